"""Float64 CPU oracle of the GSA layer's backward pass.

TEST INFRASTRUCTURE ONLY (like gsa_oracle.py): only the tests may import it;
the product path never does, and it shares no code with the CUDA path.

The notes train the layer end to end ("Speed3R: Sparse Feed-forward 3D
Reconstruction Models", Paper-Notes CVPR 2026, GSA core design); they define
only the forward.  The backward is therefore its mathematical gradient: the
forward below restates the steps of gsa_oracle.gsa_head in torch (CPU,
float64) with the region selection held fixed (TopKSelect is a discrete
choice and passes no gradient), and torch's reverse-mode differentiation
(a library primitive) gives the gradients of every input.
  pool -> compressed attention -> (selection with the given regions) ->
  upsample -> gate -> blend;  special tokens over every token.
Pinned by tests/test_oracle_backward.py: its forward equals gsa_oracle's on
the same inputs, and its gradients match central finite differences.
"""
from __future__ import annotations

import numpy as np
import torch


def _valid(grid_h, grid_w, Hp, Wp):
    return (torch.arange(Hp)[:, None] < grid_h) & (torch.arange(Wp)[None, :] < grid_w)


def forward_head(q_spec, k_spec, v_spec, q_img, k_img, v_img, w_g, idx, *, grid_h, grid_w, pool_s,
                 fixed_frames=(), gate_mode="learned", softmax_scale=None):
    """Torch float64 forward of one head with fixed regions idx [R][k].
    Tensors as in gsa_oracle.gsa_head.  Returns (o_img [F][Hp][Wp][d], o_spec [F*ns][d])."""
    F, Hp, Wp, d = q_img.shape
    ns = q_spec.shape[1]
    s = pool_s
    scale = 1.0 / np.sqrt(d) if not softmax_scale else float(softmax_scale)
    valid = _valid(grid_h, grid_w, Hp, Wp)
    vmask = valid[None, :, :, None].to(q_img.dtype)

    def pool(x):
        sums = (x * vmask).reshape(F, Hp // s, s, Wp // s, s, d).sum(dim=(2, 4))
        cnt = valid.reshape(Hp // s, s, Wp // s, s).sum(dim=(1, 3)).to(x.dtype)
        return (sums / cnt[None, :, :, None]).reshape(-1, d)

    qc, kc, vc = pool(q_img), pool(k_img), pool(v_img)
    oc = torch.softmax(qc @ kc.T * scale, dim=-1) @ vc                     # [R][d]

    # selection: window r's queries attend to the tokens of its regions (+ fixed context)
    rx = Wp // s
    R = qc.shape[0]
    r = torch.arange(R)
    f, rr = r // ((Hp // s) * rx), r % ((Hp // s) * rx)
    wi, wj = rr // rx, rr % rx
    a = torch.arange(s)
    ty = wi[:, None, None] * s + a[None, :, None]                           # [R][s][1]
    tx = wj[:, None, None] * s + a[None, None, :]                           # [R][1][s]
    qtok = ((f[:, None, None] * Hp + ty) * Wp + tx).reshape(R, s * s)
    qvalid = ((ty < grid_h) & (tx < grid_w)).reshape(R, s * s)
    sel = torch.as_tensor(np.asarray(idx), dtype=torch.long)               # [R][k]
    kf_, kr = sel // ((Hp // s) * rx), sel % ((Hp // s) * rx)
    ki, kj = kr // rx, kr % rx
    ky = ki[:, :, None, None] * s + a[None, None, :, None]
    kx = kj[:, :, None, None] * s + a[None, None, None, :]
    ktok = ((kf_[:, :, None, None] * Hp + ky) * Wp + kx).reshape(R, -1)      # [R][k*s*s]
    kvalid = ((ky < grid_h) & (kx < grid_w)).reshape(R, -1)
    qf, kff, vff = q_img.reshape(-1, d), k_img.reshape(-1, d), v_img.reshape(-1, d)
    q = qf[qtok]                                                            # [R][s*s][d]
    sc = torch.einsum("rqd,rkd->rqk", q, kff[ktok]) * scale
    sc = sc.masked_fill(~kvalid[:, None, :], float("-inf"))
    vals = vff[ktok]
    if len(fixed_frames):
        fk, fv = [], []
        for fr in fixed_frames:
            fk += [k_spec[fr], k_img[fr][valid]]
            fv += [v_spec[fr], v_img[fr][valid]]
        fk, fv = torch.cat(fk), torch.cat(fv)
        sc = torch.cat([sc, torch.einsum("rqd,nd->rqn", q, fk) * scale], dim=2)
        vals = torch.cat([vals, fv[None].expand(R, -1, -1)], dim=1)
    osel = torch.einsum("rqk,rkd->rqd", torch.softmax(sc, dim=-1), vals)    # [R][s*s][d]

    ocu = oc[:, None, :].expand_as(osel)
    if gate_mode == "comp_only":
        g = torch.ones_like(q)
    elif gate_mode == "sel_only":
        g = torch.zeros_like(q)
    else:
        g = torch.sigmoid(q @ w_g.T)
    ow = (g * ocu + (1 - g) * osel) * qvalid[..., None].to(q.dtype)
    o_img = torch.zeros(F * Hp * Wp, d, dtype=q.dtype).index_put((qtok.reshape(-1),), ow.reshape(-1, d))

    kall = torch.cat([k_spec.reshape(-1, d), k_img.reshape(-1, d)])
    vall = torch.cat([v_spec.reshape(-1, d), v_img.reshape(-1, d)])
    kv = torch.cat([torch.ones(F * ns, dtype=torch.bool), valid.reshape(-1).repeat(F)])
    ss = (q_spec.reshape(-1, d) @ kall.T * scale).masked_fill(~kv[None, :], float("-inf"))
    o_spec = torch.softmax(ss, dim=-1) @ vall
    return o_img.reshape(F, Hp, Wp, d), o_spec


NAMES = ("q_spec", "k_spec", "v_spec", "q_img", "k_img", "v_img", "w_g")


def backward_head(arrays, idx, d_o_img, d_o_spec, **kw):
    """arrays: dict of float64 numpy arrays of one head (NAMES); idx [R][k];
    d_o_img [F][Hp][Wp][d], d_o_spec [F*ns][d] (or [F][ns][d]).  Returns the
    outputs and the gradient of <o_img, d_o_img> + <o_spec, d_o_spec> with
    respect to every input (float64 numpy, keys 'd' + name)."""
    t = {n: torch.tensor(np.asarray(arrays[n], dtype=np.float64), requires_grad=True) for n in NAMES}
    o_img, o_spec = forward_head(*(t[n] for n in NAMES), idx, **kw)
    loss = (o_img * torch.as_tensor(np.asarray(d_o_img, dtype=np.float64))).sum()
    if o_spec.numel():
        loss = loss + (o_spec * torch.as_tensor(np.asarray(d_o_spec, dtype=np.float64).reshape(o_spec.shape))).sum()
    loss.backward()
    out = {"o_img": o_img.detach().numpy(), "o_spec": o_spec.detach().numpy()}
    for n in NAMES:
        gr = t[n].grad
        out["d" + n] = np.zeros(t[n].shape) if gr is None else gr.numpy()
    return out


def attention_backward_rows(q, k, v, d_o, scale, *, q_rows, k_cols, chunk=64):
    """Gradients of O = softmax(q k^T * scale) v at selected rows and key columns,
    in float64 numpy, for attention sizes that autograd cannot hold at once.

    The closed form of the softmax-attention gradient (the same step the
    backward of every attention of the layer takes):
        P = softmax(S), S = q k^T * scale,  O = P v,  D_i = sum_c dO_ic O_ic,
        dS = P o (dO v^T - D),  dq = scale dS k,  dk = scale dS^T q,  dv = P^T dO.
    dq is returned for the query rows q_rows, dk and dv for the key columns
    k_cols (these sum over every query, processed `chunk` rows at a time).
    Pinned in tests/test_oracle_backward.py against torch autograd.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    d_o = np.asarray(d_o, dtype=np.float64)
    q_rows = np.asarray(q_rows)
    k_cols = np.asarray(k_cols)
    row_set = {int(r): i for i, r in enumerate(q_rows)}
    dq = np.zeros((len(q_rows), q.shape[1]))
    dk = np.zeros((len(k_cols), k.shape[1]))
    dv = np.zeros((len(k_cols), v.shape[1]))
    for r0 in range(0, q.shape[0], chunk):
        rows = slice(r0, min(r0 + chunk, q.shape[0]))
        s = (q[rows] @ k.T) * scale
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        o = p @ v
        dd = (d_o[rows] * o).sum(axis=1, keepdims=True)
        ds = p * (d_o[rows] @ v.T - dd)
        dk += scale * ds[:, k_cols].T @ q[rows]
        dv += p[:, k_cols].T @ d_o[rows]
        for i in range(rows.start, rows.stop):
            j = row_set.get(i)
            if j is not None:
                dq[j] = scale * ds[i - rows.start] @ k
    return {"dq": dq, "dk": dk, "dv": dv}

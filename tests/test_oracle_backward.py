"""Pins of the backward oracle: its torch forward restates the numpy oracle
(equal outputs on the same inputs and regions), and its gradients match
central finite differences of that forward."""
import numpy as np
import pytest
import torch

import oracle
from oracle import gsa_backward_oracle as bo


def _inputs(F, grid, pad, ns, d, seed, fixed=()):
    rng = np.random.default_rng(seed)
    Hp, Wp = pad
    a = {}
    for n in ("q_img", "k_img", "v_img"):
        x = rng.standard_normal((F, Hp, Wp, d)) * 0.7
        x[:, grid[0]:] = 1000.0
        x[:, :, grid[1]:] = 1000.0
        a[n] = x
    for n in ("q_spec", "k_spec", "v_spec"):
        a[n] = rng.standard_normal((F, ns, d)) * 0.7
    a["w_g"] = rng.standard_normal((d, d)) / np.sqrt(d)
    return a


CASES = [
    dict(F=3, grid=(4, 6), pad=(4, 6), ns=2, d=8, s=2, k=3, fixed=(), gate="learned"),
    dict(F=4, grid=(5, 5), pad=(6, 6), ns=1, d=8, s=2, k=2, fixed=(1,), gate="learned"),
    dict(F=2, grid=(4, 4), pad=(4, 4), ns=2, d=8, s=2, k=2, fixed=(), gate="sel_only"),
    dict(F=2, grid=(4, 4), pad=(4, 4), ns=0, d=8, s=4, k=1, fixed=(), gate="comp_only"),
    # 8x8 windows on a padded grid with a fixed frame (the GPU backward's four-row-block case)
    dict(F=3, grid=(7, 8), pad=(8, 8), ns=1, d=8, s=8, k=1, fixed=(1,), gate="learned"),
]


@pytest.mark.parametrize("c", CASES)
def test_torch_forward_equals_numpy_oracle(c):
    a = _inputs(c["F"], c["grid"], c["pad"], c["ns"], c["d"], 1, c["fixed"])
    kw = dict(grid_h=c["grid"][0], grid_w=c["grid"][1], pool_s=c["s"], fixed_frames=c["fixed"], gate_mode=c["gate"])
    ref = oracle.gsa_head(a["q_spec"], a["k_spec"], a["v_spec"], a["q_img"], a["k_img"], a["v_img"], a["w_g"],
                          topk=c["k"], **kw)
    t = [torch.tensor(a[n]) for n in bo.NAMES]
    o_img, o_spec = bo.forward_head(*t, ref["idx"], **kw)
    np.testing.assert_allclose(o_img.numpy(), ref["o_img"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(o_spec.numpy(), ref["o_spec"].reshape(o_spec.shape), rtol=0, atol=1e-12)


@pytest.mark.parametrize("c", CASES[:3] + CASES[4:])
def test_gradients_match_central_differences(c):
    a = _inputs(c["F"], c["grid"], c["pad"], c["ns"], c["d"], 2, c["fixed"])
    kw = dict(grid_h=c["grid"][0], grid_w=c["grid"][1], pool_s=c["s"], fixed_frames=c["fixed"], gate_mode=c["gate"])
    ref = oracle.gsa_head(a["q_spec"], a["k_spec"], a["v_spec"], a["q_img"], a["k_img"], a["v_img"], a["w_g"],
                          topk=c["k"], **kw)
    idx = ref["idx"]
    rng = np.random.default_rng(3)
    dimg = rng.standard_normal(ref["o_img"].shape)
    dspec = rng.standard_normal(ref["o_spec"].shape)
    res = bo.backward_head(a, idx, dimg, dspec, **kw)

    def loss(arr):
        t = [torch.tensor(arr[n]) for n in bo.NAMES]
        oi, osp = bo.forward_head(*t, idx, **kw)
        return float((oi.numpy() * dimg).sum() + (osp.numpy() * dspec.reshape(osp.shape)).sum())

    eps = 1e-6
    valid = oracle.valid_grid(c["grid"][0], c["grid"][1], *c["pad"])
    for n in bo.NAMES:
        shape = a[n].shape
        for _ in range(6):
            pos = tuple(rng.integers(0, m) for m in shape)
            if n.endswith("_img") and not valid[pos[1], pos[2]]:
                assert res["d" + n][pos] == 0.0          # pads get no gradient
                continue
            up, dn = {k: v.copy() for k, v in a.items()}, {k: v.copy() for k, v in a.items()}
            up[n][pos] += eps
            dn[n][pos] -= eps
            fd = (loss(up) - loss(dn)) / (2 * eps)
            assert abs(fd - res["d" + n][pos]) <= 1e-6 * max(1.0, abs(fd)), (n, pos, fd, res["d" + n][pos])


def test_attention_backward_rows_matches_autograd():
    """The closed-form row/column gradients of one softmax attention equal torch
    autograd of O = softmax(q k^T s) v (all rows and columns, several chunk sizes)."""
    rng = np.random.default_rng(7)
    nq, nk, d, scale = 37, 53, 16, 0.31
    q, k, v, d_o = (rng.standard_normal(sh) for sh in ((nq, d), (nk, d), (nk, d), (nq, d)))
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    o = torch.softmax(tq @ tk.T * scale, dim=1) @ tv
    o.backward(torch.tensor(d_o))
    rows = np.array([0, 5, 17, 36])
    cols = np.array([1, 2, 30, 52])
    for chunk in (8, 64):
        got = bo.attention_backward_rows(q, k, v, d_o, scale, q_rows=rows, k_cols=cols, chunk=chunk)
        np.testing.assert_allclose(got["dq"], tq.grad.numpy()[rows], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(got["dk"], tk.grad.numpy()[cols], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(got["dv"], tv.grad.numpy()[cols], rtol=1e-12, atol=1e-12)

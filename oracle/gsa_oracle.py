"""Plain float64 CPU oracle of Speed3R's Global Sparse Attention (GSA) layer.

TEST INFRASTRUCTURE ONLY.  This file defines what the layer computes so that
the CUDA path can be checked against it.  Only the tests, the smoke check and
the benchmark's CPU-baseline leg may import it; the product path never does.
It shares no code with the CUDA path (it imports numpy and nothing else).

Source: "Speed3R: Sparse Feed-forward 3D Reconstruction Models" (Paper-Notes,
CVPR 2026), section "全局稀疏注意力（GSA）核心设计" (GSA core design) and its
subsections "压缩分支" (compression branch), "选择分支" (selection branch),
"门控聚合" (gated aggregation), and "Speed3R-VGGT 适配" (VGGT adaptation).
Below these are cited as [notes, <section>].

Per head h, independently (the pages treat attention per head implicitly):
  1. pool      Q/K/V_comp = s x s non-overlapping mean of Q/K/V_img
  2. comp      O'_comp = softmax(Q_comp K_comp^T / sqrt(d)) V_comp
  3. guide     S_guide = Q_comp K_comp^T (unscaled);  TopKSelect per compressed row
  4. select    O_sel[t] = softmax(q_t K_sel^T / sqrt(d)) V_sel, keys = tokens of the
               selected regions of t's window (+ VGGT fixed context)
  5. upsample  O_comp[t] = O'_comp[region(t)]
  6. gate      g = sigmoid(W_g q_t);  O_img = g * O_comp + (1-g) * O_sel
  7. special   O_spec = softmax(Q_spec K^T / sqrt(d)) V over every token
Readings taken where the pages are silent (each is listed in the design notes):
  * softmax scale 1/sqrt(d) in every attention; the guide scores are unscaled;
  * one top-k per compressed query row, over regions; ties -> lower region index;
  * the own region is a candidate like any other;
  * VGGT: candidates exclude every fixed-context frame (default), the key set adds
    every valid image token and every special token of the fixed frames;
  * padded grids: pools average valid tokens only, pad keys are never attended,
    pad queries output 0;
  * the gate is a per-head d x d matrix without bias, g per channel.
Parity status: every function here is pinned by tests/test_oracle_pins.py
(special cases, brute force, invariants); the layer as a whole has no printed
worked example on the pages, so end-to-end values are pinned only through
those special cases.
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


# ----------------------------------------------------------------------------
# generic pieces
# ----------------------------------------------------------------------------
def softmax_rows(x: np.ndarray) -> np.ndarray:
    """Row softmax in float64; rows that are all -inf are not allowed."""
    m = np.max(x, axis=-1, keepdims=True)
    e = np.exp(x - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def attention(q, k, v, scale, key_valid=None):
    """softmax(q k^T * scale) v, with invalid keys excluded.

    [notes, 特殊 token 全注意力 (special-token full attention), the
    equation O_spec = softmax(Q_spec K^T / sqrt(d_k)) V] gives the form that
    every Attention(.) of the layer follows.
    """
    s = (q @ k.T) * scale
    if key_valid is not None:
        s = np.where(key_valid[None, :], s, NEG_INF)
    return softmax_rows(s) @ v


def valid_grid(grid_h, grid_w, pad_h, pad_w) -> np.ndarray:
    """[pad_h][pad_w] bool: True where a patch token is real (not padding)."""
    return (np.arange(pad_h)[:, None] < grid_h) & (np.arange(pad_w)[None, :] < grid_w)


# ----------------------------------------------------------------------------
# 1. pooling   [notes, 压缩分支: s x s non-overlapping average pooling,
#               M'_img = M_img / s^2]
# ----------------------------------------------------------------------------
def pool(x_img: np.ndarray, grid_h: int, grid_w: int, s: int) -> np.ndarray:
    """x_img [F][Hp][Wp][d] -> x_comp [F*(Hp/s)*(Wp/s)][d].

    Region r = f*(Hp/s)*(Wp/s) + i*(Wp/s) + j covers rows s*i..s*i+s-1 and
    cols s*j..s*j+s-1 of frame f; its value is the mean of its valid tokens.
    """
    F, Hp, Wp, d = x_img.shape
    assert Hp % s == 0 and Wp % s == 0
    valid = valid_grid(grid_h, grid_w, Hp, Wp)
    xs = np.where(valid[None, :, :, None], x_img, 0.0)
    sums = xs.reshape(F, Hp // s, s, Wp // s, s, d).sum(axis=(2, 4))
    cnt = valid.reshape(Hp // s, s, Wp // s, s).sum(axis=(1, 3)).astype(np.float64)
    assert np.all(cnt > 0), "every region needs at least one valid token"
    return (sums / cnt[None, :, :, None]).reshape(F * (Hp // s) * (Wp // s), d)


# ----------------------------------------------------------------------------
# 3. top-k   [notes, 选择分支: TopKSelect(S_guide) per query -> region indices]
# ----------------------------------------------------------------------------
def topk_bruteforce(scores_row: np.ndarray, cand: np.ndarray, k: int) -> np.ndarray:
    """The k best candidate regions of one row: score descending, then index
    ascending.  Full sort; the definition itself."""
    idx = np.nonzero(cand)[0]
    order = np.lexsort((idx, -scores_row[idx]))
    return idx[order[:k]]


def topk_rows(scores: np.ndarray, cand: np.ndarray, k: int):
    """Exact top-k of every row of `scores` [n][R] over candidate columns.

    Same result as topk_bruteforce row by row.  Each row is first narrowed to
    the columns scoring at least a lower bound B of its (k+1)-th best candidate
    score, then those columns are sorted by (score desc, index asc).  B is the
    (k+1)-th largest of the row's block maxima (columns in 128 blocks): at least
    k+1 blocks hold a value >= B, so at least k+1 candidates score >= B and every
    column of the top k+1 (ties of the k-th value included) survives the cut.
    Returns (idx [n][k], gap_rel [n]) where gap_rel is
    (s_k - s_{k+1}) / max(|s_k|, 1e-30) over the candidate scores (inf when
    there is no (k+1)-th candidate).
    """
    n, R = scores.shape
    ncand = int(cand.sum())
    assert 1 <= k <= ncand
    s = scores if cand.all() else np.where(cand[None, :], scores, NEG_INF)
    out = np.empty((n, k), dtype=np.int64)
    gap = np.full(n, np.inf)
    kk = min(k + 1, ncand)
    nb = min(128, R)
    starts = (np.arange(nb) * R) // nb                                # nb non-empty column blocks
    bmax = np.maximum.reduceat(s, starts, axis=1)                     # [n][nb]
    cnt = (bmax > NEG_INF).sum(axis=1)
    if np.all(cnt >= kk):
        bound = -np.partition(-bmax, kk - 1, axis=1)[:, kk - 1]       # kk-th largest block max
    else:
        bound = np.full(n, NEG_INF)                                   # few candidate blocks: no cut
    for i in range(n):
        cols = np.nonzero(s[i] >= bound[i])[0]
        cols = cols[s[i, cols] > NEG_INF] if bound[i] == NEG_INF else cols
        order = np.lexsort((cols, -s[i, cols]))
        out[i] = cols[order[:k]]
        if ncand > k:
            sk = s[i, cols[order[k - 1]]]
            sk1 = s[i, cols[order[k]]]
            gap[i] = (sk - sk1) / max(abs(sk), 1e-30)
    return out, gap


def candidate_regions(num_frames, regions_per_frame, fixed_frames) -> np.ndarray:
    """[R] bool: regions eligible for the dynamic top-k.

    pi^3: every region.  VGGT [notes, Speed3R-VGGT 适配]: the dynamic top-k
    draws from frames outside the fixed global context.
    """
    cand = np.ones(num_frames * regions_per_frame, dtype=bool)
    for f in fixed_frames:
        cand[f * regions_per_frame:(f + 1) * regions_per_frame] = False
    return cand


# ----------------------------------------------------------------------------
# 4. selection   [notes, 选择分支: O_sel = Attention(Q_img, K_sel, V_sel); the
#                 queries of one compression window share one KV set]
# ----------------------------------------------------------------------------
def region_tokens(regions: np.ndarray, Hp: int, Wp: int, s: int):
    """Flat image-token indices (into [F*Hp*Wp]) of the given regions.

    regions [...] -> tokens [..., s*s] in row-major order inside the region,
    plus (y, x) of each token for validity checks.
    """
    rpf = (Hp // s) * (Wp // s)
    f = regions // rpf
    i = (regions % rpf) // (Wp // s)
    j = regions % (Wp // s)
    a = np.arange(s)
    y = i[..., None, None] * s + a[:, None]          # [..., s, 1]
    x = j[..., None, None] * s + a[None, :]          # [..., 1, s]
    y, x = np.broadcast_arrays(y, x)
    tok = (f[..., None, None] * Hp + y) * Wp + x
    sh = regions.shape + (s * s,)
    return tok.reshape(sh), y.reshape(sh), x.reshape(sh)


def fixed_context_keys(k_img, v_img, k_spec, v_spec, fixed_frames, grid_h, grid_w):
    """Keys/values of the VGGT fixed global context: every special token and
    every valid image token of each fixed frame [notes, Speed3R-VGGT 适配:
    all tokens of the reference frame and of frames sampled every 100]."""
    F, Hp, Wp, d = k_img.shape
    valid = valid_grid(grid_h, grid_w, Hp, Wp).reshape(-1)
    ks, vs = [], []
    for f in fixed_frames:
        ks.append(k_spec[f]); vs.append(v_spec[f])
        ks.append(k_img[f].reshape(-1, d)[valid]); vs.append(v_img[f].reshape(-1, d)[valid])
    if not ks:
        return np.zeros((0, d)), np.zeros((0, d))
    return np.concatenate(ks), np.concatenate(vs)


def selection_attention(q_img, k_img, v_img, idx, windows, *, grid_h, grid_w, s,
                        scale, fixed_k=None, fixed_v=None, batch=256):
    """O_sel for the query tokens of `windows` (compressed-row indices).

    q_img/k_img/v_img [F][Hp][Wp][d]; idx [R][k] selected regions per window
    (only rows in `windows` are read).  Returns o [len(windows)][s*s][d] and the
    tokens' flat indices [len(windows)][s*s] and validity.
    """
    F, Hp, Wp, d = q_img.shape
    qf = q_img.reshape(-1, d); kf = k_img.reshape(-1, d); vf = v_img.reshape(-1, d)
    windows = np.asarray(windows)
    qtok, qy, qx = region_tokens(windows, Hp, Wp, s)
    qvalid = (qy < grid_h) & (qx < grid_w)
    out = np.zeros((len(windows), s * s, d))
    nfix = 0 if fixed_k is None else fixed_k.shape[0]
    for b0 in range(0, len(windows), batch):
        w = windows[b0:b0 + batch]
        sel = idx[w]                                          # [B][k]
        ktok, ky, kx = region_tokens(sel, Hp, Wp, s)          # [B][k][s*s]
        B = len(w)
        ktok = ktok.reshape(B, -1)
        kvalid = ((ky < grid_h) & (kx < grid_w)).reshape(B, -1)
        q = qf[qtok[b0:b0 + B]]                               # [B][s*s][d]
        sc = np.einsum("bqd,bkd->bqk", q, kf[ktok]) * scale
        sc = np.where(kvalid[:, None, :], sc, NEG_INF)
        if nfix:
            sf = np.einsum("bqd,nd->bqn", q, fixed_k) * scale
            sc = np.concatenate([sc, sf], axis=2)
        p = softmax_rows(sc)
        o = np.einsum("bqk,bkd->bqd", p[:, :, :ktok.shape[1]], vf[ktok])
        if nfix:
            o += np.einsum("bqn,nd->bqd", p[:, :, ktok.shape[1]:], fixed_v)
        out[b0:b0 + B] = o
    out = np.where(qvalid[..., None], out, 0.0)
    return out, qtok, qvalid


def selection_attention_union(q_img, k_img, v_img, k_spec, v_spec, idx, windows, *,
                              grid_h, grid_w, s, scale, fixed_frames):
    """Alternative VGGT reading (oracle flag only; tiny inputs): the key set is
    the set union of the selected regions' tokens and the fixed context, with no
    duplicated key.  Used with candidates that exclude only frame 0."""
    F, Hp, Wp, d = q_img.shape
    valid = valid_grid(grid_h, grid_w, Hp, Wp).reshape(-1)
    nimg = F * Hp * Wp
    qf = q_img.reshape(-1, d)
    kall = np.concatenate([k_img.reshape(-1, d), k_spec.reshape(-1, d)])
    vall = np.concatenate([v_img.reshape(-1, d), v_spec.reshape(-1, d)])
    ns = k_spec.shape[1]
    base = np.zeros(nimg + F * ns, dtype=bool)
    for f in fixed_frames:
        base[f * Hp * Wp:(f + 1) * Hp * Wp] = valid
        base[nimg + f * ns: nimg + (f + 1) * ns] = True
    windows = np.asarray(windows)
    qtok, qy, qx = region_tokens(windows, Hp, Wp, s)
    qvalid = (qy < grid_h) & (qx < grid_w)
    out = np.zeros((len(windows), s * s, d))
    for wi, w in enumerate(windows):
        m = base.copy()
        ktok, ky, kx = region_tokens(idx[w], Hp, Wp, s)
        m[ktok[(ky < grid_h) & (kx < grid_w)]] = True
        out[wi] = attention(qf[qtok[wi]], kall, vall, scale, m)
    out = np.where(qvalid[..., None], out, 0.0)
    return out, qtok, qvalid


# ----------------------------------------------------------------------------
# 6. gate    [notes, 门控聚合: g = sigmoid(W_g Q_img),
#             O_img = g * O_comp + (1 - g) * O_sel]
# ----------------------------------------------------------------------------
def sigmoid(x):
    with np.errstate(over="ignore"):      # exp(+large) -> inf -> g = 0 exactly
        return 1.0 / (1.0 + np.exp(-x))


def gate_blend(q, o_comp, o_sel, w_g, gate_mode="learned"):
    """q, o_comp, o_sel [n][d]; w_g [d][d] (row = output channel)."""
    if gate_mode == "comp_only":
        g = np.ones_like(q)
    elif gate_mode == "sel_only":
        g = np.zeros_like(q)
    else:
        g = sigmoid(q @ w_g.T)
    return g * o_comp + (1.0 - g) * o_sel


# ----------------------------------------------------------------------------
# the whole layer, one head at a time
# ----------------------------------------------------------------------------
def gsa_head(q_spec, k_spec, v_spec, q_img, k_img, v_img, w_g, *, grid_h, grid_w,
             pool_s, topk, fixed_frames=(), gate_mode="learned", softmax_scale=None,
             forced_idx=None, windows=None, spec_rows=None, candidates="exclude_fixed"):
    """One head of the GSA layer.

    q_spec/k_spec/v_spec [F][n_spec][d]; q_img/k_img/v_img [F][Hp][Wp][d];
    w_g [d][d].  `windows` restricts the image path to some compressed rows
    (default: all); `spec_rows` restricts the special path to some special-token
    rows (default: all).  `forced_idx` [R][k] replaces the top-k result (rows
    outside `windows` are ignored).  Returns a dict of float64 arrays.
    """
    F, Hp, Wp, d = q_img.shape
    ns = q_spec.shape[1]
    s = pool_s
    scale = 1.0 / np.sqrt(d) if not softmax_scale else float(softmax_scale)
    rpf = (Hp // s) * (Wp // s)
    R = F * rpf
    valid = valid_grid(grid_h, grid_w, Hp, Wp)

    # 1. pool
    qc = pool(q_img, grid_h, grid_w, s)
    kc = pool(k_img, grid_h, grid_w, s)
    vc = pool(v_img, grid_h, grid_w, s)
    win = np.arange(R) if windows is None else np.asarray(windows)

    # 2. compressed attention over every region (rows restricted to `win`)
    oc = attention(qc[win], kc, vc, scale)

    # 3. guide scores and top-k
    if candidates == "exclude_fixed":
        cand = candidate_regions(F, rpf, fixed_frames)
    else:  # "exclude_reference": the alternative reading, frame 0 only
        cand = candidate_regions(F, rpf, (0,) if fixed_frames else ())
    guide = qc[win] @ kc.T
    idx_w, gap_w = topk_rows(guide, cand, topk)
    idx = np.full((R, topk), -1, dtype=np.int64)
    idx[win] = idx_w
    gap = np.full(R, np.nan)
    gap[win] = gap_w
    use_idx = idx if forced_idx is None else np.asarray(forced_idx)

    # 4. selection
    if candidates == "exclude_fixed":
        fk, fv = fixed_context_keys(k_img, v_img, k_spec, v_spec, fixed_frames,
                                    grid_h, grid_w)
        osel, qtok, qvalid = selection_attention(
            q_img, k_img, v_img, use_idx, win, grid_h=grid_h, grid_w=grid_w, s=s,
            scale=scale, fixed_k=fk if len(fixed_frames) else None, fixed_v=fv)
    else:
        osel, qtok, qvalid = selection_attention_union(
            q_img, k_img, v_img, k_spec, v_spec, use_idx, win, grid_h=grid_h,
            grid_w=grid_w, s=s, scale=scale, fixed_frames=fixed_frames)

    # 5. upsample + 6. gate
    ocomp_up = np.broadcast_to(oc[:, None, :], osel.shape)
    qf = q_img.reshape(-1, d)[qtok]
    oimg_w = gate_blend(qf.reshape(-1, d), ocomp_up.reshape(-1, d), osel.reshape(-1, d),
                        w_g, gate_mode).reshape(osel.shape)
    oimg_w = np.where(qvalid[..., None], oimg_w, 0.0)

    # 7. special tokens attend to every special token and every valid image token
    kall = np.concatenate([k_spec.reshape(-1, d), k_img.reshape(-1, d)])
    vall = np.concatenate([v_spec.reshape(-1, d), v_img.reshape(-1, d)])
    kvalid = np.concatenate([np.ones(F * ns, dtype=bool), np.tile(valid.reshape(-1), F)])
    qs = q_spec.reshape(-1, d)
    srows = np.arange(F * ns) if spec_rows is None else np.asarray(spec_rows)
    ospec = attention(qs[srows], kall, vall, scale, kvalid) if len(srows) else np.zeros((0, d))

    res = dict(q_comp=qc, k_comp=kc, v_comp=vc, windows=win, o_comp_prime=oc,
               idx=idx, gap=gap, o_sel=osel, o_img_windows=oimg_w, tokens=qtok,
               token_valid=qvalid, spec_rows=srows, o_spec=ospec)
    if windows is None:
        o_img = np.zeros((F * Hp * Wp, d))
        o_img[qtok.reshape(-1)] = oimg_w.reshape(-1, d)
        o_sel_full = np.zeros((F * Hp * Wp, d))
        o_sel_full[qtok.reshape(-1)] = osel.reshape(-1, d)
        res["o_img"] = o_img.reshape(F, Hp, Wp, d)
        res["o_sel_full"] = o_sel_full.reshape(F, Hp, Wp, d)
    return res


def gsa_forward(q_spec, k_spec, v_spec, q_img, k_img, v_img, w_g, **kw):
    """All heads: inputs carry a leading head axis.  Returns per-head results
    stacked along axis 0 for o_img [H][F][Hp][Wp][d], o_spec [H][F*n_spec][d],
    idx [H][R][k], o_comp_prime [H][R][d], gap [H][R] and the pooled tensors."""
    H = q_img.shape[0]
    per = [gsa_head(q_spec[h], k_spec[h], v_spec[h], q_img[h], k_img[h], v_img[h],
                    w_g[h], **kw) for h in range(H)]
    keys = ["q_comp", "k_comp", "v_comp", "o_comp_prime", "idx", "gap", "o_spec"]
    if "o_img" in per[0]:
        keys += ["o_img", "o_sel_full"]
    return {k: np.stack([p[k] for p in per]) for k in keys}


# ----------------------------------------------------------------------------
# dense global attention of the same tokens (the speedup comparison)
# ----------------------------------------------------------------------------
def dense_token_layout_valid(num_frames, num_special, grid_h, grid_w, pad_h, pad_w):
    """[F*(n_spec + Hp*Wp)] bool for the dense layout: per frame the special
    tokens, then the padded image grid."""
    v = valid_grid(grid_h, grid_w, pad_h, pad_w).reshape(-1)
    per = np.concatenate([np.ones(num_special, dtype=bool), v])
    return np.tile(per, num_frames)


def dense_attention(q, k, v, key_valid=None, rows=None, softmax_scale=None):
    """Dense global attention softmax(Q K^T / sqrt(d)) V of one head over every
    token [notes, 推理延迟对比: the "Full Attn." baseline]; `rows` restricts
    the query rows."""
    d = q.shape[1]
    scale = 1.0 / np.sqrt(d) if not softmax_scale else float(softmax_scale)
    qq = q if rows is None else q[np.asarray(rows)]
    return attention(qq, k, v, scale, key_valid)

"""Pins of the CPU oracle against facts fixed by the method's definition and by
mathematics (no GPU).  Each test would fail under a plausible slip in the
oracle: a dropped term, a wrong scale, a transposed operand, a wrong region
order, a wrong tie rule, a leaking pad.

The special cases come from "Speed3R: Sparse Feed-forward 3D Reconstruction
Models" (Paper-Notes, CVPR 2026), GSA core design: with s = 1 the compression
branch is dense attention; with top-k = every region the selection branch is
dense attention; forcing the gate isolates each branch.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from gsa_inputs import CONFIGS, GSAConfig, make_inputs, to_f64_numpy


def _np_inputs(cfg, seed=0):
    x = make_inputs(cfg, seed=seed)
    return {k: to_f64_numpy(v) for k, v in x.items()}


def _sdpa(q, k, v, mask=None, scale=None):
    """torch's reference attention in float64 on CPU (an independent routine)."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(a)) for a in (q, k, v))
    m = None if mask is None else torch.from_numpy(np.broadcast_to(mask, (q.shape[0], k.shape[0])).copy())
    return torch.nn.functional.scaled_dot_product_attention(
        tq[None], tk[None], tv[None], attn_mask=None if m is None else m[None], scale=scale)[0].numpy()


def _textbook_attention(q, k, v, scale):
    """Per-query loop: weights exp(q.k*scale) normalised, then the weighted sum."""
    out = np.zeros((q.shape[0], v.shape[1]))
    for i in range(q.shape[0]):
        sc = [float(np.dot(q[i], k[j])) * scale for j in range(k.shape[0])]
        mx = max(sc)
        w = [math.exp(t - mx) for t in sc]
        z = sum(w)
        for j in range(k.shape[0]):
            out[i] += (w[j] / z) * v[j]
    return out


SMALL = GSAConfig("small", 3, 6, 6, 6, 6, 2, 2, 16, 2, 3, "fp32")
SMALL_PAD = GSAConfig("small_pad", 3, 5, 7, 6, 8, 2, 2, 16, 2, 3, "fp32")
SMALL_S1 = GSAConfig("small_s1", 2, 3, 4, 3, 4, 1, 1, 16, 1, 2, "fp32")
SMALL_VGGT = GSAConfig("small_vggt", 5, 3, 3, 4, 4, 2, 1, 16, 2, 3, "fp32", (0, 3))


def _run(cfg, a, **kw):
    return oracle.gsa_forward(a["q_spec"], a["k_spec"], a["v_spec"], a["q_img"], a["k_img"],
                              a["v_img"], a["w_g"], grid_h=cfg.grid_h, grid_w=cfg.grid_w,
                              pool_s=cfg.pool_s, topk=kw.pop("topk", cfg.topk),
                              fixed_frames=cfg.fixed_frames, **kw)


# ---------------------------------------------------------------- pooling
@pytest.mark.parametrize("cfg", [SMALL, SMALL_PAD, SMALL_VGGT])
def test_pool_equals_loop_mean(cfg):
    a = _np_inputs(cfg)
    x = a["k_img"][0]
    F, Hp, Wp, d = x.shape
    s = cfg.pool_s
    got = oracle.pool(x, cfg.grid_h, cfg.grid_w, s)
    r = 0
    for f in range(F):
        for i in range(Hp // s):
            for j in range(Wp // s):
                toks = [x[f, y, xx] for y in range(i * s, i * s + s) for xx in range(j * s, j * s + s)
                        if y < cfg.grid_h and xx < cfg.grid_w]
                np.testing.assert_allclose(got[r], np.mean(toks, axis=0), rtol=1e-13, atol=1e-13)
                r += 1
    assert r == got.shape[0]


def test_pool_s1_is_identity():
    a = _np_inputs(SMALL_S1)
    x = a["q_img"][0]
    np.testing.assert_array_equal(oracle.pool(x, 3, 4, 1), x.reshape(-1, x.shape[-1]))


# ---------------------------------------------------------------- generic attention
def test_attention_textbook_and_library():
    rng = np.random.default_rng(1)
    q, k, v = rng.normal(size=(5, 8)), rng.normal(size=(7, 8)), rng.normal(size=(7, 3))
    sc = 1 / math.sqrt(8)
    got = oracle.attention(q, k, v, sc)
    np.testing.assert_allclose(got, _textbook_attention(q, k, v, sc), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got, _sdpa(q, k, v), rtol=1e-12, atol=1e-12)
    # a key shift adds the same constant to every score of a row: no change
    u = rng.normal(size=8)
    np.testing.assert_allclose(oracle.attention(q, k + u, v, sc), got, rtol=1e-11, atol=1e-11)
    # an invalid key is exactly absent
    mask = np.array([1, 1, 0, 1, 1, 1, 0], dtype=bool)
    np.testing.assert_allclose(oracle.attention(q, k, v, sc, mask),
                               _textbook_attention(q, k[mask], v[mask], sc), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- compression branch
def test_compression_s1_equals_dense_image_attention():
    cfg = SMALL_S1
    a = _np_inputs(cfg)
    r = _run(cfg, a)
    d = cfg.head_dim
    for h in range(cfg.num_heads):
        q = a["q_img"][h].reshape(-1, d); k = a["k_img"][h].reshape(-1, d); v = a["v_img"][h].reshape(-1, d)
        np.testing.assert_allclose(r["o_comp_prime"][h], _sdpa(q, k, v), rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(r["o_comp_prime"][h], _textbook_attention(q, k, v, 1 / math.sqrt(d)),
                                   rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------------- top-k
def test_topk_rows_equals_bruteforce_sort_with_ties():
    rng = np.random.default_rng(7)
    n, R, k = 40, 50, 6
    sc = rng.integers(-4, 5, size=(n, R)).astype(np.float64)   # many exact ties
    sc[:5] = 0.0                                             # all-tie rows
    cand = rng.random(R) > 0.2
    idx, gap = oracle.topk_rows(sc, cand, k)
    for i in range(n):
        want = sorted([j for j in range(R) if cand[j]], key=lambda j: (-sc[i, j], j))[:k]
        assert list(idx[i]) == want
        assert list(oracle.topk_bruteforce(sc[i], cand, k)) == want
        rest = sorted([sc[i, j] for j in range(R) if cand[j]], reverse=True)
        sk, sk1 = rest[k - 1], rest[k]
        assert gap[i] == pytest.approx((sk - sk1) / max(abs(sk), 1e-30))
    assert np.all(idx[:5] == np.nonzero(cand)[0][:k])   # ties -> lowest indices


def test_topk_rows_wide_rows_against_bruteforce():
    """Rows much wider than the 128 column blocks topk_rows narrows with: the
    best values crowded into one block, exact ties at the k-th place, whole
    blocks that are not candidates, and rows with fewer candidate blocks than
    k+1."""
    rng = np.random.default_rng(11)
    n, R, k = 24, 3000, 32
    sc = rng.integers(-50, 50, size=(n, R)).astype(np.float64)
    sc[0, 100:140] = 1000.0 + np.arange(40) // 3             # the top 40 inside one block, with ties
    sc[1, :] = 0.0
    sc[1, 2000:2010] = 5.0                                   # 10 winners, then a 2990-way tie
    sc[2] = rng.normal(size=R)
    cand = np.ones(R, dtype=bool)
    cand[500:900] = False                                    # whole blocks excluded
    sparse = np.zeros(R, dtype=bool)
    sparse[[3, 7, 2999, 1500, 1501] + list(range(40, 80))] = True   # candidates in few blocks
    for c in (cand, sparse):
        idx, gap = oracle.topk_rows(sc, c, k)
        for i in range(n):
            want = oracle.topk_bruteforce(sc[i], c, k)
            assert list(idx[i]) == list(want)
            rest = np.sort(sc[i, c])[::-1]
            assert gap[i] == pytest.approx((rest[k - 1] - rest[k]) / max(abs(rest[k - 1]), 1e-30))


def test_topk_continuous_and_scale_invariant():
    rng = np.random.default_rng(3)
    sc = rng.normal(size=(30, 200))
    cand = np.ones(200, dtype=bool)
    idx, _ = oracle.topk_rows(sc, cand, 10)
    want = np.argsort(-sc, axis=1, kind="stable")[:, :10]
    assert np.array_equal(idx, want)
    idx2, _ = oracle.topk_rows(sc * 3.7 + 0.0, cand, 10)
    assert np.array_equal(idx, idx2)


def test_topk_all_candidates_returns_everything():
    rng = np.random.default_rng(4)
    sc = rng.normal(size=(6, 9))
    cand = np.ones(9, dtype=bool)
    idx, gap = oracle.topk_rows(sc, cand, 9)
    assert all(sorted(r) == list(range(9)) for r in idx)
    assert np.all(np.isinf(gap))


def test_guide_scores_are_pooled_dot_products():
    """Top-k of one row equals the brute-force top-k of the unscaled pooled dots."""
    cfg = SMALL
    a = _np_inputs(cfg)
    r = _run(cfg, a)
    qc = oracle.pool(a["q_img"][1], cfg.grid_h, cfg.grid_w, cfg.pool_s)
    kc = oracle.pool(a["k_img"][1], cfg.grid_h, cfg.grid_w, cfg.pool_s)
    for row in range(qc.shape[0]):
        sc = np.array([float(np.dot(qc[row], kc[j])) for j in range(kc.shape[0])])
        want = sorted(range(len(sc)), key=lambda j: (-sc[j], j))[:cfg.topk]
        assert list(r["idx"][1, row]) == want


# ---------------------------------------------------------------- selection branch
@pytest.mark.parametrize("cfg", [SMALL, SMALL_PAD])
def test_selection_with_all_regions_equals_dense_image_attention(cfg):
    a = _np_inputs(cfg)
    R = cfg.num_regions
    r = _run(cfg, a, topk=R, gate_mode="sel_only")
    d = cfg.head_dim
    valid = oracle.valid_grid(cfg.grid_h, cfg.grid_w, cfg.pad_h, cfg.pad_w).reshape(-1)
    valid = np.tile(valid, cfg.num_frames)
    for h in range(cfg.num_heads):
        q = a["q_img"][h].reshape(-1, d); k = a["k_img"][h].reshape(-1, d); v = a["v_img"][h].reshape(-1, d)
        want = _sdpa(q, k, v, mask=valid[None, :])
        got = r["o_sel_full"][h].reshape(-1, d)
        np.testing.assert_allclose(got[valid], want[valid], rtol=1e-10, atol=1e-10)
        np.testing.assert_array_equal(got[~valid], 0.0)
        np.testing.assert_allclose(r["o_img"][h].reshape(-1, d), got, rtol=0, atol=0)


def test_vggt_all_candidates_equals_dense_over_images_and_fixed_specials():
    cfg = SMALL_VGGT
    a = _np_inputs(cfg)
    rpf = cfg.regions_per_frame
    ncand = cfg.num_regions - rpf * len(cfg.fixed_frames)
    d, F, ns = cfg.head_dim, cfg.num_frames, cfg.num_special
    valid = np.tile(oracle.valid_grid(cfg.grid_h, cfg.grid_w, cfg.pad_h, cfg.pad_w).reshape(-1), F)
    spec_ok = np.zeros(F * ns, dtype=bool)
    for f in cfg.fixed_frames:
        spec_ok[f * ns:(f + 1) * ns] = True
    for mode in ("exclude_fixed", "exclude_reference"):
        k_all = ncand if mode == "exclude_fixed" else cfg.num_regions - rpf
        r = _run(cfg, a, topk=k_all, gate_mode="sel_only", candidates=mode)
        for h in range(cfg.num_heads):
            q = a["q_img"][h].reshape(-1, d)
            k = np.concatenate([a["k_img"][h].reshape(-1, d), a["k_spec"][h].reshape(-1, d)])
            v = np.concatenate([a["v_img"][h].reshape(-1, d), a["v_spec"][h].reshape(-1, d)])
            mask = np.concatenate([valid, spec_ok])
            want = _sdpa(q, k, v, mask=mask[None, :])
            got = r["o_img"][h].reshape(-1, d)
            np.testing.assert_allclose(got[valid], want[valid], rtol=1e-10, atol=1e-10)


def test_vggt_fixed_frames_never_selected():
    cfg = SMALL_VGGT
    a = _np_inputs(cfg)
    r = _run(cfg, a)
    frames = r["idx"] // cfg.regions_per_frame
    assert not np.isin(frames, cfg.fixed_frames).any()


def test_forced_index_reproduces_selection():
    cfg = SMALL_PAD
    a = _np_inputs(cfg)
    r = _run(cfg, a)
    h = 0
    hr = oracle.gsa_head(a["q_spec"][h], a["k_spec"][h], a["v_spec"][h], a["q_img"][h], a["k_img"][h],
                         a["v_img"][h], a["w_g"][h], grid_h=cfg.grid_h, grid_w=cfg.grid_w,
                         pool_s=cfg.pool_s, topk=cfg.topk, forced_idx=r["idx"][h])
    np.testing.assert_array_equal(hr["o_img"], r["o_img"][h])
    # a different forced set changes the selection output
    other = np.roll(r["idx"][h], 1, axis=0)
    hr2 = oracle.gsa_head(a["q_spec"][h], a["k_spec"][h], a["v_spec"][h], a["q_img"][h], a["k_img"][h],
                          a["v_img"][h], a["w_g"][h], grid_h=cfg.grid_h, grid_w=cfg.grid_w,
                          pool_s=cfg.pool_s, topk=cfg.topk, forced_idx=other)
    assert np.abs(hr2["o_sel_full"] - r["o_sel_full"][h]).max() > 1e-3


def test_selection_window_closed_form_zero_query():
    """q = 0 gives uniform weights: O_sel is the plain mean of the selected
    regions' valid value tokens, and the gate is sigmoid(0) = 1/2."""
    cfg = SMALL_PAD
    a = _np_inputs(cfg)
    a["q_img"][:] = 0.0
    r = _run(cfg, a)
    s, Hp, Wp, d = cfg.pool_s, cfg.pad_h, cfg.pad_w, cfg.head_dim
    # all guide scores are 0 -> ties -> the lowest region indices win
    assert np.all(r["idx"] == np.arange(cfg.topk))
    toks = []
    for reg in range(cfg.topk):
        f, rem = divmod(reg, (Hp // s) * (Wp // s))
        i, j = divmod(rem, Wp // s)
        toks += [(f, y, x) for y in range(i * s, i * s + s) for x in range(j * s, j * s + s)
                 if y < cfg.grid_h and x < cfg.grid_w]
    for h in range(cfg.num_heads):
        mean_v = np.mean([a["v_img"][h][t] for t in toks], axis=0)
        np.testing.assert_allclose(r["o_sel_full"][h, 0, 0, 0], mean_v, rtol=1e-12, atol=1e-12)
        vc = oracle.pool(a["v_img"][h], cfg.grid_h, cfg.grid_w, s)
        np.testing.assert_allclose(r["o_comp_prime"][h, 0], vc.mean(axis=0), rtol=1e-12, atol=1e-12)
        want = 0.5 * vc.mean(axis=0) + 0.5 * mean_v
        np.testing.assert_allclose(r["o_img"][h, 0, 0, 0], want, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- gate
def test_gate_modes_isolate_branches():
    cfg = SMALL_PAD
    a = _np_inputs(cfg)
    s, d = cfg.pool_s, cfg.head_dim
    rc = _run(cfg, a, gate_mode="comp_only")
    rs = _run(cfg, a, gate_mode="sel_only")
    valid = oracle.valid_grid(cfg.grid_h, cfg.grid_w, cfg.pad_h, cfg.pad_w)
    for h in range(cfg.num_heads):
        up = rc["o_comp_prime"][h].reshape(cfg.num_frames, cfg.pad_h // s, cfg.pad_w // s, d)
        up = np.repeat(np.repeat(up, s, axis=1), s, axis=2)
        up = np.where(valid[None, :, :, None], up, 0.0)
        np.testing.assert_allclose(rc["o_img"][h], up, rtol=0, atol=1e-15)
        np.testing.assert_array_equal(rs["o_img"][h], rs["o_sel_full"][h])
    a0 = dict(a); a0["w_g"] = np.zeros_like(a["w_g"])
    r0 = _run(cfg, a0)
    np.testing.assert_allclose(r0["o_img"], 0.5 * (rc["o_img"] + rs["o_img"]), rtol=1e-12, atol=1e-12)


def test_gate_orientation_row_is_output_channel():
    """W_g with one large entry W[c_out, c_in] and q[c_in] > 0 drives g[c_out]
    to 1 (comp branch) and leaves every other channel at g = 1/2."""
    cfg = SMALL
    a = _np_inputs(cfg)
    c_out, c_in = 3, 11
    a["w_g"][:] = 0.0
    a["w_g"][:, c_out, c_in] = 1e4
    a["q_img"][..., c_in] = np.abs(a["q_img"][..., c_in]) + 1.0
    r = _run(cfg, a)
    rc = _run(cfg, a, gate_mode="comp_only")
    rs = _run(cfg, a, gate_mode="sel_only")
    np.testing.assert_allclose(r["o_img"][..., c_out], rc["o_img"][..., c_out], rtol=1e-12, atol=1e-12)
    others = [c for c in range(cfg.head_dim) if c != c_out]
    np.testing.assert_allclose(r["o_img"][..., others],
                               0.5 * (rc["o_img"][..., others] + rs["o_img"][..., others]),
                               rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- invariants
@pytest.mark.parametrize("cfg", [SMALL, SMALL_PAD, SMALL_VGGT])
def test_constant_value_gives_constant_output(cfg):
    a = _np_inputs(cfg)
    c = np.linspace(-1, 1, cfg.head_dim)
    valid = oracle.valid_grid(cfg.grid_h, cfg.grid_w, cfg.pad_h, cfg.pad_w)
    a["v_img"][:] = np.where(valid[None, None, :, :, None], c, 1000.0)
    a["v_spec"][:] = c
    r = _run(cfg, a)
    got = r["o_img"][:, :, valid, :]
    np.testing.assert_allclose(got, np.broadcast_to(c, got.shape), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["o_spec"], np.broadcast_to(c, r["o_spec"].shape), rtol=1e-12, atol=1e-12)


def test_frame_permutation_equivariance():
    cfg = SMALL
    a = _np_inputs(cfg)
    r = _run(cfg, a)
    perm = np.array([2, 0, 1])
    b = {k: (v[:, perm] if k != "w_g" else v) for k, v in a.items()}
    rb = _run(cfg, b)
    np.testing.assert_allclose(rb["o_img"], r["o_img"][:, perm], rtol=1e-12, atol=1e-12)
    rpf = cfg.regions_per_frame
    inv = np.argsort(perm)     # old frame f sits at new position inv[f]
    def relabel(idx):
        return inv[idx // rpf] * rpf + idx % rpf
    R = cfg.num_regions
    old_rows = np.concatenate([np.arange(rpf) + f * rpf for f in perm])
    gap = r["gap"][:, old_rows]
    for h in range(cfg.num_heads):
        for new_row, old_row in enumerate(old_rows):
            if gap[h, new_row] > 1e-9:
                assert sorted(rb["idx"][h, new_row]) == sorted(relabel(r["idx"][h, old_row]))


@pytest.mark.parametrize("cfg", [SMALL_PAD, SMALL_VGGT])
def test_pad_values_do_not_leak(cfg):
    a = _np_inputs(cfg)
    r = _run(cfg, a)
    valid = oracle.valid_grid(cfg.grid_h, cfg.grid_w, cfg.pad_h, cfg.pad_w)
    b = {k: v.copy() for k, v in a.items()}
    rng = np.random.default_rng(5)
    for t in ("q_img", "k_img", "v_img"):
        b[t][:, :, ~valid, :] = rng.normal(size=b[t][:, :, ~valid, :].shape) * 50
    rb = _run(cfg, b)
    np.testing.assert_array_equal(rb["o_img"], r["o_img"])
    np.testing.assert_array_equal(rb["o_spec"], r["o_spec"])
    np.testing.assert_array_equal(r["o_img"][:, :, ~valid, :], 0.0)


# ---------------------------------------------------------------- special tokens, dense
@pytest.mark.parametrize("cfg", [SMALL, SMALL_PAD])
def test_special_tokens_equal_dense_attention(cfg):
    a = _np_inputs(cfg)
    r = _run(cfg, a)
    d = cfg.head_dim
    valid = np.tile(oracle.valid_grid(cfg.grid_h, cfg.grid_w, cfg.pad_h, cfg.pad_w).reshape(-1),
                    cfg.num_frames)
    for h in range(cfg.num_heads):
        k = np.concatenate([a["k_spec"][h].reshape(-1, d), a["k_img"][h].reshape(-1, d)])
        v = np.concatenate([a["v_spec"][h].reshape(-1, d), a["v_img"][h].reshape(-1, d)])
        mask = np.concatenate([np.ones(cfg.num_spec, dtype=bool), valid])
        want = _sdpa(a["q_spec"][h].reshape(-1, d), k, v, mask=mask[None, :])
        np.testing.assert_allclose(r["o_spec"][h], want, rtol=1e-11, atol=1e-11)


def test_dense_attention_layout_and_mask():
    cfg = SMALL_PAD
    lay = oracle.dense_token_layout_valid(cfg.num_frames, cfg.num_special, cfg.grid_h, cfg.grid_w,
                                          cfg.pad_h, cfg.pad_w)
    per = cfg.num_special + cfg.pad_h * cfg.pad_w
    assert lay.shape == (cfg.num_frames * per,)
    for f, t in itertools.product(range(cfg.num_frames), range(per)):
        if t < cfg.num_special:
            assert lay[f * per + t]
        else:
            y, x = divmod(t - cfg.num_special, cfg.pad_w)
            assert lay[f * per + t] == (y < cfg.grid_h and x < cfg.grid_w)
    rng = np.random.default_rng(0)
    q, k, v = (rng.normal(size=(lay.size, 16)) for _ in range(3))
    rows = np.array([0, 5, 17])
    np.testing.assert_allclose(oracle.dense_attention(q, k, v, lay, rows=rows),
                               _sdpa(q[rows], k, v, mask=lay[None, :]), rtol=1e-12, atol=1e-12)


def test_window_subset_matches_full_run():
    cfg = SMALL_PAD
    a = _np_inputs(cfg)
    full = _run(cfg, a)
    h = 1
    win = np.array([0, 4, 7, 11])
    sub = oracle.gsa_head(a["q_spec"][h], a["k_spec"][h], a["v_spec"][h], a["q_img"][h], a["k_img"][h],
                          a["v_img"][h], a["w_g"][h], grid_h=cfg.grid_h, grid_w=cfg.grid_w,
                          pool_s=cfg.pool_s, topk=cfg.topk, windows=win, spec_rows=[1, 3])
    d = cfg.head_dim
    flat = full["o_img"][h].reshape(-1, d)
    np.testing.assert_allclose(sub["o_img_windows"].reshape(-1, d), flat[sub["tokens"].reshape(-1)],
                               rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(sub["idx"][win], full["idx"][h][win])
    np.testing.assert_allclose(sub["o_spec"], full["o_spec"][h][[1, 3]], rtol=1e-13, atol=1e-13)


def test_named_workloads_sizes():
    c = CONFIGS
    assert c["tiny_fp32"].num_img_valid == 256 and c["tiny_fp32"].num_regions == 64
    assert c["pi3_f32"].num_img_valid == 41472 and c["pi3_f32"].num_regions == 2592
    assert c["pi3_f128"].num_img_valid == 165888
    assert c["vggt_f256"].num_img_valid == 350464 and c["vggt_f256"].num_regions == 25600
    assert c["vggt_f256"].fixed_frames == (0, 100, 200)
    assert c["pi3_f1000"].num_img_valid == 1296000 and c["pi3_f1000"].num_regions == 81000

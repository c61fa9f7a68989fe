"""gsa_backward on the GPU against the backward oracle (float64 autograd of
the layer with the GPU's region selection held fixed).

Tolerance (bf16 contexts): the GPU rounds P, dS, dO_sel and the gate
gradient to bf16 (relative 2^-9 each) and accumulates in fp32, so each
gradient must have relative L2 error <= 2e-2 and max-abs error <= 2e-2 times
max(1, its largest magnitude)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import gsa_backward_oracle as bo
import sparse_global_attention_b200 as gsa
from gsa_inputs import GSAConfig, make_inputs, to_f64_numpy

pytestmark = pytest.mark.gpu

SMALL = GSAConfig("bwd_small", 3, 12, 12, 12, 12, 2, 2, 64, 4, 4, "bf16")
MULTI = GSAConfig("bwd_multi_tile", 6, 24, 24, 24, 24, 3, 2, 64, 4, 16, "bf16")
S2 = GSAConfig("bwd_s2", 2, 10, 14, 10, 14, 1, 2, 64, 2, 12, "bf16")
VGGT = GSAConfig("bwd_pad_vggt", 5, 10, 11, 12, 12, 3, 2, 64, 4, 6, "bf16", (0, 3))
# 600 regions and 528 special rows: five 128-row tiles each, so the three-stage
# TMA rings of the tcgen05 dQ and dK/dV kernels wrap around
WRAP = GSAConfig("bwd_ring_wrap", 24, 20, 20, 20, 20, 22, 2, 64, 4, 8, "bf16")
# fixed context over seven 128-key tiles with a ragged last one (3 x (3 + 17*17) = 876
# keys) on a padded grid with 2x2 windows: its dense backward (dQ added to the
# selection's, dK/dV of the packed keys scattered back) over 1,944 query slots
FIXED_TILES = GSAConfig("bwd_fixed_tiles", 6, 17, 17, 18, 18, 3, 2, 64, 2, 6, "bf16", (0, 2, 5))
# 8x8 windows (the ablation's window size): each window's 64 queries are four row
# blocks of the selection backward that add into the window's dO'_comp; a ragged grid,
# and with fixed frames the split fixed-context backward
S8 = GSAConfig("bwd_s8", 3, 14, 15, 16, 16, 2, 2, 64, 8, 3, "bf16")
S8_FIXED = GSAConfig("bwd_s8_fixed", 4, 13, 16, 16, 16, 2, 2, 64, 8, 4, "bf16", (0, 2))
CASES = [SMALL, MULTI, S2, VGGT, WRAP, FIXED_TILES, S8, S8_FIXED]


def _close(name, got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    scale = max(1.0, float(np.abs(want).max()))
    rel = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
    assert err.max() <= 2e-2 * scale, f"{name}: max-abs {err.max():.3e} (scale {scale:.3e}, rel-L2 {rel:.3e})"
    assert rel <= 2e-2, f"{name}: rel-L2 {rel:.3e}"


@pytest.mark.parametrize("gate", ["learned", "sel_only", "comp_only"])
@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_backward_matches_autograd_oracle(cfg, gate):
    if gate != "learned" and cfg is not SMALL:
        pytest.skip("forced gates on the small case only")
    x = {k: v.cuda() for k, v in make_inputs(cfg, seed=31).items()}
    gen = torch.Generator().manual_seed(5)
    dout = {"o_img": (torch.randn(x["q_img"].shape, generator=gen) * 0.5).to(torch.bfloat16).cuda(),
            "o_spec": (torch.randn(x["q_spec"].shape, generator=gen) * 0.5).to(torch.bfloat16).cuda()}
    layer = gsa.GSALayer.from_workload(cfg, gate_mode=gate)
    try:
        idx = torch.empty((cfg.num_heads, cfg.num_regions, cfg.topk), dtype=torch.int32, device="cuda")
        out = layer.forward(x, sel_idx=idx)
        gr = layer.backward(x, out, dout)
        torch.cuda.synchronize()
        assert layer.status() == 0
    finally:
        layer.close()
    kw = dict(grid_h=cfg.grid_h, grid_w=cfg.grid_w, pool_s=cfg.pool_s, fixed_frames=cfg.fixed_frames,
              gate_mode=gate)
    valid = oracle.valid_grid(cfg.grid_h, cfg.grid_w, cfg.pad_h, cfg.pad_w)
    for h in range(cfg.num_heads):
        a = {n: to_f64_numpy(x[n][h]) for n in bo.NAMES}
        d_img = dout["o_img"][h].float().cpu().numpy().astype(np.float64)
        d_img = d_img * valid[None, :, :, None]              # pad outputs are constant 0
        d_spec = dout["o_spec"][h].float().cpu().numpy().astype(np.float64)
        want = bo.backward_head(a, idx[h].cpu().numpy().astype(np.int64), d_img, d_spec, **kw)
        for n in bo.NAMES:
            if n.endswith("_spec") and cfg.num_special == 0:
                continue
            got = gr["d" + n][h].cpu().numpy()
            _close(f"head {h} d{n}", got, want["d" + n])


def test_full_size_special_branch_gradients_sampled():
    """128 frames, 16 heads: dq of sampled special rows and dk, dv of sampled
    special keys.  In this workload (no fixed frames) they come only from the
    special-token attention over 166,528 keys, so the oracle is one attention's
    closed-form gradient; the dQ kernel's ring wraps over 1,301 key tiles and the
    dK/dV kernel loops five query tiles."""
    from gsa_inputs import CONFIGS
    cfg = CONFIGS["pi3_f128"]
    assert not cfg.fixed_frames
    x = make_inputs(cfg, seed=0, device="cuda")
    gen = torch.Generator().manual_seed(5)
    dout = {"o_img": (torch.randn(x["q_img"].shape, generator=gen) * 0.5).to(torch.bfloat16).cuda(),
            "o_spec": (torch.randn(x["q_spec"].shape, generator=gen) * 0.5).to(torch.bfloat16).cuda()}
    layer = gsa.GSALayer.from_workload(cfg)
    try:
        idx = torch.empty((cfg.num_heads, cfg.num_regions, cfg.topk), dtype=torch.int32, device="cuda")
        out = layer.forward(x, sel_idx=idx)
        gr = layer.backward(x, out, dout)
        torch.cuda.synchronize()
        assert layer.status() == 0
    finally:
        layer.close()
    d = cfg.head_dim
    scale = 1.0 / np.sqrt(d)
    n = cfg.num_spec
    rng = np.random.default_rng(11)
    for h in (0, cfg.num_heads - 1):
        qs = to_f64_numpy(x["q_spec"][h]).reshape(-1, d)
        keys = np.concatenate([to_f64_numpy(x["k_spec"][h]).reshape(-1, d), to_f64_numpy(x["k_img"][h]).reshape(-1, d)])
        vals = np.concatenate([to_f64_numpy(x["v_spec"][h]).reshape(-1, d), to_f64_numpy(x["v_img"][h]).reshape(-1, d)])
        d_o = dout["o_spec"][h].float().cpu().numpy().astype(np.float64).reshape(-1, d)
        rows = np.sort(rng.choice(n, 24, replace=False))
        cols = np.sort(np.concatenate([[0, n - 1], rng.choice(np.arange(1, n - 1), 22, replace=False)]))
        want = bo.attention_backward_rows(qs, keys, vals, d_o, scale, q_rows=rows, k_cols=cols)
        _close(f"head {h} dq_spec rows", gr["dq_spec"][h].cpu().numpy().reshape(-1, d)[rows], want["dq"])
        _close(f"head {h} dk_spec keys", gr["dk_spec"][h].cpu().numpy().reshape(-1, d)[cols], want["dk"])
        _close(f"head {h} dv_spec keys", gr["dv_spec"][h].cpu().numpy().reshape(-1, d)[cols], want["dv"])


def test_full_size_compressed_branch_gradients_sampled():
    """128 frames, 16 heads, gate forced to the compressed branch: the selection
    branch gets no gradient, so for a sampled image token t in region r (16 valid
    tokens per region here)
        dq_img[t] = dq_comp[r] / 16
        dk_img[t] = dk_comp[r] / 16 + (special-token attention's dk at key t), dv alike,
    with dq/dk/dv_comp the gradients of the 10,368 x 10,368 compressed attention
    (dO'_comp[r] = sum of dO_img over r) and the special term from the attention of
    the special rows over every key."""
    from gsa_inputs import CONFIGS
    cfg = CONFIGS["pi3_f128"]
    assert cfg.grid_h == cfg.pad_h and cfg.grid_w == cfg.pad_w and not cfg.fixed_frames
    x = make_inputs(cfg, seed=2, device="cuda")
    gen = torch.Generator().manual_seed(6)
    dout = {"o_img": (torch.randn(x["q_img"].shape, generator=gen) * 0.5).to(torch.bfloat16).cuda(),
            "o_spec": (torch.randn(x["q_spec"].shape, generator=gen) * 0.5).to(torch.bfloat16).cuda()}
    layer = gsa.GSALayer.from_workload(cfg, gate_mode="comp_only")
    try:
        idx = torch.empty((cfg.num_heads, cfg.num_regions, cfg.topk), dtype=torch.int32, device="cuda")
        out = layer.forward(x, sel_idx=idx)
        gr = layer.backward(x, out, dout)
        torch.cuda.synchronize()
        assert layer.status() == 0
    finally:
        layer.close()
    d, s, F, Hp, Wp = cfg.head_dim, cfg.pool_s, cfg.num_frames, cfg.pad_h, cfg.pad_w
    scale = 1.0 / np.sqrt(d)
    rx, rpf = Wp // s, (Hp // s) * (Wp // s)
    rng = np.random.default_rng(12)
    for h in (0, cfg.num_heads - 1):
        a = {n: to_f64_numpy(x[n][h]) for n in ("q_img", "k_img", "v_img", "q_spec", "k_spec", "v_spec")}
        pooled = {n: oracle.pool(a[n], cfg.grid_h, cfg.grid_w, s).reshape(-1, d) for n in ("q_img", "k_img", "v_img")}
        d_img = dout["o_img"][h].float().cpu().numpy().astype(np.float64)
        d_comp = d_img.reshape(F, Hp // s, s, rx, s, d).sum(axis=(2, 4)).reshape(-1, d)
        tok = np.sort(rng.choice(F * Hp * Wp, 16, replace=False))
        f, rem = tok // (Hp * Wp), tok % (Hp * Wp)
        reg = f * rpf + (rem // Wp // s) * rx + (rem % Wp) // s
        comp = bo.attention_backward_rows(pooled["q_img"], pooled["k_img"], pooled["v_img"], d_comp, scale,
                                          q_rows=reg, k_cols=reg)
        n = cfg.num_spec
        keys = np.concatenate([a["k_spec"].reshape(-1, d), a["k_img"].reshape(-1, d)])
        vals = np.concatenate([a["v_spec"].reshape(-1, d), a["v_img"].reshape(-1, d)])
        d_spec = dout["o_spec"][h].float().cpu().numpy().astype(np.float64).reshape(-1, d)
        spec = bo.attention_backward_rows(a["q_spec"].reshape(-1, d), keys, vals, d_spec, scale,
                                          q_rows=np.array([], dtype=np.int64), k_cols=n + tok)
        area = float(s * s)
        _close(f"head {h} dq_img", gr["dq_img"][h].cpu().numpy().reshape(-1, d)[tok], comp["dq"] / area)
        _close(f"head {h} dk_img", gr["dk_img"][h].cpu().numpy().reshape(-1, d)[tok], comp["dk"] / area + spec["dk"])
        _close(f"head {h} dv_img", gr["dv_img"][h].cpu().numpy().reshape(-1, d)[tok], comp["dv"] / area + spec["dv"])

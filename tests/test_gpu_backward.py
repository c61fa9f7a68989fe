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
CASES = [SMALL, MULTI, S2, VGGT, WRAP]


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

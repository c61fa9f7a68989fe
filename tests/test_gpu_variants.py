"""The ablation variants ("消融实验" rows (1) and (2) of the Speed3R notes) run
less work but must produce the outputs their definitions give:
  no compressed value  O_img = O_sel (guide-only compressed branch)
  no selection branch  O_img = Upsample(O'_comp)
Each is compared with the oracle (gate forced to the branch that remains) and
with the full layer's selection and special-token outputs."""
import numpy as np
import pytest
import torch

import oracle
import sparse_global_attention_b200 as gsa
from gsa_inputs import CONFIGS, GSAConfig, make_inputs, to_f64_numpy
from gpu_helpers import assert_close

pytestmark = pytest.mark.gpu

MULTI_TILE_BF16 = GSAConfig("multi_tile_bf16", 6, 24, 24, 24, 24, 5, 2, 64, 4, 32, "bf16")
PAD_VGGT_BF16 = GSAConfig("pad_vggt_bf16", 5, 10, 11, 12, 12, 3, 2, 64, 4, 6, "bf16", (0, 3))
CASES = [CONFIGS["tiny_fp32"], PAD_VGGT_BF16, MULTI_TILE_BF16]


def _run(cfg, x, variant, with_idx=True):
    layer = gsa.GSALayer.from_workload(cfg, variant=variant)
    try:
        idx = None
        if with_idx:
            idx = torch.full((cfg.num_heads, cfg.num_regions, cfg.topk), -7, dtype=torch.int32, device="cuda")
        out = layer.forward(x, sel_idx=idx)
        torch.cuda.synchronize()
        assert layer.status() == 0
        return out, idx
    finally:
        layer.close()


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_no_compressed_value_is_the_selection_branch(cfg):
    x = {k: v.cuda() for k, v in make_inputs(cfg, seed=5).items()}
    full, idx_full = _run(cfg, x, "full")
    out, idx = _run(cfg, x, "no_comp_value")
    assert torch.equal(idx, idx_full)                       # same guide, same top-k
    assert torch.equal(out["o_spec"], full["o_spec"])
    d = cfg.head_dim
    for h in range(cfg.num_heads):
        a = {k: to_f64_numpy(v[h]) for k, v in x.items()}
        want = oracle.gsa_head(a["q_spec"], a["k_spec"], a["v_spec"], a["q_img"], a["k_img"], a["v_img"],
                               a["w_g"], grid_h=cfg.grid_h, grid_w=cfg.grid_w, pool_s=cfg.pool_s,
                               topk=cfg.topk, fixed_frames=cfg.fixed_frames, gate_mode="sel_only",
                               forced_idx=idx[h].cpu().numpy().astype(np.int64))
        tok = want["tokens"].reshape(-1)
        got = out["o_img"][h].float().cpu().numpy().reshape(-1, d)[tok]
        assert_close("O_img(no compressed value)", got, want["o_img_windows"].reshape(-1, d), cfg)


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_no_selection_is_the_upsampled_compressed_branch(cfg):
    x = {k: v.cuda() for k, v in make_inputs(cfg, seed=6).items()}
    full, _ = _run(cfg, x, "full")
    out, _ = _run(cfg, x, "no_selection", with_idx=False)
    assert torch.equal(out["o_spec"], full["o_spec"])
    d = cfg.head_dim
    for h in range(cfg.num_heads):
        a = {k: to_f64_numpy(v[h]) for k, v in x.items()}
        want = oracle.gsa_head(a["q_spec"], a["k_spec"], a["v_spec"], a["q_img"], a["k_img"], a["v_img"],
                               a["w_g"], grid_h=cfg.grid_h, grid_w=cfg.grid_w, pool_s=cfg.pool_s,
                               topk=cfg.topk, fixed_frames=cfg.fixed_frames, gate_mode="comp_only")
        tok = want["tokens"].reshape(-1)
        got = out["o_img"][h].float().cpu().numpy().reshape(-1, d)[tok]
        assert_close("O_img(no selection)", got, want["o_img_windows"].reshape(-1, d), cfg)


def test_no_selection_rejects_a_selection_output():
    cfg = PAD_VGGT_BF16
    x = {k: v.cuda() for k, v in make_inputs(cfg, seed=7).items()}
    layer = gsa.GSALayer.from_workload(cfg, variant="no_selection")
    try:
        idx = torch.zeros((cfg.num_heads, cfg.num_regions, cfg.topk), dtype=torch.int32, device="cuda")
        with pytest.raises(gsa.GSAError):
            layer.forward(x, sel_idx=idx)
    finally:
        layer.close()

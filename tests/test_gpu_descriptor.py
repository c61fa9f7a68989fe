"""FlashVGGT descriptor attention (GSA_VARIANT_DESCRIPTOR) on the GPU against
the CPU oracle: bilinear descriptors of K/V, every image and special token
attending to the descriptors of all frames plus the special tokens."""
import numpy as np
import pytest
import torch

import oracle
import sparse_global_attention_b200 as gsa
from gsa_inputs import CONFIGS, GSAConfig, make_inputs, to_f64_numpy
from gpu_helpers import assert_close

pytestmark = pytest.mark.gpu

SMALL_BF16 = GSAConfig("desc_small_bf16", 3, 12, 12, 12, 12, 2, 2, 64, 4, 4, "bf16")
PAD_BF16 = GSAConfig("desc_pad_bf16", 4, 11, 11, 12, 12, 3, 2, 64, 2, 4, "bf16")
NO_SPEC_BF16 = GSAConfig("desc_nospec_bf16", 2, 16, 16, 16, 16, 0, 1, 64, 4, 4, "bf16")
CASES = [CONFIGS["tiny_fp32"], SMALL_BF16, PAD_BF16, NO_SPEC_BF16, CONFIGS["pi3_f32"]]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_descriptor_attention_parity(cfg):
    x = {k: v.cuda() for k, v in make_inputs(cfg, seed=21).items()}
    layer = gsa.GSALayer.from_workload(cfg, variant="descriptor")
    try:
        out = layer.forward(x)
        torch.cuda.synchronize()
        assert layer.status() == 0
    finally:
        layer.close()
    d = cfg.head_dim
    heads = range(cfg.num_heads) if cfg.num_heads <= 2 else (0, cfg.num_heads - 1)
    rng = np.random.default_rng(0)
    n_img = cfg.num_frames * cfg.pad_h * cfg.pad_w
    rows = np.arange(n_img) if n_img <= 20000 else np.sort(rng.choice(n_img, 4096, replace=False))
    valid = np.tile(oracle.valid_grid(cfg.grid_h, cfg.grid_w, cfg.pad_h, cfg.pad_w), (cfg.num_frames, 1, 1)).reshape(-1)
    for h in heads:
        a = {k: to_f64_numpy(v[h]) for k, v in x.items()}
        o_img, o_spec = oracle.descriptor_attention_head(a["q_spec"], a["k_spec"], a["v_spec"], a["q_img"], a["k_img"],
                                                         a["v_img"], grid_h=cfg.grid_h, grid_w=cfg.grid_w,
                                                         r=cfg.pool_s, img_rows=rows)
        got = out["o_img"][h].float().cpu().numpy().reshape(-1, d)[rows]
        assert_close("O_img(descriptor)", got, o_img, cfg)
        assert np.all(got[~valid[rows]] == 0)
        if cfg.num_special:
            gs = out["o_spec"][h].float().cpu().numpy().reshape(-1, d)
            assert_close("O_spec(descriptor)", gs, o_spec, cfg)

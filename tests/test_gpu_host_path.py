"""gsa_forward_host: the layer on host buffers, pipelined over head chunks,
against gsa_forward on the same inputs.  The image output and the selection do
not depend on the chunking and must be bit-identical; the special-token output
uses a per-chunk key split and must agree to rounding."""
import pytest
import torch

import sparse_global_attention_b200 as gsa
from gsa_inputs import CONFIGS, GSAConfig, make_inputs

pytestmark = pytest.mark.gpu

MULTI_TILE_BF16 = GSAConfig("multi_tile_bf16", 6, 24, 24, 24, 24, 5, 2, 64, 4, 32, "bf16")
PAD_VGGT_BF16 = GSAConfig("pad_vggt_bf16", 5, 10, 11, 12, 12, 3, 2, 64, 4, 6, "bf16", (0, 3))
CASES = [CONFIGS["tiny_fp32"], MULTI_TILE_BF16, PAD_VGGT_BF16, CONFIGS["pi3_f32"]]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_host_buffers_match_device_forward(cfg):
    x_host = make_inputs(cfg, seed=11)
    x = {k: v.cuda() for k, v in x_host.items()}
    hx = {k: v.pin_memory() for k, v in x_host.items()}
    layer = gsa.GSALayer.from_workload(cfg)
    try:
        H, R, k = cfg.num_heads, cfg.num_regions, cfg.topk
        idx = torch.empty((H, R, k), dtype=torch.int32, device="cuda")
        ref = layer.forward(x, sel_idx=idx)
        torch.cuda.synchronize()
        ho = {n: torch.empty(ref[n].shape, dtype=ref[n].dtype).pin_memory() for n in ref}
        hidx = torch.empty((H, R, k), dtype=torch.int32).pin_memory()
        for _ in range(2):                                   # the second call reuses the context's copies
            for t in ho.values():
                t.fill_(7)
            hidx.fill_(-7)
            layer.forward_host(hx, ho, sel_idx=hidx)
            torch.cuda.synchronize()
            assert layer.status() == 0
            assert torch.equal(ho["o_img"], ref["o_img"].cpu())
            assert torch.equal(hidx, idx.cpu())
            if cfg.num_special:
                d = (ho["o_spec"].float() - ref["o_spec"].cpu().float()).abs().max().item()
                assert d <= (1e-5 if cfg.dtype == "fp32" else 1e-2), d
    finally:
        layer.close()

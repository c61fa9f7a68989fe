"""The allocation-free special-token entry point, checked against the
context path.

gsa_special_attention_noalloc is for callers that cannot allocate device
memory: a host program or serving engine that owns all GPU memory and hands the
layer only inputs and outputs, or a loop that cannot pay for an allocation's
synchronisation.  It keeps its partial results in the library's static device
array, which every call shares.  Here it must return what gsa_forward returns
for the special tokens, within the bf16 tolerance of the other tests, on two
calls in a row (the second call finds the first call's partials in the array),
and it must refuse a request whose partials would not fit.
"""
import numpy as np
import pytest
import torch

import sparse_global_attention_b200 as gsa
from gsa_inputs import CONFIGS, GSAConfig, make_inputs

pytestmark = pytest.mark.gpu

PADDED = GSAConfig("noalloc_pad", 5, 10, 11, 12, 12, 3, 2, 64, 4, 6, "bf16")


def _close(got, want):
    g = got.float().cpu().numpy().astype(np.float64)
    w = want.float().cpu().numpy().astype(np.float64)
    max_abs = float(np.abs(g - w).max())
    rel = float(np.linalg.norm(g - w) / max(np.linalg.norm(w), 1e-30))
    assert max_abs <= 2e-2 and rel <= 1e-2, (max_abs, rel)


def _noalloc(cfg, x, out, **over):
    a = dict(num_heads=cfg.num_heads, num_frames=cfg.num_frames, num_special=cfg.num_special,
             grid_h=cfg.grid_h, grid_w=cfg.grid_w, pad_h=cfg.pad_h, pad_w=cfg.pad_w)
    a.update(over)
    return gsa.gsa_special_attention_noalloc(
        x["q_spec"].data_ptr(), x["k_spec"].data_ptr(), x["v_spec"].data_ptr(), x["k_img"].data_ptr(),
        x["v_img"].data_ptr(), out.data_ptr(), a["num_heads"], a["num_frames"], a["num_special"],
        a["grid_h"], a["grid_w"], a["pad_h"], a["pad_w"], 0.0,
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("cfg", [CONFIGS["pi3_f32"], PADDED], ids=["pi3_f32", "padded"])
def test_noalloc_special_matches_context_path(cfg):
    x = make_inputs(cfg, seed=5, device="cuda")
    layer = gsa.GSALayer.from_workload(cfg)
    ref = layer.forward(x)["o_spec"].clone()
    torch.cuda.synchronize()
    assert layer.status() == 0
    layer.close()
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        assert _noalloc(cfg, x, out) == gsa.GSA_OK
        torch.cuda.synchronize()
        _close(out, ref)


def test_noalloc_rejects_requests_beyond_its_array():
    cfg = CONFIGS["pi3_f32"]
    x = make_inputs(cfg.with_(num_heads=1), seed=0, device="cuda")
    out = torch.empty_like(x["q_spec"])
    # 1000 frames x 5 special tokens x 16 heads needs more partials than the array holds
    rc = _noalloc(cfg, x, out, num_heads=16, num_frames=1000)
    assert rc == 3   # GSA_ERR_UNSUPPORTED, nothing launched
    assert gsa.gsa_special_attention_noalloc(0, 0, 0, 0, 0, 0, 1, 1, 1, 1, 1, 1, 1) == 1

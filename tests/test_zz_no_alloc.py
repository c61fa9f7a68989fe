"""The allocation-free special-token entry point, checked against the
context path.

gsa_special_attention_noalloc is for callers that cannot allocate device
memory: a host program or serving engine that owns all GPU memory and hands the
layer only inputs and outputs, or a loop that cannot pay for an allocation's
synchronisation.  It keeps its partial results in the library's static device
array, which every call shares.  Here it must return what gsa_forward returns
for the special tokens, within the bf16 tolerance of the other tests, on two
calls in a row (the second call finds the first call's partials in the array);
its device status word must read clean after them, must carry a device-side
timeout to the host (and be cleared by the read); and it must refuse a request
whose partials would not fit.
"""
import re
import os

import numpy as np
import pytest
import torch

import sparse_global_attention_b200 as gsa
from gsa_inputs import CONFIGS, GSAConfig, make_inputs

pytestmark = pytest.mark.gpu

PADDED = GSAConfig("noalloc_pad", 5, 10, 11, 12, 12, 3, 2, 64, 4, 6, "bf16")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _close(got, want):
    g = got.float().cpu().numpy().astype(np.float64)
    w = want.float().cpu().numpy().astype(np.float64)
    max_abs = float(np.abs(g - w).max())
    rel = float(np.linalg.norm(g - w) / max(np.linalg.norm(w), 1e-30))
    assert max_abs <= 2e-2 and rel <= 1e-2, (max_abs, rel)


def _noalloc(cfg, x, out):
    return gsa.gsa_special_attention_noalloc(
        x["q_spec"].data_ptr(), x["k_spec"].data_ptr(), x["v_spec"].data_ptr(), x["k_img"].data_ptr(),
        x["v_img"].data_ptr(), out.data_ptr(), cfg.num_heads, cfg.num_frames, cfg.num_special,
        cfg.grid_h, cfg.grid_w, cfg.pad_h, cfg.pad_w, 0.0, torch.cuda.current_stream().cuda_stream)


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
    assert gsa.gsa_special_attention_noalloc_status(torch.cuda.current_stream().cuda_stream) == gsa.GSA_OK


def test_noalloc_status_carries_a_device_timeout():
    """A bounded device wait that nothing completes records its timeout in the
    allocation-free calls' status word; the read returns it and clears it, and
    the next call computes normally."""
    cfg = PADDED
    x = make_inputs(cfg, seed=6, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    ref = torch.empty_like(x["q_spec"])
    assert _noalloc(cfg, x, ref) == gsa.GSA_OK
    assert gsa.gsa_special_attention_noalloc_status(stream) == gsa.GSA_OK
    gsa.gsa_debug_expire_wait(None, 20000, stream)            # 20 ms, nothing ever arrives
    assert gsa.gsa_special_attention_noalloc_status(stream) == 6   # GSA_ERR_DEVICE_TIMEOUT
    assert gsa.gsa_special_attention_noalloc_status(stream) == gsa.GSA_OK
    out = torch.full_like(ref, float("nan"))
    assert _noalloc(cfg, x, out) == gsa.GSA_OK
    assert gsa.gsa_special_attention_noalloc_status(stream) == gsa.GSA_OK
    assert torch.equal(out, ref)


def test_noalloc_rejects_requests_beyond_its_array():
    # every special row keeps 264 bytes of partials per key split: with 16 heads x
    # 1600 frames x 5 tokens even a single split overflows the array, whatever the
    # split rule; the tensors are allocated at that shape all the same
    src = open(os.path.join(ROOT, "include", "gsa.h")).read()
    arr = re.search(r"#define GSA_NOALLOC_SCRATCH_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", src)
    assert int(arr[1]) * int(arr[2]) * int(arr[3]) == gsa.GSA_NOALLOC_SCRATCH_BYTES
    cfg = GSAConfig("noalloc_big", 1600, 4, 4, 4, 4, 5, 16, 64, 4, 1, "bf16")
    assert 256 + cfg.num_heads * cfg.num_frames * cfg.num_special * 264 > gsa.GSA_NOALLOC_SCRATCH_BYTES
    H, F, ns = cfg.num_heads, cfg.num_frames, cfg.num_special
    spec = lambda: torch.zeros(H, F, ns, 64, dtype=torch.bfloat16, device="cuda")
    img = lambda: torch.zeros(H, F, 4, 4, 64, dtype=torch.bfloat16, device="cuda")
    x = {"q_spec": spec(), "k_spec": spec(), "v_spec": spec(), "k_img": img(), "v_img": img()}
    out = spec()
    assert _noalloc(cfg, x, out) == 3          # GSA_ERR_UNSUPPORTED, nothing launched
    assert gsa.gsa_special_attention_noalloc(0, 0, 0, 0, 0, 0, 1, 1, 1, 1, 1, 1, 1) == 1

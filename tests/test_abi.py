"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, and rejects invalid configurations on the host."""
import ctypes
import os
import re

import pytest

import sparse_global_attention_b200 as gsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "gsa.h")).read()
    return sorted(set(re.findall(r"GSA_API\s+[\w\s\*]*?\b(gsa_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = gsa.load_library()
    names = _declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(gsa.EXPORTED) == names


def _cfg(**kw):
    base = dict(num_frames=4, grid_h=8, grid_w=8, num_special=1, num_heads=2, pool_s=2, topk=4,
                dtype="fp32")
    base.update(kw)
    return gsa.make_config(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=32), 2),                       # head_dim must be 64
    (dict(pool_s=3), 3),                          # unsupported pool size
    (dict(grid_h=9), 2),                          # grid not divisible by s
    (dict(topk=0), 1),
    (dict(topk=65, num_frames=64), 3),            # above 64: fp32 keeps the 64-entry list
    (dict(topk=100, num_frames=64, dtype="bf16"), 3),                      # above 64 with s = 2
    (dict(topk=129, num_frames=64, dtype="bf16", pool_s=4), 3),            # above the maximum of 128
    (dict(topk=17, num_frames=1), 2),             # more than the 16 regions
    (dict(pad_h=10, grid_h=7), 2),                # a region row with no valid token
    (dict(pad_h=6, grid_h=8), 2),                 # pad smaller than the grid
    (dict(num_frames=0), 1),
    (dict(fixed_frames=(0, 0)), 1),               # duplicated fixed frame
    (dict(fixed_frames=(5,)), 1),                 # fixed frame out of range
    (dict(fixed_frames=(0, 1, 2, 3)), 2),         # no candidate region left
    (dict(gate_mode=7), 1),
    (dict(softmax_scale=-1.0), 1),
    (dict(variant=4), 1),                         # no such variant
    (dict(variant=-1), 1),
])
def test_invalid_configs_are_rejected_on_the_host(kw, code):
    cfg = _cfg(**kw)
    assert gsa.gsa_create_status(cfg) == code
    assert gsa.gsa_workspace_bytes(cfg) == 0


def test_top128_is_accepted_for_bf16_4x4_windows():
    cfg = _cfg(topk=128, num_frames=64, dtype="bf16", pool_s=4)
    assert gsa.gsa_workspace_bytes(cfg) > 0


def test_workspace_bytes_of_named_workloads():
    from gsa_inputs import CONFIGS
    for name, w in CONFIGS.items():
        cfg = gsa.make_config(num_frames=w.num_frames, grid_h=w.grid_h, grid_w=w.grid_w,
                              pad_h=w.pad_h, pad_w=w.pad_w, num_special=w.num_special,
                              num_heads=w.num_heads, pool_s=w.pool_s, topk=w.topk, dtype=w.dtype,
                              fixed_frames=w.fixed_frames)
        b = gsa.gsa_workspace_bytes(cfg)
        assert b > 0, name
        # the workspace at least holds O_sel and the pooled tensors
        esize = 2 if w.dtype == "bf16" else 4
        assert b >= w.num_heads * w.num_img_slots * 64 * esize
    assert gsa.load_library().gsa_workspace_bytes(None) == 0


def test_strerror_and_null_safety():
    assert gsa.gsa_strerror(0) == "ok"
    assert "shape" in gsa.gsa_strerror(2)
    assert gsa.gsa_strerror(999) == "unknown status"
    lib = gsa.load_library()
    lib.gsa_destroy(None)                         # NULL-safe
    assert lib.gsa_get_status(None) == 1
    fn = lib.gsa_debug_expire_wait
    fn.argtypes = [ctypes.c_void_p, ctypes.c_uint, ctypes.c_void_p]
    assert fn(None, 0, None) == 1                 # limit out of range: GSA_ERR_INVALID_ARG, nothing launched
    assert lib.gsa_forward(None, *([None] * 11)) == 1

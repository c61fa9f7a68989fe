"""Thin Python binding of the GSA C ABI (include/gsa.h).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
libgsa_b200.so.  The functions carry the C names (gsa_create, gsa_forward,
gsa_dense_forward, gsa_destroy, ...) and take plain device pointers, which the
`GSALayer` convenience class extracts from torch tensors.  There is no CPU
fallback: if the shared library is missing, loading fails loudly.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgsa_b200.so")

GSA_OK = 0
GSA_BF16, GSA_FP32 = 0, 1
GSA_GATE_LEARNED, GSA_GATE_COMP_ONLY, GSA_GATE_SEL_ONLY = 0, 1, 2
GATE_MODES = {"learned": 0, "comp_only": 1, "sel_only": 2}
VARIANTS = {"full": 0, "no_comp_value": 1, "no_selection": 2, "descriptor": 3}
GSA_PROFILE_TIMES, GSA_PROFILE_KEEP_OSEL = 1, 2
GSA_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024     # the static array of the allocation-free calls
EXPORTED = ("gsa_create", "gsa_workspace_bytes", "gsa_forward", "gsa_dense_forward",
            "gsa_get_intermediate", "gsa_set_profiling", "gsa_get_kernel_times",
            "gsa_get_status", "gsa_strerror", "gsa_destroy", "gsa_special_attention_noalloc",
            "gsa_special_attention_noalloc_status",
            "gsa_debug_expire_wait", "gsa_forward_host", "gsa_backward")


class gsa_config(ctypes.Structure):
    _fields_ = [
        ("num_frames", ctypes.c_int), ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
        ("pad_h", ctypes.c_int), ("pad_w", ctypes.c_int), ("num_special", ctypes.c_int),
        ("num_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("pool_s", ctypes.c_int),
        ("topk", ctypes.c_int), ("dtype", ctypes.c_int),
        ("fixed_frames", ctypes.POINTER(ctypes.c_int)), ("num_fixed_frames", ctypes.c_int),
        ("gate_mode", ctypes.c_int), ("softmax_scale", ctypes.c_float),
        ("variant", ctypes.c_int),
    ]


class GSAError(RuntimeError):
    pass


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libgsa_b200.so (built by `python -m sparse_global_attention_b200.build`)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"GSA CUDA library not built: {path} is missing "
                          f"(run `python -m sparse_global_attention_b200.build`)")
    lib = ctypes.CDLL(path)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.gsa_create.argtypes = [ctypes.POINTER(gsa_config), ctypes.POINTER(vp)]
    lib.gsa_create.restype = i
    lib.gsa_workspace_bytes.argtypes = [ctypes.POINTER(gsa_config)]
    lib.gsa_workspace_bytes.restype = sz
    lib.gsa_forward.argtypes = [vp] * 10 + [vp, vp]
    lib.gsa_forward.restype = i
    lib.gsa_dense_forward.argtypes = [vp, vp, vp, vp, vp, vp]
    lib.gsa_dense_forward.restype = i
    lib.gsa_get_intermediate.argtypes = [vp, i, ctypes.POINTER(vp), ctypes.POINTER(sz)]
    lib.gsa_get_intermediate.restype = i
    lib.gsa_set_profiling.argtypes = [vp, i]
    lib.gsa_set_profiling.restype = i
    lib.gsa_get_kernel_times.argtypes = [vp, ctypes.POINTER(ctypes.c_float),
                                         ctypes.POINTER(ctypes.c_char_p), i]
    lib.gsa_get_kernel_times.restype = i
    lib.gsa_get_status.argtypes = [vp]
    lib.gsa_get_status.restype = i
    lib.gsa_strerror.argtypes = [i]
    lib.gsa_strerror.restype = ctypes.c_char_p
    lib.gsa_destroy.argtypes = [vp]
    lib.gsa_destroy.restype = None
    _lib = lib
    return lib


def _check(rc: int, what: str):
    if rc != GSA_OK:
        msg = load_library().gsa_strerror(rc).decode()
        raise GSAError(f"{what} failed: {msg} (status {rc})")


def make_config(*, num_frames, grid_h, grid_w, pad_h=None, pad_w=None, num_special=0,
                num_heads=1, head_dim=64, pool_s=4, topk=32, dtype="bf16",
                fixed_frames: Sequence[int] = (), gate_mode="learned",
                softmax_scale=0.0, variant="full") -> gsa_config:
    c = gsa_config()
    c.num_frames, c.grid_h, c.grid_w = num_frames, grid_h, grid_w
    c.pad_h = grid_h if pad_h is None else pad_h
    c.pad_w = grid_w if pad_w is None else pad_w
    c.num_special, c.num_heads, c.head_dim = num_special, num_heads, head_dim
    c.pool_s, c.topk = pool_s, topk
    c.dtype = GSA_BF16 if dtype == "bf16" else GSA_FP32
    fixed = (ctypes.c_int * max(1, len(fixed_frames)))(*fixed_frames)
    c._fixed_keepalive = fixed
    c.fixed_frames = ctypes.cast(fixed, ctypes.POINTER(ctypes.c_int)) if fixed_frames else None
    c.num_fixed_frames = len(fixed_frames)
    c.gate_mode = GATE_MODES[gate_mode] if isinstance(gate_mode, str) else int(gate_mode)
    c.softmax_scale = float(softmax_scale)
    c.variant = VARIANTS[variant] if isinstance(variant, str) else int(variant)
    return c


# ---- the C names, with pointers as Python ints ------------------------------------
def gsa_create(cfg: gsa_config) -> int:
    ctx = ctypes.c_void_p()
    _check(load_library().gsa_create(ctypes.byref(cfg), ctypes.byref(ctx)), "gsa_create")
    return ctx.value


def gsa_create_status(cfg: gsa_config) -> int:
    """gsa_create's status without raising (the context, if any, is destroyed)."""
    lib = load_library()
    ctx = ctypes.c_void_p()
    rc = lib.gsa_create(ctypes.byref(cfg), ctypes.byref(ctx))
    if ctx.value:
        lib.gsa_destroy(ctx)
    return rc


def gsa_workspace_bytes(cfg: gsa_config) -> int:
    return load_library().gsa_workspace_bytes(ctypes.byref(cfg))


def gsa_forward(ctx, q_spec, k_spec, v_spec, q_img, k_img, v_img, w_g, o_spec, o_img,
                sel_idx_out=0, stream=0):
    _check(load_library().gsa_forward(ctx, q_spec, k_spec, v_spec, q_img, k_img, v_img, w_g,
                                      o_spec, o_img, sel_idx_out or None, stream or None),
           "gsa_forward")


def gsa_dense_forward(ctx, q, k, v, o, stream=0):
    _check(load_library().gsa_dense_forward(ctx, q, k, v, o, stream or None), "gsa_dense_forward")


def gsa_get_intermediate(ctx, which: int):
    p, n = ctypes.c_void_p(), ctypes.c_size_t()
    _check(load_library().gsa_get_intermediate(ctx, which, ctypes.byref(p), ctypes.byref(n)),
           "gsa_get_intermediate")
    return p.value, n.value


def gsa_set_profiling(ctx, flags):
    """flags: GSA_PROFILE_TIMES (per-kernel CUDA-event timing) | GSA_PROFILE_KEEP_OSEL;
    True/False mean GSA_PROFILE_TIMES / 0."""
    _check(load_library().gsa_set_profiling(ctx, int(flags)), "gsa_set_profiling")


def gsa_get_kernel_times(ctx, cap: int = 16):
    ms = (ctypes.c_float * cap)()
    names = (ctypes.c_char_p * cap)()
    n = load_library().gsa_get_kernel_times(ctx, ms, names, cap)
    if n < 0:
        _check(-n, "gsa_get_kernel_times")
    return [(names[i].decode(), float(ms[i])) for i in range(n)]


def gsa_get_status(ctx) -> int:
    return load_library().gsa_get_status(ctx)


def gsa_debug_expire_wait(ctx, limit_us: int, stream=None):
    """Failure-detection self-test: a device wait that runs out after limit_us
    and records GSA_ERR_DEVICE_TIMEOUT in the context's error word (ctx None:
    in the status word of the allocation-free calls on the current device)."""
    fn = load_library().gsa_debug_expire_wait
    fn.argtypes = [ctypes.c_void_p, ctypes.c_uint, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    _check(fn(ctx, int(limit_us), stream or None), "gsa_debug_expire_wait")


def gsa_strerror(code: int) -> str:
    return load_library().gsa_strerror(code).decode()


def gsa_destroy(ctx):
    if ctx:
        load_library().gsa_destroy(ctx)


def gsa_special_attention_noalloc_status(stream=0) -> int:
    """Device status word of the allocation-free calls on the current device
    (synchronises `stream`, returns the code and clears it)."""
    fn = load_library().gsa_special_attention_noalloc_status
    fn.argtypes = [ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn(stream or None)


def gsa_special_attention_noalloc(q_spec, k_spec, v_spec, k_img, v_img, o_spec, num_heads,
                                  num_frames, num_special, grid_h, grid_w, pad_h, pad_w,
                                  softmax_scale=0.0, stream=0) -> int:
    """Special-token attention for callers that cannot allocate device memory
    (a host that owns all GPU memory, or a loop that cannot pay for an
    allocation's synchronisation): no context, partials in the library's static
    device array.  Pointers as ints; returns the C status code."""
    lib = load_library()
    fn = lib.gsa_special_attention_noalloc
    fn.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 7 + [ctypes.c_float, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn(q_spec, k_spec, v_spec, k_img, v_img, o_spec, num_heads, num_frames, num_special,
              grid_h, grid_w, pad_h, pad_w, float(softmax_scale), stream or None)


# ---- torch convenience wrapper (marshalling only) ------------------------------------
class GSALayer:
    """Owns one gsa_ctx; takes torch CUDA tensors and passes their pointers."""

    def __init__(self, cfg: gsa_config):
        self.cfg = cfg
        self.ctx = gsa_create(cfg)

    @classmethod
    def from_workload(cls, w, gate_mode="learned", topk: Optional[int] = None, **kw):
        """Build from a workload description with the fields of gsa_inputs.GSAConfig."""
        return cls(make_config(num_frames=w.num_frames, grid_h=w.grid_h, grid_w=w.grid_w,
                               pad_h=w.pad_h, pad_w=w.pad_w, num_special=w.num_special,
                               num_heads=w.num_heads, head_dim=w.head_dim, pool_s=w.pool_s,
                               topk=w.topk if topk is None else topk, dtype=w.dtype,
                               fixed_frames=w.fixed_frames, gate_mode=gate_mode, **kw))

    @property
    def num_regions(self) -> int:
        c = self.cfg
        return c.num_frames * (c.pad_h // c.pool_s) * (c.pad_w // c.pool_s)

    def forward(self, x, out=None, sel_idx=None, stream=None):
        """x: dict with q_img/k_img/v_img/q_spec/k_spec/v_spec/w_g torch tensors."""
        import torch
        if out is None:
            out = {"o_img": torch.empty_like(x["q_img"]), "o_spec": torch.empty_like(x["q_spec"])}
        for k in ("q_img", "k_img", "v_img", "q_spec", "k_spec", "v_spec", "w_g"):
            t = x[k]
            if not (t.is_cuda and t.is_contiguous()):
                raise GSAError(f"{k} must be a contiguous CUDA tensor")
        st = stream if stream is not None else torch.cuda.current_stream().cuda_stream
        has_spec = x["q_spec"].numel() > 0
        gsa_forward(self.ctx,
                    x["q_spec"].data_ptr() if has_spec else 0,
                    x["k_spec"].data_ptr() if has_spec else 0,
                    x["v_spec"].data_ptr() if has_spec else 0,
                    x["q_img"].data_ptr(), x["k_img"].data_ptr(), x["v_img"].data_ptr(),
                    x["w_g"].data_ptr(), out["o_spec"].data_ptr() if has_spec else 0,
                    out["o_img"].data_ptr(), 0 if sel_idx is None else sel_idx.data_ptr(), st)
        return out

    def forward_host(self, hx, hout, sel_idx=None, stream=None):
        """The layer on host tensors (gsa_forward_host): hx/hout hold CPU tensors
        with the layouts of forward(); pinned memory lets the copies overlap the
        compute.  Asynchronous on the stream like forward()."""
        import torch
        for k in ("q_img", "k_img", "v_img", "q_spec", "k_spec", "v_spec", "w_g"):
            t = hx[k]
            if t.is_cuda or not t.is_contiguous():
                raise GSAError(f"{k} must be a contiguous host tensor")
        st = stream if stream is not None else torch.cuda.current_stream().cuda_stream
        has_spec = hx["q_spec"].numel() > 0
        fn = load_library().gsa_forward_host
        fn.argtypes = [ctypes.c_void_p] * 12
        fn.restype = ctypes.c_int
        _check(fn(self.ctx,
                  hx["q_spec"].data_ptr() if has_spec else None,
                  hx["k_spec"].data_ptr() if has_spec else None,
                  hx["v_spec"].data_ptr() if has_spec else None,
                  hx["q_img"].data_ptr(), hx["k_img"].data_ptr(), hx["v_img"].data_ptr(),
                  hx["w_g"].data_ptr(), hout["o_spec"].data_ptr() if has_spec else None,
                  hout["o_img"].data_ptr(), None if sel_idx is None else sel_idx.data_ptr(), st or None),
               "gsa_forward_host")
        return hout

    def backward(self, x, out, dout, stream=None):
        """gsa_backward after forward(x) -> out: dout = {"o_img", "o_spec"} output
        gradients (context dtype).  Returns float32 gradients of every input:
        dq_img, dk_img, dv_img, dq_spec, dk_spec, dv_spec, dw_g."""
        import torch
        st = stream if stream is not None else torch.cuda.current_stream().cuda_stream
        gr = {"dq_img": x["q_img"], "dk_img": x["k_img"], "dv_img": x["v_img"], "dq_spec": x["q_spec"],
              "dk_spec": x["k_spec"], "dv_spec": x["v_spec"], "dw_g": x["w_g"]}
        gr = {k: torch.empty(v.shape, dtype=torch.float32, device=v.device) for k, v in gr.items()}
        has_spec = x["q_spec"].numel() > 0
        p = lambda t: t.data_ptr() if (t is not None and t.numel() > 0) else None
        fn = load_library().gsa_backward
        fn.argtypes = [ctypes.c_void_p] * 19
        fn.restype = ctypes.c_int
        _check(fn(self.ctx, p(x["q_spec"]), p(x["k_spec"]), p(x["v_spec"]), p(x["q_img"]), p(x["k_img"]),
                  p(x["v_img"]), p(x["w_g"]), p(out["o_spec"]) if has_spec else None,
                  p(dout["o_spec"]) if has_spec else None, p(dout["o_img"]),
                  p(gr["dq_spec"]), p(gr["dk_spec"]), p(gr["dv_spec"]), p(gr["dq_img"]), p(gr["dk_img"]),
                  p(gr["dv_img"]), p(gr["dw_g"]), st or None), "gsa_backward")
        return gr

    def dense(self, q, k, v, o=None, stream=None):
        import torch
        o = torch.empty_like(q) if o is None else o
        st = stream if stream is not None else torch.cuda.current_stream().cuda_stream
        gsa_dense_forward(self.ctx, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), st)
        return o

    def intermediate(self, which: int, dtype, shape):
        """Copy an intermediate of the last forward into a new torch tensor."""
        import torch
        ptr, nbytes = gsa_get_intermediate(self.ctx, which)
        torch.cuda.current_stream().synchronize()
        out = _raw_u8(ptr, nbytes).clone().view(dtype).reshape(shape)
        return out

    def status(self) -> int:
        return gsa_get_status(self.ctx)

    def close(self):
        gsa_destroy(self.ctx)
        self.ctx = None

    def __del__(self):
        try:
            if getattr(self, "ctx", None):
                self.close()
        except Exception:
            pass


def _raw_u8(ptr: int, nbytes: int):
    import torch

    class _Holder:
        __cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1", "data": (ptr, False),
                                    "version": 3, "strides": None}
    return torch.as_tensor(_Holder(), device="cuda")

"""Seeded synthetic inputs for the GSA layer: shapes and random tensors only.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark. It holds no arithmetic of the method: it describes the workloads
(frame count, patch grid, token counts, pool size, top-k) and draws the Q/K/V,
special-token and gate tensors from seeded generators. Nothing here pools,
scores, selects, attends or gates.

Workloads stand in for the multi-view token sets the Speed3R pages evaluate on
(RE10K, CO3Dv2, Tanks & Temples, ...; none are available offline): each frame's
image tokens come from a smooth 16-dim latent field made of 8 Gaussian bumps,
shared by every frame up to a random per-frame shift, mapped to Q/K/V by a
random 16x64 matrix per head and tensor, plus 0.1 N(0,1) noise.

Layouts (row-major, contiguous):
  image tokens   [H][F][pad_h][pad_w][d]   (pad rows/cols hold 1000.0)
  special tokens [H][F][num_special][d]
  gate weights   [H][d][d]                 (row = output channel)
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Tuple

import torch

PAD_VALUE = 1000.0
LATENT_DIM = 16
NUM_BUMPS = 8


@dataclasses.dataclass(frozen=True)
class GSAConfig:
    name: str
    num_frames: int
    grid_h: int          # valid patch rows per frame
    grid_w: int          # valid patch cols per frame
    pad_h: int           # stored rows per frame (>= grid_h, divisible by pool_s)
    pad_w: int           # stored cols per frame
    num_special: int     # special tokens per frame (camera + registers)
    num_heads: int
    head_dim: int
    pool_s: int
    topk: int
    dtype: str           # "bf16" or "fp32"
    fixed_frames: Tuple[int, ...] = ()   # VGGT fixed global context frames

    # ---- derived sizes (pure bookkeeping) ----
    @property
    def regions_per_frame(self) -> int:
        return (self.pad_h // self.pool_s) * (self.pad_w // self.pool_s)

    @property
    def num_regions(self) -> int:
        return self.num_frames * self.regions_per_frame

    @property
    def num_img_valid(self) -> int:
        return self.num_frames * self.grid_h * self.grid_w

    @property
    def num_img_slots(self) -> int:
        return self.num_frames * self.pad_h * self.pad_w

    @property
    def num_spec(self) -> int:
        return self.num_frames * self.num_special

    def with_(self, **kw) -> "GSAConfig":
        return dataclasses.replace(self, **kw)


def _vggt_fixed(num_frames: int) -> Tuple[int, ...]:
    return tuple(f for f in range(num_frames) if f % 100 == 0)


# The five workloads: a tiny fp32 case, three pi^3-style bf16 cases at 32, 128
# and 1000 frames, and a VGGT-style case with a padded grid and fixed context.
CONFIGS: Dict[str, GSAConfig] = {
    "tiny_fp32": GSAConfig("tiny_fp32", 4, 8, 8, 8, 8, 1, 2, 64, 2, 4, "fp32"),
    "pi3_f32": GSAConfig("pi3_f32", 32, 36, 36, 36, 36, 5, 16, 64, 4, 32, "bf16"),
    "pi3_f128": GSAConfig("pi3_f128", 128, 36, 36, 36, 36, 5, 16, 64, 4, 32, "bf16"),
    "vggt_f256": GSAConfig("vggt_f256", 256, 37, 37, 40, 40, 5, 16, 64, 4, 32, "bf16",
                           _vggt_fixed(256)),
    "pi3_f1000": GSAConfig("pi3_f1000", 1000, 36, 36, 36, 36, 5, 16, 64, 4, 32, "bf16"),
}
CONFIG_ORDER = ["tiny_fp32", "pi3_f32", "pi3_f128", "vggt_f256", "pi3_f1000"]


def _gen(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1_000_003 + int(stream))
    return g


def _latent_field(cfg: GSAConfig, seed: int, device) -> torch.Tensor:
    """z [F][grid_h][grid_w][16] in fp32: 8 Gaussian bumps, per-frame shift."""
    g = _gen(seed, 1, device)
    Hv, Wv, F = cfg.grid_h, cfg.grid_w, cfg.num_frames
    amp = torch.randn(NUM_BUMPS, LATENT_DIM, generator=g, device=device)
    ctr = torch.rand(NUM_BUMPS, 2, generator=g, device=device) * torch.tensor(
        [float(Wv), float(Hv)], device=device)
    sig = (0.1 + 0.15 * torch.rand(NUM_BUMPS, generator=g, device=device)) * float(min(Hv, Wv))
    shift = (torch.rand(F, 2, generator=g, device=device) - 0.5) * 0.5 * torch.tensor(
        [float(Wv), float(Hv)], device=device)
    xs = torch.arange(Wv, device=device, dtype=torch.float32) + 0.5
    ys = torch.arange(Hv, device=device, dtype=torch.float32) + 0.5
    z = torch.zeros(F, Hv, Wv, LATENT_DIM, device=device)
    for b in range(NUM_BUMPS):
        dx = xs[None, None, :] - ctr[b, 0] - shift[:, 0, None, None]   # [F,1,Wv]
        dy = ys[None, :, None] - ctr[b, 1] - shift[:, 1, None, None]   # [F,Hv,1]
        w = torch.exp(-(dx * dx + dy * dy) / (2.0 * sig[b] * sig[b]))  # [F,Hv,Wv]
        z += w[..., None] * amp[b]
    return z


def make_inputs(cfg: GSAConfig, seed: int = 0, device="cpu",
                heads=None) -> Dict[str, torch.Tensor]:
    """Draw one seeded input set for `cfg`.

    Returns a dict of tensors in the config's dtype (bf16 inputs are rounded
    to nearest-even from fp32): q_img/k_img/v_img [H][F][pad_h][pad_w][d],
    q_spec/k_spec/v_spec [H][F][num_special][d], w_g [H][d][d].
    `heads` restricts generation to a subset of heads (same values as in the
    full draw, since every head has its own generator stream).
    """
    dev = torch.device(device)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    H, F, d = cfg.num_heads, cfg.num_frames, cfg.head_dim
    Hv, Wv, Hp, Wp, ns = cfg.grid_h, cfg.grid_w, cfg.pad_h, cfg.pad_w, cfg.num_special
    heads = list(range(H)) if heads is None else list(heads)
    z = _latent_field(cfg, seed, dev)
    gs = _gen(seed, 2, dev)
    spec_lat = torch.randn(F, max(ns, 1), LATENT_DIM, generator=gs, device=dev)[:, :ns]
    out = {}
    for ti, name in enumerate(("q", "k", "v")):
        img = torch.empty(len(heads), F, Hp, Wp, d, dtype=dt, device=dev)
        spec = torch.empty(len(heads), F, ns, d, dtype=dt, device=dev)
        for hi, h in enumerate(heads):
            g = _gen(seed, 100 + 3 * h + ti, dev)
            amap = torch.randn(LATENT_DIM, d, generator=g, device=dev) * 0.25
            noise = torch.randn(F, Hv, Wv, d, generator=g, device=dev) * 0.1
            t = torch.matmul(z, amap) + noise
            full = torch.full((F, Hp, Wp, d), PAD_VALUE, device=dev)
            full[:, :Hv, :Wv, :] = t
            img[hi] = full.to(dt)
            sn = torch.randn(F, ns, d, generator=g, device=dev) * 0.1
            spec[hi] = (torch.matmul(spec_lat, amap) + sn).to(dt)
            del t, full, noise
        out[name + "_img"] = img
        out[name + "_spec"] = spec
    wg = torch.empty(len(heads), d, d, dtype=dt, device=dev)
    for hi, h in enumerate(heads):
        g = _gen(seed, 10_000 + h, dev)
        wg[hi] = (torch.randn(d, d, generator=g, device=dev) * 0.125).to(dt)
    out["w_g"] = wg
    return out


def to_f64_numpy(t: torch.Tensor):
    """Exact widening of a (bf16 or fp32) tensor to a float64 numpy array."""
    return t.detach().to("cpu", torch.float64).numpy()

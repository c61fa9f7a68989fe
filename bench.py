#!/usr/bin/env python
"""Benchmark of the B200 GSA layer (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--config pi3_f1000] [--dense full|off] [--no-e2e]

A step is one full GSA forward (pool, compressed attention + streaming top-k,
selection, upsample/gate/blend, special tokens) over the
1000-frame pi^3-style workload (1000 frames x 36x36 patches + 5 special tokens
per frame, 16 heads, d=64, s=4, top-32), inputs resident in HBM.  Inputs are
7.9 GB per GPU, far above the 126 MB L2, so no flush is needed between steps.
Under torchrun every rank runs its own independent copy of the workload (the
layer has no cross-GPU exchange; heads and layers are independent), so per-GPU
work is fixed as N grows ("weak" scaling) and `value` sums all ranks.

--impl reference times the CPU oracle (fp64 numpy, as it stands) on a bounded
sample of the same workload and reports the same metric; the other ranks of a
multi-rank launch exit without work.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from datetime import timedelta

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GSA layer image tokens/s at 1000 views; % of bf16 peak; speedup vs dense attn"
UNIT = "image tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 << 20
FLUSH_BYTES = 256 << 20

# kernels of one step (names reported by gsa_get_kernel_times) and how each is graded
TENSOR_KERNELS = {"comp_attn_topk", "special", "fixed_attn", "dense"}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(cfg):
    return (f"{cfg.name}: {cfg.num_frames} frames x {cfg.grid_h}x{cfg.grid_w} patch grid"
            + (f" (padded {cfg.pad_h}x{cfg.pad_w})" if (cfg.pad_h, cfg.pad_w) != (cfg.grid_h, cfg.grid_w) else "")
            + f" + {cfg.num_special} special tokens/frame, {cfg.num_heads} heads, d={cfg.head_dim},"
            f" s={cfg.pool_s}, top-{cfg.topk}" + (f", fixed frames {list(cfg.fixed_frames)}" if cfg.fixed_frames else ""))


def algorithmic_work(cfg, kc):
    """Per-launch algorithmic FLOPs and compulsory HBM bytes of each kernel."""
    H, d = cfg.num_heads, cfg.head_dim
    R = cfg.num_regions
    M = cfg.num_img_valid
    slots = cfg.num_img_slots
    Ms = cfg.num_spec
    e = 2 if cfg.dtype == "bf16" else 4
    s2 = cfg.pool_s ** 2
    nfix_keys = len(cfg.fixed_frames) * (cfg.num_special + cfg.grid_h * cfg.grid_w)
    keys_sel = cfg.topk * s2 + nfix_keys
    w = {}
    # pool reads Q/K/V once and writes bf16 Q/K/V_comp plus the bf16 low parts of Q/K_comp
    w["pool"] = {"flops": 0.0,
                 "bytes": 3.0 * H * slots * d * e + 5.0 * H * R * d * e}
    # the guide scores take three bf16 products (hi*hi + hi*lo + lo*hi); the
    # algorithmic count is the plain 4*d per (query, key) pair of one attention
    w["comp_attn_topk"] = {"flops": 4.0 * d * R * R * H,
                           "bytes": 5.0 * H * R * d * e + H * R * d * 4 + H * R * kc * 4}
    w["selection"] = {"flops": 4.0 * d * M * keys_sel * H,
                      # Q_img + O_sel + every image token's K/V once + idx
                      "bytes": 2.0 * H * slots * d * e + 2.0 * H * slots * d * e + H * R * cfg.topk * 4}
    w["epilogue"] = {"flops": 2.0 * d * d * M * H,
                     "bytes": 3.0 * H * slots * d * e + H * R * d * 4 + H * d * d * e}
    # selection with the upsample/gate/blend fused: reads Q, every image token's K/V once,
    # O'_comp and the region lists; writes O_img
    w["selection_gate"] = {"flops": w["selection"]["flops"] + w["epilogue"]["flops"],
                           "bytes": 4.0 * H * slots * d * e + H * R * d * 4 + H * R * cfg.topk * 4}
    if nfix_keys and cfg.dtype == "bf16":
        # the fixed context runs apart: gather of its K/V (read + write), one dense attention
        # of every image query over it (reads Q, writes the fp32 output and its LSE); the
        # selection then attends only the selected regions and reads that output back
        w["fixed_attn"] = {"flops": 4.0 * d * M * nfix_keys * H,
                           "bytes": 6.0 * H * nfix_keys * d * e + H * slots * d * (e + 4) + H * slots * 4}
        w["selection_gate"]["flops"] -= w["fixed_attn"]["flops"]
        w["selection_gate"]["bytes"] += H * slots * (d + 1) * 4
    w["special"] = {"flops": 4.0 * d * Ms * (Ms + M) * H, "bytes": 2.0 * H * (Ms + slots) * d * e + 2.0 * H * Ms * d * e}
    w["special_merge"] = {"flops": 0.0, "bytes": 0.0}
    w["dense"] = {"flops": 4.0 * d * (M + Ms) ** 2 * H, "bytes": 4.0 * H * (slots + Ms) * d * e}
    return w


# the sources each timed kernel is compiled from (a traffic record is used only while
# the hash of its kernel's sources matches the one recorded with it)
_ATTN_SRC = ("attn_tc.cu", "tc_ptx.cuh", "gsa_common.cuh", "gsa_kernels.h")
KERNEL_SOURCES = {
    "comp_attn_topk": _ATTN_SRC, "special": _ATTN_SRC, "fixed_attn": _ATTN_SRC, "dense": _ATTN_SRC,
    "selection_gate": ("select.cu", "sel_tc.cu", "tc_ptx.cuh", "gsa_common.cuh", "gsa_kernels.h"),
    "sel_union": ("sel_tc.cu", "gsa_common.cuh", "gsa_kernels.h"),
    "pool": ("pool.cu", "gsa_common.cuh", "gsa_kernels.h"),
    "special_merge": ("merge.cu", "gsa_common.cuh", "gsa_kernels.h"),
}


def kernel_source_sha(kernel="comp_attn_topk"):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_global_attention_b200", "csrc")
    for n in KERNEL_SOURCES.get(kernel, _ATTN_SRC):
        p = os.path.join(csrc, n)
        if not os.path.exists(p):
            continue
        with open(p, "rb") as f:
            h.update(n.encode())
            h.update(f.read())
    return h.hexdigest()[:12]


def read_traffic(kernel, workload, compulsory=None):
    """DRAM bytes per launch of `kernel` from an ncu capture of its current sources
    (profiles/ncu_traffic.txt: `kernel workload bytes source_sha`).  A record of
    this workload is used as it stands.  Otherwise, given `compulsory` = {workload
    name: algorithmic bytes of one launch}, a record of a smaller workload of the
    same kernel is scaled by the ratio of the two launches' compulsory bytes.
    Returns (bytes, note) or (None, None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(p):
        return None, None
    sha = kernel_source_sha(kernel)
    recs = {}
    with open(p) as f:
        for line in f:
            parts = line.split()
            if len(parts) == 4 and not line.startswith("#") and parts[0] == kernel and parts[3] == sha:
                recs[parts[1]] = float(parts[2])
    if workload in recs:
        return recs[workload], f"ncu capture of {workload}"
    for w, b in recs.items():
        if compulsory and w in compulsory and workload in compulsory and compulsory[w] > 0:
            return b * compulsory[workload] / compulsory[w], (
                f"ncu capture of {w}, scaled x{compulsory[workload] / compulsory[w]:.2f} by compulsory bytes")
    return None, None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, ValueError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 7:
                continue
            try:
                sm.append(float(p[0]))
                mx = max(mx, float(p[1]))
            except ValueError:
                continue
            for n, v in zip(names, p[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(v, dist=None, device="cpu"):
    """Largest value of `v` over all ranks (every rank gets it); the per-step
    time of a multi-GPU run is the slowest rank's."""
    if dist is None:
        return float(v)
    import torch
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(world, tokens_per_rank, ms_max):
    """Whole-job image tokens/s: every rank processes its own workload (weak
    scaling), the job takes as long as its slowest rank."""
    return world * tokens_per_rank / (ms_max / 1e3)


# ---------------------------------------------------------------------------------------
# the CPU oracle as the baseline / reference arm
# ---------------------------------------------------------------------------------------
def oracle_sample(cfg, head_arrays, nwin, seed=0):
    """Time the oracle on head 0: the head's full pooling plus `nwin` windows
    (compressed row, top-k, selection, gate) and a proportional number of
    special rows; extrapolate to the whole layer (every window of every head)."""
    import numpy as np
    import oracle
    a = head_arrays
    rng = np.random.default_rng(seed)
    R = cfg.num_regions
    win = np.sort(rng.choice(R, size=min(nwin, R), replace=False))
    nspec = max(1, int(round(cfg.num_spec * len(win) / R))) if cfg.num_special else 0
    srows = np.sort(rng.choice(cfg.num_spec, size=nspec, replace=False)) if nspec else np.zeros(0, int)
    t0 = time.perf_counter()
    for t in ("q_img", "k_img", "v_img"):
        oracle.pool(a[t], cfg.grid_h, cfg.grid_w, cfg.pool_s)
    t_pool = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.gsa_head(a["q_spec"], a["k_spec"], a["v_spec"], a["q_img"], a["k_img"], a["v_img"], a["w_g"],
                    grid_h=cfg.grid_h, grid_w=cfg.grid_w, pool_s=cfg.pool_s, topk=cfg.topk,
                    fixed_frames=cfg.fixed_frames, windows=win, spec_rows=srows)
    t_all = time.perf_counter() - t0
    t_win = max(t_all - t_pool, 1e-9)
    per_head = t_pool + t_win * (R / len(win))
    layer_s = per_head * cfg.num_heads
    return {"layer_s": layer_s, "sample_s": t_pool + t_all, "windows": len(win), "spec_rows": nspec}


def cpu_info():
    cores = len(os.sched_getaffinity(0))
    threads = None
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        blas = [f"{i.get('internal_api')}:{i.get('num_threads')}" for i in info if i.get("user_api") == "blas"]
        threads = max([i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"] or [cores])
        return cores, threads, ",".join(blas)
    except Exception:
        return cores, cores, "unknown"


def host_head_arrays(cfg, x, h=0):
    from gsa_inputs import to_f64_numpy
    return {k: to_f64_numpy(v[h]) for k, v in x.items()}


def run_reference(args, cfg, rank, world):
    """--impl reference: the CPU oracle as it stands, bounded samples of the workload."""
    if rank != 0:
        return None
    from gsa_inputs import make_inputs
    x = make_inputs(cfg, seed=0, device="cpu", heads=[0])
    a = host_head_arrays(cfg, x, 0)
    del x
    nwin = args.ref_windows
    for _ in range(args.warmup):
        oracle_sample(cfg, a, nwin)
    times, samples = [], []
    for i in range(args.steps):
        r = oracle_sample(cfg, a, nwin, seed=i)
        times.append(r["layer_s"])
        samples.append(r["sample_s"])
    layer_s = statistics.median(times)
    value = cfg.num_img_valid / layer_s
    cores, threads, blas = cpu_info()
    sample = (f"head 0 of {cfg.num_heads}: full pooling of the head + {nwin} random windows (compressed row,"
              f" top-k, selection, gate) + proportional special rows; time extrapolated x{cfg.num_regions}/{nwin}"
              f" windows and x{cfg.num_heads} heads; median of {args.steps} samples ({statistics.median(samples):.1f}"
              f" s each); BLAS {blas}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": layer_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": workload_desc(cfg), "parallelism": "cpu oracle, rank 0"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    return line


# ---------------------------------------------------------------------------------------
# the B200 arm
# ---------------------------------------------------------------------------------------
def run_b200(args, cfg, rank, world, local, dist):
    import torch
    import sparse_global_attention_b200 as gsa
    from gsa_inputs import make_inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    x = make_inputs(cfg, seed=rank, device=dev)
    layer = gsa.GSALayer.from_workload(cfg)
    out = {"o_img": torch.empty_like(x["q_img"]), "o_spec": torch.empty_like(x["q_spec"])}
    stream = torch.cuda.current_stream()

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        layer.forward(x, out=out)
    torch.cuda.synchronize()
    st = layer.status()
    if st != 0:
        raise RuntimeError(f"device status {st} during warm-up: {gsa.gsa_strerror(st)}")

    # ---- timed region: K steps, inputs resident in HBM ------------------------
    # inputs far above the 126 MB L2 need no flush; smaller workloads get a 256 MB
    # write before every step, outside each step's own pair of events
    in_bytes = sum(t.numel() * t.element_size() for t in x.values())
    flush = in_bytes < 4 * L2_BYTES
    fbuf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush else None
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        if flush:
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for a0, a1 in evs:
                fbuf.fill_(1)
                a0.record(stream)
                layer.forward(x, out=out)
                a1.record(stream)
            torch.cuda.synchronize()
            step_ms = sum(a0.elapsed_time(a1) for a0, a1 in evs) / args.steps
        else:
            e0.record(stream)
            for _ in range(args.steps):
                layer.forward(x, out=out)
            e1.record(stream)
            torch.cuda.synchronize()
            step_ms = e0.elapsed_time(e1) / args.steps
    barrier()
    ms = max_over_ranks(step_ms, dist, dev)
    del fbuf
    value = throughput(world, cfg.num_img_valid, ms)

    # ---- per-kernel times (CUDA events recorded by the library on its stream) --
    gsa.gsa_set_profiling(layer.ctx, True)
    per = {}
    nprof = max(1, min(args.steps, 5))
    for _ in range(nprof):
        layer.forward(x, out=out)
        for name, t in gsa.gsa_get_kernel_times(layer.ctx):
            per.setdefault(name, []).append(t)
    gsa.gsa_set_profiling(layer.ctx, False)
    kernel_ms = {k: statistics.mean(v) for k, v in per.items()}
    launches_per_step = len(kernel_ms)
    kc = cfg.topk

    pk, pk_kind = peaks()
    work = algorithmic_work(cfg, kc)
    kernels = {}
    for k, t in kernel_ms.items():
        w = work.get(k, {"flops": 0.0, "bytes": 0.0})
        ent = {"ms": round(t, 4)}
        if w["flops"]:
            ent["tflops"] = round(w["flops"] / (t / 1e3) / 1e12, 2)
        if w["bytes"]:
            ent["gbs"] = round(w["bytes"] / (t / 1e3) / 1e9, 1)
        kernels[k] = ent
    # compulsory bytes of each kernel on the smaller workloads whose ncu captures may be scaled
    from gsa_inputs import CONFIGS as _C
    comp_bytes = {}
    for wn in ("pi3_f128", "pi3_f32", "vggt_f256", cfg.name):
        if wn in _C or wn == cfg.name:
            wc = cfg if wn == cfg.name else _C[wn]
            comp_bytes[wn] = algorithmic_work(wc, wc.topk)
    for k in kernels:
        tr, note = read_traffic(k, cfg.name, {w: comp_bytes[w].get(k, {"bytes": 0.0})["bytes"] for w in comp_bytes})
        if tr is not None:
            kernels[k]["traffic"] = round(tr)
            kernels[k]["traffic_source"] = note
            if work.get(k, {}).get("bytes"):
                kernels[k]["traffic_over_compulsory"] = round(tr / work[k]["bytes"], 3)
    dom = max(kernel_ms, key=kernel_ms.get)
    # steps of a few hundred ms run at full clocks: the burst bf16 figure is the peak;
    # the sustained (power-capped, seconds-long) figure is kept as a second fraction
    tpeak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    tpeak_sus = pk.get("bf16_tflops_sustained")
    if dom in TENSOR_KERNELS:
        ach = work[dom]["flops"] / (kernel_ms[dom] / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": round(ach, 2), "peak": tpeak, "unit": "TFLOP/s"}
    else:
        ach = work[dom]["bytes"] / (kernel_ms[dom] / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = round(ach / roof["peak"], 4)
    roof["kernel"] = dom
    roof["peak_source"] = f"{pk_kind} ({'bf16 burst' if roof['bound'] == 'tensor' else 'copy'})"
    if roof["bound"] == "tensor" and tpeak_sus:
        roof["frac_of_sustained"] = round(ach / tpeak_sus, 4)
    roof["traffic"] = kernels[dom].get("traffic")
    roof["traffic_source"] = kernels[dom].get("traffic_source")
    roof["compulsory_bytes"] = round(work[dom]["bytes"])
    tensor_flops = sum(work[k]["flops"] for k in ("comp_attn_topk", "special", "selection", "epilogue"))
    pct_peak = tensor_flops / (ms / 1e3) / 1e12 / tpeak
    # whole-layer roofline fraction: each launched kernel's own roofline time
    # (the larger of FLOPs / bf16 peak and bytes / copy peak), summed, over the step time
    roof_ms = 0.0
    for k in kernel_ms:
        w = work.get(k, {"flops": 0.0, "bytes": 0.0})
        roof_ms += 1e3 * max(w["flops"] / (tpeak * 1e12), w["bytes"] / (pk["hbm_gbs"] * 1e9))
    layer_roof = round(roof_ms / ms, 4)

    # ---- dense global attention of the same shape (speedup denominator) ---------
    dense = None
    if args.dense != "off" and rank == 0:
        H, F, d = cfg.num_heads, cfg.num_frames, cfg.head_dim

        def dense_layout(spec, img):
            return torch.cat([spec, img.reshape(H, F, -1, d)], dim=2).reshape(H, -1, d).contiguous()

        del out
        torch.cuda.empty_cache()
        qd, kd, vd = (dense_layout(x[n + "_spec"], x[n + "_img"]) for n in "qkv")
        od = torch.empty_like(qd)
        small = gsa.GSALayer.from_workload(cfg.with_(num_frames=2, fixed_frames=()))   # warms the dense kernel
        small.dense(qd[:, :2 * (cfg.num_special + cfg.pad_h * cfg.pad_w)].contiguous(),
                    kd[:, :2 * (cfg.num_special + cfg.pad_h * cfg.pad_w)].contiguous(),
                    vd[:, :2 * (cfg.num_special + cfg.pad_h * cfg.pad_w)].contiguous())
        torch.cuda.synchronize()
        small.close()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        layer.dense(qd, kd, vd, od)
        d1.record(stream)
        torch.cuda.synchronize()
        dms = d0.elapsed_time(d1)
        dfl = work["dense"]["flops"]
        dense = {"ms": round(dms, 2), "tflops": round(dfl / (dms / 1e3) / 1e12, 1),
                 "frac": round(dfl / (dms / 1e3) / 1e12 / tpeak, 4), "reps": 1}
        # context only: PyTorch's own attention (its default backend) on one head of
        # the same dense shape, bf16, no mask (this workload has no pad tokens)
        if cfg.grid_h == cfg.pad_h and cfg.grid_w == cfg.pad_w:
            import torch.nn.functional as tnf
            qh, kh, vh = (t[:1].unsqueeze(0) for t in (qd, kd, vd))
            with torch.cuda.stream(stream):
                tnf.scaled_dot_product_attention(qh, kh, vh)
                s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                s0.record(stream)
                for _ in range(2):
                    tnf.scaled_dot_product_attention(qh, kh, vh)
                s1.record(stream)
            torch.cuda.synchronize()
            sms = s0.elapsed_time(s1) / 2
            sfl = dfl / H
            dense["torch_sdpa_one_head"] = {"ms": round(sms, 2), "tflops": round(sfl / (sms / 1e3) / 1e12, 1)}
        del qd, kd, vd, od
        torch.cuda.empty_cache()
        out = {"o_img": torch.empty_like(x["q_img"]), "o_spec": torch.empty_like(x["q_spec"])}
    else:
        pass
    if dist is not None:
        barrier()

    # ---- end to end through the public API with host buffers ---------------------
    e2e = None
    if not args.no_e2e:
        if "out" not in locals() or out is None:
            out = {"o_img": torch.empty_like(x["q_img"]), "o_spec": torch.empty_like(x["q_spec"])}
        hx = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in x.items()}
        for k in hx:
            hx[k].copy_(x[k])
        ho = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in out.items()}
        h2d = sum(t.numel() * t.element_size() for t in hx.values())
        d2h = sum(t.numel() * t.element_size() for t in ho.values())

        def e2e_step():
            # gsa_forward_host: pinned host inputs in, pinned host outputs out, the
            # copies overlapped with the layer chunk by chunk over the heads
            layer.forward_host(hx, ho)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ke = max(1, min(args.steps, 5))
        f0.record(stream)
        for _ in range(ke):
            e2e_step()
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ems = max_over_ranks(f0.elapsed_time(f1) / ke, dist, dev)
        e2e = {"value": throughput(world, cfg.num_img_valid, ems), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": round(ems, 3), "steps": ke}

    st = layer.status()
    if st != 0:
        raise RuntimeError(f"device status {st}: {gsa.gsa_strerror(st)}")

    # ---- the oracle on the host cores (rank 0, N = 1 only) --------------------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        a = host_head_arrays(cfg, x, 0)
        r = oracle_sample(cfg, a, args.cpu_windows)
        cores, threads, blas = cpu_info()
        cpu = {"value": cfg.num_img_valid / r["layer_s"], "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": (f"head 0 of {cfg.num_heads} of the same inputs: full pooling of the head + "
                          f"{r['windows']} random windows (compressed row, top-k, selection, gate) + "
                          f"{r['spec_rows']} special rows, {r['sample_s']:.1f} s of CPU work, extrapolated to "
                          f"all windows and heads; BLAS {blas}; {cores} cores visible")}

    # ---- backward pass (optional): gradients of every input, selection held fixed ----
    backward = None
    if args.backward:
        dout = {k: (torch.randn(v.shape, device=dev) * 0.5).to(v.dtype) for k, v in out.items()}
        fwd = layer.forward(x, out=out)
        for _ in range(2):
            gr = layer.backward(x, fwd, dout)
        torch.cuda.synchronize()
        barrier()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        for _ in range(3):
            gr = layer.backward(x, fwd, dout)
        b1.record(stream)
        torch.cuda.synchronize()
        barrier()
        bms = max_over_ranks(b0.elapsed_time(b1) / 3, dist, dev)
        gsa.gsa_set_profiling(layer.ctx, True)
        gr = layer.backward(x, fwd, dout)
        bk = {n: round(t, 3) for n, t in gsa.gsa_get_kernel_times(layer.ctx)}
        gsa.gsa_set_profiling(layer.ctx, False)
        st = layer.status()
        if st != 0:
            raise RuntimeError(f"device status {st} in the backward: {gsa.gsa_strerror(st)}")
        d = cfg.head_dim
        H = cfg.num_heads
        fl = {"bwd_comp_attn": 10.0 * d * cfg.num_regions ** 2 * H,
              "bwd_selection_gate": 10.0 * d * cfg.num_img_valid * cfg.topk * cfg.pool_s ** 2 * H,
              "bwd_special": 10.0 * d * cfg.num_spec * (cfg.num_spec + cfg.num_img_valid) * H}
        kern = {n: ({"ms": t, "tflops": round(fl[n] / (t / 1e3) / 1e12, 1)} if n in fl else {"ms": t})
                for n, t in bk.items()}
        backward = {"ms": round(bms, 3), "vs_forward": round(bms / ms, 2),
                    "flops_convention": "10*d per (query, key) pair and attention (S, dP, dQ, dK, dV)",
                    "kernels": kern}
        del gr, dout

    layer.close()

    # ---- ablation variants of the notes' table, same inputs (optional) -------------
    ablations = None
    if args.ablations:
        ablations = {}
        specs = [("no_comp_value", dict(variant="no_comp_value")), ("no_selection", dict(variant="no_selection")),
                 ("top8", dict(topk=8)), ("top16", dict(topk=16)), ("top64", dict(topk=64)),
                 ("top128", dict(topk=128)),
                 ("flashvggt_descriptor_attention", dict(variant="descriptor")), ("windows8x8", None)]
        for name, kw in specs:
            if kw is None:
                # 8x8 windows: the grid padded to a multiple of 8, inputs drawn for that layout
                pad = lambda n: (n + 7) // 8 * 8
                wcfg = cfg.with_(pool_s=8, pad_h=pad(cfg.grid_h), pad_w=pad(cfg.grid_w))
                del x, out
                torch.cuda.empty_cache()
                x = make_inputs(wcfg, seed=rank, device=dev)
                out = {"o_img": torch.empty_like(x["q_img"]), "o_spec": torch.empty_like(x["q_spec"])}
                lay = gsa.GSALayer.from_workload(wcfg)
            else:
                lay = gsa.GSALayer.from_workload(cfg, **kw)
            for _ in range(2):
                lay.forward(x, out=out)
            torch.cuda.synchronize()
            barrier()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            for _ in range(3):
                lay.forward(x, out=out)
            a1.record(stream)
            torch.cuda.synchronize()
            barrier()
            st = lay.status()
            lay.close()
            if st != 0:
                raise RuntimeError(f"device status {st} in ablation {name}: {gsa.gsa_strerror(st)}")
            ams = max_over_ranks(a0.elapsed_time(a1) / 3, dist, dev)
            ablations[name] = {"ms": round(ams, 3), "vs_full": round(ams / ms, 3)}
            if name == "flashvggt_descriptor_attention":
                # every image and special token against (F * Hd * Wd descriptors + special tokens)
                nd = cfg.num_frames * (cfg.grid_h // cfg.pool_s) * (cfg.grid_w // cfg.pool_s) + cfg.num_spec
                fl = 4.0 * cfg.head_dim * cfg.num_heads * (cfg.num_frames * cfg.pad_h * cfg.pad_w + cfg.num_spec) * nd
                tf = fl / (ams / 1e3) / 1e12
                ablations[name].update({"tflops": round(tf, 1), "frac_of_burst_bf16": round(tf / tpeak, 4)})

    if rank != 0:
        return None
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
        "config": {"workload": workload_desc(cfg), "image_tokens": cfg.num_img_valid,
                   "special_tokens": cfg.num_spec, "regions": cfg.num_regions,
                   "l2": (f"inputs {in_bytes / 1e9:.2f} GB per GPU >> 126 MB L2: no flush between steps" if not flush
                          else f"inputs {in_bytes / 1e6:.0f} MB: a {FLUSH_BYTES >> 20} MB write before every step, "
                               "outside the step's events"),
                   "parallelism": f"{world} independent replica(s), one per GPU, no collective on the data path"},
        "roofline": roof, "pct_bf16_peak": round(pct_peak, 4), "layer_roofline_frac": layer_roof,
        "speedup_vs_dense": (round(dense["ms"] / ms, 2) if dense else None), "dense": dense,
        "kernels": kernels, "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(), "e2e": e2e, "cpu_baseline": cpu,
    }
    if ablations is not None:
        line["ablations"] = ablations
    if backward is not None:
        line["backward"] = backward
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--config", default="pi3_f1000")
    ap.add_argument("--dense", default="full", choices=["full", "off"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="also time gsa_backward (gradients of every input) on the same inputs")
    ap.add_argument("--ablations", action="store_true",
                    help="also time the layer variants of the ablation table (no compressed value, "
                         "no selection, top-8/16/64, 8x8 windows), test-time top-128 and FlashVGGT's "
                         "descriptor attention on the same inputs")
    # the same sample size for the cpu_baseline leg and the reference arm, so that
    # their extrapolations agree
    ap.add_argument("--cpu-windows", type=int, default=1024)
    ap.add_argument("--ref-windows", type=int, default=1024)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "b200":
        args.warmup = 3

    from gsa_inputs import CONFIGS
    cfg = CONFIGS[args.config]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if args.impl == "reference":
        line = run_reference(args, cfg, rank, world)
    else:
        if world > 1:
            import torch
            import torch.distributed as dist_mod
            torch.cuda.set_device(local)
            dist_mod.init_process_group("nccl", timeout=timedelta(seconds=300),
                                        device_id=torch.device("cuda", local))
            dist = dist_mod
        line = run_b200(args, cfg, rank, world, local, dist)
        if dist is not None:
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()

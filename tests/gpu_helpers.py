"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
the CPU oracle on the same seeded inputs, and compare with the stated bars.

Acceptance (per output tensor): bf16 configs max-abs <= 2e-2 and relative L2
<= 1e-2; fp32 configs max-abs <= 1e-4.  Selected regions: for every
compressed row whose oracle gap (s_k - s_{k+1}) / |s_k| exceeds 1e-3 the GPU's
set must equal the oracle's; the outputs of every window are compared with an
oracle run forced to the GPU's selection (identical sets where the gap rule
applies, the GPU's valid choice elsewhere).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sparse_global_attention_b200 as gsa
from gsa_inputs import make_inputs, to_f64_numpy

GAP = 1e-3


def tol(cfg):
    return (1e-4, None) if cfg.dtype == "fp32" else (2e-2, 1e-2)


def assert_close(name, got, want, cfg, mask=None):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    if mask is not None:
        got, want = got[mask], want[mask]
    err = np.abs(got - want)
    max_abs, rel_tol = tol(cfg)
    mx = float(err.max()) if err.size else 0.0
    rel = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
    assert mx <= max_abs, f"{name}: max-abs error {mx:.3e} > {max_abs:g} (rel-L2 {rel:.3e})"
    if rel_tol is not None:
        assert rel <= rel_tol, f"{name}: rel-L2 error {rel:.3e} > {rel_tol:g}"
    return mx, rel


def run_gpu(cfg, x, gate_mode="learned", topk=None):
    """One gsa_forward through the C ABI; returns outputs and intermediates on the host."""
    layer = gsa.GSALayer.from_workload(cfg, gate_mode=gate_mode, topk=topk)
    gsa.gsa_set_profiling(layer.ctx, gsa.GSA_PROFILE_KEEP_OSEL)   # keep O_sel for the checks
    k = cfg.topk if topk is None else topk
    R = cfg.num_regions
    H = cfg.num_heads
    idx = torch.full((H, R, k), -7, dtype=torch.int32, device="cuda")
    out = layer.forward(x, sel_idx=idx)
    torch.cuda.synchronize()
    st = layer.status()
    assert st == 0, f"device status {st}: {gsa.gsa_strerror(st)}"
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    res = {
        "o_img": out["o_img"], "o_spec": out["o_spec"], "idx": idx,
        "q_comp": layer.intermediate(0, dt, (H, R, 64)),
        "k_comp": layer.intermediate(1, dt, (H, R, 64)),
        "v_comp": layer.intermediate(2, dt, (H, R, 64)),
        "o_comp_prime": layer.intermediate(3, torch.float32, (H, R, 64)),
        "idx_ws": layer.intermediate(4, torch.int32, (H, R, k)),
        "o_sel": layer.intermediate(5, dt, (H, cfg.num_frames, cfg.pad_h, cfg.pad_w, 64)),
        "q_comp_lo": layer.intermediate(6, dt, (H, R, 64)),
        "k_comp_lo": layer.intermediate(7, dt, (H, R, 64)),
    }
    layer.close()
    return res


def head_arrays(x, h):
    return {k: to_f64_numpy(v[h]) for k, v in x.items()}


def check_idx_gap_rule(gpu_idx, ora_idx, gap, rows=None):
    """Sets equal where the oracle's k-th / (k+1)-th gap exceeds GAP.
    Returns the number of rows checked and the number under the threshold."""
    rows = np.arange(gpu_idx.shape[0]) if rows is None else np.asarray(rows)
    checked = under = 0
    for r in rows:
        assert len(set(gpu_idx[r].tolist())) == gpu_idx.shape[1], f"row {r}: duplicate regions"
        if gap[r] > GAP:
            assert sorted(gpu_idx[r].tolist()) == sorted(ora_idx[r].tolist()), (
                f"row {r}: selected regions differ (gap {gap[r]:.3e})")
            checked += 1
        else:
            under += 1
    return checked, under


def compare_head(cfg, x, res, h, windows=None, spec_rows=None, gate_mode="learned", topk=None):
    """Compare head h of a GPU run with the oracle (all or sampled windows)."""
    a = head_arrays(x, h)
    k = cfg.topk if topk is None else topk
    gidx = res["idx"][h].cpu().numpy().astype(np.int64)
    kw = dict(grid_h=cfg.grid_h, grid_w=cfg.grid_w, pool_s=cfg.pool_s, topk=k,
              fixed_frames=cfg.fixed_frames, gate_mode=gate_mode, windows=windows,
              spec_rows=spec_rows)
    nat = oracle.gsa_head(a["q_spec"], a["k_spec"], a["v_spec"], a["q_img"], a["k_img"], a["v_img"],
                          a["w_g"], **kw)
    win = nat["windows"]
    # selected regions: valid, distinct, candidate frames only, gap rule
    assert gidx[win].min() >= 0 and gidx[win].max() < cfg.num_regions
    if cfg.fixed_frames:
        assert not np.isin(gidx[win] // cfg.regions_per_frame, cfg.fixed_frames).any()
    checked, under = check_idx_gap_rule(gidx, nat["idx"], nat["gap"], rows=win)
    # pooled tensors (fp32 copies are the exact means up to fp32 rounding)
    assert_close("Q_comp", res["q_comp"][h].float().cpu().numpy(), nat["q_comp"], cfg)
    assert_close("V_comp", res["v_comp"][h].float().cpu().numpy(), nat["v_comp"], cfg)
    # bf16 contexts carry the pooled Q/K as hi + lo pairs: together ~16 significant bits
    for name, key in (("q", "q_comp"), ("k", "k_comp")):
        hi = res[key][h].double().cpu().numpy()
        both = hi + res[key + "_lo"][h].double().cpu().numpy() if cfg.dtype == "bf16" else hi
        bound = 2.0 ** -15 * np.abs(nat[key]) + 1e-6
        assert np.all(np.abs(both - nat[key]) <= bound), f"{name}_comp hi+lo split"
    # compressed attention rows
    assert_close("O'_comp", res["o_comp_prime"][h].cpu().numpy()[win], nat["o_comp_prime"], cfg)
    # selection branch and layer output, oracle forced to the GPU's selection
    forced = oracle.gsa_head(a["q_spec"], a["k_spec"], a["v_spec"], a["q_img"], a["k_img"],
                             a["v_img"], a["w_g"], forced_idx=gidx, **kw)
    tok = forced["tokens"].reshape(-1)
    d = cfg.head_dim
    osel = res["o_sel"][h].float().cpu().numpy().reshape(-1, d)[tok]
    assert_close("O_sel", osel, forced["o_sel"].reshape(-1, d), cfg)
    oimg = res["o_img"][h].float().cpu().numpy().reshape(-1, d)[tok]
    assert_close("O_img", oimg, forced["o_img_windows"].reshape(-1, d), cfg)
    if cfg.num_special:
        ospec = res["o_spec"][h].float().cpu().numpy().reshape(-1, d)[forced["spec_rows"]]
        assert_close("O_spec", ospec, forced["o_spec"], cfg)
    return checked, under

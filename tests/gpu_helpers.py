"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
the CPU oracle on the same seeded inputs, and compare with the stated bars.

Acceptance (per output tensor): bf16 configs max-abs <= 2e-2 and relative L2
<= 1e-2; fp32 configs max-abs <= 1e-4.  Selected regions, per compressed row,
with s_k the oracle's k-th best candidate score:
  * gap rule: where (s_k - s_{k+1}) / |s_k| exceeds 1e-3, the GPU's set equals
    the oracle's;
  * every other row (a near tie at the k-th place) is checked for validity:
    every region the GPU chose scores at least s_k - tol in exact arithmetic,
    and every candidate scoring above s_k + tol is among the GPU's choices, with
    tol = 1e-3 |s_k| + 2^-14 |q_r| max_j |k_j|.  The second term covers the
    on-chip guide scores' own error (the bf16 hi/lo split is accurate to about
    2^-17 |q||k|), which can exceed 1e-3 |s_k| on rows whose k-th score is
    close to zero;
  * every chosen region is distinct and a candidate (not in a fixed frame).
The outputs of every window are compared with an oracle run forced to the GPU's
selection (identical sets where the gap rule applies, a valid choice elsewhere).
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


def check_index_rows(gpu_idx, scores, cand, k, qnorm, kmax, label="", verbose=True):
    """Selected regions of every row of `scores` [n][R] (exact fp64 guide scores
    of the rows, all candidate columns) against the oracle's top-k.

    gpu_idx [n][k]; cand [R] bool; qnorm [n] = |q_r|; kmax = max_j |k_j|.
    Rows over the 1e-3 relative gap must match the oracle's set exactly; every
    other row must be a valid top-k within tol (see the module docstring).
    Returns (rows checked exactly, rows checked for validity)."""
    gpu_idx = np.asarray(gpu_idx, dtype=np.int64)
    n = gpu_idx.shape[0]
    ora_idx, gap = oracle.topk_rows(scores, cand, k)
    assert gpu_idx.min() >= 0 and gpu_idx.max() < scores.shape[1], f"{label}: region index out of range"
    assert cand[gpu_idx].all(), f"{label}: a chosen region is not a candidate"
    srt = np.sort(gpu_idx, axis=1)
    assert (srt[:, 1:] != srt[:, :-1]).all(), f"{label}: duplicate regions in a row"
    exact = gap > GAP
    bad = np.nonzero(exact & (np.sort(ora_idx, axis=1) != srt).any(axis=1))[0]
    assert bad.size == 0, (f"{label}: selected regions differ on {bad.size} rows over the gap "
                           f"(first row {bad[0]}, gap {gap[bad[0]]:.3e})")
    s_k = np.take_along_axis(scores, ora_idx[:, -1:], axis=1)[:, 0]
    tol = 1e-3 * np.abs(s_k) + 2.0 ** -14 * qnorm * kmax
    chosen = np.take_along_axis(scores, gpu_idx, axis=1)
    low = np.nonzero((chosen < (s_k - tol)[:, None]).any(axis=1))[0]
    assert low.size == 0, (f"{label}: row {low[0]} chose a region scoring "
                           f"{chosen[low[0]].min():.6g} < s_k - tol = {s_k[low[0]] - tol[low[0]]:.6g}")
    must = scores > (s_k + tol)[:, None]              # candidates clearly above the k-th place
    if not cand.all():
        must &= cand[None, :]
    hit = np.take_along_axis(must, gpu_idx, axis=1).sum(axis=1)
    miss = np.nonzero(hit != must.sum(axis=1))[0]
    assert miss.size == 0, f"{label}: row {miss[0]} misses a region scoring above s_k + tol"
    under = int((~exact).sum())
    if verbose:
        print(f"[index] {label}: {n} rows, {n - under} over the 1e-3 gap (sets identical), "
              f"{under} near ties ({under / max(n, 1):.1%}) checked for validity")
    return n - under, under


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
    # selected regions: exact where the gap rule applies, a valid top-k elsewhere
    cand = oracle.candidate_regions(cfg.num_frames, cfg.regions_per_frame, cfg.fixed_frames)
    scores = nat["q_comp"][win] @ nat["k_comp"].T
    kmax = float(np.linalg.norm(nat["k_comp"], axis=1).max())
    checked, under = check_index_rows(gidx[win], scores, cand, k, np.linalg.norm(nat["q_comp"][win], axis=1),
                                      kmax, label=f"{cfg.name} head {h}")
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

"""The GPU tests' top-k index check (gpu_helpers.check_index_rows), run on the
CPU against answers built from the oracle: it must accept the oracle's own
selection and a valid swap at a near tie, and reject a plausible mistake in a
selection (a wrong region, a duplicate, a region of a fixed frame, a region
missing above the k-th place).  The rule it applies: [Speed3R notes, 选择分支]
TopKSelect of S_guide per compressed row, ties to the lower region index."""
import numpy as np
import pytest

import oracle
from gpu_helpers import check_index_rows
from gsa_inputs import CONFIGS, make_inputs, to_f64_numpy


@pytest.fixture(scope="module")
def rows():
    cfg = CONFIGS["pi3_f32"]
    x = make_inputs(cfg, seed=0, heads=[0])
    qc = oracle.pool(to_f64_numpy(x["q_img"][0]), cfg.grid_h, cfg.grid_w, cfg.pool_s)
    kc = oracle.pool(to_f64_numpy(x["k_img"][0]), cfg.grid_h, cfg.grid_w, cfg.pool_s)
    r = np.arange(0, qc.shape[0], 7)[:300]
    scores = qc[r] @ kc.T
    cand = np.ones(kc.shape[0], dtype=bool)
    return scores, cand, np.linalg.norm(qc[r], axis=1), float(np.linalg.norm(kc, axis=1).max())


def _check(rows, idx, k=32, cand=None):
    scores, c, qn, km = rows
    return check_index_rows(idx, scores, c if cand is None else cand, k, qn, km, label="cpu", verbose=False)


def test_accepts_the_oracle_selection_and_counts_near_ties(rows):
    scores, cand, _, _ = rows
    idx, gap = oracle.topk_rows(scores, cand, 32)
    exact, under = _check(rows, idx)
    assert exact + under == scores.shape[0]
    assert under == int((gap <= 1e-3).sum()) and 0 < under < scores.shape[0]


def test_accepts_a_swap_inside_a_near_tie(rows):
    scores, cand, _, _ = rows
    idx, _ = oracle.topk_rows(scores, cand, 33)
    # the row whose 32nd and 33rd scores are closest: exchanging them is a valid top-32
    order = np.argsort(np.abs(np.take_along_axis(scores, idx[:, 31:32], 1)[:, 0]
                              - np.take_along_axis(scores, idx[:, 32:33], 1)[:, 0]))
    r = int(order[0])
    sel = idx[:, :32].copy()
    sel[r, 31] = idx[r, 32]
    _check(rows, sel)


def test_rejects_a_wrong_region_over_the_gap(rows):
    scores, cand, _, _ = rows
    idx, gap = oracle.topk_rows(scores, cand, 32)
    r = int(np.nonzero(gap > 1e-3)[0][0])
    bad = idx.copy()
    bad[r, 0] = int(np.argmin(scores[r]))
    with pytest.raises(AssertionError):
        _check(rows, bad)


def test_rejects_a_low_region_in_a_near_tie_row(rows):
    scores, cand, _, _ = rows
    idx, gap = oracle.topk_rows(scores, cand, 32)
    r = int(np.nonzero(gap <= 1e-3)[0][0])
    bad = idx.copy()
    bad[r, 5] = int(np.argsort(scores[r])[len(scores[r]) // 2])     # a median-scoring region
    with pytest.raises(AssertionError):
        _check(rows, bad)


def test_rejects_duplicates_and_non_candidates(rows):
    scores, cand, _, _ = rows
    idx, _ = oracle.topk_rows(scores, cand, 32)
    dup = idx.copy()
    dup[3, 1] = dup[3, 0]
    with pytest.raises(AssertionError):
        _check(rows, dup)
    fixed = cand.copy()
    fixed[idx[0, 0]] = False                       # as if its frame were a fixed-context frame
    with pytest.raises(AssertionError):
        _check(rows, idx, cand=fixed)

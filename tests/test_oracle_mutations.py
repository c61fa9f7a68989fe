"""The oracle's pins have teeth: plant a plausible mistake in the oracle (on
the CPU, by swapping one of its functions for a wrong variant) and check that
the matching pin fails."""
import numpy as np
import pytest

import oracle
import oracle.gsa_oracle as go
import test_oracle_pins as pins


def _pool_transposed(x_img, grid_h, grid_w, s):
    F, Hp, Wp, d = x_img.shape
    good = _ORIG["pool"](x_img, grid_h, grid_w, s)
    g = good.reshape(F, Hp // s, Wp // s, d)
    return np.ascontiguousarray(np.swapaxes(g, 1, 2)).reshape(-1, d) if Hp == Wp else g[:, ::-1].reshape(-1, d)


def _attention_no_scale(q, k, v, scale, key_valid=None):
    return _ORIG["attention"](q, k, v, 1.0, key_valid)


def _topk_ties_high_index(scores, cand, k):
    idx, gap = _ORIG["topk_rows"](scores, cand, k)
    out = idx.copy()
    for i in range(scores.shape[0]):
        cols = np.nonzero(cand)[0]
        order = np.lexsort((-cols, -scores[i, cols]))
        out[i] = cols[order[:k]]
    return out, gap


def _gate_transposed(q, o_comp, o_sel, w_g, gate_mode="learned"):
    return _ORIG["gate_blend"](q, o_comp, o_sel, w_g.T, gate_mode)


def _gate_swapped(q, o_comp, o_sel, w_g, gate_mode="learned"):
    return _ORIG["gate_blend"](q, o_sel, o_comp, w_g, gate_mode)


def _pool_counts_pads(x_img, grid_h, grid_w, s):
    return _ORIG["pool"](x_img, x_img.shape[1], x_img.shape[2], s)


_ORIG = {n: getattr(go, n) for n in ("pool", "attention", "topk_rows", "gate_blend")}

CASES = [
    ("pool", _pool_transposed, lambda: pins.test_pool_equals_loop_mean(pins.SMALL)),
    ("pool", _pool_counts_pads, lambda: pins.test_pool_equals_loop_mean(pins.SMALL_PAD)),
    ("attention", _attention_no_scale, pins.test_compression_s1_equals_dense_image_attention),
    ("attention", _attention_no_scale, lambda: pins.test_special_tokens_equal_dense_attention(pins.SMALL)),
    ("topk_rows", _topk_ties_high_index, pins.test_selection_window_closed_form_zero_query),
    ("gate_blend", _gate_transposed, pins.test_gate_orientation_row_is_output_channel),
    ("gate_blend", _gate_swapped, pins.test_gate_modes_isolate_branches),
]


@pytest.mark.parametrize("name,mutant,pin", CASES, ids=[f"{c[0]}-{c[1].__name__}" for c in CASES])
def test_planted_mistake_fails_its_pin(monkeypatch, name, mutant, pin):
    monkeypatch.setattr(go, name, mutant)
    monkeypatch.setattr(oracle, name, mutant)
    with pytest.raises(AssertionError):
        pin()

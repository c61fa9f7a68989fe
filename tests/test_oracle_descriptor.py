"""Pins of the descriptor-attention oracle (FlashVGGT notes: bilinear
descriptors, descriptor attention) against facts outside the oracle: a
library resize routine, closed forms, and the r = 1 reduction to dense
attention."""
import numpy as np
import pytest
import torch

import oracle


@pytest.mark.parametrize("h,w,r", [(8, 8, 4), (36, 36, 4), (37, 37, 4), (12, 20, 2), (9, 7, 3), (16, 16, 8)])
def test_bilinear_resize_matches_torch_interpolate(h, w, r):
    rng = np.random.default_rng(h * 100 + w + r)
    x = rng.standard_normal((h, w, 5))
    got = oracle.bilinear_resize(x, h // r, w // r)
    t = torch.from_numpy(x).permute(2, 0, 1)[None]
    want = torch.nn.functional.interpolate(t, size=(h // r, w // r), mode="bilinear", align_corners=False,
                                           antialias=False)[0].permute(1, 2, 0).numpy()
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_resize_of_a_ramp_samples_the_half_pixel_centres():
    # x[y, x] = y: the output row i holds its sample coordinate (i + 1/2) * H / h - 1/2
    H, W, h = 37, 6, 9
    x = np.broadcast_to(np.arange(H, dtype=np.float64)[:, None, None], (H, W, 1))
    got = oracle.bilinear_resize(x, h, 3)[:, 0, 0]
    want = np.clip((np.arange(h) + 0.5) * H / h - 0.5, 0, H - 1)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_resize_keeps_constants():
    x = np.full((10, 14, 3), 2.5)
    np.testing.assert_allclose(oracle.bilinear_resize(x, 2, 3), 2.5, rtol=0, atol=1e-14)


def _inputs(F=3, grid=(7, 9), pad=(8, 12), ns=2, d=8, seed=0):
    rng = np.random.default_rng(seed)
    Hp, Wp = pad
    img = [rng.standard_normal((F, Hp, Wp, d)) for _ in range(3)]
    for t in img:                                            # pads hold a sentinel that must never leak
        t[:, grid[0]:, :, :] = 1000.0
        t[:, :, grid[1]:, :] = 1000.0
    spec = [rng.standard_normal((F, ns, d)) for _ in range(3)]
    return spec, img


def test_r1_descriptor_attention_is_dense_attention_over_valid_tokens():
    (qs, ks, vs), (qi, ki, vi) = _inputs()
    gh, gw = 7, 9
    o_img, o_spec = oracle.descriptor_attention_head(qs, ks, vs, qi, ki, vi, grid_h=gh, grid_w=gw, r=1)
    d = qi.shape[-1]
    F, Hp, Wp = qi.shape[:3]
    valid = np.tile(oracle.valid_grid(gh, gw, Hp, Wp), (F, 1, 1)).reshape(-1)
    keys = np.concatenate([ki.reshape(-1, d)[valid], ks.reshape(-1, d)])
    vals = np.concatenate([vi.reshape(-1, d)[valid], vs.reshape(-1, d)])
    want = oracle.attention(qi.reshape(-1, d)[valid], keys, vals, 1 / np.sqrt(d))
    np.testing.assert_allclose(o_img[valid], want, rtol=0, atol=1e-12)
    assert np.all(o_img[~valid] == 0)
    want_s = oracle.attention(qs.reshape(-1, d), keys, vals, 1 / np.sqrt(d))
    np.testing.assert_allclose(o_spec, want_s, rtol=0, atol=1e-12)


def test_descriptors_ignore_pad_values():
    (qs, ks, vs), (qi, ki, vi) = _inputs(seed=3)
    a = oracle.descriptors(ki, 7, 9, 2)
    ki2 = ki.copy()
    ki2[:, 7:, :, :] = -5.0
    ki2[:, :, 9:, :] = 7.0
    np.testing.assert_array_equal(a, oracle.descriptors(ki2, 7, 9, 2))
    assert a.shape == (3 * 3 * 4, ki.shape[-1])


def test_constant_values_give_that_constant():
    (qs, ks, vs), (qi, ki, vi) = _inputs(seed=4)
    vi[...] = 0.75
    vs[...] = 0.75
    o_img, o_spec = oracle.descriptor_attention_head(qs, ks, vs, qi, ki, vi, grid_h=7, grid_w=9, r=2)
    F, Hp, Wp = qi.shape[:3]
    valid = np.tile(oracle.valid_grid(7, 9, Hp, Wp), (F, 1, 1)).reshape(-1)
    np.testing.assert_allclose(o_img[valid], 0.75, rtol=0, atol=1e-12)
    np.testing.assert_allclose(o_spec, 0.75, rtol=0, atol=1e-12)


# ---- the pins have teeth: plausible mistakes planted in the oracle fail them ----
import oracle.flashvggt_oracle as fo  # noqa: E402

_RW = fo.resize_weights


def _align_corners(n_in, n_out):
    pos = np.arange(n_out, dtype=np.float64) * ((n_in - 1) / max(n_out - 1, 1))
    i0 = np.minimum(np.floor(pos).astype(np.int64), n_in - 1)
    return i0, np.minimum(i0 + 1, n_in - 1), pos - i0


def _no_half_pixel(n_in, n_out):
    pos = np.arange(n_out, dtype=np.float64) * (n_in / n_out)
    i0 = np.minimum(np.floor(pos).astype(np.int64), n_in - 1)
    return i0, np.minimum(i0 + 1, n_in - 1), pos - i0


def _swapped_weights(n_in, n_out):
    i0, i1, w = _RW(n_in, n_out)
    return i0, i1, 1.0 - w


@pytest.mark.parametrize("mutant", [_align_corners, _no_half_pixel, _swapped_weights],
                         ids=lambda f: f.__name__)
def test_planted_resize_mistake_fails_a_pin(monkeypatch, mutant):
    monkeypatch.setattr(fo, "resize_weights", mutant)
    failed = 0
    for pin in (lambda: test_bilinear_resize_matches_torch_interpolate(37, 37, 4),
                test_resize_of_a_ramp_samples_the_half_pixel_centres):
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed >= 1

"""Plain float64 CPU oracle of FlashVGGT's descriptor attention.

TEST INFRASTRUCTURE ONLY, like gsa_oracle.py: only the tests, the smoke check
and the benchmark's CPU-baseline leg may import it; the product path never
does.  It imports numpy and nothing else, and shares no code with the CUDA
path.

Source: "FlashVGGT: Efficient and Scalable Visual Geometry Transformers with
Compressed Descriptor Attention" (Paper-Notes, CVPR 2026), key designs
"空间压缩描述符Token" (spatially compressed descriptor tokens: bilinear
interpolation of each frame's (H, W) token grid to (H/r, W/r)) and
"描述符注意力机制" (descriptor attention: full-resolution tokens are the
queries, the compressed descriptors the keys/values).  Cited below as
[FlashVGGT notes, <design>].

Readings taken where the pages are silent (listed in the design notes):
  * "bilinear interpolation" is the half-pixel-centre convention: output i of
    n_out samples the input at (i + 1/2) * n_in / n_out - 1/2, clamped below at
    0, and blends the two neighbours (the last one repeats at the border); the
    output size is floor(n_in / r);
  * it is applied to K and V (linear with weights summing to 1, so it commutes
    with the K/V projections); on padded grids only the valid Hv x Wv grid is
    resized;
  * every image token and every special token is a query; the keys are the
    descriptors of every frame followed by every special token ("plus the aux
    tokens"); softmax scale 1/sqrt(d); pad queries output 0.
Parity status: pinned by tests/test_oracle_descriptor.py (a library resize
routine, closed forms on constant and linear fields, r = 1 reducing to dense
attention).
"""
from __future__ import annotations

import numpy as np

from .gsa_oracle import attention


def resize_weights(n_in: int, n_out: int):
    """Per output index: the two input indices and the weight of the second.

    [FlashVGGT notes, 空间压缩描述符Token: "双线性插值"] with the half-pixel
    convention stated in the module docstring."""
    pos = (np.arange(n_out, dtype=np.float64) + 0.5) * (n_in / n_out) - 0.5
    pos = np.maximum(pos, 0.0)
    i0 = np.minimum(np.floor(pos).astype(np.int64), n_in - 1)
    i1 = np.minimum(i0 + 1, n_in - 1)
    return i0, i1, pos - i0


def bilinear_resize(x: np.ndarray, h_out: int, w_out: int) -> np.ndarray:
    """x [H][W][d] -> [h_out][w_out][d]: resize along y, then along x."""
    y0, y1, wy = resize_weights(x.shape[0], h_out)
    x0, x1, wx = resize_weights(x.shape[1], w_out)
    rows = x[y0] * (1.0 - wy)[:, None, None] + x[y1] * wy[:, None, None]
    return rows[:, x0] * (1.0 - wx)[None, :, None] + rows[:, x1] * wx[None, :, None]


def descriptors(x_img: np.ndarray, grid_h: int, grid_w: int, r: int) -> np.ndarray:
    """x_img [F][Hp][Wp][d] -> [F*(grid_h//r)*(grid_w//r)][d], frame by frame
    from the valid grid only."""
    F, _, _, d = x_img.shape
    hd, wd = grid_h // r, grid_w // r
    out = [bilinear_resize(x_img[f, :grid_h, :grid_w], hd, wd).reshape(hd * wd, d) for f in range(F)]
    return np.concatenate(out, axis=0)


def descriptor_attention_head(q_spec, k_spec, v_spec, q_img, k_img, v_img, *, grid_h, grid_w, r,
                              img_rows=None, spec_rows=None):
    """One head of descriptor attention.

    q/k/v_img [F][Hp][Wp][d], q/k/v_spec [F][ns][d].  Returns (o_img, o_spec):
    o_img [F*Hp*Wp][d] (or the rows img_rows of it), pad rows 0; o_spec
    [F*ns][d] (or spec_rows).  [FlashVGGT notes, 描述符注意力机制: queries are
    the full-resolution tokens, keys/values the descriptors (and the aux
    tokens).]"""
    F, Hp, Wp, d = q_img.shape
    scale = 1.0 / np.sqrt(d)
    kk = np.concatenate([descriptors(k_img, grid_h, grid_w, r), k_spec.reshape(-1, d)], axis=0)
    vv = np.concatenate([descriptors(v_img, grid_h, grid_w, r), v_spec.reshape(-1, d)], axis=0)
    qi = q_img.reshape(-1, d)
    valid = np.tile((np.arange(Hp)[:, None] < grid_h) & (np.arange(Wp)[None, :] < grid_w), (F, 1, 1)).reshape(-1)
    rows = np.arange(F * Hp * Wp) if img_rows is None else np.asarray(img_rows)
    o_img = attention(qi[rows], kk, vv, scale) * valid[rows][:, None]
    qs = q_spec.reshape(-1, d)
    srows = np.arange(qs.shape[0]) if spec_rows is None else np.asarray(spec_rows)
    o_spec = attention(qs[srows], kk, vv, scale) if qs.shape[0] else np.zeros((0, d))
    return o_img, o_spec

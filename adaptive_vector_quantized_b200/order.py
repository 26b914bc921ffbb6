"""Token orders on an image grid, and two diagnostics of how query tiles
follow the image ("AVQ-Attention: Adaptive Vector-Quantized Attention",
Sec. 4.2 and Fig. 3: tokens along a generalised Hilbert curve so that tiles
of consecutive tokens are compact; Sec. H, Table 8: Gilbert vs raster vs
random order).

Host-side helpers: the curve itself is `avq_gilbert_order` of the C library;
`avq_permute` applies an order to device tensors.
"""
from __future__ import annotations

import numpy as np


def grid_order(width: int, height: int, kind: str = "gilbert", rng=None) -> np.ndarray:
    """Raster index (y * width + x) of the t-th token: 'gilbert' (generalised
    Hilbert curve), 'raster' (row by row) or 'random' (a permutation drawn
    from `rng`)."""
    if kind == "gilbert":
        from . import avq_gilbert_order

        return avq_gilbert_order(width, height).numpy().astype(np.int64)
    if kind == "raster":
        return np.arange(width * height, dtype=np.int64)
    if kind == "random":
        rng = np.random.default_rng() if rng is None else rng
        return rng.permutation(width * height).astype(np.int64)
    raise ValueError(kind)


def tile_locality(order, width: int, height: int, tile: int) -> dict:
    """Compactness of the tiles of `tile` consecutive tokens of `order`:
    `boundary` = mean number of grid edges between a tile's cells and cells
    of other tiles, divided by that of a square of the same area (4 sqrt(T));
    `bbox_fill` = mean of (cells / bounding-box area).  A compact tile has a
    small boundary; a thin strip or a scattered set a large one."""
    order = np.asarray(order, dtype=np.int64)
    n = width * height
    if order.shape != (n,):
        raise ValueError("order must hold every cell once")
    tile_of = np.empty(n, dtype=np.int64)
    tile_of[order] = np.arange(n) // tile
    grid = tile_of.reshape(height, width)
    cut = np.zeros(int(tile_of.max()) + 1)
    for a, b in ((grid[:, 1:], grid[:, :-1]), (grid[1:, :], grid[:-1, :])):
        diff = a != b
        np.add.at(cut, a[diff], 1)
        np.add.at(cut, b[diff], 1)
    sizes = np.bincount(tile_of)
    ys, xs = np.divmod(np.arange(n), width)
    fills = []
    for t in range(len(sizes)):
        m = tile_of == t
        area = (xs[m].max() - xs[m].min() + 1) * (ys[m].max() - ys[m].min() + 1)
        fills.append(sizes[t] / area)
    return dict(boundary=float(np.mean(cut / (4.0 * np.sqrt(sizes)))),
                bbox_fill=float(np.mean(fills)))


def selection_capture(importance, P: int) -> float:
    """Mean over query blocks of the share of the block's importance (Eq. 7)
    held by its top-P parents: sum of the P largest w_j(I) / sum_j w_j(I).
    Since sum_j w_j(I) = |I|, it is the fraction of the block's parent-level
    softmax mass that refinement reaches."""
    w = np.asarray(importance, dtype=np.float64)
    w = w.reshape(-1, w.shape[-1])
    tot = w.sum(axis=1)
    top = np.sort(w, axis=1)[:, ::-1][:, :P].sum(axis=1)
    keep = tot > 0
    return float(np.mean(top[keep] / tot[keep]))

"""Oracle for the generalised Hilbert ("Gilbert") token order.

Test infrastructure, like the rest of this package: only the tests, the
smoke check and the bench's CPU-baseline leg use it.

"AVQ-Attention: Adaptive Vector-Quantized Attention", Sec. 4.2 and Fig. 3:
image tokens are reordered along a generalised Hilbert curve so that tiles
of consecutive tokens are compact 2-D regions on grids of any size (the
28 x 28 patch grid of Fig. 3).  The pages give no construction (they cite a
third-party repository, whose code is not used here); the plainest reading
is a Hamiltonian path of the grid graph with unit steps that reduces to the
Hilbert curve on 2^k x 2^k grids.  This is a plain restatement of that
construction, written independently of the library's C version:

  walk(corner, travel direction u with la cells, side direction v with lb cells)
  visits every cell of the la x lb block once, from `corner` to
  corner + (la - 1) u.  By the chessboard colouring such a path exists iff
  la is even or la and lb are both odd; each step below keeps that true:
    lb == 1          a line along u
    la == 2          along v, one step along u, back along -v
    la >= 2 lb or lb == 2
                     two blocks along u, cut at a = la // 2 (moved to an even
                     value when lb is even)
    otherwise        the Hilbert "U": near strip of b rows (b = lb // 2 moved
                     to an even value in [2, lb - 1]); its first a = la // 2
                     columns along v, then the far strip (lb - b rows) along u,
                     then the near strip's last la - a columns back along -v.
The whole grid starts at (0, 0) and runs along the longer side when that
side admits a path (even, or both sides odd), else along the other.

Pins (tests): every cell once, unit steps, equality with the textbook
Hilbert curve on 2^k x 2^k grids, and tile compactness against raster order.
"""
from __future__ import annotations

import numpy as np


def _walk(out, W, x, y, u, la, v, lb):
    ux, uy = u
    vx, vy = v
    if lb == 1:
        for i in range(la):
            out.append((y + i * uy) * W + x + i * ux)
        return
    if la == 2:
        for j in range(lb):
            out.append((y + j * vy) * W + x + j * vx)
        for j in reversed(range(lb)):
            out.append((y + uy + j * vy) * W + x + ux + j * vx)
        return
    if la >= 2 * lb or lb == 2:
        a = la // 2
        if lb % 2 == 0 and a % 2 == 1:
            a = a - 1 if a - 1 >= 2 else a + 1
        _walk(out, W, x, y, u, a, v, lb)
        _walk(out, W, x + a * ux, y + a * uy, u, la - a, v, lb)
        return
    b = lb // 2
    if b % 2 == 1:
        b = b + 1 if b + 1 <= lb - 1 else b - 1
    a = la // 2
    _walk(out, W, x, y, v, b, u, a)
    _walk(out, W, x + b * vx, y + b * vy, u, la, v, lb - b)
    _walk(out, W, x + (la - 1) * ux + (b - 1) * vx, y + (la - 1) * uy + (b - 1) * vy,
          (-vx, -vy), b, (-ux, -uy), la - a)


def gilbert_order(width: int, height: int) -> np.ndarray:
    """Raster index (y * width + x) of the t-th cell of the curve."""
    if width < 1 or height < 1:
        raise ValueError("grid sides must be positive")
    out: list[int] = []
    if width >= height:
        along_x = width % 2 == 0 or height % 2 == 1
    else:
        along_x = not (height % 2 == 0 or width % 2 == 1)
    if along_x:
        _walk(out, width, 0, 0, (1, 0), width, (0, 1), height)
    else:
        _walk(out, width, 0, 0, (0, 1), height, (1, 0), width)
    return np.asarray(out, dtype=np.int64)

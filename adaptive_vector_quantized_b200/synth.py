"""Seeded synthetic inputs for AVQ attention.

This module is shared by the CUDA path (bench, smoke, GPU tests) and by the
oracle's tests.  It holds none of the method's arithmetic: only random draws,
rounding to the run dtype and token layouts on an image grid.

Workloads follow the shapes of the paper "AVQ-Attention: Adaptive
Vector-Quantized Attention": head dim 64, 12 or 16 heads, codebooks labelled
M0/P/C such as 64/16/8 (Sec. 5, Table 2), tokens of an image grid reordered
along a space-filling curve (Sec. 4.2, Fig. 3).  No dataset is used; the
recipes below stand in for ImageNet/ADE20K/COCO activations.

Codebook recipe (keeps the parent-child constraint of Sec. 4.1, Eq. 5 exact
in every dtype): parents are N(0,1) draws and child offsets N(0, sigma_c^2)
draws, both rounded to the 2^-6 grid; offsets are centred in integer grid
units so that they sum to exactly zero; every value is kept below 4 in
magnitude, so it has at most 8 significant bits and is exact in bf16, fp32
and fp64.  Hence parent == mean(children) holds exactly.
"""
from __future__ import annotations

import math

import numpy as np
import torch

GRID_UNITS = 64  # values live on the 2^-6 grid
GRID_LIMIT = 255  # |value| <= 255/64 < 4  ->  <= 8 significant bits

# Named workloads.  dtype "f32" or "bf16"; keys: "tree" (each key is a random
# tree node plus noise), "regions" (a Voronoi region map on a side x side
# image grid, each region labelled with one tree node).
CONFIGS = {
    "tiny": dict(dtype="f32", B=1, H=1, N=1024, d=64, M0=16, C=4, P=4, block=64,
                 keys="tree", key_sigma=0.1, sigma_c=0.3, two_pass=False),
    "vit": dict(dtype="bf16", B=2, H=12, N=4096, d=64, M0=64, C=8, P=16, block=128,
                keys="regions", side=64, key_sigma=0.1, noise=0.0, order="hilbert",
                sigma_c=0.3, two_pass=False),
    "long": dict(dtype="bf16", B=1, H=16, N=65536, d=64, M0=64, C=8, P=16, block=128,
                 keys="regions", side=256, key_sigma=0.1, noise=0.1, order="hilbert",
                 sigma_c=0.3, two_pass=False),
    "largecb": dict(dtype="bf16", B=1, H=8, N=16384, d=128, M0=256, C=8, P=32, block=128,
                    keys="tree", key_sigma=0.1, sigma_c=0.3, two_pass=True),
    # the paper's 224 x 224 ViT shape: a 28 x 28 patch grid (N = 784, not a
    # multiple of the query block) along the generalised Hilbert curve
    "vit28": dict(dtype="bf16", B=2, H=12, N=784, d=64, M0=64, C=8, P=16, block=128,
                  keys="regions", grid=(28, 28), key_sigma=0.1, noise=0.0, order="gilbert",
                  sigma_c=0.3, two_pass=False),
    # depth-3 tree (the conclusion's "deeper hierarchies"): 64 parents, 512
    # children, 4096 grandchildren; P parents refined, then P of their children
    "deep3": dict(dtype="bf16", B=1, H=8, N=16384, d=64, M0=64, C=8, P=16, P2=16, block=128,
                  keys="tree3", key_sigma=0.03, sigma_c=0.3, sigma_g=0.1, noise=0.0, depth=3),
}
CONFIG_SEEDS = {"tiny": 1000, "vit": 1001, "long": 1002, "largecb": 1003, "sweep": 1004, "vit28": 1005,
                "deep3": 1006}


def sweep_config(P: int, N: int, order: str = "hilbert", flat192: bool = False) -> dict:
    """One point of the P x N sweep (H=8, d=64, 64/P/8) or the flat 192-codeword VQ."""
    side = int(round(math.sqrt(N)))
    if side * side != N:
        raise ValueError("sweep N must be a square grid")
    cfg = dict(dtype="bf16", B=1, H=8, N=N, d=64, M0=64, C=8, P=P, block=128,
               keys="regions", side=side, key_sigma=0.1, noise=0.1, order=order,
               sigma_c=0.3, two_pass=False)
    if flat192:
        cfg.update(M0=192, C=0, P=0)
    return cfg


def get_config(name: str, **overrides) -> dict:
    if name not in CONFIGS:
        raise KeyError(name)
    cfg = dict(CONFIGS[name])
    cfg.update(overrides)
    return cfg


def m_total(M0: int, C: int) -> int:
    """Number of codewords in the two-level tree: M0 parents plus C children each."""
    return M0 * (1 + C)


def hilbert_cells(side: int) -> np.ndarray:
    """Raster index (y*side + x) of the t-th cell along a Hilbert curve.

    Textbook quadrant-rotation construction for a 2^k x 2^k grid.
    """
    if side < 1 or side & (side - 1):
        raise ValueError("side must be a power of two")
    t = np.arange(side * side, dtype=np.int64)
    x = np.zeros_like(t)
    y = np.zeros_like(t)
    s = 1
    rem = t.copy()
    while s < side:
        rx = (rem // 2) & 1
        ry = (rem ^ rx) & 1
        flip = (ry == 0) & (rx == 1)
        x = np.where(flip, s - 1 - x, x)
        y = np.where(flip, s - 1 - y, y)
        swap = ry == 0
        x, y = np.where(swap, y, x), np.where(swap, x, y)
        x = x + s * rx
        y = y + s * ry
        rem = rem // 4
        s *= 2
    return (y * side + x).astype(np.int64)


def _round_dtype(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(dtype)


def _centred_offsets(rng, C: int, d: int, sigma: float):
    """C offsets [C, d] in grid units, N(0, sigma^2) draws rounded to the
    grid and shifted (in whole units) so that they sum to exactly zero."""
    off = np.rint(rng.standard_normal((C, d)) * sigma * GRID_UNITS).astype(np.int64)
    tot = off.sum(axis=0)
    q = np.floor_divide(tot, C)
    r = tot - q * C  # 0 <= r < C
    off -= q[None, :]
    off -= (np.arange(C)[:, None] < r[None, :]).astype(np.int64)
    return off


def make_codebook(rng: np.random.Generator, H: int, M0: int, C: int, d: int,
                  sigma_c: float = 0.3):
    """Parents [H,M0,d] and children [H,M0,C,d] in grid units (int64) with
    sum_c children == C * parent exactly (offsets centred in integer units)."""
    par = np.clip(np.rint(rng.standard_normal((H, M0, d)) * GRID_UNITS),
                  -GRID_LIMIT + 64, GRID_LIMIT - 64).astype(np.int64)
    if C == 0:
        return par, np.zeros((H, M0, 0, d), dtype=np.int64)
    child = np.empty((H, M0, C, d), dtype=np.int64)
    for h in range(H):
        for m in range(M0):
            for _ in range(1000):
                ch = par[h, m][None, :] + _centred_offsets(rng, C, d, sigma_c)
                if np.abs(ch).max() <= GRID_LIMIT:
                    break
            else:  # pragma: no cover - astronomically unlikely
                raise RuntimeError("could not draw children inside the grid limit")
            child[h, m] = ch
    return par, child


def make_codebook3(rng: np.random.Generator, H: int, M0: int, C: int, d: int,
                   sigma_c: float = 0.3, sigma_g: float = 0.1):
    """A depth-3 tree in grid units: parents [H,M0,d], children [H,M0,C,d],
    grandchildren [H,M0,C,C,d]; every child is exactly the mean of its
    grandchildren and every parent of its children (centred integer offsets),
    all values at most 8 significant bits (exact in bf16)."""
    par, child = make_codebook(rng, H, M0, C, d, sigma_c)
    gc = np.empty((H, M0, C, C, d), dtype=np.int64)
    for h in range(H):
        for m in range(M0):
            for c in range(C):
                for _ in range(1000):
                    g = child[h, m, c][None, :] + _centred_offsets(rng, C, d, sigma_g)
                    if np.abs(g).max() <= GRID_LIMIT:
                        break
                else:  # pragma: no cover - astronomically unlikely
                    raise RuntimeError("could not draw grandchildren inside the grid limit")
                gc[h, m, c] = g
    return par, child, gc


def m_total3(M0: int, C: int) -> int:
    """Codewords of the depth-3 tree: M0 parents, M0*C children, M0*C*C grandchildren."""
    return M0 + M0 * C + M0 * C * C


def make_inputs3(cfg: dict, seed: int) -> dict:
    """Inputs of a depth-3 forward: as make_inputs, plus grandchildren
    [H,M0,C,C,d].  Keys: a uniform parent, then a uniform level (parent,
    child or grandchild) and a uniform node of that level below the parent,
    plus N(0, key_sigma^2) noise; a fraction `noise` of keys ~U(-3,3)^d."""
    B, H, N, d, M0, C = (cfg[k] for k in ("B", "H", "N", "d", "M0", "C"))
    dtype = cfg["dtype"]
    s_code, s_key, s_q, s_v = np.random.SeedSequence(seed).spawn(4)
    rng_key = np.random.default_rng(s_key)
    par_i, ch_i, gc_i = make_codebook3(np.random.default_rng(s_code), H, M0, C, d,
                                       cfg.get("sigma_c", 0.3), cfg.get("sigma_g", 0.1))
    par_f, ch_f, gc_f = (x.astype(np.float64) / GRID_UNITS for x in (par_i, ch_i, gc_i))
    K = np.empty((B, H, N, d), dtype=np.float32)
    sigma = cfg.get("key_sigma", 0.03)
    for b in range(B):
        for h in range(H):
            p = rng_key.integers(0, M0, N)
            lvl = rng_key.integers(0, 3, N)
            c = rng_key.integers(0, C, N)
            g = rng_key.integers(0, C, N)
            base = np.where((lvl == 0)[:, None], par_f[h][p],
                            np.where((lvl == 1)[:, None], ch_f[h][p, c], gc_f[h][p, c, g]))
            base = base + rng_key.standard_normal((N, d)) * sigma
            frac = cfg.get("noise", 0.0)
            if frac > 0:
                sel = rng_key.random(N) < frac
                base[sel] = rng_key.uniform(-3.0, 3.0, size=(int(sel.sum()), d))
            K[b, h] = base.astype(np.float32)
    Q = np.random.default_rng(s_q).standard_normal((B, H, N, d), dtype=np.float32)
    V = np.random.default_rng(s_v).standard_normal((B, H, N, d), dtype=np.float32)
    return dict(
        Q=_round_dtype(Q, dtype), K=_round_dtype(K, dtype), V=_round_dtype(V, dtype),
        parents=_round_dtype(par_f, dtype), children=_round_dtype(ch_f, dtype),
        grandchildren=_round_dtype(gc_f, dtype),
        B=B, H=H, N=N, d=d, M0=M0, C=C, P=cfg["P"], P2=cfg.get("P2", cfg["P"]), block=cfg["block"],
        scale=1.0 / math.sqrt(d), dtype=dtype, depth=3,
    )


def _tree_nodes(M0: int, C: int):
    """(parent, child) pairs of every tree node; child == -1 for the parent itself."""
    nodes = [(m, -1) for m in range(M0)]
    nodes += [(m, c) for m in range(M0) for c in range(C)]
    return nodes


def _pick_nodes(rng, count, M0, C):
    """Random tree nodes: a uniform parent, then uniform over {parent, its C children}."""
    p = rng.integers(0, M0, size=count)
    c = rng.integers(-1, C, size=count) if C > 0 else np.full(count, -1)
    return p, c


def _node_vectors(par_f, child_f, h, p, c):
    out = par_f[h][p].copy()
    moved = c >= 0
    if moved.any():
        out[moved] = child_f[h][p[moved], c[moved]]
    return out


def _region_nodes(rng, width, height, n_seeds, M0, C, order):
    """Tree node of every token: Voronoi regions of random seeds on the
    width x height grid, tokens taken along the requested order (hilbert
    (2^k square grids), gilbert (any grid), raster or random)."""
    from scipy.spatial import cKDTree

    if width == height:
        seeds = rng.uniform(0.0, width, size=(n_seeds, 2))
    else:
        seeds = rng.uniform(0.0, 1.0, size=(n_seeds, 2)) * np.array([width, height])
    sp, sc = _pick_nodes(rng, n_seeds, M0, C)
    yy, xx = np.divmod(np.arange(width * height), width)
    cells = np.stack([xx + 0.5, yy + 0.5], axis=1)
    _, nearest = cKDTree(seeds).query(cells)
    if order == "hilbert":
        if width != height:
            raise ValueError("the hilbert order needs a square 2^k grid; use gilbert")
        tok = hilbert_cells(width)
    elif order == "gilbert":
        from .order import grid_order

        tok = grid_order(width, height, "gilbert")
    elif order == "raster":
        tok = np.arange(width * height)
    elif order == "random":
        tok = rng.permutation(width * height)
    else:
        raise ValueError(order)
    return sp[nearest[tok]], sc[nearest[tok]]


def make_inputs(cfg: dict, seed: int) -> dict:
    """All inputs of one AVQ forward: Q, K, V [B,H,N,d], parents [H,M0,d],
    children [H,M0,C,d] as CPU tensors in the run dtype, plus the run scalars."""
    B, H, N, d, M0, C = (cfg[k] for k in ("B", "H", "N", "d", "M0", "C"))
    dtype = cfg["dtype"]
    ss = np.random.SeedSequence(seed)
    s_code, s_key, s_q, s_v = ss.spawn(4)
    rng_code = np.random.default_rng(s_code)
    rng_key = np.random.default_rng(s_key)
    rng_q = np.random.default_rng(s_q)
    rng_v = np.random.default_rng(s_v)

    par_i, child_i = make_codebook(rng_code, H, M0, C, d, cfg.get("sigma_c", 0.3))
    par_f = (par_i / GRID_UNITS).astype(np.float32)
    child_f = (child_i / GRID_UNITS).astype(np.float32)

    K = np.empty((B, H, N, d), dtype=np.float32)
    sigma = cfg.get("key_sigma", 0.1)
    q_gain = float(cfg.get("q_coherent", 0.0))
    nodes = np.empty((B, H, N, d), dtype=np.float32) if q_gain > 0 else None
    for b in range(B):
        for h in range(H):
            if cfg["keys"] == "regions":
                W, Hg = cfg["grid"] if "grid" in cfg else (cfg["side"], cfg["side"])
                assert W * Hg == N
                p, c = _region_nodes(rng_key, W, Hg, 4 * M0, M0, C, cfg.get("order", "hilbert"))
            elif cfg["keys"] == "tree":
                p, c = _pick_nodes(rng_key, N, M0, C)
            else:
                raise ValueError(cfg["keys"])
            base = _node_vectors(par_f, child_f, h, p, c)
            if nodes is not None:
                nodes[b, h] = base
            base += rng_key.standard_normal((N, d), dtype=np.float32) * np.float32(sigma)
            frac = cfg.get("noise", 0.0)
            if frac > 0:
                sel = rng_key.random(N) < frac
                base[sel] = rng_key.uniform(-3.0, 3.0, size=(int(sel.sum()), d)).astype(np.float32)
            K[b, h] = base
    Q = rng_q.standard_normal((B, H, N, d), dtype=np.float32)
    if nodes is not None:  # queries that look at their own region: q = g * node + N(0, 1)
        Q += np.float32(q_gain) * nodes
    V = rng_v.standard_normal((B, H, N, d), dtype=np.float32)

    return dict(
        Q=_round_dtype(Q, dtype), K=_round_dtype(K, dtype), V=_round_dtype(V, dtype),
        parents=_round_dtype(par_f, dtype), children=_round_dtype(child_f, dtype),
        B=B, H=H, N=N, d=d, M0=M0, C=C, P=cfg["P"], block=cfg["block"],
        scale=1.0 / math.sqrt(d), dtype=dtype, two_pass=bool(cfg.get("two_pass", False)),
    )

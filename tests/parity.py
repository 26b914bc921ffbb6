"""Comparison rules between the CUDA path and the oracle.

- Assignments and counts are bit-exact, except keys whose oracle decision is
  a near-tie: where another candidate is within 1e-5*(|k|^2 + |c|^2) of the
  chosen one (at the parent choice or at the child/parent decision), the GPU
  may pick either; statistics are then compared with statistics recomputed
  from the GPU's own assignments.
- Top-P sets are bit-exact, except the tie band: parents whose oracle
  importance is within 1e-5 (relative) of the P-th largest may be in or out;
  everything above the band must be selected and nothing below it.  The
  output is then compared with the oracle rerun on the GPU's selection.
- O within max-abs 1e-4*max|V| (fp32 path) or 2e-2*max|V| (bf16 inputs with
  fp32 accumulation).
"""
from __future__ import annotations

import numpy as np

ASSIGN_BAND = 1e-5
TOPP_BAND = 1e-5
O_TOL = {"f32": 1e-4, "bf16": 2e-2}
# Value sums are fp32 sums of up to N terms in an order fixed by the schedule;
# the bound is relative to the sum of magnitudes of the summed values.
VSUM_TOL = 2e-5


def _f64(a):
    if hasattr(a, "detach"):
        import torch

        a = a.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


def acceptable_code(k, parents_h, children_h, g, M0, C, band=ASSIGN_BAND):
    """Is code g an acceptable answer for key k within the near-tie band?"""
    dp = ((parents_h - k[None]) ** 2).sum(-1)
    pg = g if g < M0 else (g - M0) // C
    tol_p = band * (k @ k + parents_h[pg] @ parents_h[pg])
    if dp[pg] > dp.min() + tol_p:
        return False
    if C == 0:
        return g < M0
    ch = children_h[pg]
    dc = ((ch - k[None]) ** 2).sum(-1)
    if g >= M0:
        c = (g - M0) - pg * C
        tol_c = band * (k @ k + ch[c] @ ch[c])
        return dc[c] <= dc.min() + tol_c and dc[c] <= dp[pg] + tol_c
    cbest = int(dc.argmin())
    tol_c = band * (k @ k + ch[cbest] @ ch[cbest])
    return dc.min() >= dp[pg] - tol_c


def check_assign(gpu_assign, oracle_assign, K, parents, children):
    """Returns the number of accepted near-tie disagreements; raises on any other."""
    gpu_assign = np.asarray(gpu_assign)
    oracle_assign = np.asarray(oracle_assign)
    bad = np.argwhere(gpu_assign != oracle_assign)
    if len(bad) == 0:
        return 0
    K = _f64(K)
    par = _f64(parents)
    ch = _f64(children)
    M0 = par.shape[1]
    C = ch.shape[2]
    Mt = M0 * (1 + C)
    assert ((gpu_assign >= 0) & (gpu_assign < Mt)).all(), "code out of range"
    for b, h, j in bad:
        g = int(gpu_assign[b, h, j])
        ok = acceptable_code(K[b, h, j], par[h], ch[h], g, M0, C)
        assert ok, f"key {(int(b), int(h), int(j))}: GPU code {g}, oracle {int(oracle_assign[b, h, j])}"
    assert len(bad) <= max(8, gpu_assign.size // 1000), f"{len(bad)} near-tie disagreements"
    return len(bad)


def check_stats(gpu_vsum, gpu_counts, ref_vsum, ref_counts, abs_vsum):
    """Counts bit-exact; value sums within VSUM_TOL of the summed magnitudes."""
    gpu_counts = np.asarray(gpu_counts)
    assert (gpu_counts == np.asarray(ref_counts)).all(), "counts differ"
    err = np.abs(_f64(gpu_vsum) - ref_vsum)
    lim = VSUM_TOL * abs_vsum + 1e-6
    worst = np.unravel_index(np.argmax(err - lim), err.shape)
    assert (err <= lim).all(), f"vsum off at {worst}: {err[worst]} > {lim[worst]}"


def topp_band(w, P, band=TOPP_BAND):
    """(must, may) masks over the parents for one block's oracle importance."""
    ws = np.sort(w)[::-1]
    t = ws[P - 1]
    tol = band * abs(t)
    must = w > t + tol
    may = np.abs(w - t) <= tol
    return must, may


def check_sel(gpu_sel, oracle_imp, P):
    """GPU selection against the oracle's importance with the tie band.
    Returns the number of blocks whose selection differs from the oracle's."""
    gpu_sel = np.asarray(gpu_sel)
    if P == 0:
        return 0
    differ = 0
    for idx in np.ndindex(*gpu_sel.shape[:-1]):
        s = gpu_sel[idx]
        w = oracle_imp[idx]
        assert len(set(s.tolist())) == P, f"block {idx}: duplicate parents {s}"
        assert ((s >= 0) & (s < w.shape[0])).all()
        must, may = topp_band(w, P)
        chosen = np.zeros_like(must)
        chosen[s] = True
        assert (chosen[must]).all(), f"block {idx}: missed a parent above the tie band"
        assert not (chosen & ~must & ~may).any(), f"block {idx}: picked a parent below the band"
        ref = np.lexsort((np.arange(w.shape[0]), -w))[:P]
        differ += int(sorted(ref.tolist()) != sorted(s.tolist()))
    return differ


def check_order(gpu_sel, gpu_imp):
    """The selection lists parents in descending importance."""
    gpu_sel = np.asarray(gpu_sel)
    if gpu_sel.shape[-1] < 2:
        return
    w = np.take_along_axis(np.asarray(gpu_imp), gpu_sel.astype(np.int64), axis=-1)
    assert (np.diff(w, axis=-1) <= 0).all(), "selection not in descending importance"


def check_output(gpu_O, ref_O, V, dtype, rows=None):
    """max |O_gpu - O_ref| <= tol * max|V| over the compared rows."""
    g = _f64(gpu_O)
    r = np.asarray(ref_O)
    if rows is not None:
        g = g[rows]
        r = r[rows]
    vmax = float(np.abs(_f64(V)).max())
    err = float(np.nanmax(np.abs(g - r)))
    assert np.isfinite(g).all(), "non-finite output"
    assert err <= O_TOL[dtype] * vmax, f"O error {err} > {O_TOL[dtype]} * {vmax}"
    return err / vmax


def acceptable_code3(k, parents_h, children_h, gc_h, g, M0, C, band=ASSIGN_BAND):
    """Is depth-3 code g acceptable for key k within the near-tie band, at each
    of the descent's decisions (parent choice, child vs parent, grandchild vs
    child)?  children_h [M0,C,d], gc_h [M0*C,C,d]."""
    M1 = M0 * C
    if g < M0:
        pg, cg, gg = g, -1, -1
    elif g < M0 + M1:
        pg, cg, gg = (g - M0) // C, g - M0, -1
    else:
        cg = (g - M0 - M1) // C
        pg, gg = cg // C, (g - M0 - M1) % C
    dp = ((parents_h - k[None]) ** 2).sum(-1)
    if dp[pg] > dp.min() + band * (k @ k + parents_h[pg] @ parents_h[pg]):
        return False
    dc = ((children_h[pg] - k[None]) ** 2).sum(-1)
    if cg < 0:
        cb = int(dc.argmin())
        return dc.min() >= dp[pg] - band * (k @ k + children_h[pg][cb] @ children_h[pg][cb])
    c = cg - pg * C
    tol_c = band * (k @ k + children_h[pg][c] @ children_h[pg][c])
    if not (dc[c] <= dc.min() + tol_c and dc[c] <= dp[pg] + tol_c):
        return False
    dg = ((gc_h[cg] - k[None]) ** 2).sum(-1)
    if gg < 0:
        gb = int(dg.argmin())
        return dg.min() >= dc[c] - band * (k @ k + gc_h[cg][gb] @ gc_h[cg][gb])
    tol_g = band * (k @ k + gc_h[cg][gg] @ gc_h[cg][gg])
    return dg[gg] <= dg.min() + tol_g and dg[gg] <= dc[c] + tol_g


def check_assign3(gpu_assign, oracle_assign, K, parents, children, grandchildren):
    """Depth-3 codes: bit-exact outside the near-tie band."""
    gpu_assign = np.asarray(gpu_assign)
    bad = np.argwhere(gpu_assign != np.asarray(oracle_assign))
    if len(bad) == 0:
        return 0
    K, par, ch, gc = _f64(K), _f64(parents), _f64(children), _f64(grandchildren)
    M0, C = par.shape[1], ch.shape[2]
    Mt = M0 + M0 * C + M0 * C * C
    assert ((gpu_assign >= 0) & (gpu_assign < Mt)).all(), "code out of range"
    for b, h, j in bad:
        g = int(gpu_assign[b, h, j])
        ok = acceptable_code3(K[b, h, j], par[h], ch[h], gc[h].reshape(M0 * C, C, -1), g, M0, C)
        assert ok, f"key {(int(b), int(h), int(j))}: GPU code {g}, oracle {int(oracle_assign[b, h, j])}"
    assert len(bad) <= max(8, gpu_assign.size // 1000), f"{len(bad)} near-tie disagreements"
    return len(bad)

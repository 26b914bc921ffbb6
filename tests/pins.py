"""Pins of the oracle: checks against what the paper and the mathematics fix.

Each `pin_*` takes an `oracle.Oracle` and raises AssertionError on a
mismatch.  They are run against the real oracle (test_oracle_pins.py) and
against deliberately broken copies of it (test_oracle_mutations.py), to show
that a plausible mistake anywhere in the oracle fails at least one of them.
References are to "AVQ-Attention: Adaptive Vector-Quantized Attention".
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

from adaptive_vector_quantized_b200 import synth
from oracle import brute

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b)) / max(1e-300, np.max(np.abs(b))))


# small seeded cases (sizes that finish in well under a second) --------------
def case_tiny():
    return synth.make_inputs(synth.get_config("tiny"), 11)


def case_regions():
    cfg = dict(dtype="bf16", B=1, H=2, N=1024, d=64, M0=16, C=8, P=4, block=128,
               keys="regions", side=32, key_sigma=0.1, noise=0.1, order="hilbert",
               sigma_c=0.3)
    return synth.make_inputs(cfg, 12)


def case_wide():
    cfg = dict(dtype="bf16", B=1, H=1, N=300, d=128, M0=32, C=8, P=8, block=64,
               keys="tree", key_sigma=0.1, sigma_c=0.3)
    return synth.make_inputs(cfg, 13)


CASES = (case_tiny, case_regions, case_wide)


def _run(orc, inp, P=None, block=None, sel=None):
    P = inp["P"] if P is None else P
    block = inp["block"] if block is None else block
    assign, vsum, counts, dec = orc.quantize(inp["K"], inp["V"], inp["parents"], inp["children"])
    O, s, imp = orc.attention(inp["Q"], inp["parents"], inp["children"], vsum, counts,
                              P, block, inp["scale"], sel=sel)
    return assign, vsum, counts, O, s, imp


# ---------------------------------------------------------------------------
def pin_hand_worked(orc):
    """Hand-derived d=2 example (Alg. 1, Alg. 2, Eqs. 7-9, Eq. 18)."""
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_d2.json")))
    par = np.array(g["parents"])[None]
    ch = np.array(g["children"])[None]
    K = np.array(g["keys"])[None, None]
    V = np.array(g["values"])[None, None]
    Q = np.array(g["queries"])[None, None]
    env = {"v0": V[0, 0, 0], "v1": V[0, 0, 1], "v2": V[0, 0, 2], "exp": math.exp}
    ev = lambda s: np.asarray(eval(s, {"__builtins__": {}}, env), dtype=np.float64)  # noqa: E731
    exp = g["expected"]
    assign, vsum, counts, _ = orc.quantize(K, V, par, ch)
    assert assign[0, 0].tolist() == exp["codes"], assign
    assert counts[0, 0].tolist() == exp["counts"], counts
    for row, expr in exp["vsum"].items():
        assert _rel(vsum[0, 0, int(row)], ev(expr) + 0.0) < 1e-15 or np.all(ev(expr) == vsum[0, 0, int(row)])
    O, sel, imp = orc.attention(Q, par, ch, vsum, counts, 1, 1, g["scale"])
    for i, expr in enumerate(exp["Y_P1"]):
        assert _rel(O[0, 0, i], ev(expr)) < 1e-13, (i, O[0, 0, i], ev(expr))
    assert sel[0, 0].tolist() == exp["sel_P1_block1"]
    O3, sel3, imp3 = orc.attention(Q, par, ch, vsum, counts, 1, 3, g["scale"])
    for j, expr in enumerate(exp["importance_block3"]):
        assert abs(imp3[0, 0, 0, j] - float(ev(expr))) < 1e-13
    assert _rel(O3[0, 0], O[0, 0]) < 1e-13
    O0, _, _ = orc.attention(Q, par, ch, vsum, counts, 0, 1, g["scale"])
    for i, expr in enumerate(exp["Y_P0"]):
        assert _rel(O0[0, 0, i], ev(expr)) < 1e-13, (i, O0[0, 0, i], ev(expr))


def pin_assign_brute(orc):
    """Alg. 1 codes equal a vectorised full-distance-table assignment."""
    for mk in CASES:
        inp = mk()
        assign, _, _, _ = orc.quantize(inp["K"], inp["V"], inp["parents"], inp["children"])
        ref = brute.assign_brute(inp["K"], inp["parents"], inp["children"])
        assert (assign == ref).all(), (mk.__name__, int((assign != ref).sum()))


def pin_aggregate(orc):
    """Eq. 3 statistics of the two-level tree, plus their invariants."""
    for mk in CASES:
        inp = mk()
        M0, C, N = inp["M0"], inp["C"], inp["N"]
        assign, vsum, counts, _ = orc.quantize(inp["K"], inp["V"], inp["parents"], inp["children"])
        vs_ref, ns_ref = brute.aggregate_brute(assign, inp["V"], M0, C)
        assert (counts == ns_ref).all()
        assert _rel(vsum, vs_ref) < 1e-12
        V = brute._f64(inp["V"])
        # every key counts once at the parent level: sum_p n_p = N, sum_p Vbar_p = sum_j V_j
        assert (counts[..., :M0].sum(-1) == N).all()
        assert _rel(vsum[..., :M0, :].sum(-2), V.sum(-2)) < 1e-10
        # children hold a subset of their parent's keys (Eq. 15: n_stay >= 0)
        if C > 0:
            ch_counts = counts[..., M0:].reshape(*counts.shape[:-1], M0, C).sum(-1)
            assert (ch_counts <= counts[..., :M0]).all()
            moved = assign >= M0
            assert (counts[..., M0:].sum(-1) == moved.sum(-1)).all()


def pin_aggregate_given_codes(orc):
    """The aggregation of Algorithm 1 for codes made elsewhere (the checker of
    GPU statistics, Eq. 3): a parent holds every key of its cluster, a child
    only the keys that moved to it.
    - hand-made code lists with the statistics written out by hand, one with
      children (including a code of the last child) and one flat (C = 0);
    - brute-force aggregation of the oracle's own codes on the seeded cases;
    - Algorithm 1's own statistics when given Algorithm 1's codes."""
    # M0 = 3, C = 2: children of parent m are codes 3 + 2m and 4 + 2m.
    codes = np.array([0, 3, 4, 8, 2, 5, 1, 8, 7], dtype=np.int32)
    N = codes.size
    V = np.stack([2.0 ** np.arange(N), -np.arange(N, dtype=np.float64)], -1)[None, None]
    vs, ns = orc.aggregate(codes[None, None], V, 3, 2)
    # parents: 0 <- keys 0,1,2; 1 <- keys 5,6; 2 <- keys 3,4,7,8
    # children: 3 <- key 1; 4 <- key 2; 5 <- key 5; 7 <- key 8; 8 <- keys 3,7
    want_n = [3, 2, 4, 1, 1, 1, 0, 1, 2]
    want_v = {0: [1 + 2 + 4, -(0 + 1 + 2)], 1: [32 + 64, -(5 + 6)],
              2: [8 + 16 + 128 + 256, -(3 + 4 + 7 + 8)], 3: [2, -1], 4: [4, -2],
              5: [32, -5], 6: [0, 0], 7: [256, -8], 8: [8 + 128, -(3 + 7)]}
    assert ns[0, 0].tolist() == want_n, ns
    for x, v in want_v.items():
        assert vs[0, 0, x].tolist() == [float(t) for t in v], (x, vs[0, 0, x])
    # flat codebook: M0 = 4, C = 0
    flat = np.array([3, 0, 3, 1], dtype=np.int32)
    Vf = np.arange(8, dtype=np.float64).reshape(1, 1, 4, 2)
    vs, ns = orc.aggregate(flat[None, None], Vf, 4, 0)
    assert ns[0, 0].tolist() == [1, 1, 0, 2]
    assert vs[0, 0].tolist() == [[2, 3], [6, 7], [0, 0], [0 + 4, 1 + 5]]
    for mk in CASES:
        inp = mk()
        M0, C = inp["M0"], inp["C"]
        assign, vsum_q, counts_q, _ = orc.quantize(inp["K"], inp["V"], inp["parents"], inp["children"])
        vs, ns = orc.aggregate(assign, inp["V"], M0, C)
        vs_ref, ns_ref = brute.aggregate_brute(assign, inp["V"], M0, C)
        assert (ns == ns_ref).all(), mk.__name__
        assert _rel(vs, vs_ref) < 1e-12, mk.__name__
        assert (ns == counts_q).all(), mk.__name__
        assert _rel(vs, vsum_q) < 1e-12, mk.__name__


def pin_representative(orc):
    """Sec. C identity: AVQ output equals exact softmax attention over the
    representative keys, for several P including P = M0."""
    for mk in CASES:
        inp = mk()
        for P in sorted({1, inp["P"], inp["M0"]}):
            assign, vsum, counts, O, sel, _ = _run(orc, inp, P=P)
            Y = brute.representative_attention(inp["Q"], assign, inp["V"], inp["parents"],
                                               inp["children"], sel, inp["block"], inp["scale"])
            assert _rel(O, Y) < 1e-10, (mk.__name__, P, _rel(O, Y))


def pin_rescale_exercised(orc):
    """The representative check above covers the online-max merge of
    Algorithm 2 only if some selected non-empty child logit exceeds the
    parent max; make sure the regions case has such rows."""
    inp = case_regions()
    assign, vsum, counts, O, sel, _ = _run(orc, inp)
    Q = brute._f64(inp["Q"])
    par = brute._f64(inp["parents"])
    ch = brute._f64(inp["children"])
    M0, C, blk = inp["M0"], inp["C"], inp["block"]
    found = 0
    for h in range(inp["H"]):
        s = inp["scale"] * Q[0, h] @ par[h].T
        live = counts[0, h, :M0] > 0
        m = np.where(live[None], s, -np.inf).max(1)
        for b in range(sel.shape[2]):
            for p in sel[0, h, b]:
                sc = inp["scale"] * Q[0, h, b * blk:(b + 1) * blk] @ ch[h, p].T
                nz = counts[0, h, M0 + p * C: M0 + (p + 1) * C] > 0
                found += int((np.where(nz[None], sc, -np.inf) > m[b * blk:(b + 1) * blk, None]).any())
    assert found > 0
    Y = brute.representative_attention(inp["Q"], assign, inp["V"], inp["parents"],
                                       inp["children"], sel, blk, inp["scale"])
    assert _rel(O, Y) < 1e-10


def pin_flat_p0(orc):
    """P = 0 is fixed-codebook VQ attention over the parents (Eq. 4); C = 0
    (a flat codebook) is the same for any P."""
    inp = case_regions()
    assign, vsum, counts, O, _, _ = _run(orc, inp, P=0)
    M0 = inp["M0"]
    Y = brute.flat_vq_attention(inp["Q"], inp["parents"], vsum[..., :M0, :], counts[..., :M0],
                                inp["scale"])
    assert _rel(O, Y) < 1e-10
    cfg = dict(dtype="bf16", B=1, H=1, N=700, d=64, M0=48, C=0, P=5, block=64,
               keys="tree", key_sigma=0.1)
    flat = synth.make_inputs(cfg, 21)
    assign, vsum, counts, O, _, _ = _run(orc, flat)
    assert (assign < 48).all()
    Y = brute.flat_vq_attention(flat["Q"], flat["parents"], vsum, counts, flat["scale"])
    assert _rel(O, Y) < 1e-10


def _exact_codebook_case(rng, on_children: bool):
    H, M0, C, d, N = 1, 12, 4, 8, 240
    par, ch = synth.make_codebook(rng, H, M0, C, d, sigma_c=0.1)
    par = par / 64.0
    ch = ch / 64.0
    if on_children:
        p = rng.integers(0, M0, N)
        c = rng.integers(0, C, N)
        K = ch[0][p, c]
    else:
        K = par[0][rng.integers(0, M0, N)]
    Q = rng.standard_normal((1, H, N, d))
    V = rng.standard_normal((1, H, N, d))
    return Q, K[None, None], V, par, ch


def pin_exact_codebook(orc):
    """A codebook holding every distinct key reproduces exact attention (Eq. 1):
    keys on the parents give exact attention for any P; keys on the children
    give it for P = M0."""
    rng = np.random.default_rng(31)
    Q, K, V, par, ch = _exact_codebook_case(rng, on_children=False)
    Y = brute.exact_attention(Q, K, V, 0.5)
    for P in (0, 3, 12):
        assign, vsum, counts, _ = orc.quantize(K, V, par, ch)
        assert (assign < 12).all()
        O, _, _ = orc.attention(Q, par, ch, vsum, counts, P, 32, 0.5)
        assert _rel(O, Y) < 1e-10, (P, _rel(O, Y))
    Q, K, V, par, ch = _exact_codebook_case(rng, on_children=True)
    assign, vsum, counts, _ = orc.quantize(K, V, par, ch)
    assert (assign >= 12).all()
    O, _, _ = orc.attention(Q, par, ch, vsum, counts, 12, 32, 0.5)
    assert _rel(O, brute.exact_attention(Q, K, V, 0.5)) < 1e-10


def pin_importance(orc):
    """Eq. 7 equals the block sum of each parent's flat-VQ softmax mass, and
    sums to the block size."""
    for mk in CASES:
        inp = mk()
        assign, vsum, counts, O, sel, imp = _run(orc, inp)
        W = brute.importance_brute(inp["Q"], inp["parents"], counts, inp["block"], inp["scale"])
        assert _rel(imp, W) < 1e-12
        N, blk = inp["N"], inp["block"]
        sizes = np.array([min(blk, N - b * blk) for b in range(imp.shape[2])], dtype=np.float64)
        assert np.allclose(imp.sum(-1), sizes[None, None, :], rtol=1e-12)


def _topp_ref(w, P):
    order = np.lexsort((np.arange(w.shape[-1]), -w))  # descending, ties to lower index
    return order[:P]


def pin_topp(orc):
    """Top-P: the P largest importances, descending, ties to the lower index."""
    for mk in CASES:
        inp = mk()
        _, _, _, _, sel, imp = _run(orc, inp)
        for idx in np.ndindex(*sel.shape[:3]):
            assert sel[idx].tolist() == _topp_ref(imp[idx], inp["P"]).tolist()
    # exact ties: zero queries make every logit 0; equal counts make every w equal
    M0, C, d = 8, 2, 4
    rng = np.random.default_rng(41)
    par, ch = synth.make_codebook(rng, 1, M0, C, d)
    par, ch = par / 64.0, ch / 64.0
    K = np.repeat(par[0], 4, axis=0)[None, None]
    V = rng.standard_normal(K.shape)
    Q = np.zeros_like(K)
    assign, vsum, counts, _ = orc.quantize(K, V, par, ch)
    _, sel, imp = orc.attention(Q, par, ch, vsum, counts, 3, 32, 1.0)
    assert np.all(imp[0, 0, 0] == imp[0, 0, 0, 0])
    assert sel[0, 0, 0].tolist() == [0, 1, 2]


def pin_relabel(orc):
    """Relabelling parents (with their child runs) permutes the selection and
    leaves the output unchanged."""
    inp = case_tiny()
    M0, C = inp["M0"], inp["C"]
    assign, vsum, counts, O, sel, imp = _run(orc, inp)
    perm = np.random.default_rng(51).permutation(M0)
    inv = np.argsort(perm)
    par2 = inp["parents"][:, perm]
    ch2 = inp["children"][:, perm]
    assign2, vsum2, counts2, O2, sel2, imp2 = _run(orc, dict(inp, parents=par2, children=ch2))
    assert _rel(O2, O) < 1e-12
    for idx in np.ndindex(*sel.shape[:3]):
        w = np.sort(imp[idx])[::-1]
        if abs(w[inp["P"] - 1] - w[inp["P"]]) <= 1e-9 * w[inp["P"] - 1]:
            continue
        assert sorted(perm[sel2[idx]].tolist()) == sorted(sel[idx].tolist())
    par_code = np.where(assign < M0, assign, (assign - M0) // C)
    par_code2 = np.where(assign2 < M0, assign2, (assign2 - M0) // C)
    assert (perm[par_code2] == par_code).all()
    assert (counts2[..., :M0] == counts[..., :M0][..., perm]).all()
    assert (inv[perm] == np.arange(M0)).all()


def pin_key_permutation(orc):
    """Counts and sums do not depend on the order of the keys; codes move with them."""
    inp = case_regions()
    assign, vsum, counts, _ = orc.quantize(inp["K"], inp["V"], inp["parents"], inp["children"])
    perm = np.random.default_rng(61).permutation(inp["N"])
    assign2, vsum2, counts2, _ = orc.quantize(inp["K"][:, :, perm], inp["V"][:, :, perm],
                                              inp["parents"], inp["children"])
    assert (assign2 == assign[:, :, perm]).all()
    assert (counts2 == counts).all()
    assert _rel(vsum2, vsum) < 1e-12


def pin_keys_on_codewords(orc):
    """A key placed exactly on a codeword is assigned to it."""
    inp = case_tiny()
    M0, C = inp["M0"], inp["C"]
    par = brute._f64(inp["parents"])
    ch = brute._f64(inp["children"])
    codes = np.arange(M0 * (1 + C))
    K = np.concatenate([par[0], ch[0].reshape(M0 * C, -1)])[None, None]
    V = np.zeros_like(K)
    assign, _, _, _ = orc.quantize(K, V, par, ch)
    assert (assign[0, 0] == codes).all()


def pin_strict_ties(orc):
    """Ties: equal parents -> lower index (argmin); a child must be strictly
    closer than the best child so far (first child wins) and strictly closer
    than the parent (the two strict comparisons of Algorithm 1)."""
    par = np.array([[[0.0, 0.0], [10.0, 10.0]]])
    ch = np.array([[[[1, 1], [1, -1], [-1, 1], [-1, -1]],
                    [[11, 11], [11, 9], [9, 11], [9, 9]]]], dtype=np.float64)
    K = np.array([[1.0, 0.0],    # parent 0 at 1, children 0 and 1 at 1: stays
                  [1.2, 0.0],    # children 0 and 1 tie at 1.04 < 1.44: child 0 -> code 2
                  [5.0, 5.0],    # both parents at 50: lower index; children of 0 at 32 -> code 2
                  [0.0, 0.0],    # on parent 0
                  [-1.2, 0.0]])  # children 2 and 3 tie: child 2 -> code 4
    K = K[None, None]
    V = np.ones_like(K)
    assign, _, _, _ = orc.quantize(K, V, par, ch)
    assert assign[0, 0].tolist() == [0, 2, 2, 0, 4], assign


def pin_masking(orc):
    """Eq. 18 and Sec. D: an empty child or parent with a huge logit neither
    sets the running max nor produces inf*0; the output is still the
    representative-key attention."""
    par = np.array([[[0.0, 0.0], [-60.0, 0.0], [50.0, 0.0]]])
    ch = np.array([[[[30.0, 0.0], [-30.0, 0.0]],
                    [[-61.0, 0.0], [-59.0, 0.0]],
                    [[49.0, 0.0], [51.0, 0.0]]]])
    rng = np.random.default_rng(71)
    stay = np.stack([rng.uniform(-0.5, 0.5, 6), rng.uniform(-0.5, 0.5, 6)], 1)
    moved = np.array([[-29.9, 0.0], [-29.95, 0.1]])
    far = np.array([[-60.0, 0.2], [-60.1, 0.0]])
    K = np.concatenate([stay, moved, far])[None, None]
    N = K.shape[2]
    V = rng.standard_normal((1, 1, N, 2))
    Q = np.tile(np.array([40.0, 0.0]), (N, 1))[None, None]
    assign, vsum, counts, _ = orc.quantize(K, V, par, ch)
    assert counts[0, 0, 2] == 0 and counts[0, 0, 3] == 0, counts  # parent 2 and child (0,0) empty
    assert counts[0, 0, 4] == 2
    O, sel, _ = orc.attention(Q, par, ch, vsum, counts, 1, N, 1.0)
    assert sel[0, 0, 0].tolist() == [0]
    assert np.isfinite(O).all()
    Y = brute.representative_attention(Q, assign, V, par, ch, sel, N, 1.0)
    assert _rel(O, Y) < 1e-12


def pin_counting(orc):
    """Codebook size and per-block code count of the paper's configurations."""
    g = json.load(open(os.path.join(GOLDEN, "counting.json")))
    for row in g["mtotal"]:
        assert synth.m_total(row["M0"], row["C"]) == row["Mtotal"]
    for row in g["codes_per_query"]:
        assert row["M0"] + row["P"] * row["C"] == row["codes"]
    # the oracle's statistics are laid out over the same M0*(1+C) codes
    inp = case_tiny()
    _, vsum, counts, _ = orc.quantize(inp["K"], inp["V"], inp["parents"], inp["children"])
    assert counts.shape[-1] == synth.m_total(inp["M0"], inp["C"])


def pin_tiled_importance(orc):
    """Tiled importance with the count-extrapolated denominator (Sec. B,
    Eqs. 13-14), parents in tiles of `tile` codes:
    - over the first tile Z~ = Z(0) N / N_seen(0), so that tile's importances
      sum to |I| N_seen(0) / N whatever the logits;
    - at the last tile N_seen = N and Z~ is the exact denominator, so the last
      tile's importances equal Eq. 7's;
    - with constant logits (Q = 0) every A is 1 and Z~ = N for every tile, so
      all importances equal Eq. 7's;
    - the selection is the top-P of the tiled importances."""
    for mk, tile in ((case_regions, 8), (case_wide, 8), (case_wide, 16)):
        inp = mk()
        assign, vsum, counts, _ = orc.quantize(inp["K"], inp["V"], inp["parents"], inp["children"])
        M0, P, blk, N = inp["M0"], inp["P"], inp["block"], inp["N"]
        args = (inp["parents"], inp["children"], vsum, counts, P, blk, inp["scale"])
        _, sel_t, imp_t = orc.attention(inp["Q"], *args, tile=tile)
        _, _, imp_x = orc.attention(inp["Q"], *args)
        nblk = imp_t.shape[2]
        sizes = np.array([min(blk, N - b * blk) for b in range(nblk)], dtype=np.float64)
        nseen0 = counts[..., :tile].sum(-1).astype(np.float64)     # [B,H]
        ntot = counts[..., :M0].sum(-1).astype(np.float64)         # [B,H] == N
        assert np.all(ntot == N)
        want = sizes[None, None, :] * (nseen0 / ntot)[..., None]
        assert np.allclose(imp_t[..., :tile].sum(-1), want, rtol=1e-11, atol=1e-300)
        last = (M0 - 1) // tile * tile
        assert _rel(imp_t[..., last:], imp_x[..., last:]) < 1e-12
        for b in range(imp_t.shape[0]):
            for h in range(imp_t.shape[1]):
                for k in range(nblk):
                    assert np.array_equal(sel_t[b, h, k], _topp_ref(imp_t[b, h, k], P))
        Q0 = np.zeros(tuple(inp["Q"].shape), dtype=np.float64)
        _, _, imp_t0 = orc.attention(Q0, *args, tile=tile)
        _, _, imp_x0 = orc.attention(Q0, *args)
        assert _rel(imp_t0, imp_x0) < 1e-12
        assert not np.allclose(imp_t, imp_x, rtol=1e-6)  # the approximation is exercised


def _update_case(orc, lam, seed):
    """Eq. 3 statistics of the keys of case_regions, a positive EMA prior."""
    inp = case_regions()
    assign, ksum, counts, _ = orc.quantize(inp["K"], inp["K"], inp["parents"], inp["children"])
    rng = np.random.default_rng(seed)
    H, M0, C, d = inp["H"], inp["M0"], inp["C"], inp["d"]
    Mt = M0 * (1 + C)
    S0 = rng.standard_normal((H, Mt, d))
    N0 = rng.uniform(0.5, 4.0, (H, Mt))
    out = orc.codebook_update(ksum, counts, S0, N0, inp["parents"], inp["children"], lam)
    return inp, assign, ksum, counts, S0, N0, out


def pin_codebook_update(orc):
    """Sec. A: Eq. 11 EMA (lambda = 0 gives the step's own statistics, so the
    parents are the plain means of their clusters, computed here from the keys
    and codes; lambda = 1 keeps the state); Eq. 12 restores
    sum_c C_pc = C C_p; and it is the minimiser of sum_c N_c |C_pc - M_c|^2
    under that constraint (checked against a direct least-squares solve)."""
    for lam in (0.0, 0.9, 1.0):
        inp, assign, ksum, counts, S0, N0, (S1, N1, po, co) = _update_case(orc, lam, 21)
        H, M0, C, d = inp["H"], inp["M0"], inp["C"], inp["d"]
        # EMA
        assert _rel(N1, lam * N0 + (1 - lam) * counts.sum(0)) < 1e-14
        assert _rel(S1, lam * S0 + (1 - lam) * ksum.sum(0)) < 1e-14
        if lam == 0.0:
            K = np.asarray(inp["K"].float().numpy(), dtype=np.float64)
            for h in range(H):
                par = np.where(assign[0, h] < M0, assign[0, h], (assign[0, h] - M0) // C)
                for p_ in range(M0):
                    sel = par == p_
                    if sel.any():
                        assert _rel(po[h, p_], K[0, h][sel].mean(0)) < 1e-12
        # constraint (Eq. 5 restored)
        assert np.allclose(co.sum(2), C * po, rtol=0, atol=1e-10 * max(1.0, np.abs(po).max()))
        # minimiser: eliminate the last child and solve the weighted least squares
        for h in range(H):
            for p_ in range(0, M0, 5):
                xs = [M0 + p_ * C + c for c in range(C)]
                n = N1[h, xs]
                if not (n > 0).all():
                    continue
                M = S1[h, xs] / n[:, None]
                # unknowns y_0..y_{C-2}; y_{C-1} = C C_p - sum y_c
                A = np.zeros((C, C - 1))
                bvec = np.zeros((C, d))
                for c in range(C - 1):
                    A[c, c] = math.sqrt(n[c])
                    bvec[c] = math.sqrt(n[c]) * M[c]
                A[C - 1, :] = -math.sqrt(n[C - 1])
                bvec[C - 1] = math.sqrt(n[C - 1]) * (M[C - 1] - C * po[h, p_])
                y, *_ = np.linalg.lstsq(A, bvec, rcond=None)
                ref = np.vstack([y, C * po[h, p_] - y.sum(0)])
                assert _rel(co[h, p_], ref) < 1e-9


def pin_codebook_massless(orc):
    """Readings for codes without mass: a massless child keeps its position
    and the others absorb the displacement; with no massive child all C
    children shift by the same amount; the constraint holds either way."""
    rng = np.random.default_rng(22)
    B, H, M0, C, d = 1, 1, 2, 4, 3
    Mt = M0 * (1 + C)
    par = rng.standard_normal((H, M0, d))
    ch = rng.standard_normal((H, M0, C, d))
    ksum = rng.standard_normal((B, H, Mt, d))
    counts = np.zeros((B, H, Mt))
    counts[0, 0, 0] = 5
    counts[0, 0, M0 + 0] = 2
    counts[0, 0, M0 + 1] = 3          # parent 0: children 2 and 3 massless
    counts[0, 0, 1] = 4               # parent 1: no child has mass
    for x in range(Mt):
        if counts[0, 0, x] == 0:
            ksum[0, 0, x] = 0.0
    S1, N1, po, co = orc.codebook_update(ksum, counts, np.zeros((H, Mt, d)), np.zeros((H, Mt)), par, ch, 0.0)
    assert np.allclose(co[0, 0, 2], ch[0, 0, 2]) and np.allclose(co[0, 0, 3], ch[0, 0, 3])
    assert np.allclose(co.sum(2), C * po, atol=1e-12)
    shift = ch[0, 1] - co[0, 1]
    assert np.allclose(shift, shift[0][None, :], atol=1e-12)
    assert np.allclose(po[0, 1], ksum[0, 0, 1] / 4)


# ---- depth-3 tree (Sec. 6, "deeper hierarchies") ----------------------------
def case3_small():
    cfg = dict(dtype="bf16", B=1, H=2, N=600, d=32, M0=8, C=4, P=3, P2=4, block=128,
               key_sigma=0.03)
    return synth.make_inputs3(cfg, 14)


def case3_wide():
    cfg = dict(dtype="f32", B=1, H=1, N=700, d=64, M0=16, C=8, P=4, P2=6, block=64,
               key_sigma=0.03, noise=0.05)
    return synth.make_inputs3(cfg, 15)


CASES3 = (case3_small, case3_wide)


def _run3(orc, inp, P=None, P2=None, sel=None, sel2=None):
    P = inp["P"] if P is None else P
    P2 = inp["P2"] if P2 is None else P2
    a, vs, ns, _ = orc.quantize3(inp["K"], inp["V"], inp["parents"], inp["children"], inp["grandchildren"])
    O, s1, s2, w1, w2 = orc.attention3(inp["Q"], inp["parents"], inp["children"], inp["grandchildren"],
                                        vs, ns, P, P2, inp["block"], inp["scale"], sel=sel, sel2=sel2)
    return a, vs, ns, O, s1, s2, w1, w2


def pin3_assign_brute(orc):
    """Depth-3 codes equal the full distance-table descent (Alg. 1, one level deeper)."""
    for mk in CASES3:
        inp = mk()
        a, _, _, _ = orc.quantize3(inp["K"], inp["V"], inp["parents"], inp["children"], inp["grandchildren"])
        ref = brute.assign_brute3(inp["K"], inp["parents"], inp["children"], inp["grandchildren"])
        assert (a == ref).all(), (mk.__name__, int((a != ref).sum()))
        M0, C = inp["M0"], inp["C"]
        assert (a >= M0 + M0 * C).any() and ((a >= M0) & (a < M0 + M0 * C)).any() and (a < M0).any()


def pin3_strict_ties(orc):
    """Depth-3 ties by hand (d = 2, one parent, C = 3): a key equally far from
    two grandchildren takes the first; a key whose best grandchild is exactly
    as far as its child stays at the child (the strict comparisons of
    Algorithm 1, one level down)."""
    par = np.array([[[0.0, 0.0]]])
    ch = np.array([[[[2.0, 0.0], [-2.0, 0.0], [0.0, 0.0]]]])
    gc = np.array([[[[[3.0, 1.0], [3.0, -1.0], [0.0, 0.0]],
                     [[-3.0, 1.0], [-3.0, -1.0], [0.0, 0.0]],
                     [[1.0, 0.0], [-1.0, 0.0], [0.0, 0.0]]]]])
    assert np.array_equal(gc.mean(3), ch) and np.array_equal(ch.mean(2), par)
    K = np.array([[3.2, 0.0],    # child 0 (1.44 < 10.24); grandchildren 0 and 1 tie at 1.04 -> g0
                  [3.0, 0.0],    # child 0 at 1; best grandchild also at 1: stays at child 0
                  [-3.2, 0.0],   # child 1, its grandchild 0
                  [0.0, 0.0],    # on the parent: no child strictly closer
                  [0.9, 0.0]])   # child 2 coincides with the parent, equally far: stays at the parent
    a, _, _, _ = orc.quantize3(K[None, None], np.ones((1, 1, 5, 2)), par, ch, gc)
    # codes: parent 0; children 1..3; grandchild (c, g) at 4 + 3 c + g
    assert a[0, 0].tolist() == [4, 1, 7, 0, 0], a


def pin3_aggregate(orc):
    """Depth-3 statistics (Eq. 3 at three levels) and their invariants."""
    for mk in CASES3:
        inp = mk()
        M0, C, N = inp["M0"], inp["C"], inp["N"]
        M1 = M0 * C
        a, vs, ns, _ = orc.quantize3(inp["K"], inp["V"], inp["parents"], inp["children"], inp["grandchildren"])
        vs_ref, ns_ref = brute.aggregate_brute3(a, inp["V"], M0, C)
        assert (ns == ns_ref).all()
        assert _rel(vs, vs_ref) < 1e-12
        assert (ns[..., :M0].sum(-1) == N).all()
        ch = ns[..., M0:M0 + M1].reshape(*ns.shape[:-1], M0, C).sum(-1)
        gc = ns[..., M0 + M1:].reshape(*ns.shape[:-1], M1, C).sum(-1)
        assert (ch <= ns[..., :M0]).all() and (gc <= ns[..., M0:M0 + M1]).all()
        assert (gc.sum(-1) == (a >= M0 + M1).sum(-1)).all()


def pin3_representative(orc):
    """Depth-3 output equals exact softmax attention over representative keys
    (the Sec. C identity applied at both levels), for several (P, P2)."""
    for mk in CASES3:
        inp = mk()
        M0, C = inp["M0"], inp["C"]
        for P, P2 in ((1, 1), (inp["P"], inp["P2"]), (M0, M0 * C), (inp["P"], 0)):
            a, vs, ns, O, s1, s2, _, _ = _run3(orc, inp, P=P, P2=P2)
            Y = brute.representative_attention3(inp["Q"], a, inp["V"], inp["parents"], inp["children"],
                                                inp["grandchildren"], s1, s2, inp["block"], inp["scale"])
            assert _rel(O, Y) < 1e-10, (mk.__name__, P, P2, _rel(O, Y))


def pin3_limits(orc):
    """P = 0 is flat VQ attention over the parents (Eq. 4); P2 = 0 is the
    depth-2 method on the same parent and child statistics."""
    inp = case3_small()
    M0, C = inp["M0"], inp["C"]
    a, vs, ns, O, _, _, _, _ = _run3(orc, inp, P=0, P2=0)
    Y = brute.flat_vq_attention(inp["Q"], inp["parents"], vs[..., :M0, :], ns[..., :M0], inp["scale"])
    assert _rel(O, Y) < 1e-10
    a, vs, ns, O, s1, _, _, _ = _run3(orc, inp, P2=0)
    k2 = M0 + M0 * C
    O2, s2d, _ = orc.attention(inp["Q"], inp["parents"], inp["children"], vs[..., :k2, :], ns[..., :k2],
                               inp["P"], inp["block"], inp["scale"])
    assert (s2d == s1).all()
    assert _rel(O, O2) < 1e-12


def pin3_exact_codebook(orc):
    """Keys placed on the grandchildren, every parent and every child refined:
    exact attention (Eq. 1).  Keys on the children with every parent refined:
    exact attention for any P2."""
    rng = np.random.default_rng(33)
    H, M0, C, d, N = 1, 6, 3, 8, 200
    par, ch, gc = synth.make_codebook3(rng, H, M0, C, d, sigma_c=0.4, sigma_g=0.1)
    par, ch, gc = par / 64.0, ch / 64.0, gc / 64.0
    Q = rng.standard_normal((1, H, N, d))
    V = rng.standard_normal((1, H, N, d))
    pick = rng.integers(0, M0 * C * C, N)
    K = gc[0].reshape(M0 * C * C, d)[pick][None, None]
    a, vs, ns, _ = orc.quantize3(K, V, par, ch, gc)
    assert (a >= M0 + M0 * C).all()
    O, _, _, _, _ = orc.attention3(Q, par, ch, gc, vs, ns, M0, M0 * C, 64, 0.5)
    assert _rel(O, brute.exact_attention(Q, K, V, 0.5)) < 1e-10
    K = ch[0].reshape(M0 * C, d)[rng.integers(0, M0 * C, N)][None, None]
    a, vs, ns, _ = orc.quantize3(K, V, par, ch, gc)
    assert ((a >= M0) & (a < M0 + M0 * C)).all()
    for P2 in (0, 2, M0 * C):
        O, _, _, _, _ = orc.attention3(Q, par, ch, gc, vs, ns, M0, P2, 64, 0.5)
        assert _rel(O, brute.exact_attention(Q, K, V, 0.5)) < 1e-10


def pin3_child_importance(orc):
    """The refined children's importance is the block sum of the softmax mass
    that attention over the depth-2 representatives puts on each child's
    keys; it never exceeds the block's rows; the second selection is the
    top-P2 of it, ties to the lower child code."""
    for mk in CASES3:
        inp = mk()
        a, vs, ns, O, s1, s2, w1, w2 = _run3(orc, inp)
        W = brute.child_mass3(inp["Q"], a, inp["parents"], inp["children"], inp["grandchildren"], s1,
                              inp["block"], inp["scale"])
        assert _rel(w2, W) < 1e-10
        N, blk = inp["N"], inp["block"]
        sizes = np.array([min(blk, N - k * blk) for k in range(w2.shape[2])], dtype=np.float64)
        assert (w2.sum(-1) <= sizes[None, None, :] * (1 + 1e-12)).all()
        C, M0 = inp["C"], inp["M0"]
        for idx in np.ndindex(*s2.shape[:3]):
            codes = (M0 + s1[idx][:, None] * C + np.arange(C)[None, :]).reshape(-1)
            order = np.lexsort((codes, -w2[idx]))[: inp["P2"]]
            assert s2[idx].tolist() == codes[order].tolist()
    # exact ties: zero queries, one key on every grandchild (equal counts per level)
    rng = np.random.default_rng(44)
    M0, C, d = 4, 3, 8
    par, ch, gc = synth.make_codebook3(rng, 1, M0, C, d, sigma_c=0.2, sigma_g=0.05)
    # parents pushed apart (offsets kept, so the means still hold exactly)
    big = 8 * par
    ch, gc = ch - par[:, :, None] + big[:, :, None], gc - par[:, :, None, None] + big[:, :, None, None]
    par, ch, gc = big / 64.0, ch / 64.0, gc / 64.0
    K = gc[0].reshape(M0 * C * C, d)[None, None]
    V = rng.standard_normal(K.shape)
    Q = np.zeros_like(K)
    a, vs, ns, _ = orc.quantize3(K, V, par, ch, gc)
    assert (a[0, 0] == M0 + M0 * C + np.arange(M0 * C * C)).all()  # every key on its grandchild
    _, s1, s2, _, w2 = orc.attention3(Q, par, ch, gc, vs, ns, 2, 3, 64, 1.0)
    assert s1[0, 0, 0].tolist() == [0, 1]
    assert np.all(w2[0, 0, 0] == w2[0, 0, 0, 0])
    assert s2[0, 0, 0].tolist() == [M0, M0 + 1, M0 + 2]


def pin3_zero_offsets(orc):
    """Grandchildren equal to their child: no key moves to a grandchild (the
    move needs a strictly smaller distance), and refining children changes
    nothing."""
    inp = dict(case3_small())
    gc = inp["grandchildren"].clone()
    gc[:] = inp["children"][..., None, :]
    inp["grandchildren"] = gc
    a, vs, ns, O, _, _, _, _ = _run3(orc, inp)
    M0, C = inp["M0"], inp["C"]
    assert (a < M0 + M0 * C).all() and (ns[..., M0 + M0 * C:] == 0).all()
    _, _, _, O0, _, _, _, _ = _run3(orc, inp, P2=0)
    assert _rel(O, O0) < 1e-12


ALL_PINS = [pin_hand_worked, pin_assign_brute, pin_aggregate, pin_aggregate_given_codes,
            pin_representative,
            pin_rescale_exercised, pin_flat_p0, pin_exact_codebook, pin_importance, pin_topp,
            pin_relabel, pin_key_permutation, pin_keys_on_codewords, pin_strict_ties,
            pin_masking, pin_counting, pin_tiled_importance, pin_codebook_update,
            pin_codebook_massless, pin3_assign_brute, pin3_strict_ties, pin3_aggregate, pin3_representative,
            pin3_limits, pin3_exact_codebook, pin3_child_importance, pin3_zero_offsets]

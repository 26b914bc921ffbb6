"""Generalised Hilbert ("Gilbert") token order (Sec. 4.2, Fig. 3) and the
tile diagnostics (Sec. H, Table 8): the C helper against the oracle's
restatement, the oracle against what the curve must satisfy, and the
diagnostics on the 28 x 28 grid."""
import numpy as np
import pytest

import adaptive_vector_quantized_b200 as avq
from adaptive_vector_quantized_b200 import order, synth
from oracle import curve

SIZES = [(w, h) for w in range(1, 33) for h in range(1, 33)] + [(28, 28), (30, 30), (100, 37), (37, 100),
                                                                 (255, 2), (2, 255), (1, 300), (256, 256)]


def _check_curve(o, W, H):
    o = np.asarray(o)
    assert o.shape == (W * H,)
    assert np.array_equal(np.sort(o), np.arange(W * H)), "every cell once"
    assert o[0] == 0, "starts at (0, 0)"
    x, y = o % W, o // W
    if W * H > 1:
        assert np.all(np.abs(np.diff(x)) + np.abs(np.diff(y)) == 1), "unit steps"
        end = (int(x[-1]), int(y[-1]))
        assert end in ((W - 1, 0), (0, H - 1)), "ends at the next corner of a side"


@pytest.mark.parametrize("W,H", SIZES)
def test_oracle_curve_is_a_unit_step_path(W, H):
    _check_curve(curve.gilbert_order(W, H), W, H)


@pytest.mark.parametrize("side", [1, 2, 4, 8, 16, 32, 64, 128])
def test_oracle_curve_is_hilbert_on_power_of_two_squares(side):
    assert np.array_equal(curve.gilbert_order(side, side), synth.hilbert_cells(side))


def test_library_curve_equals_oracle():
    for W, H in SIZES:
        assert np.array_equal(avq.avq_gilbert_order(W, H).numpy(), curve.gilbert_order(W, H)), (W, H)
    for bad in ((0, 4), (4, 0), (-1, 3)):
        with pytest.raises(avq.AVQError):
            avq.avq_gilbert_order(*bad)


def _mutant_no_reverse(out, W, x, y, u, la, v, lb):
    """Planted mistake: the near strip's last columns walked without turning
    the side direction around (the "U" does not close)."""
    ux, uy = u
    vx, vy = v
    if lb == 1 or la == 2 or la >= 2 * lb or lb == 2:
        return ORIG_WALK(out, W, x, y, u, la, v, lb)
    b = lb // 2
    if b % 2 == 1:
        b = b + 1 if b + 1 <= lb - 1 else b - 1
    a = la // 2
    _mutant_no_reverse(out, W, x, y, v, b, u, a)
    _mutant_no_reverse(out, W, x + b * vx, y + b * vy, u, la, v, lb - b)
    _mutant_no_reverse(out, W, x + (la - 1) * ux, y + (la - 1) * uy, v, b, (-ux, -uy), la - a)


def _mutant_odd_cut(out, W, x, y, u, la, v, lb):
    """Planted mistake: a long block cut in the middle even when that leaves
    an odd number of columns next to an even side."""
    ux, uy = u
    if lb != 1 and la != 2 and (la >= 2 * lb or lb == 2):
        a = la // 2
        _mutant_odd_cut(out, W, x, y, u, a, v, lb)
        _mutant_odd_cut(out, W, x + a * ux, y + a * uy, u, la - a, v, lb)
        return
    return ORIG_WALK(out, W, x, y, u, la, v, lb)


ORIG_WALK = curve._walk


@pytest.mark.parametrize("mutant", [_mutant_no_reverse, _mutant_odd_cut])
def test_pins_catch_planted_mistakes(monkeypatch, mutant):
    monkeypatch.setattr(curve, "_walk", mutant)
    caught = False
    for W, H in [(28, 28), (30, 30), (12, 6), (10, 4), (64, 64)]:
        try:
            o = curve.gilbert_order(W, H)
            _check_curve(o, W, H)
            if W == H and W & (W - 1) == 0:
                assert np.array_equal(o, synth.hilbert_cells(W))
        except (AssertionError, IndexError, ValueError, RecursionError):
            caught = True
    assert caught


@pytest.mark.parametrize("W,H", [(28, 28), (30, 30), (64, 64)])
@pytest.mark.parametrize("tile", [32, 64, 128])
def test_gilbert_tiles_are_compact(W, H, tile):
    g = order.tile_locality(order.grid_order(W, H, "gilbert"), W, H, tile)
    r = order.tile_locality(order.grid_order(W, H, "raster"), W, H, tile)
    q = order.tile_locality(order.grid_order(W, H, "random", np.random.default_rng(0)), W, H, tile)
    assert g["boundary"] < r["boundary"] < q["boundary"]
    assert g["boundary"] < 1.1  # about the perimeter of a square of the same area


def test_tile_locality_reference_values():
    # raster tiles of one full row of a 16 x 16 grid: 2 x 16 edges to other
    # tiles (first and last rows: 16), square reference 4 * 4
    r = order.tile_locality(np.arange(256), 16, 16, 16)
    assert r["bbox_fill"] == 1.0
    assert abs(r["boundary"] - np.mean([16] + [32] * 14 + [16]) / 16.0) < 1e-12


def test_selection_capture_definition():
    w = np.array([[[4.0, 3.0, 2.0, 1.0], [0.0, 0.0, 5.0, 5.0]]])
    assert abs(order.selection_capture(w, 1) - np.mean([0.4, 0.5])) < 1e-12
    assert abs(order.selection_capture(w, 4) - 1.0) < 1e-12


def test_capture_follows_the_order():
    """Queries that look at their own region: top-P parents hold more of a
    block's mass when its queries are a compact region (Gilbert) than a
    strip (raster), and much more than when they are scattered (random);
    with queries independent of the grid the order does not matter."""
    import oracle as orc_mod

    orc = orc_mod.default()
    caps = {}
    for g in (0.0, 1.0):
        for kind in ("gilbert", "raster", "random"):
            cfg = dict(dtype="f32", B=1, H=2, N=784, d=64, M0=16, C=4, P=4, block=64, keys="regions",
                       grid=(28, 28), key_sigma=0.1, noise=0.0, order=kind, sigma_c=0.3, q_coherent=g)
            inp = synth.make_inputs(cfg, 7)
            _, vs, n, _ = orc.quantize(inp["K"], inp["V"], inp["parents"], inp["children"])
            _, _, imp = orc.attention(inp["Q"], inp["parents"], inp["children"], vs, n, 4, 64, inp["scale"])
            caps[g, kind] = order.selection_capture(imp, 4)
    assert caps[1.0, "gilbert"] > caps[1.0, "raster"] > caps[1.0, "random"] + 0.1
    spread = [caps[0.0, k] for k in ("gilbert", "raster", "random")]
    assert max(spread) - min(spread) < 0.01

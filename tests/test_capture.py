"""Capture diagnostic of the large-codebook selection study (CPU): the
brute-force true attention mass per parent and the capture of a selection
(Sec. B, Table 5; Table 6's "capture")."""
import numpy as np

import oracle
from adaptive_vector_quantized_b200 import synth
from oracle import brute
from tests.table5_capture import capture_row


def _small():
    cfg = dict(dtype="bf16", B=1, H=2, N=600, d=32, M0=32, C=4, P=6, block=128, keys="tree",
               key_sigma=0.1, sigma_c=0.3, q_coherent=1.0)
    return synth.make_inputs(cfg, 77)


def test_mass_is_a_distribution_per_row():
    inp = _small()
    orc = oracle.default()
    assign, _, _, _ = orc.quantize(inp["K"], inp["V"], inp["parents"], inp["children"])
    mass = brute.parent_attention_mass(inp["Q"], inp["K"], assign, inp["M0"], inp["C"],
                                       inp["block"], inp["scale"])
    N, blk = inp["N"], inp["block"]
    sizes = np.array([min(blk, N - k * blk) for k in range(mass.shape[2])], dtype=np.float64)
    assert np.allclose(mass.sum(-1), sizes[None, None], rtol=1e-12)
    all_sel = np.broadcast_to(np.arange(inp["M0"]), mass.shape)
    assert abs(brute.top_p_capture(mass, all_sel, N, blk) - 1.0) < 1e-12


def test_exact_selection_captures_most():
    r = capture_row(_small(), tiles=(8, 16))
    for k, v in r.items():
        assert 0.0 < v <= r["exact"] + 1e-12, (k, v, r["exact"])

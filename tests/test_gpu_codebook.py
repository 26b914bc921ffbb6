"""Codebook update (Sec. A, Eqs. 11-12) on the GPU against the float64 oracle,
through the C ABI: EMA state to fp32 rounding, updated codebook to the
rounding of its dtype, and the parent = mean-of-children constraint."""
import numpy as np
import pytest
import torch

import adaptive_vector_quantized_b200 as avq
import oracle
from adaptive_vector_quantized_b200 import synth

pytestmark = pytest.mark.gpu

CASES = {
    "vit_h3_bf16": (synth.get_config("vit", B=2, H=3), 1001, 0.9, "random"),
    "vit_h3_bf16_empty_prior": (synth.get_config("vit", B=1, H=3), 1001, 0.5, "zero"),
    "tiny_f32": (synth.get_config("tiny"), 1000, 0.25, "random"),
}


@pytest.mark.parametrize("case", list(CASES))
def test_codebook_update(case):
    cfg, seed, lam, prior = CASES[case]
    inp = synth.make_inputs(cfg, seed)
    dev = "cuda"
    K = inp["K"].to(dev)
    par = inp["parents"].to(dev).contiguous()
    ch = inp["children"].to(dev).contiguous()
    # the keys' Eq. 3 statistics: avq_quantize with the keys as values
    assign, ksum, counts = avq.avq_quantize(K, K, par, ch)
    H, M0, C, d = inp["H"], inp["M0"], inp["C"], inp["d"]
    Mt = M0 * (1 + C)
    rng = np.random.default_rng(7)
    if prior == "random":
        S0 = rng.standard_normal((H, Mt, d)).astype(np.float32)
        N0 = rng.uniform(0.5, 4.0, (H, Mt)).astype(np.float32)
    else:
        S0 = np.zeros((H, Mt, d), np.float32)
        N0 = np.zeros((H, Mt), np.float32)
    S = torch.from_numpy(S0).to(dev)
    Nst = torch.from_numpy(N0).to(dev)
    p_in, c_in = par.clone(), ch.clone()
    avq.avq_codebook_update(ksum, counts, S, Nst, par, ch, lam)
    assert avq.last_kernels() == "codebook_update"
    avq.avq_check_device()
    torch.cuda.synchronize()
    rS, rN, rp, rc = oracle.default().codebook_update(ksum.cpu(), counts.cpu(), S0, N0, p_in.cpu(),
                                                      c_in.cpu(), lam)
    gS, gN = S.cpu().double().numpy(), Nst.cpu().double().numpy()
    assert np.allclose(gN, rN, rtol=1e-6, atol=1e-6)
    assert np.abs(gS - rS).max() <= 1e-5 * max(1.0, np.abs(rS).max())
    gp = par.cpu().double().numpy()
    gc = ch.cpu().double().numpy()
    # tolerance: fp32 arithmetic (means and projection), then the dtype's rounding
    rnd = 2.0 ** -8 if inp["dtype"] == "bf16" else 1e-5
    scale = max(1.0, np.abs(rp).max(), np.abs(rc).max())
    assert np.abs(gp - rp).max() <= rnd * scale, np.abs(gp - rp).max()
    assert np.abs(gc - rc).max() <= rnd * scale, np.abs(gc - rc).max()
    # Eq. 5 restored (to the dtype's rounding of C + 1 values)
    assert np.abs(gc.sum(2) - C * gp).max() <= (C + 1) * rnd * scale

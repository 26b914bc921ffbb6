"""avq_quantize_noalloc (stage 1 through the library's static scratch) against
avq_quantize (stage 1 through a caller workspace), both called through the C
ABI on the GPU.  Two calls of the no-alloc entry in a row, the second into
outputs filled with garbage, must both agree with the workspace call:
assignments and counts bit-exact (same kernels, same decisions), value sums
within the stage-1 tolerance of the summed magnitudes (the float additions
are atomic, so their order differs from call to call)."""
import numpy as np
import pytest
import torch

import adaptive_vector_quantized_b200 as avq
import oracle
from adaptive_vector_quantized_b200 import synth
from tests import parity
from tests.gpu_helpers import to_dev

pytestmark = pytest.mark.gpu


def _cfg(**kw):
    base = dict(dtype="bf16", B=1, H=2, N=1000, d=64, M0=32, C=8, P=8, block=128, keys="tree",
                key_sigma=0.1, sigma_c=0.3, two_pass=False)
    base.update(kw)
    return base


CASES = {
    "vit": (synth.get_config("vit"), 1001),
    "largecb_small": (synth.get_config("largecb", H=2, N=2048), 1003),
    "ragged_65": (_cfg(N=65, M0=16), 11),
    "c0": (_cfg(N=700, M0=16, C=0, P=0), 17),
    "f32_d128": (_cfg(dtype="f32", N=1500, d=128, M0=24, C=4), 16),
    "long": (synth.get_config("long"), 1002),
}


def _scratch_bytes(H, M0, C, d):
    Mt = M0 * (1 + C)
    r = lambda x: (x + 255) // 256 * 256
    return r(H * Mt * d * 2) + r(H * Mt * 4)


@pytest.mark.parametrize("case", list(CASES))
def test_noalloc_matches_workspace_call(case):
    cfg, seed = CASES[case]
    inp = synth.make_inputs(cfg, seed)
    d = to_dev(inp)
    ch = d["children"] if inp["C"] > 0 else None
    assert _scratch_bytes(inp["H"], inp["M0"], inp["C"], inp["d"]) <= 8 << 20

    a_ref, v_ref, n_ref = avq.avq_quantize(d["K"], d["V"], d["parents"], ch)
    k_ref = avq.last_kernels()
    avq.avq_check_device()

    results = []
    a1, v1, n1 = avq.avq_quantize_noalloc(d["K"], d["V"], d["parents"], ch)
    k1 = avq.last_kernels()
    avq.avq_check_device()
    results.append((a1.cpu().numpy(), v1.cpu().numpy(), n1.cpu().numpy()))
    # second call in a row, into outputs that hold garbage
    a2 = torch.full_like(a1, -7)
    v2 = torch.full_like(v1, float("nan"))
    n2 = torch.full_like(n1, 12345)
    avq.avq_quantize_noalloc(d["K"], d["V"], d["parents"], ch, assign=a2, vsum=v2, counts=n2)
    k2 = avq.last_kernels()
    avq.avq_check_device()
    torch.cuda.synchronize()
    results.append((a2.cpu().numpy(), v2.cpu().numpy(), n2.cpu().numpy()))

    # the same kernels as the workspace call (tensor-core path where it applies)
    assert k1 == k_ref and k2 == k_ref, (k_ref, k1, k2)
    if inp["dtype"] == "bf16":
        assert "assign_tc" in k1

    ra, rv, rn = a_ref.cpu().numpy(), v_ref.cpu().numpy(), n_ref.cpu().numpy()
    abs_vs, _ = oracle.default().aggregate(ra, np.abs(oracle._f64(inp["V"])), inp["M0"], inp["C"])
    for a, v, n in results:
        assert (a == ra).all(), "assignments differ from the workspace call"
        assert (n == rn).all(), "counts differ from the workspace call"
        err = np.abs(v.astype(np.float64) - rv.astype(np.float64))
        lim = parity.VSUM_TOL * abs_vs + 1e-6
        assert np.isfinite(v).all()
        assert (err <= lim).all(), float((err - lim).max())

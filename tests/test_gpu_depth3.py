"""The depth-3 tree on the GPU against the float64 oracle, through the C ABI
(needs a B200).  Same rules as the two-level parity tests: codes bit-exact
outside the near-tie band (at each of the three decisions), counts
bit-exact, value sums within the summed-magnitude bound, both selections
exact outside the importance tie band (the second one judged on the oracle
rerun with the GPU's parent selection), O within the dtype's tolerance of the
oracle rerun on the GPU's two selections."""
import numpy as np
import pytest
import torch

import adaptive_vector_quantized_b200 as avq
import oracle
from adaptive_vector_quantized_b200 import synth
from oracle import brute
from tests import parity

pytestmark = pytest.mark.gpu


def _cfg(**kw):
    base = dict(dtype="bf16", B=1, H=2, N=1000, d=64, M0=16, C=8, P=4, P2=6, block=128,
                key_sigma=0.03, sigma_c=0.3, sigma_g=0.1)
    base.update(kw)
    return base


CASES = {
    "bf16_ragged": (_cfg(), 61),
    "f32_d128_b64": (_cfg(dtype="f32", N=700, d=128, M0=8, C=4, P=3, P2=5, block=64), 62),
    "bf16_noise": (_cfg(N=1536, noise=0.1, P=5, P2=3), 63),
    "p2_zero": (_cfg(N=512, P2=0), 64),
    "p_zero": (_cfg(N=512, P=0, P2=0), 65),
    "c1": (_cfg(N=300, C=1, P=4, P2=2), 66),
    "all_children": (_cfg(N=400, M0=4, C=3, P=4, P2=12), 67),
    "bf16_d128": (_cfg(N=900, d=128, M0=32, P=6, P2=7), 68),
    "bf16_m48_full": (_cfg(N=700, M0=48, P=16, P2=16), 69),
    "bf16_p20": (_cfg(N=600, M0=32, P=20, P2=4), 70),
    "bf16_b64": (_cfg(N=500, block=64), 71),
    "bf16_b2": (_cfg(B=2, N=300, M0=32, P=5, P2=9), 72),
    "bf16_p1": (_cfg(N=400, P=1, P2=1), 73),
    "bf16_p2_all": (_cfg(N=500, M0=16, P=2, P2=16), 74),
    "bf16_sparse": (_cfg(N=40, M0=64, P=16, P2=16), 75),
}


def tc_route(inp):
    """Shapes whose stage 1 takes the tensor-core route by default: bf16,
    C = 8, the two-level codebook image within one CTA's shared memory."""
    return inp["dtype"] == "bf16" and inp["C"] == 8 and inp["M0"] <= 64


def tc_route2(inp, P, P2):
    """Shapes whose depth-3 attention takes the tensor-core kernel by default."""
    return (inp["dtype"] == "bf16" and inp["C"] == 8 and inp["block"] == 128 and inp["M0"] % 16 == 0
            and inp["M0"] <= 64 and P <= 16 and P2 <= 16)


def run_gpu3(inp, P=None, P2=None, path=None):
    P = inp["P"] if P is None else P
    P2 = inp["P2"] if P2 is None else P2
    d = {k: inp[k].cuda().contiguous() for k in ("Q", "K", "V", "parents", "children", "grandchildren")}
    old = avq.avq_set_path(avq.AVQ_PATH_AUTO if path is None else path)
    try:
        assign, vsum, counts = avq.avq_quantize3(d["K"], d["V"], d["parents"], d["children"],
                                                 d["grandchildren"])
        k1 = avq.last_kernels()
        O, sel, sel2, imp, imp2 = avq.avq_attention3(d["Q"], d["parents"], d["children"], d["grandchildren"],
                                                     vsum, counts, P, P2, inp["block"], inp["scale"],
                                                     importance=True)
        k2 = avq.last_kernels()
    finally:
        avq.avq_set_path(old)
    avq.avq_check_device()
    torch.cuda.synchronize()
    return dict(assign=assign.cpu().numpy(), vsum=vsum.cpu().numpy(), counts=counts.cpu().numpy(),
                O=O.cpu(), sel=sel.cpu().numpy(), sel2=sel2.cpu().numpy(), imp=imp.cpu().numpy(),
                imp2=imp2.cpu().numpy(), kernels=k1 + " " + k2)


def check3(inp, res, P=None, P2=None):
    orc = oracle.default()
    P = inp["P"] if P is None else P
    P2 = inp["P2"] if P2 is None else P2
    M0, C = inp["M0"], inp["C"]
    args = (inp["parents"], inp["children"], inp["grandchildren"])
    o_assign, _, _, _ = orc.quantize3(inp["K"], inp["V"], *args)
    ties = parity.check_assign3(res["assign"], o_assign, inp["K"], *args)
    ref_vs, ref_n = brute.aggregate_brute3(res["assign"], inp["V"], M0, C)
    abs_vs, _ = brute.aggregate_brute3(res["assign"], inp["V"].abs(), M0, C)
    parity.check_stats(res["vsum"], res["counts"], ref_vs, ref_n, abs_vs)
    # parents' importance and selection on the GPU's statistics
    _, _, _, o_imp, _ = orc.attention3(inp["Q"], *args, ref_vs, ref_n, P, P2, inp["block"], inp["scale"])
    rel = np.abs(res["imp"] - o_imp) / (np.abs(o_imp) + 1e-6)
    assert rel.max() <= 1e-4, rel.max()
    parity.check_sel(res["sel"], o_imp, P)
    # children's importance and the second selection on the GPU's parent selection
    _, _, _, _, o_imp2 = orc.attention3(inp["Q"], *args, ref_vs, ref_n, P, P2, inp["block"], inp["scale"],
                                        sel=res["sel"])
    if P * C > 0:
        g2 = res["imp2"][..., :P * C]
        rel2 = np.abs(g2 - o_imp2) / (np.abs(o_imp2) + 1e-6)
        assert rel2.max() <= 1e-4, rel2.max()
    if P2 > 0:
        # child codes -> candidate slots (the order of sel, C each)
        cand = M0 + res["sel"][..., :, None] * C + np.arange(C)
        cand = cand.reshape(*res["sel"].shape[:-1], P * C)
        slots = np.empty_like(res["sel2"])
        for idx in np.ndindex(*res["sel2"].shape[:-1]):
            lut = {int(c): u for u, c in enumerate(cand[idx])}
            slots[idx] = [lut[int(c)] for c in res["sel2"][idx]]
        parity.check_sel(slots, o_imp2, P2)
    O_ref, _, _, _, _ = orc.attention3(inp["Q"], *args, ref_vs, ref_n, P, P2, inp["block"], inp["scale"],
                                       sel=res["sel"] if P > 0 else None,
                                       sel2=res["sel2"] if P2 > 0 else None)
    err = parity.check_output(res["O"], O_ref, inp["V"], inp["dtype"])
    return dict(near_tie_keys=ties, O_rel_err=err)


@pytest.mark.parametrize("route", ["auto", "simt"])
@pytest.mark.parametrize("case", list(CASES))
def test_depth3_parity(case, route):
    cfg, seed = CASES[case]
    inp = synth.make_inputs3(cfg, seed)
    if route == "simt":
        res = run_gpu3(inp, path=avq.AVQ_PATH_SIMT)
        assert "assign3_simt" in res["kernels"] and "attention3_simt" in res["kernels"]
    else:
        res = run_gpu3(inp)
        if tc_route(inp):
            assert "assign_tc_wg" in res["kernels"] and "assign3_grandchildren" in res["kernels"]
        else:
            assert "assign3_simt" in res["kernels"]
        want = "attention3_tc" if tc_route2(inp, inp["P"], inp["P2"]) else "attention3_simt"
        assert want in res["kernels"], res["kernels"]
    M0, C = inp["M0"], inp["C"]
    a = res["assign"]
    if case not in ("c1", "bf16_sparse"):
        assert (a >= M0 + M0 * C).any() and (a < M0).any()  # every level is reached
    if case == "bf16_sparse":  # most parents and children hold no key
        assert (res["counts"][..., :M0] == 0).sum() > M0 // 2
    print(case, res["kernels"], check3(inp, res))


@pytest.mark.parametrize("route", ["auto", "simt"])
def test_depth3_workload_sampled_invariants(route):
    """The bench's depth-3 workload (B=1, H=8, N=16384, 64/16/16, C=8): full
    parity on two heads, invariants on all; the default (tensor-core) stage 1
    and the CUDA-core one."""
    cfg = synth.get_config("deep3")
    inp = synth.make_inputs3(cfg, synth.CONFIG_SEEDS["deep3"])
    res = run_gpu3(inp, path=avq.AVQ_PATH_SIMT if route == "simt" else None)
    assert ("assign_tc_wg" in res["kernels"]) == (route == "auto")
    assert ("attention3_tc" in res["kernels"]) == (route == "auto")
    N, M0, C = inp["N"], inp["M0"], inp["C"]
    M1 = M0 * C
    n = res["counts"]
    assert (n[..., :M0].sum(-1) == N).all()
    assert (n[..., M0:M0 + M1].sum(-1) == (res["assign"] >= M0).sum(-1)).all()
    assert (n[..., M0 + M1:].sum(-1) == (res["assign"] >= M0 + M1).sum(-1)).all()
    sizes = np.minimum(inp["block"], N - np.arange(res["imp"].shape[2]) * inp["block"])
    assert np.allclose(res["imp"].sum(-1), sizes[None, None, :], rtol=1e-4)
    sub = dict(inp)
    for k in ("Q", "K", "V"):
        sub[k] = inp[k][:, :2].contiguous()
    sub["parents"], sub["children"], sub["grandchildren"] = (inp[k][:2] for k in ("parents", "children",
                                                                                   "grandchildren"))
    sub["H"] = 2
    res2 = {k: (v[:, :2] if isinstance(v, np.ndarray) else v) for k, v in res.items()}
    res2["O"] = res["O"][:, :2]
    print("deep3", res["kernels"], check3(sub, res2))


def test_depth3_equals_depth2_when_p2_is_zero():
    """With P2 = 0 the depth-3 output equals the two-level output on the same
    parents, children and (parent and child) statistics, on the GPU."""
    cfg, seed = CASES["bf16_ragged"]
    inp = synth.make_inputs3(cfg, seed)
    res = run_gpu3(inp, P2=0)
    M0, C = inp["M0"], inp["C"]
    k2 = M0 + M0 * C
    vs = torch.from_numpy(np.ascontiguousarray(res["vsum"][:, :, :k2])).cuda()
    ns = torch.from_numpy(np.ascontiguousarray(res["counts"][:, :, :k2])).cuda()
    old = avq.avq_set_path(avq.AVQ_PATH_SIMT)
    try:
        O2, sel2d, _ = avq.avq_attention(inp["Q"].cuda(), inp["parents"].cuda(), inp["children"].cuda(), vs, ns,
                                         inp["P"], inp["block"], inp["scale"])
    finally:
        avq.avq_set_path(old)
    torch.cuda.synchronize()
    assert np.array_equal(sel2d.cpu().numpy(), res["sel"])
    diff = (O2.cpu().float() - res["O"].float()).abs().max().item()
    assert diff <= 2e-2 * float(inp["V"].float().abs().max())


def test_depth3_tc_route_refusals():
    """Forcing the tensor-core route on a depth-3 shape it does not cover
    (f32, or C != 8) is refused before any launch."""
    for name in ("f32_d128_b64", "all_children"):
        cfg, seed = CASES[name]
        inp = synth.make_inputs3(cfg, seed)
        d = {k: inp[k].cuda().contiguous() for k in ("K", "V", "parents", "children", "grandchildren")}
        old = avq.avq_set_path(avq.AVQ_PATH_TC)
        try:
            with pytest.raises(RuntimeError):
                avq.avq_quantize3(d["K"], d["V"], d["parents"], d["children"], d["grandchildren"])
        finally:
            avq.avq_set_path(old)
    avq.avq_check_device()


def test_depth3_tc_rescale_paths():
    """Children far above the parents' maximum and grandchildren far above the
    children's (logit gaps up to 64 against the reference-maximum margin of
    2^24): the tensor-core kernel's rescale branch at both levels, against
    the oracle."""
    H, M0, C, d, N = 1, 16, 8, 64, 512
    rng = np.random.default_rng(7)
    par = np.zeros((H, M0, d), dtype=np.float32)
    par[0, :, 2:] = np.rint(rng.standard_normal((M0, d - 2)) * 8) / 8
    steps = [4, -4, 3, -3, 2, -2, 1, -1]
    offc = np.zeros((C, d), dtype=np.float32)
    offc[:, 0] = steps
    ch = par[:, :, None, :] + offc[None, None]
    offg = np.zeros((C, d), dtype=np.float32)
    offg[:, 1] = steps
    gc = ch[:, :, :, None, :] + offg[None, None, None]
    assert np.array_equal(ch.mean(2), par) and np.array_equal(gc.mean(3), ch)
    pick_p = rng.integers(0, M0, N)
    pick_c = rng.integers(0, 2, N) * 2  # children 0 or 2: far along +e0
    pick_g = rng.integers(0, 2, N) * 2  # grandchildren 0 or 2: far along +e1
    K = gc[0][pick_p, pick_c, pick_g][None, None]
    Q = np.zeros((1, H, N, d), dtype=np.float32)
    Q[..., 0] = 16.0
    Q[..., 1] = 16.0
    Q[..., 2:] = np.rint(rng.standard_normal((N, d - 2)) * 4) / 16
    V = rng.standard_normal((1, H, N, d)).astype(np.float32)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16)  # noqa: E731
    inp = dict(Q=t(Q), K=t(K), V=t(V), parents=t(par), children=t(ch), grandchildren=t(gc), B=1, H=H, N=N,
               d=d, M0=M0, C=C, P=4, P2=6, block=128, scale=1.0, dtype="bf16", depth=3)
    res = run_gpu3(inp)
    assert "attention3_tc" in res["kernels"]
    assert (res["assign"] >= M0 + M0 * C).all()  # every key at a grandchild
    print("rescale3", res["kernels"], check3(inp, res))

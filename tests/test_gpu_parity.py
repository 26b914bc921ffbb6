"""CUDA path against the float64 oracle, through the C ABI (needs a B200).

Sizes are chosen so that the oracle finishes in seconds while still spanning
several tiles and a ragged tail; the full-size workloads are checked on
sampled query blocks plus full assignment/statistics checks.
"""
import numpy as np
import pytest
import torch

import adaptive_vector_quantized_b200 as avq
import oracle
from adaptive_vector_quantized_b200 import synth
from tests import gpu_helpers as gh
from tests import parity

pytestmark = pytest.mark.gpu

PATHS = {"simt": avq.AVQ_PATH_SIMT, "auto": avq.AVQ_PATH_AUTO}


def _cfg(**kw):
    base = dict(dtype="bf16", B=1, H=2, N=2048, d=64, M0=64, C=8, P=16, block=128,
                keys="tree", key_sigma=0.1, sigma_c=0.3, two_pass=False)
    base.update(kw)
    return base


CASES = {
    "tiny": (synth.get_config("tiny"), 1000),
    "vit_h3": (synth.get_config("vit", B=1, H=3), 1001),
    "vit_full": (synth.get_config("vit"), 1001),
    "largecb_small": (synth.get_config("largecb", H=2, N=2048), 1003),
    "ragged_1000_b64": (_cfg(N=1000, block=64, M0=32, P=8), 7),
    "ragged_1000_b128": (_cfg(N=1000, block=128, M0=32, P=8), 8),
    "ragged_d128": (_cfg(N=777, d=128, M0=48, C=4, P=5), 9),
    "n1": (_cfg(N=1, M0=16, P=4), 10),
    "n65": (_cfg(N=65, M0=16, P=4, block=64), 11),
    "m0_1": (_cfg(N=512, M0=1, P=1), 12),
    "c1": (_cfg(N=512, M0=16, C=1, P=4), 13),
    "p_eq_m0": (_cfg(N=1024, M0=16, P=16), 14),
    "p0": (_cfg(N=1024, M0=16, P=0), 15),
    "flat192": (synth.sweep_config(0, 4096, flat192=True), 1004),
    "f32_d128": (_cfg(dtype="f32", N=1500, d=128, M0=24, C=4, P=6, block=64), 16),
    "sweep_p4_random": (synth.sweep_config(4, 4096, "random"), 1004),
    "sweep_p64_hilbert": (synth.sweep_config(64, 4096, "hilbert"), 1004),
    # 28 x 28 patch grid along the generalised Hilbert curve (784 tokens: a
    # ragged last query block); the second with queries that look at their
    # own region, so that blocks select few, heavy parents
    "vit28": (synth.get_config("vit28"), 1005),
    "vit28_coherent_q": (synth.get_config("vit28", B=1, q_coherent=1.0), 1005),
    # 80 heads x 8 blocks (the last one partial) = 640 units: more units than
    # the persistent attention grid has CTAs, so CTAs walk two units each and
    # some of them end on a partial block; P = 13 pads the second chunk
    "multi_unit_ragged": (_cfg(H=80, N=1000, P=13), 17),
    # d = 128 with one parent tile: the one-tile attention kernel's two
    # 64-column halves (Q, O, codeword and value atoms), with the children in
    # shared memory (M0 = 32) or read from L2 (M0 = 64) in the assignment
    "d128_m64": (_cfg(H=3, N=1536, d=128, M0=64, P=16), 19),
    "d128_m32_ragged": (_cfg(H=2, N=1000, d=128, M0=32, P=5), 20),
    "d128_m48": (_cfg(H=2, N=777, d=128, M0=48, P=7), 21),
    "d128_m16": (_cfg(H=2, N=300, d=128, M0=16, P=3), 22),
    # two parent tiles at d = 64: the general attention kernel's two sweeps
    "m0_128_d64": (_cfg(H=2, N=1024, M0=128, P=16), 23),
}


@pytest.fixture(scope="module")
def inputs():
    cache = {}

    def get(name):
        if name not in cache:
            cfg, seed = CASES[name]
            cache[name] = synth.make_inputs(cfg, seed)
        return cache[name]

    return get


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("case", list(CASES))
def test_forward_parity(inputs, case, path):
    inp = inputs(case)
    res = gh.gpu_forward(inp, path=PATHS[path])
    diag = gh.check_forward(inp, res)
    print(case, path, res["kernels"], diag)


def _forward_tc_attention(inp, **kw):
    try:
        return gh.gpu_forward(inp, apath=avq.AVQ_PATH_TC, **kw)
    except avq.AVQError as e:
        if e.status == avq.AVQ_ERR_UNSUPPORTED:
            pytest.skip("no tensor-core attention kernel for this case")
        raise


@pytest.mark.parametrize("case", list(CASES))
def test_forward_parity_tc_both(inputs, case):
    """Both stages forced onto the tcgen05 kernels."""
    inp = inputs(case)
    try:
        res = gh.gpu_forward(inp, path=avq.AVQ_PATH_TC)
    except avq.AVQError as e:
        if e.status == avq.AVQ_ERR_UNSUPPORTED:
            pytest.skip("no tensor-core kernel for this case")
        raise
    assert "assign_tc" in res["kernels"] and "attention_tc" in res["kernels"]
    diag = gh.check_forward(inp, res)
    print(case, "tc-both", res["kernels"], diag)


@pytest.mark.parametrize("case", list(CASES))
def test_forward_parity_tc_attention(inputs, case):
    inp = inputs(case)
    res = _forward_tc_attention(inp)
    assert "attention_tc" in res["kernels"]
    diag = gh.check_forward(inp, res)
    print(case, "tc-attention", res["kernels"], diag)


def test_tc_attention_rescale_path():
    """Non-empty children whose logits exceed the parents' max by far more than
    the reference-max margin: the TMEM rescale branch must reproduce the oracle."""
    H, M0, C, d, N = 1, 16, 8, 64, 512
    rng = np.random.default_rng(5)
    par = np.zeros((H, M0, d), dtype=np.float32)
    par[0, :, 1:] = np.rint(rng.standard_normal((M0, d - 1)) * 8) / 8
    off = np.zeros((C, d), dtype=np.float32)
    off[:, 0] = [4, -4, 3, -3, 2, -2, 1, -1]
    ch = par[:, :, None, :] + off[None, None]
    assert np.array_equal(ch.mean(2), par)
    pick_p = rng.integers(0, M0, N)
    pick_c = rng.integers(0, 2, N) * 2  # children 0 or 2: far along +e0
    K = ch[0][pick_p, pick_c][None, None]
    Q = np.zeros((1, H, N, d), dtype=np.float32)
    Q[..., 0] = 16.0
    Q[..., 1:] = np.rint(rng.standard_normal((N, d - 1)) * 4) / 16
    V = rng.standard_normal((1, H, N, d)).astype(np.float32)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16)  # noqa: E731
    inp = dict(Q=t(Q), K=t(K), V=t(V), parents=t(par), children=t(ch), B=1, H=H, N=N, d=d,
               M0=M0, C=C, P=4, block=128, scale=1.0, dtype="bf16", two_pass=False)
    res = _forward_tc_attention(inp)
    diag = gh.check_forward(inp, res)
    print("rescale", res["kernels"], diag)


def test_tc_attention_far_below_children():
    """Non-empty children whose logits lie far below the maximum (2^x with x
    below -126 after the rescale, where the exponential evaluated on the FMA
    pipe is clamped), next to children far above it (the rescale branch): no
    NaN, and the oracle's output."""
    H, M0, C, d, N = 1, 16, 8, 64, 512
    rng = np.random.default_rng(6)
    par = np.zeros((H, M0, d), dtype=np.float32)
    par[0, :, 1:] = np.rint(rng.standard_normal((M0, d - 1)) * 8) / 8
    off = np.zeros((C, d), dtype=np.float32)
    off[:, 0] = [-6, -6, 2, 2, 2, 2, 2, 2]  # children 0 and 1 take the FMA-pipe exponential
    ch = par[:, :, None, :] + off[None, None]
    assert np.array_equal(ch.mean(2), par)
    pick_p = rng.integers(0, M0, N)
    pick_c = rng.integers(0, 2, N) * 2  # children 0 (far below) or 2 (far above)
    K = ch[0][pick_p, pick_c][None, None]
    Q = np.zeros((1, H, N, d), dtype=np.float32)
    Q[..., 0] = 16.0
    Q[..., 1:] = np.rint(rng.standard_normal((N, d - 1)) * 4) / 16
    V = rng.standard_normal((1, H, N, d)).astype(np.float32)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16)  # noqa: E731
    inp = dict(Q=t(Q), K=t(K), V=t(V), parents=t(par), children=t(ch), B=1, H=H, N=N, d=d,
               M0=M0, C=C, P=M0, block=128, scale=1.0, dtype="bf16", two_pass=False)
    res = _forward_tc_attention(inp)
    assert not torch.isnan(res["O"]).any()
    gh.check_forward(inp, res)


@pytest.mark.parametrize("P", [3, 13, 24, 40, 64])
def test_tc_attention_chunking(inputs, P):
    """Tensor-core attention with P not a multiple of 8 (a padded child slot)
    and with more than two chunks of 8 parents (staging buffers reused)."""
    inp = inputs("vit_h3")
    res = _forward_tc_attention(inp, P=P)
    assert "attention_tc" in res["kernels"]
    gh.check_forward(inp, res, P=P)


def test_tc_m0_48(inputs):
    """M0 = 48: a parent count that is not a power of two on both tensor-core stages."""
    cfg = _cfg(N=1000, M0=48, P=7)
    inp = synth.make_inputs(cfg, 18)
    res = gh.gpu_forward(inp, path=avq.AVQ_PATH_TC)
    assert "assign_tc" in res["kernels"] and "attention_tc" in res["kernels"]
    gh.check_forward(inp, res)


@pytest.mark.parametrize("P,block", [(0, 128), (1, 64), (8, 128), (64, 64)])
def test_vit_p_and_block_variants(inputs, P, block):
    inp = inputs("vit_h3")
    for path in PATHS.values():
        res = gh.gpu_forward(inp, P=P, block=block, path=path)
        gh.check_forward(inp, res, P=P, block=block)


def test_extrapolated_denominator(inputs):
    """Sec. B, Eqs. 13-14 on the tensor-core kernel: importance and selection
    against the oracle's tiled importance (tiles of 64 parents), O against the
    oracle rerun on the GPU's selection; the selection differs from the exact
    one somewhere, so the approximation is exercised."""
    inp = inputs("largecb_small")
    res = gh.gpu_forward(inp, two_pass=avq.AVQ_DENOM_EXTRAPOLATED, path=avq.AVQ_PATH_TC)
    assert "attention_tc " in res["kernels"] + " "
    gh.check_forward(inp, res, tile=64)
    exact = gh.gpu_forward(inp, two_pass=avq.AVQ_DENOM_TWO_PASS, path=avq.AVQ_PATH_TC)
    assert not np.array_equal(res["imp"], exact["imp"])


def test_two_pass_equals_single_pass(inputs):
    inp = inputs("largecb_small")
    a = gh.gpu_forward(inp, two_pass=True)
    b = gh.gpu_forward(inp, two_pass=False)
    gh.check_forward(inp, a)
    gh.check_forward(inp, b)
    assert np.array_equal(a["assign"], b["assign"])


def _sample_blocks(inp, n, seed):
    rng = np.random.default_rng(seed)
    nblk = (inp["N"] + inp["block"] - 1) // inp["block"]
    BH = inp["B"] * inp["H"]
    pick = rng.choice(BH * nblk, size=min(n, BH * nblk), replace=False)
    blocks = [(int(u // nblk), int(u % nblk)) for u in pick]
    blocks.append((BH - 1, nblk - 1))  # always include the last block
    return blocks


@pytest.mark.parametrize("name", ["long", "largecb"])
def test_full_size_sampled(name):
    cfg = synth.get_config(name)
    inp = synth.make_inputs(cfg, synth.CONFIG_SEEDS[name])
    res = gh.gpu_forward(inp)
    diag = gh.check_forward(inp, res, blocks=_sample_blocks(inp, 48, 5))
    # invariants that hold at any size
    N, M0 = inp["N"], inp["M0"]
    assert (res["counts"][..., :M0].sum(-1) == N).all()
    moved = (res["assign"] >= M0).sum(-1)
    assert (res["counts"][..., M0:].sum(-1) == moved).all()
    imp_sums = res["imp"].sum(-1)
    sizes = np.minimum(inp["block"], N - np.arange(imp_sums.shape[-1]) * inp["block"])
    assert np.allclose(imp_sums, sizes[None, None, :], rtol=1e-4)
    print(name, res["kernels"], diag)


def test_deterministic_mode(inputs):
    inp = inputs("vit_h3")
    dev = gh.to_dev(inp)
    a = gh.gpu_forward(inp, deterministic=True, dev=dev)
    b = gh.gpu_forward(inp, deterministic=True, dev=dev)
    c = gh.gpu_forward(inp, deterministic=False, dev=dev)
    assert np.array_equal(a["vsum"].view(np.uint32), b["vsum"].view(np.uint32))
    assert np.array_equal(a["counts"], c["counts"])
    assert np.array_equal(a["O"].view(torch.int16).numpy(), b["O"].view(torch.int16).numpy())
    gh.check_forward(inp, a)
    assert "det_" in a["kernels"]


@pytest.mark.parametrize("case", ["tiny", "multi_chunk"])
def test_deterministic_matches_fixed_order_sum(inputs, case):
    """The deterministic value sums are the plain sequential fp32 sums of each
    (parent, child) segment in key order, and parents add stay + children.
    That definition names no launch shape, so equality with it on a case of
    several sort chunks, heads and batches (N = 5000, d = 128) is what makes
    the result independent of the GPU's size."""
    if case == "tiny":
        inp = inputs("tiny")
    else:
        inp = synth.make_inputs(_cfg(B=2, H=2, N=5000, d=128, M0=32, P=8), 21)
    a = gh.gpu_forward(inp, deterministic=True)
    V = inp["V"].float().numpy().astype(np.float32)
    M0, C = inp["M0"], inp["C"]
    zero = np.zeros(V.shape[-1], dtype=np.float32)
    for b in range(inp["B"]):
        for h in range(inp["H"]):
            codes = a["assign"][b, h]
            seg = {}
            for j, code in enumerate(codes):
                key = int(code)
                seg[key] = np.float32(seg.get(key, zero) + V[b, h, j])
            for p in range(M0):
                tot = seg.get(p, zero)
                for c in range(C):
                    ch = seg.get(M0 + p * C + c, zero)
                    assert np.array_equal(a["vsum"][b, h, M0 + p * C + c], ch)
                    tot = np.float32(tot + ch)
                assert np.array_equal(a["vsum"][b, h, p], tot)


def test_permute_roundtrip_and_definition():
    torch.manual_seed(0)
    for rows, cols, dt in [(4096, 64, torch.bfloat16), (1000, 8, torch.float32), (7, 128, torch.bfloat16)]:
        X = torch.randn(3, rows, cols).to(dt).cuda()
        perm = torch.randperm(rows, dtype=torch.int64)
        idx = perm.to(torch.int32).cuda()
        Y = avq.avq_permute(X, idx)
        Z = avq.avq_permute(Y, idx, inverse=True)
        torch.cuda.synchronize()
        Xc = X.cpu().numpy() if dt == torch.float32 else X.cpu().view(torch.int16).numpy()
        Yc = Y.cpu().numpy() if dt == torch.float32 else Y.cpu().view(torch.int16).numpy()
        Zc = Z.cpu().numpy() if dt == torch.float32 else Z.cpu().view(torch.int16).numpy()
        assert np.array_equal(Yc, Xc[:, perm.numpy()])  # Y[b, i] = X[b, idx[i]]
        assert np.array_equal(Zc, Xc)
    side = 64
    order = avq.avq_hilbert_order(side).cuda()
    X = torch.arange(side * side * 8, dtype=torch.float32).reshape(1, side * side, 8).cuda()
    Y = avq.avq_permute(X, order)
    assert torch.equal(Y.cpu()[0, :, 0] / 8, order.cpu().float())
    # the 28 x 28 grid along the generalised Hilbert curve, and back
    order = avq.avq_gilbert_order(28, 28).cuda()
    X = torch.arange(784 * 8, dtype=torch.float32).reshape(1, 784, 8).cuda()
    Y = avq.avq_permute(X, order)
    Z = avq.avq_permute(Y, order, inverse=True)
    assert torch.equal(Y.cpu()[0, :, 0] / 8, order.cpu().float())
    assert torch.equal(Z.cpu(), X.cpu())


def test_permute_refuses_out_of_range_indices():
    """An index outside [0, rows) is not followed: its row is skipped and the
    bounds bit of the device error word is set (reported as AVQ_ERR_DEVICE and
    cleared by the check).  X and Y are views into larger buffers, so even a
    check that failed to skip would only touch mapped memory."""
    avq.avq_check_device()
    rows, cols, batch = 300, 64, 2
    big_x = torch.randn(batch, rows + 8, cols, dtype=torch.float32, device="cuda")
    X = big_x[:, :rows].contiguous()
    idx_h = torch.randperm(rows, dtype=torch.int64).to(torch.int32)
    bad_at = (17, 203)
    idx_h[bad_at[0]] = rows   # one past the end
    idx_h[bad_at[1]] = -1     # negative
    idx = idx_h.cuda()
    sentinel = -12345.0
    for inverse in (False, True):
        Y = torch.full_like(X, sentinel)
        avq.avq_permute(X, idx, inverse=inverse, Y=Y)
        with pytest.raises(avq.AVQError) as ei:
            avq.avq_check_device()
        assert ei.value.status == avq.AVQ_ERR_DEVICE
        avq.avq_check_device()  # the word was cleared
        Xc, Yc = X.cpu(), Y.cpu()
        ok = [i for i in range(rows) if i not in bad_at]
        for b in range(batch):
            for i in ok:
                j = int(idx_h[i])
                if inverse:
                    assert torch.equal(Yc[b, j], Xc[b, i])
                else:
                    assert torch.equal(Yc[b, i], Xc[b, j])
            if inverse:  # the destinations the bad entries would have named stay untouched
                missing = sorted(set(range(rows)) - {int(idx_h[i]) for i in ok})
                for j in missing:
                    assert bool((Yc[b, j] == sentinel).all())
            else:
                for i in bad_at:
                    assert bool((Yc[b, i] == sentinel).all())


def test_device_error_word_clean():
    avq.avq_check_device()


@pytest.mark.parametrize("M0,C", [(192, 0), (128, 8)])
def test_p0_without_importance_one_sweep(M0, C):
    """P = 0 and no importance output over several parent tiles: nothing
    depends on the importance denominator, so the kernel takes one sweep with
    a running maximum; O equals the oracle's (Eq. 4) and the two-sweep run's."""
    inp = synth.make_inputs(_cfg(N=1000, M0=M0, C=C, P=0), 31)
    d = gh.to_dev(inp)
    ch = d["children"] if C > 0 else None
    assign, vsum, counts = avq.avq_quantize(d["K"], d["V"], d["parents"], ch)
    O1, _, _ = avq.avq_attention(d["Q"], d["parents"], ch, vsum, counts, 0, inp["block"], inp["scale"])
    k = avq.last_kernels()
    O2, _, _ = avq.avq_attention(d["Q"], d["parents"], ch, vsum, counts, 0, inp["block"], inp["scale"],
                                 importance=True)
    avq.avq_check_device()
    torch.cuda.synchronize()
    assert "attention_tc" in k
    orc = oracle.default()
    ref_vs, ref_n = orc.aggregate(assign.cpu().numpy(), inp["V"], M0, C)
    O_ref, _, _ = orc.attention(inp["Q"], inp["parents"], inp["children"], ref_vs, ref_n, 0, inp["block"],
                                inp["scale"])
    parity.check_output(O1.cpu(), O_ref, inp["V"], inp["dtype"])
    parity.check_output(O2.cpu(), O_ref, inp["V"], inp["dtype"])

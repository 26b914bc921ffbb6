"""The C-ABI library loads, exports what include/avq.h declares, and rejects
bad arguments on the host before touching a GPU (CPU only)."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import adaptive_vector_quantized_b200 as avq
from adaptive_vector_quantized_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "avq.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(avq_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert "avq_quantize" in names and "avq_attention" in names and "avq_permute" in names
    L = avq.lib()
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", avq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(avq_\w+)$", out, flags=re.M))
    assert set(names) <= exported, set(names) - exported


def test_status_strings_and_version():
    assert avq.status_string(0) == "AVQ_OK"
    assert avq.status_string(6) == "AVQ_ERR_WORKSPACE"
    assert avq.status_string(99) == "AVQ_ERR_UNKNOWN"
    assert avq.avq_version() >= 100


def test_set_path():
    old = avq.avq_set_path(avq.AVQ_PATH_SIMT)
    assert old == avq.AVQ_PATH_AUTO
    assert avq.avq_set_path(avq.AVQ_PATH_AUTO) == avq.AVQ_PATH_SIMT
    with pytest.raises(ValueError):
        avq.avq_set_path(7)


def _q(dims, K=0x1000, V=0x2000, par=0x3000, ch=0x4000, a=0x5000, vs=0x6000, n=0x7000,
       dt=avq.AVQ_BF16, det=0, ws=None, wsb=0):
    L = avq.lib()
    d = None if dims is None else ctypes.byref(dims)
    return L.avq_quantize(d, dt, K, V, par, ch, a, vs, n, det, ws, wsb, None)


def _a(dims, P=4, block=128, scale=0.125, Q=0x1000, par=0x3000, ch=0x4000, vs=0x6000, n=0x7000,
       O=0x8000, sel=0x9000, imp=None, dt=avq.AVQ_BF16, two_pass=0):
    L = avq.lib()
    return L.avq_attention(ctypes.byref(dims), dt, Q, par, ch, vs, n, P, block, scale, two_pass, O,
                           sel, imp, None, 0, None)


def test_host_validation_rejects_before_launch():
    ok = avq.avq_dims(1, 2, 1024, 64, 16, 4)
    E = avq
    assert _q(None) == E.AVQ_ERR_INVALID_ARG
    assert _q(ok, dt=5) == E.AVQ_ERR_INVALID_ARG
    assert _q(avq.avq_dims(1, 2, 0, 64, 16, 4)) == E.AVQ_ERR_INVALID_ARG
    assert _q(avq.avq_dims(1, 2, 64, 96, 16, 4)) == E.AVQ_ERR_UNSUPPORTED
    assert _q(avq.avq_dims(1, 2, 64, 64, 300, 4)) == E.AVQ_ERR_UNSUPPORTED
    assert _q(avq.avq_dims(1, 2, 64, 64, 16, 9)) == E.AVQ_ERR_UNSUPPORTED
    assert _q(avq.avq_dims(2, 32768, 1, 64, 16, 4)) == E.AVQ_ERR_UNSUPPORTED  # B*H above 65535
    assert "65535" in avq.last_error()
    assert _q(avq.avq_dims(1, 1024, 1 << 21, 64, 16, 4)) == E.AVQ_ERR_UNSUPPORTED  # B*H*N >= 2^31
    assert _q(ok, K=None) == E.AVQ_ERR_INVALID_ARG
    assert "K is NULL" in avq.last_error()
    assert _q(ok, V=0x2004) == E.AVQ_ERR_INVALID_ARG
    assert "16-byte" in avq.last_error()
    assert _q(ok, ch=None) == E.AVQ_ERR_INVALID_ARG
    assert _q(ok, det=1) == E.AVQ_ERR_WORKSPACE
    assert _q(ok, det=1, ws=0x10010, wsb=1 << 30) == E.AVQ_ERR_INVALID_ARG  # not 256-aligned
    assert _a(ok, P=17) == E.AVQ_ERR_INVALID_ARG
    assert _a(ok, P=-1) == E.AVQ_ERR_INVALID_ARG
    assert _a(ok, block=32) == E.AVQ_ERR_UNSUPPORTED
    assert _a(ok, scale=0.0) == E.AVQ_ERR_INVALID_ARG
    assert _a(ok, scale=float("inf")) == E.AVQ_ERR_INVALID_ARG
    assert _a(ok, sel=None) == E.AVQ_ERR_INVALID_ARG
    assert _a(ok, O=None) == E.AVQ_ERR_INVALID_ARG
    assert _a(ok, imp=0x123) == E.AVQ_ERR_INVALID_ARG
    L = avq.lib()
    assert L.avq_permute(0x1000, 0x2000, 0x3000, 1, 10, 24, 0, None) == E.AVQ_ERR_INVALID_ARG
    assert L.avq_permute(0x1000, 0x2000, 0x1040, 1, 10, 16, 0, None) == E.AVQ_ERR_INVALID_ARG  # overlap
    assert L.avq_permute(0x1000, None, 0x90000, 1, 10, 16, 0, None) == E.AVQ_ERR_INVALID_ARG


def test_workspace_sizes():
    d = avq.avq_dims(1, 16, 65536, 64, 64, 8)
    assert avq.avq_workspace_size(d, avq.AVQ_BF16, deterministic=True) > 0
    assert avq.avq_workspace_size(None if False else d, avq.AVQ_F32, deterministic=False) >= 0


def test_hilbert_order_matches_textbook_curve():
    for side in (1, 2, 8, 64, 256):
        got = avq.avq_hilbert_order(side).numpy()
        assert np.array_equal(got, synth.hilbert_cells(side))
    with pytest.raises(avq.AVQError):
        avq.avq_hilbert_order(12)


def test_noalloc_quantize_host_checks():
    """The no-alloc stage-1 entry rejects, before any launch, a codebook whose
    tensor-core image exceeds its static scratch, and bad pointers."""
    L = avq.lib()
    big = avq.avq_dims(1, 64, 1024, 128, 256, 8)  # 64 * 2304 * 128 * 2 bytes > 8 MiB
    st = L.avq_quantize_noalloc(ctypes.byref(big), avq.AVQ_BF16, 0x1000, 0x2000, 0x3000, 0x4000,
                                0x5000, 0x6000, 0x7000, None)
    assert st == 6, avq.last_error()
    assert "static scratch" in avq.last_error()
    ok = avq.avq_dims(1, 16, 1024, 64, 64, 8)
    st = L.avq_quantize_noalloc(ctypes.byref(ok), avq.AVQ_BF16, None, 0x2000, 0x3000, 0x4000,
                                0x5000, 0x6000, 0x7000, None)
    assert st == 1 and "K is NULL" in avq.last_error()
    st = L.avq_quantize_noalloc(ctypes.byref(ok), avq.AVQ_BF16, 0x1008, 0x2000, 0x3000, 0x4000,
                                0x5000, 0x6000, 0x7000, None)
    assert st == 1 and "aligned" in avq.last_error()
    st = L.avq_quantize_noalloc(None, avq.AVQ_BF16, 0x1000, 0x2000, 0x3000, 0x4000, 0x5000,
                                0x6000, 0x7000, None)
    assert st == 1


def test_denominator_modes_host_checks():
    """two_pass outside {0, 1, 2} is an argument error; the extrapolated
    denominator over several parent tiles needs the tensor-core kernel."""
    E = avq
    big = avq.avq_dims(1, 2, 1024, 64, 128, 8)
    assert _a(big, two_pass=3) == E.AVQ_ERR_INVALID_ARG
    assert _a(big, two_pass=-1) == E.AVQ_ERR_INVALID_ARG
    old = avq.avq_set_path(avq.AVQ_PATH_SIMT)
    try:
        assert _a(big, two_pass=E.AVQ_DENOM_EXTRAPOLATED) == E.AVQ_ERR_UNSUPPORTED
        assert "tensor-core" in avq.last_error()
    finally:
        avq.avq_set_path(old)


def test_codebook_update_host_checks():
    """lambda outside [0, 1] and missing buffers are rejected before launch."""
    L = avq.lib()
    d = avq.avq_dims(1, 2, 1, 64, 16, 8)
    args = (0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None)
    assert L.avq_codebook_update(ctypes.byref(d), avq.AVQ_BF16, 1.5, *args) == avq.AVQ_ERR_INVALID_ARG
    assert L.avq_codebook_update(ctypes.byref(d), avq.AVQ_BF16, -0.1, *args) == avq.AVQ_ERR_INVALID_ARG
    assert L.avq_codebook_update(ctypes.byref(d), avq.AVQ_BF16, 0.5, None, *args[1:]) == avq.AVQ_ERR_INVALID_ARG
    assert "ksum" in avq.last_error()
    assert L.avq_codebook_update(None, avq.AVQ_BF16, 0.5, *args) == avq.AVQ_ERR_INVALID_ARG


def test_wait_selftest_host_checks():
    """The bounded-wait self-test rejects an out-of-range limit before any launch."""
    L = avq.lib()
    for bad in (0, -5, 1000001):
        assert L.avq_selftest_wait(bad, None) == avq.AVQ_ERR_INVALID_ARG


def test_exp2_selftest_host_checks():
    """The exp2 self-test rejects null pointers, odd or out-of-range lengths and
    misaligned pointers before any launch (no pointer is dereferenced)."""
    L = avq.lib()
    ok = ctypes.c_void_p(0x10000)
    assert L.avq_selftest_exp2(None, ok, 2, None) == avq.AVQ_ERR_INVALID_ARG
    assert L.avq_selftest_exp2(ok, None, 2, None) == avq.AVQ_ERR_INVALID_ARG
    for bad_n in (3, -2, (1 << 30) + 2):
        assert L.avq_selftest_exp2(ok, ok, bad_n, None) == avq.AVQ_ERR_INVALID_ARG
    assert L.avq_selftest_exp2(ctypes.c_void_p(0x10004), ok, 2, None) == avq.AVQ_ERR_INVALID_ARG


def test_fault_injection_before_launch(monkeypatch):
    """AVQ_FAULT makes the named entry points fail after their argument checks
    and before any launch (host only: nothing reaches a GPU)."""
    import ctypes

    L = avq.lib()
    fake = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced
    d = avq.avq_dims(1, 2, 256, 64, 16, 8)
    calls = {
        "quantize": lambda: L.avq_quantize(ctypes.byref(d), avq.AVQ_BF16, fake, fake, fake, fake, fake,
                                           fake, fake, 0, fake, ctypes.c_size_t(1 << 40), None),
        "attention": lambda: L.avq_attention(ctypes.byref(d), avq.AVQ_BF16, fake, fake, fake, fake, fake,
                                             4, 128, ctypes.c_float(0.125), 0, fake, fake, None, fake,
                                             ctypes.c_size_t(1 << 40), None),
        "codebook_update": lambda: L.avq_codebook_update(ctypes.byref(d), avq.AVQ_BF16, ctypes.c_float(0.9),
                                                         fake, fake, fake, fake, fake, fake, None),
        "permute": lambda: L.avq_permute(fake, fake, ctypes.c_void_p(0x20000000), 1, 64, 128, 0, None),
        "quantize3": lambda: L.avq_quantize3(ctypes.byref(d), avq.AVQ_BF16, fake, fake, fake, fake, fake,
                                             fake, fake, fake, None),
        "attention3": lambda: L.avq_attention3(ctypes.byref(d), avq.AVQ_BF16, fake, fake, fake, fake, fake,
                                               fake, 4, 8, 128, ctypes.c_float(0.125), fake, fake, fake,
                                               None, None, None),
    }
    for entry, call in calls.items():
        monkeypatch.setenv("AVQ_FAULT", entry)
        assert call() == avq.AVQ_ERR_CUDA, entry
        assert "injected" in avq.last_error()
    monkeypatch.setenv("AVQ_FAULT", "all")
    for entry, call in calls.items():
        assert call() == avq.AVQ_ERR_CUDA, entry
    # argument checks still come first
    monkeypatch.setenv("AVQ_FAULT", "all")
    assert L.avq_permute(None, fake, fake, 1, 64, 128, 0, None) == avq.AVQ_ERR_INVALID_ARG


def test_depth3_host_checks():
    """The depth-3 entry points reject bad arguments before any launch."""
    L = avq.lib()
    fake = ctypes.c_void_p(0x10000)
    d = avq.avq_dims(1, 2, 256, 64, 16, 8)
    d0 = avq.avq_dims(1, 2, 256, 64, 16, 0)
    q3 = lambda dims, gc=fake: L.avq_quantize3(ctypes.byref(dims), avq.AVQ_BF16, fake, fake, fake, fake, gc,  # noqa: E731
                                                fake, fake, fake, None)
    assert q3(d0) == avq.AVQ_ERR_INVALID_ARG and "C >= 1" in avq.last_error()
    assert q3(d, None) == avq.AVQ_ERR_INVALID_ARG and "grandchildren" in avq.last_error()
    assert q3(d, ctypes.c_void_p(0x10004)) == avq.AVQ_ERR_INVALID_ARG

    def a3(P, P2, block=128, sel2=fake):
        return L.avq_attention3(ctypes.byref(d), avq.AVQ_BF16, fake, fake, fake, fake, fake, fake, P, P2,
                                block, ctypes.c_float(0.125), fake, fake, sel2, None, None, None)
    assert a3(17, 0) == avq.AVQ_ERR_INVALID_ARG            # P > M0
    assert a3(4, 33) == avq.AVQ_ERR_INVALID_ARG            # P2 > P*C
    assert a3(4, -1) == avq.AVQ_ERR_INVALID_ARG
    assert a3(4, 4, block=96) == avq.AVQ_ERR_UNSUPPORTED
    assert a3(4, 4, sel2=None) == avq.AVQ_ERR_INVALID_ARG and "sel2" in avq.last_error()
    old = avq.avq_set_path(avq.AVQ_PATH_TC)
    try:
        # the tensor-core kernels: attention with block 128 and P, P2 <= 16;
        # the assignment with C == 8 and bf16
        assert a3(4, 4, block=64) == avq.AVQ_ERR_UNSUPPORTED
        assert a3(4, 20) == avq.AVQ_ERR_UNSUPPORTED
        assert q3(avq.avq_dims(1, 2, 256, 64, 16, 4)) == avq.AVQ_ERR_UNSUPPORTED
        assert L.avq_quantize3(ctypes.byref(d), avq.AVQ_F32, fake, fake, fake, fake, fake, fake, fake, fake,
                               None) == avq.AVQ_ERR_UNSUPPORTED
    finally:
        avq.avq_set_path(old)

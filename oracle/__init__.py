"""Float64 CPU oracle for AVQ-Attention (test infrastructure only).

Only the tests, `__graft_entry__.smoke()` and the benchmark's CPU-baseline leg
(and its `--impl reference` arm) may import this package.  The product path
(the `adaptive_vector_quantized_b200` package and its CUDA library) never
imports, links or runs anything here, and this package imports nothing from
the product.

`avq_oracle.c` is the oracle proper: Algorithm 1 (VQ Precompute, Sec. 4.2)
and Algorithm 2 (Flash AVQ-Attention, Sec. 4.3) of "AVQ-Attention: Adaptive
Vector-Quantized Attention", step by step in float64.  `brute.py` holds
independently written closed forms used to pin it (representative-key
softmax of Sec. C, flat VQ attention of Eq. 4, exact attention of Eq. 1).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "avq_oracle.c")
LIB = os.path.join(HERE, "libavq_oracle.so")
_lock = threading.Lock()


def build(src: str = SRC, out: str = LIB, force: bool = False) -> str:
    """Compile the C oracle with gcc (-O2, OpenMP) into a shared library."""
    with _lock:
        if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
            return out
        tmp = out + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", src, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
        return out


_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)
_I64 = ctypes.POINTER(ctypes.c_int64)


def _p(a, t):
    return None if a is None else a.ctypes.data_as(t)


def _f64(a) -> np.ndarray:
    """Exact float64 copy of a numpy array or a CPU torch tensor (bf16/fp32 widen exactly)."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu")
        import torch  # local: only for dtype conversion of CPU tensors

        a = a.to(torch.float64).numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


class Oracle:
    """ctypes front end of one compiled oracle library."""

    def __init__(self, lib_path: str | None = None):
        self.path = lib_path or build()
        lib = ctypes.CDLL(self.path)
        lib.avq_oracle_quantize.argtypes = [ctypes.c_int] * 6 + [_D, _D, _D, _D, _I32, _D, _I64, _D]
        lib.avq_oracle_quantize.restype = None
        lib.avq_oracle_aggregate.argtypes = [ctypes.c_int] * 5 + [_I32, _D, _D, _I64]
        lib.avq_oracle_aggregate.restype = None
        lib.avq_oracle_attention.argtypes = ([ctypes.c_int] * 8 + [ctypes.c_double, _D, _D, _D, _D, _D,
                                             _I32, _I32, ctypes.c_int, _D, _I32, _D])
        lib.avq_oracle_attention.restype = None
        lib.avq_oracle_attention_tiled.argtypes = lib.avq_oracle_attention.argtypes + [ctypes.c_int]
        lib.avq_oracle_attention_tiled.restype = None
        lib.avq_oracle_codebook_update.argtypes = [ctypes.c_int] * 5 + [ctypes.c_double] + [_D] * 8
        lib.avq_oracle_codebook_update.restype = None
        lib.avq_oracle_quantize3.argtypes = [ctypes.c_int] * 6 + [_D] * 5 + [_I32, _D, _I64, _D]
        lib.avq_oracle_quantize3.restype = None
        lib.avq_oracle_attention3.argtypes = ([ctypes.c_int] * 9 + [ctypes.c_double] + [_D] * 6
                                              + [_I32, _I32, _D, _I32, _I32, _D, _D])
        lib.avq_oracle_attention3.restype = None
        lib.avq_oracle_num_threads.restype = ctypes.c_int
        lib.avq_oracle_set_threads.argtypes = [ctypes.c_int]
        lib.avq_oracle_set_threads.restype = None
        self.lib = lib

    def num_threads(self) -> int:
        return int(self.lib.avq_oracle_num_threads())

    def set_threads(self, n: int) -> None:
        """Threads of the oracle's OpenMP loops (a launcher may have set 1)."""
        self.lib.avq_oracle_set_threads(int(n))

    # ---- Algorithm 1 ---------------------------------------------------
    def quantize(self, K, V, parents, children):
        """K, V [B,H,N,d]; parents [H,M0,d]; children [H,M0,C,d].
        Returns assign [B,H,N] int32, vsum [B,H,Mt,d] f64, counts [B,H,Mt] int64,
        dec [B,H,N,4] (best/second parent distance, best/second child distance)."""
        K, V, parents, children = map(_f64, (K, V, parents, children))
        B, H, N, d = K.shape
        M0 = parents.shape[1]
        C = children.shape[2]
        Mt = M0 * (1 + C)
        assign = np.empty((B, H, N), dtype=np.int32)
        vsum = np.empty((B, H, Mt, d), dtype=np.float64)
        counts = np.empty((B, H, Mt), dtype=np.int64)
        dec = np.empty((B, H, N, 4), dtype=np.float64)
        self.lib.avq_oracle_quantize(B * H, H, N, d, M0, C, _p(K, _D), _p(V, _D),
                                     _p(parents, _D), _p(children, _D), _p(assign, _I32),
                                     _p(vsum, _D), _p(counts, _I64), _p(dec, _D))
        return assign, vsum, counts, dec

    def aggregate(self, assign, V, M0: int, C: int):
        """Statistics (the aggregation of Algorithm 1) for given final codes."""
        V = _f64(V)
        B, H, N, d = V.shape
        assign = np.ascontiguousarray(np.asarray(assign), dtype=np.int32)
        Mt = M0 * (1 + C)
        vsum = np.empty((B, H, Mt, d), dtype=np.float64)
        counts = np.empty((B, H, Mt), dtype=np.int64)
        self.lib.avq_oracle_aggregate(B * H, N, d, M0, C, _p(assign, _I32), _p(V, _D),
                                      _p(vsum, _D), _p(counts, _I64))
        return vsum, counts

    # ---- Algorithm 2 ---------------------------------------------------
    def attention(self, Q, parents, children, vsum, counts, P: int, block: int, scale: float,
                  sel=None, blocks=None, tile: int = 0):
        """Q [B,H,N,d]; vsum [B,H,Mt,d]; counts [B,H,Mt].  `sel` [B,H,nblk,P]
        overrides the top-P selection; `blocks` (list of (bh, block)) limits the
        work to those query blocks (other rows of O stay NaN).  `tile` > 0 uses
        the tiled importance with the count-extrapolated denominator (Sec. B,
        Eqs. 13-14) over parent tiles of that many codes.
        Returns O [B,H,N,d], sel [B,H,nblk,P] int32, importance [B,H,nblk,M0]."""
        Q, parents, children, vsum = map(_f64, (Q, parents, children, vsum))
        counts = _f64(counts)
        B, H, N, d = Q.shape
        M0 = parents.shape[1]
        C = children.shape[2]
        nblk = (N + block - 1) // block
        O = np.full((B, H, N, d), np.nan)
        sel_out = np.full((B, H, nblk, max(P, 0)), -1, dtype=np.int32)
        imp = np.full((B, H, nblk, M0), np.nan)
        sel_in = None
        if sel is not None:
            sel_in = np.ascontiguousarray(np.asarray(sel), dtype=np.int32).reshape(B, H, nblk, P)
        blk = None
        nlist = 0
        if blocks is not None:
            blk = np.ascontiguousarray(np.asarray(blocks, dtype=np.int32).reshape(-1, 2))
            nlist = blk.shape[0]
        self.lib.avq_oracle_attention_tiled(B * H, H, N, d, M0, C, P, block, float(scale),
                                            _p(Q, _D), _p(parents, _D), _p(children, _D),
                                            _p(vsum, _D), _p(counts, _D), _p(sel_in, _I32),
                                            _p(blk, _I32), nlist, _p(O, _D), _p(sel_out, _I32),
                                            _p(imp, _D), int(tile))
        return O, sel_out, imp


    # ---- depth-3 tree (Sec. 6, "deeper hierarchies") ------------------------
    def quantize3(self, K, V, parents, children, grandchildren):
        """Algorithm 1 one level deeper.  grandchildren [H,M0,C,C,d].  Returns
        assign [B,H,N] (codes: parents, then M0*C children, then M0*C*C
        grandchildren), vsum [B,H,Mt3,d], counts [B,H,Mt3], dec [B,H,N,6]."""
        K, V, parents, children, grandchildren = map(_f64, (K, V, parents, children, grandchildren))
        B, H, N, d = K.shape
        M0 = parents.shape[1]
        C = children.shape[2]
        Mt = M0 + M0 * C + M0 * C * C
        assign = np.empty((B, H, N), dtype=np.int32)
        vsum = np.empty((B, H, Mt, d), dtype=np.float64)
        counts = np.empty((B, H, Mt), dtype=np.int64)
        dec = np.empty((B, H, N, 6), dtype=np.float64)
        self.lib.avq_oracle_quantize3(B * H, H, N, d, M0, C, _p(K, _D), _p(V, _D), _p(parents, _D),
                                      _p(children, _D), _p(grandchildren, _D), _p(assign, _I32),
                                      _p(vsum, _D), _p(counts, _I64), _p(dec, _D))
        return assign, vsum, counts, dec

    def attention3(self, Q, parents, children, grandchildren, vsum, counts, P: int, P2: int,
                   block: int, scale: float, sel=None, sel2=None):
        """Algorithm 2 one level deeper.  Returns O [B,H,N,d], sel [B,H,nblk,P]
        (parents), sel2 [B,H,nblk,P2] (child codes), importance [B,H,nblk,M0],
        child importance [B,H,nblk,P*C] (candidates in the order of sel)."""
        Q, parents, children, grandchildren, vsum = map(_f64, (Q, parents, children, grandchildren, vsum))
        counts = _f64(counts)
        B, H, N, d = Q.shape
        M0 = parents.shape[1]
        C = children.shape[2]
        nblk = (N + block - 1) // block
        O = np.full((B, H, N, d), np.nan)
        sel_out = np.full((B, H, nblk, max(P, 0)), -1, dtype=np.int32)
        sel2_out = np.full((B, H, nblk, max(P2, 0)), -1, dtype=np.int32)
        imp = np.full((B, H, nblk, M0), np.nan)
        imp2 = np.full((B, H, nblk, max(P * C, 0)), np.nan)
        si = None if sel is None else np.ascontiguousarray(np.asarray(sel), dtype=np.int32)
        si2 = None if sel2 is None else np.ascontiguousarray(np.asarray(sel2), dtype=np.int32)
        self.lib.avq_oracle_attention3(B * H, H, N, d, M0, C, P, P2, block, float(scale), _p(Q, _D),
                                       _p(parents, _D), _p(children, _D), _p(grandchildren, _D),
                                       _p(vsum, _D), _p(counts, _D), _p(si, _I32), _p(si2, _I32),
                                       _p(O, _D), _p(sel_out, _I32), _p(sel2_out, _I32), _p(imp, _D),
                                       _p(imp2, _D))
        return O, sel_out, sel2_out, imp, imp2

    # ---- Sec. A: codebook update -----------------------------------------
    def codebook_update(self, ksum, counts, S, Nst, parents, children, lam: float):
        """ksum [B,H,Mt,d], counts [B,H,Mt]: Eq. 3 statistics of the keys;
        S [H,Mt,d], Nst [H,Mt]: EMA state; parents [H,M0,d], children
        [H,M0,C,d]: current codebook.  Returns (S', N', parents', children')."""
        ksum, counts, parents, children = map(_f64, (ksum, counts, parents, children))
        S = _f64(S).copy()
        Nst = _f64(Nst).copy()
        B, H, Mt, d = ksum.shape
        M0 = parents.shape[1]
        C = children.shape[2]
        po = np.empty_like(parents)
        co = np.empty_like(children)
        self.lib.avq_oracle_codebook_update(B, H, d, M0, C, float(lam), _p(ksum, _D), _p(counts, _D),
                                            _p(S, _D), _p(Nst, _D), _p(parents, _D),
                                            _p(children, _D), _p(po, _D), _p(co, _D))
        return S, Nst, po, co


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default

"""B200-native forward pass of AVQ-Attention (Adaptive Vector-Quantized Attention).

Thin Python binding over the C ABI of ``libavq.so`` (declared in
``include/avq.h``).  The functions keep the C names and only marshal
arguments: they check tensor dtypes/shapes/devices, allocate outputs with
torch when the caller passes none, and hand raw device pointers and the
current CUDA stream to the library.  Every step of the computation runs in
the library's CUDA kernels; there is no CPU or PyTorch fallback -- if the
library is missing the import of the first call raises.

Stage 1, ``avq_quantize``: full-tree key quantisation and aggregation
("AVQ-Attention: Adaptive Vector-Quantized Attention", Sec. 4.2, Algorithm 1).
Stage 2, ``avq_attention``: count-weighted attention over the parents with
top-P child refinement per query block (Sec. 4.3, Algorithm 2).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libavq.so")

AVQ_OK, AVQ_ERR_INVALID_ARG, AVQ_ERR_UNSUPPORTED, AVQ_ERR_CUDA = 0, 1, 2, 3
AVQ_ERR_DEVICE, AVQ_ERR_TIMEOUT, AVQ_ERR_WORKSPACE = 4, 5, 6
AVQ_F32, AVQ_BF16 = 0, 1
AVQ_PATH_AUTO, AVQ_PATH_SIMT, AVQ_PATH_TC = 0, 1, 2
AVQ_DENOM_AUTO, AVQ_DENOM_TWO_PASS, AVQ_DENOM_EXTRAPOLATED = 0, 1, 2


class AVQError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{status_string(status)}: {msg}")
        self.status = status


class avq_dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int),
                ("d", ctypes.c_int), ("M0", ctypes.c_int), ("C", ctypes.c_int)]


_lib = None
_lib_lock = threading.Lock()
_vp = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    """The loaded libavq.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        with _lib_lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise ImportError(
                        f"{LIB_PATH} is missing: build it with "
                        "`python -m adaptive_vector_quantized_b200.build`")
                L = ctypes.CDLL(LIB_PATH)
                P = ctypes.POINTER
                L.avq_quantize.argtypes = [P(avq_dims), ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp,
                                           _vp, ctypes.c_int, _vp, ctypes.c_size_t, _vp]
                L.avq_quantize_noalloc.argtypes = [P(avq_dims), ctypes.c_int, _vp, _vp, _vp, _vp,
                                                   _vp, _vp, _vp, _vp]
                L.avq_attention.argtypes = [P(avq_dims), ctypes.c_int, _vp, _vp, _vp, _vp, _vp,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                            _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
                L.avq_quantize3.argtypes = [P(avq_dims), ctypes.c_int] + [_vp] * 8 + [_vp]
                L.avq_attention3.argtypes = ([P(avq_dims), ctypes.c_int] + [_vp] * 6
                                             + [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float]
                                             + [_vp] * 5 + [_vp])
                L.avq_codebook_update.argtypes = [P(avq_dims), ctypes.c_int, ctypes.c_float, _vp, _vp,
                                                  _vp, _vp, _vp, _vp, _vp]
                L.avq_permute.argtypes = [_vp, _vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, _vp]
                L.avq_hilbert_order.argtypes = [ctypes.c_int, _vp]
                L.avq_gilbert_order.argtypes = [ctypes.c_int, ctypes.c_int, _vp]
                L.avq_selftest_wait.argtypes = [ctypes.c_int, _vp]
                L.avq_selftest_exp2.argtypes = [_vp, _vp, ctypes.c_int64, _vp]
                L.avq_workspace_size.argtypes = [P(avq_dims), ctypes.c_int, ctypes.c_int,
                                                 ctypes.c_int, ctypes.c_int, ctypes.c_int]
                L.avq_workspace_size.restype = ctypes.c_size_t
                L.avq_check_device.argtypes = [_vp]
                L.avq_set_path.argtypes = [ctypes.c_int]
                L.avq_set_path.restype = ctypes.c_int
                for name in ("avq_status_string", "avq_last_error", "avq_last_kernels"):
                    getattr(L, name).restype = ctypes.c_char_p
                L.avq_status_string.argtypes = [ctypes.c_int]
                L.avq_version.restype = ctypes.c_int
                for name in ("avq_quantize", "avq_quantize_noalloc", "avq_attention", "avq_permute",
                             "avq_quantize3", "avq_attention3",
                             "avq_hilbert_order", "avq_gilbert_order", "avq_check_device",
                             "avq_codebook_update", "avq_selftest_wait", "avq_selftest_exp2"):
                    getattr(L, name).restype = ctypes.c_int
                _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().avq_status_string(int(status)).decode()


def last_error() -> str:
    return lib().avq_last_error().decode()


def last_kernels() -> str:
    return lib().avq_last_kernels().decode()


def avq_set_path(path: int) -> int:
    old = lib().avq_set_path(int(path))
    if old < 0:
        raise ValueError(f"unknown path {path}")
    return old


def _check(status: int):
    if status != AVQ_OK:
        raise AVQError(status, last_error())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return AVQ_F32
    if t.dtype == torch.bfloat16:
        return AVQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return _vp(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return _vp(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _expect(t, name, shape, dtype, device):
    """Raise unless `t` is a contiguous CUDA tensor of this shape, dtype and device."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device} (all tensors on one GPU)")


def _dims(Q_like: torch.Tensor, parents: torch.Tensor, children) -> avq_dims:
    B, H, N, d = Q_like.shape
    Hp, M0, dp = parents.shape
    C = 0 if children is None else children.shape[2]
    if Hp != H or dp != d:
        raise ValueError("parents must be [H, M0, d]")
    if children is not None and tuple(children.shape) != (H, M0, C, d):
        raise ValueError("children must be [H, M0, C, d]")
    return avq_dims(B, H, N, d, M0, C)


def avq_workspace_size(dims: avq_dims, dtype: int, deterministic=False, two_pass=False,
                       P: int = 0, block: int = 128) -> int:
    return int(lib().avq_workspace_size(ctypes.byref(dims), int(dtype), int(bool(deterministic)),
                                        int(two_pass), int(P), int(block)))


def workspace(dims: avq_dims, dtype: int, device, deterministic=False, two_pass=False, P=0,
              block=128):
    """A device byte tensor of the size the library asks for (None when 0)."""
    n = avq_workspace_size(dims, dtype, deterministic, two_pass, P, block)
    if n == 0:
        return None
    return torch.empty(n + 256, dtype=torch.uint8, device=device)


def _ws_ptr(ws, device=None):
    if ws is None:
        return None, 0
    if device is not None and ws.device != device:
        raise ValueError(f"workspace is on {ws.device}, expected {device}")
    p = ws.data_ptr()
    off = (-p) % 256
    return _vp(p + off), ws.numel() - off


def _check_stage1(K, V, parents, children, assign, vsum, counts, Mt):
    """Shapes, dtypes and devices of stage 1's tensors: every tensor on K's
    device, V like K, codebook in K's dtype, outputs of the stated layout."""
    B, H, N, d = K.shape
    dev = K.device
    _expect(V, "V", K.shape, K.dtype, dev)
    _expect(parents, "parents", parents.shape, K.dtype, dev)
    _expect(children, "children", children.shape if children is not None else (), K.dtype, dev)
    _expect(assign, "assign", (B, H, N), torch.int32, dev)
    _expect(vsum, "vsum", (B, H, Mt, d), torch.float32, dev)
    _expect(counts, "counts", (B, H, Mt), torch.int32, dev)


def avq_quantize(K, V, parents, children, assign=None, vsum=None, counts=None,
                 deterministic=False, ws=None, stream=None):
    """Stage 1.  K, V [B,H,N,d]; parents [H,M0,d]; children [H,M0,C,d] (or None
    for C = 0).  Returns (assign [B,H,N] int32, vsum [B,H,Mt,d] fp32,
    counts [B,H,Mt] int32)."""
    dims = _dims(K, parents, children)
    dt = _dtype_code(K)
    B, H, N, d = K.shape
    Mt = dims.M0 * (1 + dims.C)
    dev = K.device
    _check_stage1(K, V, parents, children, assign, vsum, counts, Mt)
    if assign is None:
        assign = torch.empty((B, H, N), dtype=torch.int32, device=dev)
    if vsum is None:
        vsum = torch.empty((B, H, Mt, d), dtype=torch.float32, device=dev)
    if counts is None:
        counts = torch.empty((B, H, Mt), dtype=torch.int32, device=dev)
    if ws is None:
        ws = workspace(dims, dt, dev, deterministic=deterministic)
    wp, wn = _ws_ptr(ws, dev)
    with torch.cuda.device(dev):  # the library launches on the current device
        _check(lib().avq_quantize(ctypes.byref(dims), dt, _ptr(K), _ptr(V), _ptr(parents),
                                  _ptr(children), _ptr(assign), _ptr(vsum), _ptr(counts),
                                  int(bool(deterministic)), wp, wn, _stream(stream)))
    return assign, vsum, counts


def avq_quantize_noalloc(K, V, parents, children, assign=None, vsum=None, counts=None, stream=None):
    """Stage 1 through the library's static scratch instead of a workspace
    (no device memory is allocated by the call; pass `assign`, `vsum` and
    `counts` to keep this wrapper from allocating the outputs).  Calls whose
    executions may overlap on one device race on that scratch."""
    dims = _dims(K, parents, children)
    dt = _dtype_code(K)
    B, H, N, d = K.shape
    Mt = dims.M0 * (1 + dims.C)
    dev = K.device
    _check_stage1(K, V, parents, children, assign, vsum, counts, Mt)
    if assign is None:
        assign = torch.empty((B, H, N), dtype=torch.int32, device=dev)
    if vsum is None:
        vsum = torch.empty((B, H, Mt, d), dtype=torch.float32, device=dev)
    if counts is None:
        counts = torch.empty((B, H, Mt), dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):  # the scratch array and the launch are the current device's
        _check(lib().avq_quantize_noalloc(ctypes.byref(dims), dt, _ptr(K), _ptr(V), _ptr(parents),
                                          _ptr(children), _ptr(assign), _ptr(vsum), _ptr(counts),
                                          _stream(stream)))
    return assign, vsum, counts


def avq_attention(Q, parents, children, vsum, counts, P: int, block: int = 128, scale=None,
                  two_pass=False, O=None, sel=None, importance=False, ws=None, stream=None):
    """Stage 2.  Returns (O [B,H,N,d], sel [B,H,nblk,P] int32, importance
    [B,H,nblk,M0] fp32 or None).  `importance=True` asks for the importance
    output; a tensor is written in place.  `two_pass`: AVQ_DENOM_AUTO (or
    False), AVQ_DENOM_TWO_PASS (or True) or AVQ_DENOM_EXTRAPOLATED."""
    dims = _dims(Q, parents, children)
    dt = _dtype_code(Q)
    B, H, N, d = Q.shape
    nblk = (N + block - 1) // block
    dev = Q.device
    if scale is None:
        scale = d ** -0.5
    Mt = dims.M0 * (1 + dims.C)
    _expect(parents, "parents", parents.shape, Q.dtype, dev)
    _expect(children, "children", children.shape if children is not None else (), Q.dtype, dev)
    _expect(vsum, "vsum", (B, H, Mt, d), torch.float32, dev)
    _expect(counts, "counts", (B, H, Mt), torch.int32, dev)
    _expect(O, "O", Q.shape, Q.dtype, dev)
    _expect(sel, "sel", (B, H, nblk, max(P, 0)), torch.int32, dev)
    if isinstance(importance, torch.Tensor):
        _expect(importance, "importance", (B, H, nblk, dims.M0), torch.float32, dev)
    if O is None:
        O = torch.empty_like(Q)
    if sel is None:
        sel = torch.empty((B, H, nblk, max(P, 0)), dtype=torch.int32, device=dev)
    imp = None
    if isinstance(importance, torch.Tensor):
        imp = importance
    elif importance:
        imp = torch.empty((B, H, nblk, dims.M0), dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(dims, dt, dev, two_pass=two_pass, P=P, block=block)
    wp, wn = _ws_ptr(ws, dev)
    with torch.cuda.device(dev):
        _check(lib().avq_attention(ctypes.byref(dims), dt, _ptr(Q), _ptr(parents), _ptr(children),
                                   _ptr(vsum), _ptr(counts), int(P), int(block), float(scale),
                                   int(two_pass), _ptr(O), _ptr(sel) if P > 0 else None,
                                   _ptr(imp), wp, wn, _stream(stream)))
    return O, sel, imp


def m_total3(M0: int, C: int) -> int:
    """Codes of a depth-3 tree: M0 parents, M0*C children, M0*C*C grandchildren."""
    return M0 + M0 * C + M0 * C * C


def _dims3(X, parents, children, grandchildren):
    B, H, N, d = X.shape
    Hp, M0, dp = parents.shape
    if Hp != H or dp != d:
        raise ValueError("parents must be [H, M0, d]")
    C = children.shape[2]
    if tuple(children.shape) != (H, M0, C, d):
        raise ValueError("children must be [H, M0, C, d]")
    if tuple(grandchildren.shape) != (H, M0, C, C, d):
        raise ValueError("grandchildren must be [H, M0, C, C, d]")
    return avq_dims(B, H, N, d, M0, C)


def avq_quantize3(K, V, parents, children, grandchildren, assign=None, vsum=None, counts=None,
                  stream=None):
    """Stage 1 over a depth-3 tree.  K, V [B,H,N,d]; parents [H,M0,d];
    children [H,M0,C,d]; grandchildren [H,M0,C,C,d].  Returns (assign [B,H,N]
    int32, vsum [B,H,Mt3,d] fp32, counts [B,H,Mt3] int32), Mt3 = m_total3."""
    dims = _dims3(K, parents, children, grandchildren)
    dt = _dtype_code(K)
    B, H, N, d = K.shape
    Mt = m_total3(dims.M0, dims.C)
    dev = K.device
    _expect(V, "V", K.shape, K.dtype, dev)
    for t, nm in ((parents, "parents"), (children, "children"), (grandchildren, "grandchildren")):
        _expect(t, nm, t.shape, K.dtype, dev)
    _expect(assign, "assign", (B, H, N), torch.int32, dev)
    _expect(vsum, "vsum", (B, H, Mt, d), torch.float32, dev)
    _expect(counts, "counts", (B, H, Mt), torch.int32, dev)
    if assign is None:
        assign = torch.empty((B, H, N), dtype=torch.int32, device=dev)
    if vsum is None:
        vsum = torch.empty((B, H, Mt, d), dtype=torch.float32, device=dev)
    if counts is None:
        counts = torch.empty((B, H, Mt), dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().avq_quantize3(ctypes.byref(dims), dt, _ptr(K), _ptr(V), _ptr(parents), _ptr(children),
                                   _ptr(grandchildren), _ptr(assign), _ptr(vsum), _ptr(counts),
                                   _stream(stream)))
    return assign, vsum, counts


def avq_attention3(Q, parents, children, grandchildren, vsum, counts, P: int, P2: int, block: int = 128,
                   scale=None, O=None, importance=False, stream=None):
    """Stage 2 over a depth-3 tree.  Returns (O [B,H,N,d], sel [B,H,nblk,P]
    parents, sel2 [B,H,nblk,P2] child codes, importance [B,H,nblk,M0] or None,
    importance2 [B,H,nblk,P*C] or None)."""
    dims = _dims3(Q, parents, children, grandchildren)
    dt = _dtype_code(Q)
    B, H, N, d = Q.shape
    M0, C = dims.M0, dims.C
    Mt = m_total3(M0, C)
    nblk = (N + block - 1) // block
    dev = Q.device
    if scale is None:
        scale = d ** -0.5
    for t, nm in ((parents, "parents"), (children, "children"), (grandchildren, "grandchildren")):
        _expect(t, nm, t.shape, Q.dtype, dev)
    _expect(vsum, "vsum", (B, H, Mt, d), torch.float32, dev)
    _expect(counts, "counts", (B, H, Mt), torch.int32, dev)
    _expect(O, "O", Q.shape, Q.dtype, dev)
    if O is None:
        O = torch.empty_like(Q)
    sel = torch.empty((B, H, nblk, max(P, 0)), dtype=torch.int32, device=dev)
    sel2 = torch.empty((B, H, nblk, max(P2, 0)), dtype=torch.int32, device=dev)
    imp = imp2 = None
    if importance:
        imp = torch.empty((B, H, nblk, M0), dtype=torch.float32, device=dev)
        imp2 = torch.empty((B, H, nblk, max(P * C, 1)), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().avq_attention3(ctypes.byref(dims), dt, _ptr(Q), _ptr(parents), _ptr(children),
                                    _ptr(grandchildren), _ptr(vsum), _ptr(counts), int(P), int(P2),
                                    int(block), float(scale), _ptr(O), _ptr(sel) if P > 0 else None,
                                    _ptr(sel2) if P2 > 0 else None, _ptr(imp), _ptr(imp2), _stream(stream)))
    return O, sel, sel2, imp, imp2


def avq_codebook_update(ksum, counts, S, Nst, parents, children, lam: float, stream=None):
    """Codebook update (EMA statistics and constraint projection).  ksum
    [B,H,Mt,d] fp32 and counts [B,H,Mt] int32: avq_quantize's statistics of
    the keys; S [H,Mt,d] and Nst [H,Mt] fp32: EMA state, updated in place;
    parents [H,M0,d] and children [H,M0,C,d]: codebook, rewritten in place."""
    B, H, Mt, d = ksum.shape
    Hp, M0, dp = parents.shape
    C = 0 if children is None else children.shape[2]
    if Hp != H or dp != d or Mt != M0 * (1 + C):
        raise ValueError("ksum must be [B, H, M0*(1+C), d] for parents [H, M0, d]")
    if children is not None and tuple(children.shape) != (H, M0, C, d):
        raise ValueError("children must be [H, M0, C, d]")
    dims = avq_dims(B, H, 1, d, M0, C)
    dt = _dtype_code(parents)
    dev = parents.device
    _expect(ksum, "ksum", (B, H, Mt, d), torch.float32, dev)
    _expect(counts, "counts", (B, H, Mt), torch.int32, dev)
    _expect(S, "S", (H, Mt, d), torch.float32, dev)
    _expect(Nst, "Nst", (H, Mt), torch.float32, dev)
    _expect(children, "children", (H, M0, C, d), parents.dtype, dev)
    with torch.cuda.device(dev):
        _check(lib().avq_codebook_update(ctypes.byref(dims), dt, float(lam), _ptr(ksum), _ptr(counts),
                                         _ptr(S), _ptr(Nst), _ptr(parents), _ptr(children),
                                         _stream(stream)))
    return S, Nst, parents, children


def avq_permute(X, idx, inverse=False, Y=None, stream=None):
    """Gather (inverse=False: Y[b,i] = X[b,idx[i]]) or scatter back along dim -2
    of a [..., rows, cols] tensor; idx is an int32 CUDA tensor."""
    rows = X.shape[-2]
    batch = X.numel() // (rows * X.shape[-1])
    row_bytes = X.shape[-1] * X.element_size()
    _expect(idx, "idx", (rows,), torch.int32, X.device)
    _expect(Y, "Y", X.shape, X.dtype, X.device)
    if Y is None:
        Y = torch.empty_like(X)
    with torch.cuda.device(X.device):
        _check(lib().avq_permute(_ptr(X), _ptr(idx), _ptr(Y), int(batch), int(rows), int(row_bytes),
                                 int(bool(inverse)), _stream(stream)))
    return Y


def avq_hilbert_order(side: int) -> torch.Tensor:
    """Raster index of the t-th cell along a Hilbert curve (host tensor, int32)."""
    out = torch.empty(side * side, dtype=torch.int32)
    _check(lib().avq_hilbert_order(int(side), _vp(out.data_ptr())))
    return out


def avq_gilbert_order(width: int, height: int) -> torch.Tensor:
    """Raster index (y*width + x) of the t-th cell along a generalised Hilbert
    curve over a width x height grid (host tensor, int32)."""
    out = torch.empty(max(1, int(width) * int(height)), dtype=torch.int32)  # sizes checked by the library
    _check(lib().avq_gilbert_order(int(width), int(height), _vp(out.data_ptr())))
    return out


def avq_selftest_wait(timeout_us: int = 2000, stream=None):
    """Launch the bounded-wait self-test: the next avq_check_device raises
    AVQError with status AVQ_ERR_TIMEOUT."""
    _check(lib().avq_selftest_wait(int(timeout_us), _stream(stream)))


def avq_selftest_exp2(x, y=None, stream=None):
    """The FMA-pipe 2^x of the attention kernel on a contiguous fp32 CUDA
    tensor with an even number of elements; returns y (allocated if None)."""
    if not (isinstance(x, torch.Tensor) and x.is_cuda and x.dtype == torch.float32):
        raise TypeError("x must be a float32 CUDA tensor")
    if y is None:
        y = torch.empty_like(x)
    _expect(y, "y", x.shape, torch.float32, x.device)
    with torch.cuda.device(x.device):
        _check(lib().avq_selftest_exp2(_ptr(x), _ptr(y), int(x.numel()), _stream(stream)))
    return y


def avq_check_device(stream=None):
    """Synchronise the stream and raise if a kernel recorded a device-side error."""
    _check(lib().avq_check_device(_stream(stream)))


def avq_version() -> int:
    return int(lib().avq_version())

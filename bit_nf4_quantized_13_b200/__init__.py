"""B200-native QLoRA NF4 linear layer: Python binding of ``libqlora_nf4.so``.

The QLoRA hot path (Dettmers et al., arXiv:2305.14314) for one frozen linear
layer with a LoRA side path, as hand-written sm_100a CUDA kernels behind the
C ABI of ``include/qlora.h``.  This module only marshals arguments: it turns
torch CUDA tensors into device pointers, allocates outputs and workspaces
with torch, passes torch's current stream, and raises on a non-OK status.
Every step of the computation runs in the library's kernels; there is no
fallback.  The library must have been built (``python -m
bit_nf4_quantized_13_b200.build``); it is loaded on first use, and a missing
or stale library raises ImportError there.

Entry points (same names as the C ABI):
    qlora_nf4_codebook()                         -> numpy float32[16]
    qlora_quantize_nf4_dq(W)                     -> Nf4Weight
    qlora_dequantize(w, out_dtype)               -> tensor (N x K)
    qlora_linear_fwd(X, w, A, B, s)              -> (Y, T)
    qlora_linear_bwd(dY, X, w, A, B, s, T=None)  -> (dX, dA, dB)
    qlora_fp8_e4m3_encode(x)                     -> uint8 tensor
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora_nf4.so")

QLORA_OK = 0
STATUS_NAMES = {0: "QLORA_OK", 1: "QLORA_ERR_INVALID_ARG", 2: "QLORA_ERR_UNSUPPORTED",
                3: "QLORA_ERR_WORKSPACE", 4: "QLORA_ERR_CUDA", 5: "QLORA_ERR_NONFINITE",
                6: "QLORA_ERR_TIMEOUT"}
BLOCK, BLOCK2, MAX_RANK = 64, 256, 256
TYPE_NF4, TYPE_FP4, TYPE_INT4 = 0, 1, 2
QTYPES = {"nf4": TYPE_NF4, "fp4": TYPE_FP4, "int4": TYPE_INT4}


class QloraError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS_NAMES.get(status, status)}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m bit_nf4_quantized_13_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    i64, i32, vp, sz, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float
    sig = {
        "qlora_nf4_codebook": (i32, [vp]),
        "qlora_codebook": (i32, [i32, vp]),
        "qlora_quantize_4bit_dq": (i32, [i32, vp, i64, i32, i32, vp, vp, vp, vp, vp, sz, vp, vp]),
        "qlora_dequantize_4bit": (i32, [i32, vp, vp, vp, vp, i64, i32, i32, vp, i32, vp]),
        "qlora_linear_fwd_4bit": (i32, [i32, vp, i64, i64, i64, vp, vp, vp, vp, vp, vp, i32, f32, vp, vp, vp,
                                        sz, vp]),
        "qlora_linear_bwd_4bit": (i32, [i32, vp, vp, i64, i64, i64, vp, vp, vp, vp, vp, vp, i32, f32, vp, vp,
                                        vp, vp, vp, sz, vp]),
        "qlora_quantize_workspace_size": (sz, [i64]),
        "qlora_quantize_nf4_dq": (i32, [vp, i64, i32, i32, vp, vp, vp, vp, vp, sz, vp, vp]),
        "qlora_dequantize": (i32, [vp, vp, vp, vp, i64, i32, i32, vp, i32, vp]),
        "qlora_linear_fwd_workspace_size": (sz, [i64, i64, i64, i32]),
        "qlora_linear_bwd_workspace_size": (sz, [i64, i64, i64, i32]),
        "qlora_linear_fwd": (i32, [vp, i64, i64, i64, vp, vp, vp, vp, vp, vp, i32, f32, vp, vp, vp,
                                   sz, vp]),
        "qlora_linear_bwd": (i32, [vp, vp, i64, i64, i64, vp, vp, vp, vp, vp, vp, i32, f32, vp, vp,
                                   vp, vp, vp, sz, vp]),
        "qlora_fp8_e4m3_encode": (i32, [vp, vp, i64, vp]),
        "qlora_kernel_launch_count": (ctypes.c_uint64, []),
        "qlora_device_error": (i32, [i32]),
        "qlora_quantize_nf4_dq_noalloc": (i32, [vp, i64, i32, i32, vp, vp, vp, vp, vp, vp]),
        "qlora_debug_wait_timeout": (i32, [ctypes.c_uint64, vp]),
        "qlora_int8_quantize": (i32, [vp, i64, i32, vp, vp, vp, vp]),
        "qlora_int8_dequantize": (i32, [vp, vp, i64, i32, vp, vp]),
        "qlora_debug_fill": (i32, [vp, i64, ctypes.c_uint32, vp]),
        "qlora_debug_read": (i32, [vp, i64, ctypes.c_uint32, vp, vp]),
        "qlora_linear_group_fwd_workspace_size": (sz, [i64, i32, i32]),
        "qlora_linear_group_bwd_workspace_size": (sz, [i64, i32, i32]),
        "qlora_linear_group_fwd": (i32, [i32, vp, i64, i64, vp, i32, vp, vp, i32, f32, vp, vp, vp, sz, vp]),
        "qlora_linear_group_bwd": (i32, [i32, vp, vp, i64, i64, vp, i32, vp, vp, i32, f32, vp, vp, vp, vp,
                                         vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype, fn.argtypes = res, args
    return L


_lib_handle = None


def _get_lib() -> ctypes.CDLL:
    global _lib_handle
    if _lib_handle is None:
        try:
            _lib_handle = _load()
        except AttributeError as e:  # a library built from older sources
            raise ImportError(f"{LIB_PATH} is stale ({e}); rebuild it") from e
    return _lib_handle


def __getattr__(name):
    if name == "lib":
        return _get_lib()
    raise AttributeError(name)


def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, st: int) -> None:
    if st != QLORA_OK:
        raise QloraError(fn, st)


def _need_cuda(*ts):
    """Contiguous CUDA tensors, all on one device (the current one while the
    call runs: the library launches on the current device's stream)."""
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensors on different devices: {dev} and {t.device}")
    if dev is not None and dev.index is not None and dev.index != _torch().cuda.current_device():
        raise ValueError(f"tensors are on {dev} but the current device is cuda:"
                         f"{_torch().cuda.current_device()}")


def _need_dtype(dtype, **ts):
    for name, t in ts.items():
        if t is not None and t.dtype != dtype:
            raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _need_shape(name, t, shape):
    if t is not None and tuple(t.shape) != tuple(int(d) for d in shape):
        raise ValueError(f"{name} must have shape {tuple(int(d) for d in shape)}, got {tuple(t.shape)}")


def _need_weight(w, numel):
    """The four buffers of an Nf4Weight hold at least what `numel` weights need
    (the kernels read exactly that much)."""
    nb = -(-numel // BLOCK)
    need = {"codes": (numel + 1) // 2, "c2_fp8": nb, "c1": -(-nb // BLOCK2), "mean": 1}
    for name, n in need.items():
        t = getattr(w, name)
        if t.numel() < n:
            raise ValueError(f"Nf4Weight.{name} holds {t.numel()} elements, {n} needed")
    torch = _torch()
    _need_dtype(torch.uint8, codes=w.codes, c2_fp8=w.c2_fp8)
    _need_dtype(torch.float32, c1=w.c1, mean=w.mean)


def _linear_dims(X, w, A, B):
    """(M, N, K, r) of a linear call, checking that the operands agree."""
    if X.dim() != 2 or len(w.shape) != 2 or A.dim() != 2 or B.dim() != 2:
        raise ValueError("X, the weight, A and B must be 2-D")
    M, K = (int(d) for d in X.shape)
    N, Kw = (int(d) for d in w.shape)
    if Kw != K:
        raise ValueError(f"X has K = {K} columns but the weight is {N} x {Kw}")
    r = int(A.shape[0])
    _need_shape("A", A, (r, K))
    _need_shape("B", B, (N, r))
    _need_weight(w, N * K)
    torch = _torch()
    _need_dtype(torch.bfloat16, X=X, A=A, B=B)
    return M, N, K, r


def _workspace(nbytes: int, device):
    torch = _torch()
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


# ----------------------------------------------------------------- codebook

def qlora_nf4_codebook() -> np.ndarray:
    out = np.zeros(16, np.float32)
    _check("qlora_nf4_codebook", _get_lib().qlora_nf4_codebook(out.ctypes.data_as(ctypes.c_void_p)))
    return out


def qlora_codebook(qtype: int = TYPE_NF4) -> np.ndarray:
    """The 16 values of a 4-bit data type (TYPE_NF4, TYPE_FP4, TYPE_INT4)."""
    out = np.zeros(16, np.float32)
    _check("qlora_codebook", _get_lib().qlora_codebook(int(qtype), out.ctypes.data_as(ctypes.c_void_p)))
    return out


# ----------------------------------------------------------------- quantize

@dataclass
class Nf4Weight:
    """A frozen weight in the library's storage format (4 device buffers)."""
    codes: object   # uint8 [ceil(numel/2)]
    c2_fp8: object  # uint8 [ceil(numel/64)]
    c1: object      # float32 [ceil(numel/16384)]
    mean: object    # float32 [1]
    shape: tuple
    qtype: int = 0  # the 4-bit data type the codes index (TYPE_NF4 / TYPE_FP4 / TYPE_INT4)

    @property
    def numel(self) -> int:
        n = 1
        for d in self.shape:
            n *= int(d)
        return n

    def nbytes(self) -> int:
        return sum(int(t.numel() * t.element_size()) for t in (self.codes, self.c2_fp8, self.c1, self.mean))


def qlora_quantize_workspace_size(numel: int) -> int:
    return int(_get_lib().qlora_quantize_workspace_size(int(numel)))


def alloc_nf4_weight(shape, device, qtype: int = TYPE_NF4) -> Nf4Weight:
    torch = _torch()
    n = 1
    for d in shape:
        n *= int(d)
    nb = -(-n // BLOCK)
    return Nf4Weight(torch.empty((n + 1) // 2, dtype=torch.uint8, device=device),
                     torch.empty(max(nb, 1), dtype=torch.uint8, device=device),
                     torch.empty(max(-(-nb // BLOCK2), 1), dtype=torch.float32, device=device),
                     torch.zeros(1, dtype=torch.float32, device=device), tuple(int(d) for d in shape),
                     int(qtype))


def qlora_quantize_nf4_dq(W, out: Nf4Weight | None = None, ws=None, status=None,
                          stream=None, qtype: int = TYPE_NF4) -> Nf4Weight:
    """4-bit (NF4 by default) + double quantization of an fp32 CUDA tensor
    (any shape, flattened)."""
    torch = _torch()
    _need_cuda(W)
    if W.dtype != torch.float32:
        raise ValueError("W must be float32")
    n = W.numel()
    w = out if out is not None else alloc_nf4_weight(tuple(W.shape), W.device, qtype)
    w.qtype = int(qtype)
    _need_weight(w, n)
    _need_cuda(W, w.codes, w.c2_fp8, w.c1, w.mean, ws, status)
    if status is not None:
        _need_dtype(torch.int32, status=status)
    if ws is None:
        ws = _workspace(qlora_quantize_workspace_size(n), W.device)
    st = _get_lib().qlora_quantize_4bit_dq(int(qtype), _ptr(W), n, BLOCK, BLOCK2, _ptr(w.codes), _ptr(w.c2_fp8),
                                           _ptr(w.c1), _ptr(w.mean), _ptr(ws), ws.numel(), _ptr(status),
                                           _stream(stream))
    _check("qlora_quantize_4bit_dq", st)
    return w


def qlora_dequantize(w: Nf4Weight, out_dtype=None, out=None, stream=None):
    torch = _torch()
    out_dtype = out_dtype or torch.float32
    code = {torch.float32: 0, torch.bfloat16: 1}[out_dtype]
    _need_weight(w, w.numel)
    if out is None:
        out = torch.empty(w.shape, dtype=out_dtype, device=w.codes.device)
    _need_dtype(out_dtype, out=out)
    if out.numel() < w.numel:
        raise ValueError(f"out holds {out.numel()} elements, {w.numel} needed")
    _need_cuda(w.codes, w.c2_fp8, w.c1, w.mean, out)
    st = _get_lib().qlora_dequantize_4bit(int(w.qtype), _ptr(w.codes), _ptr(w.c2_fp8), _ptr(w.c1), _ptr(w.mean),
                                          w.numel, BLOCK, BLOCK2, _ptr(out), code, _stream(stream))
    _check("qlora_dequantize_4bit", st)
    return out


# ------------------------------------------------------------------- linear

def qlora_linear_fwd_workspace_size(M, N, K, r) -> int:
    return int(_get_lib().qlora_linear_fwd_workspace_size(int(M), int(N), int(K), int(r)))


def qlora_linear_bwd_workspace_size(M, N, K, r) -> int:
    return int(_get_lib().qlora_linear_bwd_workspace_size(int(M), int(N), int(K), int(r)))


def qlora_linear_fwd(X, w: Nf4Weight, A, B, s: float, Y=None, T_save=None, ws=None, stream=None):
    """Y = X W'^T + s (X A^T) B^T; returns (Y, T) with T = bf16(s X A^T)."""
    torch = _torch()
    M, N, K, r = _linear_dims(X, w, A, B)
    _need_shape("Y", Y, (M, N))
    _need_shape("T_save", T_save, (M, r))
    _need_dtype(torch.bfloat16, Y=Y, T_save=T_save)
    _need_cuda(X, A, B, Y, T_save, ws, w.codes, w.c2_fp8, w.c1, w.mean)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    if T_save is None:
        T_save = torch.empty((M, r), dtype=torch.bfloat16, device=X.device)
    if ws is None:
        ws = _workspace(qlora_linear_fwd_workspace_size(M, N, K, r), X.device)
    st = _get_lib().qlora_linear_fwd_4bit(int(w.qtype), _ptr(X), M, N, K, _ptr(w.codes), _ptr(w.c2_fp8),
                                          _ptr(w.c1), _ptr(w.mean), _ptr(A), _ptr(B), r, float(s), _ptr(Y),
                                          _ptr(T_save), _ptr(ws), ws.numel(), _stream(stream))
    _check("qlora_linear_fwd_4bit", st)
    return Y, T_save


def qlora_linear_bwd(dY, X, w: Nf4Weight, A, B, s: float, T=None, dX=None, dA=None, dB=None,
                     ws=None, want_dx: bool = True, stream=None):
    """Adapter gradients and the input gradient; no gradient for W."""
    torch = _torch()
    M, N, K, r = _linear_dims(X, w, A, B)
    _need_shape("dY", dY, (M, N))
    _need_shape("T", T, (M, r))
    _need_shape("dX", dX, (M, K))
    _need_shape("dA", dA, (r, K))
    _need_shape("dB", dB, (N, r))
    _need_dtype(torch.bfloat16, dY=dY, T=T, dX=dX, dA=dA, dB=dB)
    _need_cuda(dY, X, A, B, T, dX, dA, dB, ws, w.codes, w.c2_fp8, w.c1, w.mean)
    if want_dx and dX is None:
        dX = torch.empty((M, K), dtype=torch.bfloat16, device=X.device)
    if dA is None:
        dA = torch.empty((r, K), dtype=torch.bfloat16, device=X.device)
    if dB is None:
        dB = torch.empty((N, r), dtype=torch.bfloat16, device=X.device)
    if ws is None:
        ws = _workspace(qlora_linear_bwd_workspace_size(M, N, K, r), X.device)
    st = _get_lib().qlora_linear_bwd_4bit(int(w.qtype), _ptr(dY), _ptr(X), M, N, K, _ptr(w.codes),
                                          _ptr(w.c2_fp8), _ptr(w.c1), _ptr(w.mean), _ptr(A), _ptr(B), r,
                                          float(s), _ptr(T), _ptr(dX if want_dx else None), _ptr(dA), _ptr(dB),
                                          _ptr(ws), ws.numel(), _stream(stream))
    _check("qlora_linear_bwd_4bit", st)
    return dX, dA, dB


class _Weight4bit(ctypes.Structure):
    """The C struct qlora_weight_4bit."""
    _fields_ = [("codes", ctypes.c_void_p), ("c2_fp8", ctypes.c_void_p), ("c1", ctypes.c_void_p),
                ("mean", ctypes.c_void_p), ("N", ctypes.c_int64)]


def _group_dims(X, ws_, A_cat, B_cat):
    """(M, K, r, [N_g], descriptor array) of a group call."""
    torch = _torch()
    if not 1 <= len(ws_) <= 4:
        raise ValueError(f"a group holds 1 to 4 linears, got {len(ws_)}")
    if X.dim() != 2 or A_cat.dim() != 2 or B_cat.dim() != 2:
        raise ValueError("X, A_cat and B_cat must be 2-D")
    M, K = (int(d) for d in X.shape)
    qtype = int(ws_[0].qtype)
    ns = []
    for w in ws_:
        if len(w.shape) != 2 or int(w.shape[1]) != K:
            raise ValueError(f"every weight must be N_g x {K}, got {w.shape}")
        if int(w.qtype) != qtype:
            raise ValueError("the weights of a group share one 4-bit type")
        _need_weight(w, int(w.shape[0]) * K)
        ns.append(int(w.shape[0]))
    G = len(ws_)
    if int(A_cat.shape[0]) % G:
        raise ValueError(f"A_cat has {A_cat.shape[0]} rows, not a multiple of {G}")
    r = int(A_cat.shape[0]) // G
    _need_shape("A_cat", A_cat, (G * r, K))
    _need_shape("B_cat", B_cat, (sum(ns), r))
    _need_dtype(torch.bfloat16, X=X, A_cat=A_cat, B_cat=B_cat)
    desc = (_Weight4bit * G)(*[_Weight4bit(w.codes.data_ptr(), w.c2_fp8.data_ptr(), w.c1.data_ptr(),
                                           w.mean.data_ptr(), n) for w, n in zip(ws_, ns)])
    return M, K, r, ns, qtype, desc


def qlora_linear_group_fwd_workspace_size(M, G, r) -> int:
    return int(_get_lib().qlora_linear_group_fwd_workspace_size(int(M), int(G), int(r)))


def qlora_linear_group_bwd_workspace_size(M, G, r) -> int:
    return int(_get_lib().qlora_linear_group_bwd_workspace_size(int(M), int(G), int(r)))


def qlora_linear_group_fwd(X, weights, A_cat, B_cat, s: float, Y=None, T_save=None, ws=None, stream=None):
    """G linears on the same input (q/k/v, gate/up) as one: Y = [Y_1 .. Y_G]
    (M x sum N_g) with Y_g = X W_g'^T + s (X A_g^T) B_g^T; A_cat = [A_1; ..],
    B_cat = [B_1; ..].  Returns (Y, T) with T = [T_1 .. T_G] (M x G r)."""
    torch = _torch()
    M, K, r, ns, qtype, desc = _group_dims(X, weights, A_cat, B_cat)
    G, n_all = len(ns), sum(ns)
    _need_shape("Y", Y, (M, n_all))
    _need_shape("T_save", T_save, (M, G * r))
    _need_dtype(torch.bfloat16, Y=Y, T_save=T_save)
    _need_cuda(X, A_cat, B_cat, Y, T_save, ws, *[t for w in weights for t in (w.codes, w.c2_fp8, w.c1, w.mean)])
    if Y is None:
        Y = torch.empty((M, n_all), dtype=torch.bfloat16, device=X.device)
    if T_save is None:
        T_save = torch.empty((M, G * r), dtype=torch.bfloat16, device=X.device)
    if ws is None:
        ws = _workspace(qlora_linear_group_fwd_workspace_size(M, G, r), X.device)
    st = _get_lib().qlora_linear_group_fwd(qtype, _ptr(X), M, K, desc, G, _ptr(A_cat), _ptr(B_cat), r, float(s),
                                           _ptr(Y), _ptr(T_save), _ptr(ws), ws.numel(), _stream(stream))
    _check("qlora_linear_group_fwd", st)
    return Y, T_save


def qlora_linear_group_bwd(dY, X, weights, A_cat, B_cat, s: float, T=None, dX=None, dA_cat=None, dB_cat=None,
                           ws=None, want_dx: bool = True, stream=None):
    """Gradients of qlora_linear_group_fwd: dX = sum_g dY_g W_g' + U_g A_g,
    dA_cat = [dA_1; ..], dB_cat = [dB_1; ..]; no gradient for the weights."""
    torch = _torch()
    M, K, r, ns, qtype, desc = _group_dims(X, weights, A_cat, B_cat)
    G, n_all = len(ns), sum(ns)
    _need_shape("dY", dY, (M, n_all))
    _need_shape("T", T, (M, G * r))
    _need_shape("dX", dX, (M, K))
    _need_shape("dA_cat", dA_cat, (G * r, K))
    _need_shape("dB_cat", dB_cat, (n_all, r))
    _need_dtype(torch.bfloat16, dY=dY, T=T, dX=dX, dA_cat=dA_cat, dB_cat=dB_cat)
    _need_cuda(dY, X, A_cat, B_cat, T, dX, dA_cat, dB_cat, ws,
               *[t for w in weights for t in (w.codes, w.c2_fp8, w.c1, w.mean)])
    if want_dx and dX is None:
        dX = torch.empty((M, K), dtype=torch.bfloat16, device=X.device)
    if dA_cat is None:
        dA_cat = torch.empty((G * r, K), dtype=torch.bfloat16, device=X.device)
    if dB_cat is None:
        dB_cat = torch.empty((n_all, r), dtype=torch.bfloat16, device=X.device)
    if ws is None:
        ws = _workspace(qlora_linear_group_bwd_workspace_size(M, G, r), X.device)
    st = _get_lib().qlora_linear_group_bwd(qtype, _ptr(dY), _ptr(X), M, K, desc, G, _ptr(A_cat), _ptr(B_cat), r,
                                           float(s), _ptr(T), _ptr(dX if want_dx else None), _ptr(dA_cat),
                                           _ptr(dB_cat), _ptr(ws), ws.numel(), _stream(stream))
    _check("qlora_linear_group_bwd", st)
    return dX, dA_cat, dB_cat


def qlora_fp8_e4m3_encode(x, out=None, stream=None):
    torch = _torch()
    _need_dtype(torch.float32, x=x)
    if out is not None:
        _need_dtype(torch.uint8, out=out)
        if out.numel() < x.numel():
            raise ValueError(f"out holds {out.numel()} elements, {x.numel()} needed")
    _need_cuda(x, out)
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check("qlora_fp8_e4m3_encode",
           _get_lib().qlora_fp8_e4m3_encode(_ptr(x), _ptr(out), x.numel(), _stream(stream)))
    return out


def qlora_debug_fill(dst, value: int = 0, stream=None):
    """Measurement aid: the DRAM write ceiling (a 16-byte streaming fill of
    a contiguous CUDA tensor whose size is a multiple of 16 bytes)."""
    _need_cuda(dst)
    nbytes = dst.numel() * dst.element_size()
    if nbytes % 16:
        raise ValueError("the buffer must be a multiple of 16 bytes")
    _check("qlora_debug_fill", _get_lib().qlora_debug_fill(_ptr(dst), nbytes // 4, int(value) & 0xffffffff,
                                                           _stream(stream)))


def qlora_debug_read(src, sink, never: int = 0x9E3779B9, stream=None):
    """Measurement aid: the DRAM read ceiling (a 16-byte streaming read of a
    contiguous CUDA tensor; `sink` is a 4-byte CUDA tensor written only if
    the data folds to `never`)."""
    _need_cuda(src, sink)
    nbytes = src.numel() * src.element_size()
    if nbytes % 16:
        raise ValueError("the buffer must be a multiple of 16 bytes")
    _check("qlora_debug_read", _get_lib().qlora_debug_read(_ptr(src), nbytes // 4, int(never) & 0xffffffff,
                                                           _ptr(sink), _stream(stream)))


def qlora_device_error(reset: bool = False) -> int:
    """Sticky error word of the tensor-core kernels (0 = none, 6 = a bounded
    in-kernel wait timed out)."""
    return int(_get_lib().qlora_device_error(1 if reset else 0))


def qlora_int8_quantize(x, block: int = 64, codes=None, c=None, status=None, stream=None):
    """Block-wise Int8 absmax quantization (eq. 1): returns (codes int8, c fp32)."""
    torch = _torch()
    _need_dtype(torch.float32, x=x)
    n = x.numel()
    nb = -(-n // block)
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    if c is None:
        c = torch.empty(max(nb, 1), dtype=torch.float32, device=x.device)
    _need_dtype(torch.int8, codes=codes)
    _need_dtype(torch.float32, c=c)
    if codes.numel() < n or c.numel() < nb:
        raise ValueError("codes / c too small")
    if status is not None:
        _need_dtype(torch.int32, status=status)
    _need_cuda(x, codes, c, status)
    _check("qlora_int8_quantize", _get_lib().qlora_int8_quantize(_ptr(x), n, int(block), _ptr(codes), _ptr(c),
                                                                 _ptr(status), _stream(stream)))
    return codes, c


def qlora_int8_dequantize(codes, c, block: int = 64, out=None, stream=None):
    """Eq. (2): fp32 values from Int8 codes and the per-block constants."""
    torch = _torch()
    _need_dtype(torch.int8, codes=codes)
    _need_dtype(torch.float32, c=c)
    n = codes.numel()
    if c.numel() < -(-n // block):
        raise ValueError("c too small")
    if out is None:
        out = torch.empty(codes.shape, dtype=torch.float32, device=codes.device)
    _need_dtype(torch.float32, out=out)
    if out.numel() < n:
        raise ValueError("out too small")
    _need_cuda(codes, c, out)
    _check("qlora_int8_dequantize", _get_lib().qlora_int8_dequantize(_ptr(codes), _ptr(c), n, int(block),
                                                                     _ptr(out), _stream(stream)))
    return out


def qlora_debug_wait_timeout(limit_ns: int, stream=None) -> None:
    """Failure-detection self-test: one kernel whose bounded wait is never
    satisfied gives up after limit_ns (<= 1e9) and records QLORA_ERR_TIMEOUT
    for qlora_device_error."""
    _check("qlora_debug_wait_timeout", _get_lib().qlora_debug_wait_timeout(int(limit_ns), _stream(stream)))


def qlora_kernel_launch_count() -> int:
    """Kernels this library has launched in this process so far."""
    return int(_get_lib().qlora_kernel_launch_count())


NOALLOC_MAX_NUMEL = 1 << 28


def qlora_quantize_nf4_dq_noalloc(W, out: Nf4Weight | None = None, status=None,
                                  stream=None) -> Nf4Weight:
    """qlora_quantize_nf4_dq without a workspace: the library's built-in
    device scratch is used instead (numel <= 2^28; calls must not overlap)."""
    torch = _torch()
    _need_cuda(W)
    if W.dtype != torch.float32:
        raise ValueError("W must be float32")
    w = out if out is not None else alloc_nf4_weight(tuple(W.shape), W.device)
    _need_weight(w, W.numel())
    _need_cuda(W, w.codes, w.c2_fp8, w.c1, w.mean, status)
    if status is not None:
        _need_dtype(torch.int32, status=status)
    st = _get_lib().qlora_quantize_nf4_dq_noalloc(_ptr(W), W.numel(), BLOCK, BLOCK2, _ptr(w.codes),
                                           _ptr(w.c2_fp8), _ptr(w.c1), _ptr(w.mean), _ptr(status),
                                           _stream(stream))
    _check("qlora_quantize_nf4_dq_noalloc", st)
    return w

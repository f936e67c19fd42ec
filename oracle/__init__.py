"""CPU oracle for the QLoRA NF4 linear layer -- TEST INFRASTRUCTURE ONLY.

Plain C (``qlora_oracle.c``) reached through ctypes, with numpy arrays for
marshalling.  Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package; the product library never does.
It shares no code with the CUDA path.  See ``qlora_oracle.c`` for the
method's steps, the readings taken where the pages are silent, and the
citations.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qlora_oracle.c")
_LIB = os.path.join(_HERE, "libqlora_oracle.so")
_lock = threading.Lock()
_lib = None

OK = 0
ERR_ARG = 1
ERR_NONFINITE = 5


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE fp32/fp64, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-fexcess-precision=standard", "-pthread",
               "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            i64, vp, dbl, flt, i32 = (ctypes.c_int64, ctypes.c_void_p, ctypes.c_double,
                                      ctypes.c_float, ctypes.c_int)
            L.oracle_norm_ppf.restype = dbl
            L.oracle_norm_ppf.argtypes = [dbl]
            L.oracle_nf4_delta.restype = dbl
            L.oracle_nf4_delta.argtypes = []
            L.oracle_nf4_codebook.argtypes = [vp]
            L.oracle_fp4_codebook.argtypes = [vp]
            L.oracle_int4_codebook.argtypes = [vp]
            L.oracle_e2m1_decode.restype = dbl
            L.oracle_e2m1_decode.argtypes = [i32]
            L.oracle_quantize_nf4.restype = i32
            L.oracle_quantize_nf4.argtypes = [vp, i64, i32, vp, vp, vp]
            L.oracle_mean_exact.restype = i32
            L.oracle_mean_exact.argtypes = [vp, i64, vp, vp]
            L.oracle_double_quant.argtypes = [vp, i64, flt, i32, vp, vp]
            L.oracle_dequant_constants.argtypes = [vp, vp, flt, i64, i32, vp]
            L.oracle_dequantize.argtypes = [vp, vp, vp, flt, i64, i32, i32, vp, vp]
            L.oracle_e4m3_encode.restype = ctypes.c_uint8
            L.oracle_e4m3_encode.argtypes = [flt]
            L.oracle_e4m3_encode_array.argtypes = [vp, i64, vp]
            L.oracle_e4m3_decode.restype = flt
            L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            L.oracle_bf16_rne_array.argtypes = [vp, i64, vp]
            L.oracle_linear_fwd.restype = i32
            L.oracle_linear_fwd.argtypes = [vp, i64, i64, i64, vp, vp, vp, i64, dbl, vp, i64,
                                            vp, vp]
            L.oracle_linear_bwd.restype = i32
            L.oracle_linear_bwd.argtypes = [vp, vp, i64, i64, i64, vp, vp, vp, i64, dbl, vp,
                                            i64, vp, vp, vp]
            L.oracle_int8_quant.argtypes = [vp, i64, vp, vp]
            L.oracle_int8_dequant.argtypes = [vp, i64, flt, vp]
            L.oracle_int8_quant_blocks.argtypes = [vp, i64, i64, vp, vp]
            L.oracle_int8_dequant_blocks.argtypes = [vp, i64, i64, vp, vp]
            L.oracle_set_threads.argtypes = [i32]
            L.oracle_get_threads.restype = i32
            _lib = L
    return _lib


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def threads() -> int:
    return int(lib().oracle_get_threads())


# -- a1 --------------------------------------------------------------------
def norm_ppf(p: float) -> float:
    return float(lib().oracle_norm_ppf(float(p)))


def nf4_delta() -> float:
    return float(lib().oracle_nf4_delta())


def nf4_codebook() -> np.ndarray:
    q = np.zeros(16, np.float32)
    lib().oracle_nf4_codebook(_p(q))
    return q


QTYPES = ("nf4", "fp4", "int4")


def e2m1_decode(bits: int) -> float:
    return float(lib().oracle_e2m1_decode(int(bits)))


def codebook(qtype: str = "nf4") -> np.ndarray:
    """The 16-entry table of a 4-bit type: "nf4", "fp4" (OCP E2M1 / 6) or
    "int4" (k / 7)."""
    q = np.zeros(16, np.float32)
    fn = {"nf4": lib().oracle_nf4_codebook, "fp4": lib().oracle_fp4_codebook,
          "int4": lib().oracle_int4_codebook}[qtype]
    fn(_p(q))
    return q


# -- a2, a3 ----------------------------------------------------------------
def quantize_nf4(w, block: int = 64, qtype: str = "nf4"):
    """Returns (codes uint8[ceil(n/2)], c2 fp32[ceil(n/64)], status)."""
    w = _f32(w).reshape(-1)
    n = w.size
    nb = (n + block - 1) // block
    codes = np.zeros((n + 1) // 2, np.uint8)
    c2 = np.zeros(nb, np.float32)
    q = codebook(qtype)
    st = lib().oracle_quantize_nf4(_p(w), n, block, _p(q), _p(codes), _p(c2))
    return codes, c2, int(st)


# -- a4 --------------------------------------------------------------------
def mean_exact(c2):
    """Returns (mu fp32, RN64 of the exact sum, status)."""
    c2 = _f32(c2).reshape(-1)
    mu = np.zeros(1, np.float32)
    s = np.zeros(1, np.float64)
    st = lib().oracle_mean_exact(_p(c2), c2.size, _p(mu), _p(s))
    return np.float32(mu[0]), float(s[0]), int(st)


# -- FP8 -------------------------------------------------------------------
def e4m3_encode(x) -> np.ndarray:
    x = _f32(x).reshape(-1)
    out = np.zeros(x.size, np.uint8)
    lib().oracle_e4m3_encode_array(_p(x), x.size, _p(out))
    return out


def e4m3_decode(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint8).reshape(-1)
    L = lib()
    return np.array([L.oracle_e4m3_decode(int(v)) for v in b], dtype=np.float32)


def bf16_rne(x) -> np.ndarray:
    x = _f32(x)
    out = np.zeros(x.shape, np.uint16)
    lib().oracle_bf16_rne_array(_p(x), x.size, _p(out))
    return out


# -- a5 --------------------------------------------------------------------
def double_quant(c2, mu, block2: int = 256):
    c2 = _f32(c2).reshape(-1)
    nb = c2.size
    ng = (nb + block2 - 1) // block2
    b = np.zeros(nb, np.uint8)
    c1 = np.zeros(ng, np.float32)
    lib().oracle_double_quant(_p(c2), nb, ctypes.c_float(mu), block2, _p(b), _p(c1))
    return b, c1


def quantize_nf4_dq(w, block: int = 64, block2: int = 256, qtype: str = "nf4"):
    """The full quantization of one frozen weight: a2-a5.

    Returns a dict with codes, c2_fp8, c1, mean, and the intermediate c2."""
    codes, c2, st = quantize_nf4(w, block, qtype)
    mu, _, st2 = mean_exact(c2)
    b, c1 = double_quant(c2, mu, block2)
    return {"codes": codes, "c2_fp8": b, "c1": c1, "mean": np.float32(mu), "c2": c2,
            "status": st if st else st2}


# -- a6, a7 ----------------------------------------------------------------
def dequant_constants(c2_fp8, c1, mu, block2: int = 256) -> np.ndarray:
    b = np.ascontiguousarray(c2_fp8, np.uint8)
    c1 = _f32(c1)
    out = np.zeros(b.size, np.float32)
    lib().oracle_dequant_constants(_p(b), _p(c1), ctypes.c_float(mu), b.size, block2, _p(out))
    return out


def dequantize(codes, c2_fp8, c1, mu, numel: int, block: int = 64, block2: int = 256, qtype: str = "nf4"):
    codes = np.ascontiguousarray(codes, np.uint8)
    b = np.ascontiguousarray(c2_fp8, np.uint8)
    c1 = _f32(c1)
    q = codebook(qtype)
    out = np.zeros(numel, np.float32)
    lib().oracle_dequantize(_p(codes), _p(b), _p(c1), ctypes.c_float(mu), numel, block, block2,
                            _p(q), _p(out))
    return out


# -- a8 - a10 --------------------------------------------------------------
def linear_fwd(X, W_bf16, A, B, s, rows=None):
    """Y (fp64, len(rows) x N) and T0 = X A^T (fp64) for the selected rows."""
    X, W, A, B = _u16(X), _u16(W_bf16), _u16(A), _u16(B)
    M, K = X.shape
    N = W.shape[0]
    r = A.shape[0]
    rr = None if rows is None else np.ascontiguousarray(rows, np.int64)
    nr = M if rr is None else rr.size
    Y = np.zeros((nr, N), np.float64)
    T0 = np.zeros((nr, r), np.float64)
    st = lib().oracle_linear_fwd(_p(X), M, N, K, _p(W), _p(A), _p(B), r, float(s), _p(rr), nr,
                                 _p(Y), _p(T0))
    assert st == OK
    return Y, T0


def linear_bwd(dY, X, W_bf16, A, B, s, rows=None, want_dx=True):
    """dX (fp64, selected rows), dA (r x K), dB (N x r)."""
    dY, X, W, A, B = _u16(dY), _u16(X), _u16(W_bf16), _u16(A), _u16(B)
    M, K = X.shape
    N = W.shape[0]
    r = A.shape[0]
    rr = None if rows is None else np.ascontiguousarray(rows, np.int64)
    nr = M if rr is None else rr.size
    dX = np.zeros((nr, K), np.float64) if want_dx else None
    dA = np.zeros((r, K), np.float64)
    dB = np.zeros((N, r), np.float64)
    st = lib().oracle_linear_bwd(_p(dY), _p(X), M, N, K, _p(W), _p(A), _p(B), r, float(s),
                                 _p(rr), nr, _p(dX), _p(dA), _p(dB))
    assert st == OK
    return dX, dA, dB


# -- eq. 1 / eq. 2 (Int8, not on the NF4 path) -----------------------------
def int8_quant(x):
    x = _f32(x).reshape(-1)
    out = np.zeros(x.size, np.int8)
    c = np.zeros(1, np.float32)
    lib().oracle_int8_quant(_p(x), x.size, _p(out), _p(c))
    return out, np.float32(c[0])


def int8_dequant(xq, c):
    xq = np.ascontiguousarray(xq, np.int8)
    out = np.zeros(xq.size, np.float32)
    lib().oracle_int8_dequant(_p(xq), xq.size, ctypes.c_float(c), _p(out))
    return out


def int8_quant_blocks(x, block: int = 64):
    """Eq. (1) on consecutive blocks: (codes int8[n], c fp32[ceil(n/block)])."""
    x = _f32(x).reshape(-1)
    nb = (x.size + block - 1) // block
    out = np.zeros(x.size, np.int8)
    c = np.zeros(max(nb, 1), np.float32)
    lib().oracle_int8_quant_blocks(_p(x), x.size, block, _p(out), _p(c))
    return out, c[:nb]


def int8_dequant_blocks(xq, c, block: int = 64):
    """Eq. (2) on consecutive blocks."""
    xq = np.ascontiguousarray(xq, np.int8).reshape(-1)
    c = _f32(c)
    out = np.zeros(xq.size, np.float32)
    lib().oracle_int8_dequant_blocks(_p(xq), xq.size, block, _p(c), _p(out))
    return out

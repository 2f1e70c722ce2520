"""CPU oracle for the quantized linear layers (q8 / q4 weight-only, W8A8).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The CUDA product
path (``int8_int4_b200``) never imports it and shares no code with it.

The arithmetic lives in ``aria_oracle.c`` (plain C, fp64 GEMMs, fp32 IEEE
quotients, round-half-even); this module only marshals numpy arrays through
ctypes. Citations are to "A Quantized Native Runtime for On-Device Semantic
Audio Generation" (aria project page): "What aria is" (weights packed from
fp16 to 8 or 4 bits, the fp16 copy released), "Results" (the fp16 / q8 /
W8A8 / q4 table; W8A8 is 8-bit arithmetic on integer tensor cores) and
"Steering is real" (a direction added at one block, bit-identical at
alpha = 0). The unquantised fp16 rung of the "Results" table has a reference
too (``f16_ref``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "aria_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``aria_oracle.c`` into ``liboracle.so`` (gcc), if stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # ARIA_ORACLE_LIB: a separately compiled oracle library, used by the
            # mutation tests to run the pins against a copy with a planted mistake
            lib = ctypes.CDLL(os.environ.get("ARIA_ORACLE_LIB") or build())
            P, I64, F32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float
            sigs = {
                "orc_half_to_double": ([ctypes.c_uint16], ctypes.c_double),
                "orc_double_to_half": ([ctypes.c_double], ctypes.c_uint16),
                "orc_half_to_double_n": ([P, I64, P], None),
                "orc_double_to_half_n": ([P, I64, P], None),
                "orc_float_to_half_n": ([P, I64, P], None),
                "orc_pack_q8": ([P, I64, I64, P, P], None),
                "orc_act_quant": ([P, I64, I64, P, P], None),
                "orc_pack_q4": ([P, I64, I64, P, P], None),
                "orc_dequant_q8": ([P, P, I64, I64, P], None),
                "orc_dequant_q4": ([P, P, I64, I64, P], None),
                "orc_gemm_s32": ([P, P, I64, I64, I64, P, I64, P], ctypes.c_int),
                "orc_w8a8_out": ([P, P, P, I64, I64, P, I64, P, P, F32, P], None),
                "orc_wo_q8_ref": ([P, P, P, I64, I64, I64, P, I64, P, P, F32, P], None),
                "orc_wo_q4_ref": ([P, P, P, I64, I64, I64, P, I64, P, P, F32, P], None),
                "orc_f16_ref": ([P, P, I64, I64, I64, P, I64, P, P, F32, P], None),
            }
            for name, (args, res) in sigs.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = res
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _h(a) -> np.ndarray:
    """fp16 input as a C-contiguous uint16 bit-pattern array."""
    a = np.asarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError(f"expected float16/uint16 bits, got {a.dtype}")
    return np.ascontiguousarray(a)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(np.asarray(a, dtype=dtype))


def _rows(rows, M):
    if rows is None:
        return None, M
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    if r.size and (r.min() < 0 or r.max() >= M):
        raise IndexError("row index out of range")
    return r, r.size


# ------------------------------------------------------------------ fp16 --

def half_to_double(h) -> np.ndarray:
    """IEEE binary16 bit patterns -> float64, exact (own bit-level decode)."""
    h = _h(h)
    out = np.empty(h.shape, np.float64)
    _load().orc_half_to_double_n(_ptr(h), h.size, _ptr(out))
    return out


def double_to_half(x) -> np.ndarray:
    """float64 -> binary16 bit patterns, round to nearest even, one rounding."""
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    _load().orc_double_to_half_n(_ptr(x), x.size, _ptr(out))
    return out


def float_to_half(x) -> np.ndarray:
    """float32 -> binary16 bit patterns, round to nearest even."""
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    _load().orc_float_to_half_n(_ptr(x), x.size, _ptr(out))
    return out


# ------------------------------------------------------------------ packs --

def pack_q8(W):
    """q8 pack ("What aria is": weights from fp16 to 8 bits).

    Per output channel n: s[n] = absmax_k |W[n,k]| / 127 (fp32 quotient);
    Wq = clamp(rhe(W / s), -127, 127). Returns (Wq int8 [N,K], s fp32 [N]).
    """
    W = _h(W)
    N, K = W.shape
    Wq = np.empty((N, K), np.int8)
    s = np.empty(N, np.float32)
    _load().orc_pack_q8(_ptr(W), N, K, _ptr(Wq), _ptr(s))
    return Wq, s


def act_quant(X):
    """Per-token int8 activation quantisation (the "A8" of W8A8, "Results").

    Per token row m the q8 rule along K. Returns (Xq int8 [M,K], s_x fp32 [M]).
    """
    X = _h(X)
    M, K = X.shape
    Xq = np.empty((M, K), np.int8)
    s = np.empty(M, np.float32)
    _load().orc_act_quant(_ptr(X), M, K, _ptr(Xq), _ptr(s))
    return Xq, s


def pack_q4(W):
    """q4 group-32 pack ("What aria is": weights from fp16 to 4 bits).

    Per output channel n and group j of 32 consecutive k: s16 = fp16_rn(absmax/7),
    q = clamp(rhe(W / float(s16)), -7, 7), stored as q+8, even k in the low
    nibble. Returns (P uint8 [N,K/2], S fp16 bits uint16 [N,K/32]).
    """
    W = _h(W)
    N, K = W.shape
    if K % 32:
        raise ValueError("K must be a multiple of 32 for q4")
    P = np.zeros((N, K // 2), np.uint8)
    S = np.empty((N, K // 32), np.uint16)
    _load().orc_pack_q4(_ptr(W), N, K, _ptr(P), _ptr(S))
    return P, S


def dequant_q8(Wq, s) -> np.ndarray:
    Wq = _c(Wq, np.int8)
    s = _c(s, np.float32)
    N, K = Wq.shape
    out = np.empty((N, K), np.float64)
    _load().orc_dequant_q8(_ptr(Wq), _ptr(s), N, K, _ptr(out))
    return out


def dequant_q4(P, S) -> np.ndarray:
    P = _c(P, np.uint8)
    S = _h(S)
    N, K2 = P.shape
    out = np.empty((N, 2 * K2), np.float64)
    _load().orc_dequant_q4(_ptr(P), _ptr(S), N, 2 * K2, _ptr(out))
    return out


# ------------------------------------------------------------------ GEMMs --

def gemm_s32(Xq, Wq, rows=None) -> np.ndarray:
    """Exact int32 accumulators C[i,n] = sum_k Xq[rows[i],k]*Wq[n,k] (int64 checked)."""
    Xq = _c(Xq, np.int8)
    Wq = _c(Wq, np.int8)
    M, K = Xq.shape
    N = Wq.shape[0]
    r, R = _rows(rows, M)
    C = np.empty((R, N), np.int32)
    if _load().orc_gemm_s32(_ptr(Xq), _ptr(Wq), M, N, K, _ptr(r), R, _ptr(C)):
        raise OverflowError("int32 accumulator overflow")
    return C


def w8a8_out(C, sx, sw, bias=None, v=None, alpha=0.0, rows=None, M=None) -> np.ndarray:
    """W8A8 fp16 output bits: fp16_rn(acc*s_x[m]*s_w[n] + bias[n] + alpha*v[n]) in fp64.

    ``C`` holds the accumulators of the selected ``rows`` (all rows if None).
    """
    C = _c(C, np.int32)
    sx = _c(sx, np.float32)
    sw = _c(sw, np.float32)
    M = sx.size if M is None else M
    r, R = _rows(rows, M)
    N = sw.size
    assert C.shape == (R, N)
    Y = np.empty((R, N), np.uint16)
    _load().orc_w8a8_out(_ptr(C), _ptr(sx), _ptr(sw), M, N, _ptr(r), R,
                         _ptr(_h(bias) if bias is not None else None),
                         _ptr(_c(v, np.float32)), float(alpha), _ptr(Y))
    return Y


def w8a8(X, Wq, sw, bias=None, v=None, alpha=0.0, rows=None):
    """Whole W8A8 linear: act quant, exact int32 GEMM, fp64 epilogue -> fp16 bits."""
    Xq, sx = act_quant(X)
    C = gemm_s32(Xq, Wq, rows)
    return w8a8_out(C, sx, sw, bias, v, alpha, rows, M=Xq.shape[0])


def wo_ref(fmt, X, Wq, scales, bias=None, v=None, alpha=0.0, rows=None) -> np.ndarray:
    """Weight-only reference in fp64, not rounded: X @ dequant(W)^T + bias + alpha*v.

    fmt "q8": Wq int8 [N,K], scales fp32 [N]; fmt "q4": Wq uint8 [N,K/2], scales fp16 bits [N,K/32].
    """
    X = _h(X)
    M, K = X.shape
    r, R = _rows(rows, M)
    b = _h(bias) if bias is not None else None
    vv = _c(v, np.float32)
    lib = _load()
    if fmt == "q8":
        Wq = _c(Wq, np.int8)
        s = _c(scales, np.float32)
        N = Wq.shape[0]
        Y = np.empty((R, N), np.float64)
        lib.orc_wo_q8_ref(_ptr(X), _ptr(Wq), _ptr(s), M, N, K, _ptr(r), R,
                          _ptr(b), _ptr(vv), float(alpha), _ptr(Y))
    elif fmt == "q4":
        Wq = _c(Wq, np.uint8)
        S = _h(scales)
        N = Wq.shape[0]
        Y = np.empty((R, N), np.float64)
        lib.orc_wo_q4_ref(_ptr(X), _ptr(Wq), _ptr(S), M, N, K, _ptr(r), R,
                          _ptr(b), _ptr(vv), float(alpha), _ptr(Y))
    else:
        raise ValueError(fmt)
    return Y


def f16_ref(X, W, bias=None, v=None, alpha=0.0, rows=None) -> np.ndarray:
    """Unquantised fp16 reference ("Results": the fp16 column) in fp64, not
    rounded: X @ W^T + bias + alpha*v with X [M,K] and W [N,K] fp16."""
    X = _h(X)
    W = _h(W)
    M, K = X.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("W must be [N, K]")
    r, R = _rows(rows, M)
    Y = np.empty((R, N), np.float64)
    _load().orc_f16_ref(_ptr(X), _ptr(W), M, N, K, _ptr(r), R,
                        _ptr(_h(bias) if bias is not None else None), _ptr(_c(v, np.float32)),
                        float(alpha), _ptr(Y))
    return Y

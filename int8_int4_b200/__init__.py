"""Python binding of libaria_q.so: quantized linear layers for B200 (sm_100a).

Argument marshalling only. Every step of the path -- packing, activation
quantisation, the GEMMs and their epilogue -- runs in the library's CUDA
kernels; PyTorch provides device memory and streams. There is no CPU
fallback: if the library is missing or the tensors are not on a CUDA device,
the calls raise.

Method: "A Quantized Native Runtime for On-Device Semantic Audio Generation"
(aria project page): "What aria is" (weights packed from fp16 to 8 or 4
bits), "Results" (q8, W8A8 on integer tensor cores, q4), "Steering is real"
(a direction added at one block, bit-identical at alpha = 0). Formats and
argument rules are documented in include/aria_q.h.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libaria_q.so")

ARIA_OK = 0
STATUS = {0: "ARIA_OK", 1: "ARIA_ERR_INVALID_ARG", 2: "ARIA_ERR_UNSUPPORTED",
          3: "ARIA_ERR_MISALIGNED", 4: "ARIA_ERR_CUDA", 5: "ARIA_ERR_TIMEOUT"}
FORMATS = {"q8": 1, "q4": 2, "w8a8": 3}
API = ("aria_status_string", "aria_last_error_message", "aria_qpack_size", "aria_qpack",
       "aria_act_quant", "aria_qgemm", "aria_qgemm_s32", "aria_device_status")


class AriaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libaria_q.so (built by ``python -m int8_int4_b200.build``)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m int8_int4_b200.build`")
    lib = ctypes.CDLL(path)
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    sig = {
        "aria_status_string": ([I], ctypes.c_char_p),
        "aria_last_error_message": ([], ctypes.c_char_p),
        "aria_qpack_size": ([I, I, I64, I64, P, P], I),
        "aria_qpack": ([I, I, P, I64, I64, P, P, P], I),
        "aria_act_quant": ([P, I64, I64, P, P, P], I),
        "aria_qgemm": ([I, I, I64, I64, I64, P, P, P, P, P, P, ctypes.c_float, P, P], I),
        "aria_qgemm_s32": ([I64, I64, I64, P, P, P, P], I),
        "aria_device_status": ([P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    if path == LIB_PATH:
        _lib = lib
    return lib


def _check(status: int):
    if status != ARIA_OK:
        msg = load_library().aria_last_error_message().decode()
        raise AriaError(status, msg)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor | None, name: str, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _group(fmt: str, group):
    return (32 if fmt == "q4" else 0) if group is None else int(group)


def _expect(t, name: str, shape, dtype):
    """Shape and dtype of an argument (checked before anything reaches the device:
    the C ABI takes raw pointers and cannot see a too-small buffer)."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def check_gemm_args(fmt: str, X, Wq, scales, sx=None, bias=None, steer_vec=None, out=None):
    """The tensors of one GEMM call agree with each other and with the format
    (include/aria_q.h): X [M,K] (fp16; int8 for W8A8), Wq [N,K] int8 (q8, W8A8)
    or [N,K/2] uint8 (q4), scales fp32 [N] (q8, W8A8) or fp16 [N,K/32] (q4),
    sx fp32 [M] (W8A8 only), bias fp16 [N], steer_vec fp32 [N], out fp16 [M,N].
    Returns (M, N, K)."""
    if fmt not in FORMATS:
        raise ValueError(f"unknown format {fmt!r}")
    if X.dim() != 2 or Wq.dim() != 2:
        raise ValueError("X and Wq must be 2-D")
    M, K = X.shape
    N = Wq.shape[0]
    _expect(X, "X", (M, K), torch.int8 if fmt == "w8a8" else torch.float16)
    if fmt == "q4":
        if K % 32:
            raise ValueError("q4 needs K % 32 == 0")
        _expect(Wq, "Wq", (N, K // 2), torch.uint8)
        _expect(scales, "scales", (N, K // 32), torch.float16)
    else:
        _expect(Wq, "Wq", (N, K), torch.int8)
        _expect(scales, "scales", (N,), torch.float32)
    if fmt == "w8a8":
        if sx is None:
            raise ValueError("w8a8 needs sx")
        _expect(sx, "sx", (M,), torch.float32)
    elif sx is not None:
        raise ValueError("sx is for w8a8 only")
    _expect(bias, "bias", (N,), torch.float16)
    _expect(steer_vec, "steer_vec", (N,), torch.float32)
    _expect(out, "out", (M, N), torch.float16)
    return M, N, K


def qpack_size(fmt: str, N: int, K: int, group=None):
    wb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(load_library().aria_qpack_size(FORMATS[fmt], _group(fmt, group), N, K,
                                          ctypes.byref(wb), ctypes.byref(sb)))
    return wb.value, sb.value


def qpack(fmt: str, W: torch.Tensor, group=None, stream=None):
    """Pack fp16 W [N,K]: q8/w8a8 -> (int8 [N,K], fp32 [N]); q4 -> (uint8 [N,K/2], fp16 [N,K/32])."""
    N, K = W.shape
    g = _group(fmt, group)
    qpack_size(fmt, N, K, g)
    if fmt == "q4":
        Wq = torch.empty(N, K // 2, dtype=torch.uint8, device=W.device)
        S = torch.empty(N, K // 32, dtype=torch.float16, device=W.device)
    else:
        Wq = torch.empty(N, K, dtype=torch.int8, device=W.device)
        S = torch.empty(N, dtype=torch.float32, device=W.device)
    _check(load_library().aria_qpack(FORMATS[fmt], g, _dev(W, "W", torch.float16), N, K,
                                     Wq.data_ptr(), S.data_ptr(), _stream(stream)))
    return Wq, S


def act_quant(X: torch.Tensor, out=None, stream=None):
    """Per-token int8 quantisation of fp16 X [M,K] -> (Xq int8 [M,K], s_x fp32 [M])."""
    M, K = X.shape
    Xq, sx = out if out is not None else (
        torch.empty(M, K, dtype=torch.int8, device=X.device),
        torch.empty(M, dtype=torch.float32, device=X.device))
    _expect(Xq, "Xq", (M, K), torch.int8)
    _expect(sx, "sx", (M,), torch.float32)
    _check(load_library().aria_act_quant(_dev(X, "X", torch.float16), M, K,
                                         _dev(Xq, "Xq", torch.int8), _dev(sx, "sx", torch.float32),
                                         _stream(stream)))
    return Xq, sx


def qgemm(fmt: str, X: torch.Tensor, Wq: torch.Tensor, scales: torch.Tensor, sx=None,
          bias=None, steer_vec=None, alpha: float = 0.0, group=None, out=None, stream=None):
    """Y [M,N] fp16 = X . dequant(W)^T + bias + alpha*v (see include/aria_q.h)."""
    M, N, K = check_gemm_args(fmt, X, Wq, scales, sx, bias, steer_vec, out)
    Y = out if out is not None else torch.empty(M, N, dtype=torch.float16, device=X.device)
    xdt = torch.int8 if fmt == "w8a8" else torch.float16
    _check(load_library().aria_qgemm(
        FORMATS[fmt], _group(fmt, group), M, N, K, _dev(X, "X", xdt),
        _dev(sx, "sx", torch.float32), _dev(Wq, "Wq"), _dev(scales, "scales"),
        _dev(bias, "bias", torch.float16), _dev(steer_vec, "steer_vec", torch.float32),
        float(alpha), _dev(Y, "out"), _stream(stream)))
    return Y


def qgemm_s32(Xq: torch.Tensor, Wq: torch.Tensor, out=None, stream=None):
    """Raw int32 accumulators C [M,N] = Xq . Wq^T on the integer tensor cores."""
    M, K = Xq.shape
    N = Wq.shape[0]
    _expect(Wq, "Wq", (N, K), torch.int8)
    C = out if out is not None else torch.empty(M, N, dtype=torch.int32, device=Xq.device)
    _expect(C, "out", (M, N), torch.int32)
    _check(load_library().aria_qgemm_s32(M, N, K, _dev(Xq, "Xq", torch.int8),
                                         _dev(Wq, "Wq", torch.int8), _dev(C, "out", torch.int32),
                                         _stream(stream)))
    return C


def device_status(stream=None):
    """Synchronise the stream and raise if a kernel's bounded wait ran out."""
    _check(load_library().aria_device_status(_stream(stream)))

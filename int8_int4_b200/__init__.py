"""Python binding of libaria_q.so: quantized linear layers for B200 (sm_100a).

Argument marshalling only. Every step of the path -- packing, activation
quantisation, the GEMMs and their epilogue -- runs in the library's CUDA
kernels; PyTorch provides device memory and streams. There is no CPU
fallback: if the library is missing or the tensors are not on a CUDA device,
the calls raise.

Method: "A Quantized Native Runtime for On-Device Semantic Audio Generation"
(aria project page): "What aria is" (weights packed from fp16 to 8 or 4
bits), "Results" (fp16, q8, W8A8 on integer tensor cores, q4), "Steering is
real" (a direction added at one block, bit-identical at alpha = 0), "Live
steering while streaming" (the strength lives inside the captured graph) and
"Run it" (the steer spec site:block:file:alpha:steps). Formats and argument
rules are documented in include/aria_q.h.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libaria_q.so")

ARIA_OK = 0
STATUS = {0: "ARIA_OK", 1: "ARIA_ERR_INVALID_ARG", 2: "ARIA_ERR_UNSUPPORTED",
          3: "ARIA_ERR_MISALIGNED", 4: "ARIA_ERR_CUDA", 5: "ARIA_ERR_TIMEOUT"}
FORMATS = {"q8": 1, "q4": 2, "w8a8": 3, "f16": 4}
API = ("aria_status_string", "aria_last_error_message", "aria_qpack_size", "aria_qpack",
       "aria_act_quant", "aria_qgemm", "aria_qgemm_steer_dev", "aria_w8a8_workspace_size",
       "aria_qgemm_w8a8_fused", "aria_qgemm_w8a8_fused_noalloc", "aria_qgemm_s32",
       "aria_selftest_bounded_wait", "aria_device_status")


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
        "aria_qgemm_steer_dev": ([I, I, I64, I64, I64, P, P, P, P, P, P, P, P, P], I),
        "aria_w8a8_workspace_size": ([I64, I64, P], I),
        "aria_qgemm_w8a8_fused": ([I64, I64, I64, P, P, P, P, P, ctypes.c_float, P, P, P,
                                   ctypes.c_size_t, P], I),
        "aria_qgemm_w8a8_fused_noalloc": ([I64, I64, I64, P, P, P, P, P, ctypes.c_float, P, P, P], I),
        "aria_qgemm_s32": ([I64, I64, I64, P, P, P, P], I),
        "aria_selftest_bounded_wait": ([I64, I64, I64, P, P, P, P, P, ctypes.c_uint32, P], I),
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


def same_device(**tensors):
    """Every given tensor (None skipped) on one device; returns it. The library
    launches on the current device and encodes tensor maps from raw pointers,
    so a tensor on another GPU would be read through the wrong device."""
    dev = None
    for name, t in tensors.items():
        if t is None:
            continue
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the other arguments on {dev}")
    return dev


@contextlib.contextmanager
def _on(dev):
    """Make `dev` the current CUDA device for the library call."""
    if dev is not None and dev.type == "cuda":
        with torch.cuda.device(dev):
            yield
    else:
        yield


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


def check_gemm_args(fmt: str, X, Wq, scales, sx=None, bias=None, steer_vec=None, out=None,
                    alpha_dev=None):
    """The tensors of one GEMM call agree with each other and with the format
    (include/aria_q.h): X [M,K] (fp16; int8 for W8A8), Wq [N,K] int8 (q8, W8A8)
    or [N,K/2] uint8 (q4) or the fp16 weight [N,K] itself (f16), scales fp32
    [N] (q8, W8A8) or fp16 [N,K/32] (q4) or None (f16), sx fp32 [M] (W8A8
    only), bias fp16 [N], steer_vec fp32 [N], alpha_dev one fp32 element,
    out fp16 [M,N], all on one device. Returns (M, N, K)."""
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
    elif fmt == "f16":
        _expect(Wq, "W", (N, K), torch.float16)
        if scales is not None:
            raise ValueError("f16 weights take no scales")
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
    if alpha_dev is not None:
        if alpha_dev.numel() != 1 or alpha_dev.dtype != torch.float32:
            raise TypeError("alpha_dev must be one float32 element")
    _expect(out, "out", (M, N), torch.float16)
    same_device(X=X, Wq=Wq, scales=scales, sx=sx, bias=bias, steer_vec=steer_vec, out=out,
                alpha_dev=alpha_dev)
    return M, N, K


def qpack_size(fmt: str, N: int, K: int, group=None):
    wb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(load_library().aria_qpack_size(FORMATS[fmt], _group(fmt, group), N, K,
                                          ctypes.byref(wb), ctypes.byref(sb)))
    return wb.value, sb.value


def qpack(fmt: str, W: torch.Tensor, group=None, stream=None, out=None):
    """Pack fp16 W [N,K]: q8/w8a8 -> (int8 [N,K], fp32 [N]); q4 -> (uint8 [N,K/2], fp16 [N,K/32]).
    ``out`` = (Wq, scales) writes into existing tensors of those shapes."""
    N, K = W.shape
    g = _group(fmt, group)
    qpack_size(fmt, N, K, g)
    q4 = fmt == "q4"
    shapes = ((N, K // 2), (N, K // 32)) if q4 else ((N, K), (N,))
    dtypes = (torch.uint8, torch.float16) if q4 else (torch.int8, torch.float32)
    if out is None:
        Wq = torch.empty(*shapes[0], dtype=dtypes[0], device=W.device)
        S = torch.empty(*shapes[1], dtype=dtypes[1], device=W.device)
    else:
        Wq, S = out
        _expect(Wq, "Wq", shapes[0], dtypes[0])
        _expect(S, "scales", shapes[1], dtypes[1])
        same_device(W=W, Wq=Wq, scales=S)
    with _on(W.device):
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
    dev = same_device(X=X, Xq=Xq, sx=sx)
    with _on(dev):
        _check(load_library().aria_act_quant(_dev(X, "X", torch.float16), M, K,
                                             _dev(Xq, "Xq", torch.int8), _dev(sx, "sx", torch.float32),
                                             _stream(stream)))
    return Xq, sx


def qgemm(fmt: str, X: torch.Tensor, Wq: torch.Tensor, scales, sx=None,
          bias=None, steer_vec=None, alpha: float = 0.0, group=None, out=None, stream=None,
          alpha_dev=None):
    """Y [M,N] fp16 = X . dequant(W)^T + bias + alpha*v (see include/aria_q.h).

    fmt "f16" takes the fp16 weight [N,K] as Wq and scales=None. With
    ``alpha_dev`` (one fp32 element on the device, e.g. ``schedule[s:s+1]``)
    the strength is read from device memory when the kernel runs
    (aria_qgemm_steer_dev) and ``alpha`` is ignored."""
    if fmt != "f16" and scales is None:
        raise ValueError(f"{fmt} needs scales")
    M, N, K = check_gemm_args(fmt, X, Wq, scales, sx, bias, steer_vec, out, alpha_dev)
    Y = out if out is not None else torch.empty(M, N, dtype=torch.float16, device=X.device)
    xdt = torch.int8 if fmt == "w8a8" else torch.float16
    lib = load_library()
    args = (FORMATS[fmt], _group(fmt, group), M, N, K, _dev(X, "X", xdt),
            _dev(sx, "sx", torch.float32), _dev(Wq, "Wq"), _dev(scales, "scales"),
            _dev(bias, "bias", torch.float16), _dev(steer_vec, "steer_vec", torch.float32))
    with _on(X.device):
        if alpha_dev is not None:
            if not alpha_dev.is_cuda:
                raise ValueError("alpha_dev must be a CUDA tensor")
            _check(lib.aria_qgemm_steer_dev(*args, alpha_dev.data_ptr(), _dev(Y, "out"),
                                            _stream(stream)))
        else:
            _check(lib.aria_qgemm(*args, float(alpha), _dev(Y, "out"), _stream(stream)))
    return Y


def w8a8_workspace_size(M: int, K: int) -> int:
    n = ctypes.c_size_t()
    _check(load_library().aria_w8a8_workspace_size(M, K, ctypes.byref(n)))
    return n.value


def w8a8_workspace(M: int, K: int, device=None) -> torch.Tensor:
    """A zero-filled workspace for qgemm_w8a8_fused (uint8, 256-byte aligned:
    the caching allocator's blocks are)."""
    ws = torch.zeros(w8a8_workspace_size(M, K), dtype=torch.uint8, device=device)
    if ws.data_ptr() % 256:
        raise RuntimeError("workspace is not 256-byte aligned")
    return ws


def workspace_codes(ws: torch.Tensor, M: int, K: int):
    """Views of the token scales fp32 [M] and codes int8 [M,K] that a fused
    call leaves in its workspace (the layout of include/aria_q.h)."""
    sx_bytes = (4 * M + 255) // 256 * 256
    sx = ws[256:256 + 4 * M].view(torch.float32)
    xq = ws[256 + sx_bytes:256 + sx_bytes + M * K].view(torch.int8).view(M, K)
    return xq, sx


def qgemm_w8a8_fused(X: torch.Tensor, Wq: torch.Tensor, sw: torch.Tensor, bias=None, steer_vec=None,
                     alpha: float = 0.0, alpha_dev=None, out=None, workspace=None, stream=None):
    """W8A8 from fp16 X [M,K] in one launch: per-token quantisation inside the
    GEMM kernel (include/aria_q.h, aria_qgemm_w8a8_fused). ``workspace``: a
    zero-filled uint8 tensor of w8a8_workspace_size(M, K) bytes (see
    w8a8_workspace); calls sharing one must not overlap on the GPU."""
    M, K = X.shape
    N = Wq.shape[0]
    _expect(X, "X", (M, K), torch.float16)
    _expect(Wq, "Wq", (N, K), torch.int8)
    _expect(sw, "scales", (N,), torch.float32)
    _expect(bias, "bias", (N,), torch.float16)
    _expect(steer_vec, "steer_vec", (N,), torch.float32)
    if alpha_dev is not None and (alpha_dev.numel() != 1 or alpha_dev.dtype != torch.float32):
        raise TypeError("alpha_dev must be one float32 element")
    Y = out if out is not None else torch.empty(M, N, dtype=torch.float16, device=X.device)
    _expect(Y, "out", (M, N), torch.float16)
    if workspace is None:
        raise ValueError("qgemm_w8a8_fused needs a workspace (w8a8_workspace(M, K, device))")
    if workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise TypeError("workspace must be a contiguous uint8 tensor")
    same_device(X=X, Wq=Wq, scales=sw, bias=bias, steer_vec=steer_vec, out=Y, workspace=workspace,
                alpha_dev=alpha_dev)
    with _on(X.device):
        _check(load_library().aria_qgemm_w8a8_fused(
            M, N, K, _dev(X, "X", torch.float16), _dev(Wq, "Wq", torch.int8), _dev(sw, "scales"),
            _dev(bias, "bias", torch.float16), _dev(steer_vec, "steer_vec", torch.float32),
            float(alpha), None if alpha_dev is None else _dev(alpha_dev, "alpha_dev"),
            _dev(Y, "out"), _dev(workspace, "workspace"), workspace.numel(), _stream(stream)))
    return Y


def qgemm_w8a8_fused_noalloc(X: torch.Tensor, Wq: torch.Tensor, sw: torch.Tensor, bias=None,
                             steer_vec=None, alpha: float = 0.0, alpha_dev=None, out=None, stream=None):
    """qgemm_w8a8_fused with the library's static scratch instead of a
    workspace, for callers that must not allocate device memory while they
    run (include/aria_q.h, aria_qgemm_w8a8_fused_noalloc). ``out`` must be
    given: this call allocates nothing, not even its output."""
    M, K = X.shape
    N = Wq.shape[0]
    if out is None:
        raise ValueError("qgemm_w8a8_fused_noalloc allocates nothing: pass out=")
    _expect(X, "X", (M, K), torch.float16)
    _expect(Wq, "Wq", (N, K), torch.int8)
    _expect(sw, "scales", (N,), torch.float32)
    _expect(bias, "bias", (N,), torch.float16)
    _expect(steer_vec, "steer_vec", (N,), torch.float32)
    _expect(out, "out", (M, N), torch.float16)
    if alpha_dev is not None and (alpha_dev.numel() != 1 or alpha_dev.dtype != torch.float32):
        raise TypeError("alpha_dev must be one float32 element")
    same_device(X=X, Wq=Wq, scales=sw, bias=bias, steer_vec=steer_vec, out=out, alpha_dev=alpha_dev)
    with _on(X.device):
        _check(load_library().aria_qgemm_w8a8_fused_noalloc(
            M, N, K, _dev(X, "X", torch.float16), _dev(Wq, "Wq", torch.int8), _dev(sw, "scales"),
            _dev(bias, "bias", torch.float16), _dev(steer_vec, "steer_vec", torch.float32),
            float(alpha), None if alpha_dev is None else _dev(alpha_dev, "alpha_dev"),
            _dev(out, "out"), _stream(stream)))
    return out


def qgemm_s32(Xq: torch.Tensor, Wq: torch.Tensor, out=None, stream=None):
    """Raw int32 accumulators C [M,N] = Xq . Wq^T on the integer tensor cores."""
    M, K = Xq.shape
    N = Wq.shape[0]
    _expect(Wq, "Wq", (N, K), torch.int8)
    C = out if out is not None else torch.empty(M, N, dtype=torch.int32, device=Xq.device)
    _expect(C, "out", (M, N), torch.int32)
    dev = same_device(Xq=Xq, Wq=Wq, out=C)
    with _on(dev):
        _check(load_library().aria_qgemm_s32(M, N, K, _dev(Xq, "Xq", torch.int8),
                                             _dev(Wq, "Wq", torch.int8), _dev(C, "out", torch.int32),
                                             _stream(stream)))
    return C


def selftest_bounded_wait(Xq, sx, Wq, sw, out=None, wait_limit_us: int = 50000, stream=None):
    """Failure-detection self-test (include/aria_q.h): a W8A8 launch whose
    first pipeline stage never fills, with every bounded wait limited to
    wait_limit_us. Returns the output tensor (contents unspecified); the
    following device_status() raises AriaError with ARIA_ERR_TIMEOUT."""
    M, K = Xq.shape
    N = Wq.shape[0]
    _expect(sx, "sx", (M,), torch.float32)
    _expect(Wq, "Wq", (N, K), torch.int8)
    _expect(sw, "scales", (N,), torch.float32)
    Y = out if out is not None else torch.empty(M, N, dtype=torch.float16, device=Xq.device)
    _expect(Y, "out", (M, N), torch.float16)
    same_device(Xq=Xq, sx=sx, Wq=Wq, sw=sw, out=Y)
    with _on(Xq.device):
        _check(load_library().aria_selftest_bounded_wait(
            M, N, K, _dev(Xq, "Xq", torch.int8), _dev(sx, "sx", torch.float32), _dev(Wq, "Wq", torch.int8),
            _dev(sw, "scales", torch.float32), _dev(Y, "out"), int(wait_limit_us), _stream(stream)))
    return Y


def device_status(stream=None):
    """Synchronise the stream and raise if a kernel's bounded wait ran out."""
    _check(load_library().aria_device_status(_stream(stream)))


# ------------------------------------------------------- steering schedule --

def parse_steer_spec(spec: str) -> dict:
    """Parse a steer spec ``site:block:file:alpha:steps`` ("Run it", e.g.
    ``residual:19:directions/small/sour.atns:0.1:0-7``) into its fields.
    ``steps`` is an inclusive range ``a-b`` or a single step ``a``. The file
    is only named here: the direction itself is passed to the GEMM as a
    device vector. Raises ValueError on a malformed spec."""
    parts = spec.split(":")
    if len(parts) != 5:
        raise ValueError(f"steer spec needs 5 fields site:block:file:alpha:steps, got {spec!r}")
    site, block, path, alpha, steps = parts
    if not site:
        raise ValueError("empty steering site")
    try:
        block_i = int(block)
        alpha_f = float(alpha)
    except ValueError as e:
        raise ValueError(f"bad block or alpha in {spec!r}") from e
    if block_i < 0:
        raise ValueError("block must be >= 0")
    a, sep, b = steps.partition("-")
    try:
        s0 = int(a)
        s1 = int(b) if sep else s0
    except ValueError as e:
        raise ValueError(f"bad step range {steps!r}") from e
    if s0 < 0 or s1 < s0:
        raise ValueError(f"bad step range {steps!r}")
    return {"site": site, "block": block_i, "file": path, "alpha": alpha_f, "steps": (s0, s1)}


def steer_schedule(spec, n_steps: int) -> list:
    """Per-step strengths of a steer spec (a string or parse_steer_spec's
    dict): alpha inside the inclusive step window, 0.0 outside it (a zero
    strength skips the add, so those steps are bit-identical to unsteered
    ones). Feed it to a device tensor read through ``alpha_dev``."""
    d = parse_steer_spec(spec) if isinstance(spec, str) else spec
    s0, s1 = d["steps"]
    return [d["alpha"] if s0 <= s < s1 + 1 else 0.0 for s in range(n_steps)]

"""Host-only checks of the C ABI (no GPU needed, no kernel launched).

- libaria_q.so loads and exports every function declared in include/aria_q.h;
- argument validation rejects bad calls before touching CUDA.
"""
import ctypes
import os
import re
import subprocess

import pytest

import int8_int4_b200 as aq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "aria_q.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(aria_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from int8_int4_b200 import build
    build.build()
    return aq.load_library()


def test_header_declares_the_api():
    assert set(_declared()) == set(aq.API)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", aq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)$", out, flags=re.M))
    for name in _declared():
        assert name in exported, name
        assert getattr(lib, name)
    # nothing else leaks out with default visibility
    assert {e for e in exported if e.startswith("aria_")} == set(_declared())


def test_status_strings(lib):
    for code, name in aq.STATUS.items():
        assert lib.aria_status_string(code).decode() == name


def test_qpack_size(lib):
    assert aq.qpack_size("q8", 3072, 1024) == (3072 * 1024, 3072 * 4)
    assert aq.qpack_size("w8a8", 1536, 6144) == (1536 * 6144, 1536 * 4)
    assert aq.qpack_size("q4", 6144, 1536) == (6144 * 768, 6144 * 48 * 2)
    with pytest.raises(aq.AriaError) as e:
        aq.qpack_size("q4", 16, 48)
    assert e.value.status == 2
    with pytest.raises(aq.AriaError) as e:
        aq.qpack_size("q4", 16, 64, group=64)
    assert e.value.status == 2
    with pytest.raises(aq.AriaError) as e:
        aq.qpack_size("q8", 0, 64)
    assert e.value.status == 1


def test_validation_before_launch(lib):
    P = ctypes.c_void_p
    # NULL pointers
    assert lib.aria_qgemm(1, 0, 4, 16, 16, None, None, None, None, None, None, 0.0, None, None) == 1
    assert lib.aria_act_quant(None, 4, 16, None, None, None) == 1
    assert lib.aria_qpack(1, 0, None, 16, 16, None, None, None) == 1
    # misaligned (fake, never dereferenced: the check runs first)
    bad = P(0x1001)
    ok = P(0x10000)
    assert lib.aria_qgemm(1, 0, 4, 16, 16, bad, None, ok, ok, None, None, 0.0, ok, None) == 3
    assert lib.aria_act_quant(ok, 4, 16, bad, ok, None) == 3
    # format / argument rules
    assert lib.aria_qgemm(3, 0, 4, 16, 16, ok, None, ok, ok, None, None, 0.0, ok, None) == 1  # W8A8 w/o sx
    assert lib.aria_qgemm(1, 0, 4, 16, 16, ok, ok, ok, ok, None, None, 0.0, ok, None) == 1    # sx on q8
    assert lib.aria_qgemm(2, 16, 4, 16, 256, ok, None, ok, ok, None, None, 0.0, ok, None) == 2  # group
    assert lib.aria_qgemm(9, 0, 4, 16, 16, ok, None, ok, ok, None, None, 0.0, ok, None) == 1
    assert b"sx" in lib.aria_last_error_message() or lib.aria_last_error_message()


def test_no_cpu_path():
    import torch
    with pytest.raises(ValueError):
        aq.act_quant(torch.zeros(4, 16, dtype=torch.float16))


OK_PTR = ctypes.c_void_p(0x10000)  # aligned, never dereferenced: every case below fails validation first


@pytest.mark.parametrize("fmt,group,M,N,K,status", [
    (1, 0, 0, 16, 16, 1),            # M < 1
    (1, 0, 4, 0, 16, 1),             # N < 1
    (1, 0, 4, 16, -16, 1),           # K < 1
    (1, 0, 2 ** 31, 16, 16, 1),      # a dimension >= 2^31
    (1, 0, 4, 8, 16, 2),             # N < 16
    (1, 0, 4, 24, 16, 2),            # N % 16
    (1, 0, 4, 16, 8, 2),             # K < 16
    (1, 0, 4, 16, 40, 2),            # K % 16
    (2, 32, 4, 16, 128, 2),          # q4 GEMM: K % 256
    (3, 0, 4, 16, 24, 2),            # W8A8: K % 16
    (1, 32, 4, 16, 16, 2),           # q8 takes group 0
    (2, 0, 4, 16, 256, 2),           # q4 takes group 32
])
def test_qgemm_shape_rules(lib, fmt, group, M, N, K, status):
    sx = OK_PTR if fmt == 3 else None
    assert lib.aria_qgemm(fmt, group, M, N, K, OK_PTR, sx, OK_PTR, OK_PTR, None, None, 0.0, OK_PTR,
                          None) == status
    assert lib.aria_last_error_message()


@pytest.mark.parametrize("M,N,K,status", [(0, 16, 16, 1), (4, 24, 16, 2), (4, 16, 24, 2), (4, 16, 2 ** 31, 1)])
def test_qgemm_s32_shape_rules(lib, M, N, K, status):
    assert lib.aria_qgemm_s32(M, N, K, OK_PTR, OK_PTR, OK_PTR, None) == status


@pytest.mark.parametrize("M,K,status", [(0, 16, 1), (4, 0, 1), (4, 24, 2), (2 ** 31, 16, 1)])
def test_act_quant_shape_rules(lib, M, K, status):
    assert lib.aria_act_quant(OK_PTR, M, K, OK_PTR, OK_PTR, None) == status


@pytest.mark.parametrize("fmt,group,N,K,status", [
    (1, 0, 16, 24, 2),    # q8 pack: K % 16
    (2, 32, 16, 48, 2),   # q4 pack: K % 32
    (2, 64, 16, 64, 2),   # q4 pack: group 32 only
    (1, 0, 0, 16, 1),     # N < 1
])
def test_qpack_shape_rules(lib, fmt, group, N, K, status):
    assert lib.aria_qpack(fmt, group, OK_PTR, N, K, OK_PTR, OK_PTR, None) == status


def _args(fmt, M=8, N=32, K=256):
    import torch
    X = torch.zeros(M, K, dtype=torch.int8 if fmt == "w8a8" else torch.float16)
    if fmt == "q4":
        Wq, sc = torch.zeros(N, K // 2, dtype=torch.uint8), torch.zeros(N, K // 32, dtype=torch.float16)
    else:
        Wq, sc = torch.zeros(N, K, dtype=torch.int8), torch.zeros(N, dtype=torch.float32)
    sx = torch.zeros(M, dtype=torch.float32) if fmt == "w8a8" else None
    return dict(X=X, Wq=Wq, scales=sc, sx=sx, bias=torch.zeros(N, dtype=torch.float16),
                steer_vec=torch.zeros(N, dtype=torch.float32), out=torch.zeros(M, N, dtype=torch.float16))


@pytest.mark.parametrize("fmt", ["q8", "q4", "w8a8"])
def test_binding_accepts_consistent_arguments(fmt):
    assert aq.check_gemm_args(fmt, **_args(fmt)) == (8, 32, 256)
    a = _args(fmt)
    a.update(bias=None, steer_vec=None, out=None)
    assert aq.check_gemm_args(fmt, **a) == (8, 32, 256)


@pytest.mark.parametrize("fmt,field,bad", [
    ("q8", "Wq", ("shape", (32, 128))),          # packed for another K: the kernel would read past it
    ("q8", "scales", ("shape", (16,))),
    ("q8", "X", ("dtype", "int8")),
    ("q4", "Wq", ("shape", (32, 256))),          # a q8 pack passed as q4
    ("q4", "scales", ("dtype", "float32")),
    ("w8a8", "X", ("dtype", "float16")),          # not quantised
    ("w8a8", "sx", ("shape", (4,))),
    ("w8a8", "sx", ("none", None)),
    ("q8", "sx", ("extra", None)),
    ("q8", "bias", ("shape", (16,))),
    ("q4", "steer_vec", ("dtype", "float16")),
    ("w8a8", "out", ("shape", (8, 16))),
])
def test_binding_rejects_inconsistent_arguments(fmt, field, bad):
    import torch
    a = _args(fmt)
    kind, val = bad
    if kind == "shape":
        a[field] = torch.zeros(val, dtype=a[field].dtype)
    elif kind == "dtype":
        a[field] = a[field].to(getattr(torch, val))
    elif kind == "none":
        a[field] = None
    elif kind == "extra":
        a[field] = torch.zeros(8, dtype=torch.float32)
    with pytest.raises((ValueError, TypeError)):
        aq.check_gemm_args(fmt, **a)


# ---------------------------------------------------- later argument rules --

KMAX_I8 = (2 ** 31 - 1) // (127 * 127)       # 133144: largest K whose |acc| <= K*127^2 fits int32


def test_int8_gemm_rejects_k_that_could_wrap_int32(lib):
    k_bad = (KMAX_I8 // 16 + 1) * 16             # the first multiple of 16 above the limit
    assert k_bad * 127 * 127 > 2 ** 31 - 1
    assert lib.aria_qgemm(3, 0, 4, 16, k_bad, OK_PTR, OK_PTR, OK_PTR, OK_PTR, None, None, 0.0,
                          OK_PTR, None) == 2
    assert b"K" in lib.aria_last_error_message()
    assert lib.aria_qgemm_s32(4, 16, k_bad, OK_PTR, OK_PTR, OK_PTR, None) == 2


def test_f16_format_rules(lib):
    # fp16 weights are used as they are: no pack, no scales, no groups
    with pytest.raises(aq.AriaError) as e:
        aq.qpack_size("f16", 16, 16)
    assert e.value.status == 2
    assert lib.aria_qpack(4, 0, OK_PTR, 16, 16, OK_PTR, OK_PTR, None) == 2
    assert lib.aria_qgemm(4, 0, 4, 16, 16, OK_PTR, None, OK_PTR, OK_PTR, None, None, 0.0, OK_PTR,
                          None) == 1                                        # scales given
    assert lib.aria_qgemm(4, 32, 4, 16, 16, OK_PTR, None, OK_PTR, None, None, None, 0.0, OK_PTR,
                          None) == 2                                        # a group
    assert lib.aria_qgemm(4, 0, 4, 16, 16, OK_PTR, OK_PTR, OK_PTR, None, None, None, 0.0, OK_PTR,
                          None) == 1                                        # sx
    assert lib.aria_qgemm(4, 0, 4, 24, 16, OK_PTR, None, OK_PTR, None, None, None, 0.0, OK_PTR,
                          None) == 2                                        # N % 16


def test_device_alpha_rules(lib):
    P = ctypes.c_void_p
    # a steering vector without a device alpha
    assert lib.aria_qgemm_steer_dev(1, 0, 4, 16, 16, OK_PTR, None, OK_PTR, OK_PTR, None, OK_PTR,
                                    None, OK_PTR, None) == 1
    # alpha is one fp32 value: 4-byte alignment is required, 16 is not
    assert lib.aria_qgemm_steer_dev(1, 0, 4, 16, 16, OK_PTR, None, OK_PTR, OK_PTR, None, OK_PTR,
                                    P(0x10002), OK_PTR, None) == 3
    # the aria_qgemm rules apply unchanged
    assert lib.aria_qgemm_steer_dev(3, 0, 4, 16, 16, OK_PTR, None, OK_PTR, OK_PTR, None, OK_PTR,
                                    P(0x10004), OK_PTR, None) == 1         # W8A8 without sx
    assert lib.aria_qgemm_steer_dev(1, 0, 4, 24, 16, OK_PTR, None, OK_PTR, OK_PTR, None, OK_PTR,
                                    P(0x10004), OK_PTR, None) == 2         # N % 16


def test_binding_f16_arguments():
    import torch
    M, N, K = 8, 32, 64
    X = torch.zeros(M, K, dtype=torch.float16)
    W = torch.zeros(N, K, dtype=torch.float16)
    assert aq.check_gemm_args("f16", X, W, None) == (M, N, K)
    with pytest.raises(ValueError):
        aq.check_gemm_args("f16", X, W, torch.zeros(N, dtype=torch.float32))
    with pytest.raises(TypeError):
        aq.check_gemm_args("f16", X, W.to(torch.int8), None)


def test_binding_rejects_tensors_on_different_devices():
    """The library launches on one device and reads raw pointers: a tensor
    on another device must be refused before any call."""
    import torch
    a = _args("q8")
    a["out"] = torch.zeros(8, 32, dtype=torch.float16, device="meta")
    with pytest.raises(ValueError, match="out"):
        aq.check_gemm_args("q8", **a)
    with pytest.raises(ValueError):
        aq.same_device(X=torch.zeros(2), Y=torch.zeros(2, device="meta"))
    assert aq.same_device(X=torch.zeros(2), Y=None, Z=torch.zeros(3)) == torch.device("cpu")


def test_binding_alpha_dev_must_be_one_float():
    import torch
    a = _args("q8")
    with pytest.raises(TypeError):
        aq.check_gemm_args("q8", **a, alpha_dev=torch.zeros(2, dtype=torch.float32))
    with pytest.raises(TypeError):
        aq.check_gemm_args("q8", **a, alpha_dev=torch.zeros(1, dtype=torch.float16))
    assert aq.check_gemm_args("q8", **a, alpha_dev=torch.zeros(1, dtype=torch.float32)) == (8, 32, 256)


# --------------------------------------------- steer spec and step window --
# "Run it" (aria project page): --steer residual:19:directions/small/sour.atns:0.1:0-7

def test_parse_steer_spec_of_the_pages():
    d = aq.parse_steer_spec("residual:19:directions/small/sour.atns:0.1:0-7")
    assert d == {"site": "residual", "block": 19, "file": "directions/small/sour.atns",
                 "alpha": 0.1, "steps": (0, 7)}
    assert aq.parse_steer_spec("residual:12:v.npy:0.3:4")["steps"] == (4, 4)


@pytest.mark.parametrize("spec", ["residual:19:f:0.1", "residual:x:f:0.1:0-7", "residual:19:f:a:0-7",
                                  "residual:19:f:0.1:5-2", "residual:-1:f:0.1:0-7", ":19:f:0.1:0-7",
                                  "residual:19:f:0.1:0-"])
def test_parse_steer_spec_rejects_malformed(spec):
    with pytest.raises(ValueError):
        aq.parse_steer_spec(spec)


def test_steer_schedule_window():
    assert aq.steer_schedule("residual:12:v:0.3:0-7", 8) == [0.3] * 8
    assert aq.steer_schedule("residual:12:v:0.5:2-4", 8) == [0, 0, 0.5, 0.5, 0.5, 0, 0, 0]
    assert aq.steer_schedule("residual:12:v:0.5:6-9", 8) == [0] * 6 + [0.5, 0.5]   # clipped to the run


# ------------------------------------------------- fused W8A8 workspace ---

def test_w8a8_workspace_size(lib):
    assert aq.w8a8_workspace_size(432, 1536) == 256 + 1792 + 432 * 1536      # 4*432 -> 1792
    assert aq.w8a8_workspace_size(1, 16) == 256 + 256 + 16
    with pytest.raises(aq.AriaError):
        aq.w8a8_workspace_size(0, 16)


def test_fused_w8a8_rules(lib):
    P = ctypes.c_void_p
    need = aq.w8a8_workspace_size(4, 16)
    ws = P(0x20000)
    f = lib.aria_qgemm_w8a8_fused
    # NULL workspace, too small a workspace, misaligned workspace
    assert f(4, 16, 16, OK_PTR, OK_PTR, OK_PTR, None, None, 0.0, None, OK_PTR, None, need, None) == 1
    assert f(4, 16, 16, OK_PTR, OK_PTR, OK_PTR, None, None, 0.0, None, OK_PTR, ws, need - 1, None) == 1
    assert f(4, 16, 16, OK_PTR, OK_PTR, OK_PTR, None, None, 0.0, None, OK_PTR, P(0x20010), need, None) == 3
    # shape rules as for the W8A8 GEMM
    assert f(4, 24, 16, OK_PTR, OK_PTR, OK_PTR, None, None, 0.0, None, OK_PTR, ws, need, None) == 2
    k_bad = (KMAX_I8 // 16 + 1) * 16
    big = aq.w8a8_workspace_size(4, k_bad)
    assert f(4, 16, k_bad, OK_PTR, OK_PTR, OK_PTR, None, None, 0.0, None, OK_PTR, ws, big, None) == 2
    # a misaligned device alpha
    assert f(4, 16, 16, OK_PTR, OK_PTR, OK_PTR, None, OK_PTR, 0.0, P(0x10002), OK_PTR, ws, need,
             None) == 3


def test_workspace_codes_layout():
    import torch
    M, K = 5, 32
    ws = torch.arange(aq.w8a8_workspace_size(M, K), dtype=torch.int64).to(torch.uint8)
    xq, sx = aq.workspace_codes(ws, M, K)
    assert xq.shape == (M, K) and sx.shape == (M,)
    assert xq.view(torch.uint8)[0, 0].item() == (256 + 256) % 256           # codes after 256 + 256
    assert sx.view(torch.uint8).flatten()[0].item() == 256 % 256


def test_selftest_rules(lib):
    f = lib.aria_selftest_bounded_wait
    assert f(4, 16, 16, None, OK_PTR, OK_PTR, OK_PTR, OK_PTR, 1000, None) == 1
    assert f(4, 16, 16, OK_PTR, OK_PTR, OK_PTR, OK_PTR, OK_PTR, 0, None) == 1          # limit 0
    assert f(4, 16, 16, OK_PTR, OK_PTR, OK_PTR, OK_PTR, OK_PTR, 4000001, None) == 1    # above 4 s
    assert f(4, 16, 16, OK_PTR, OK_PTR, ctypes.c_void_p(0x10008), OK_PTR, OK_PTR, 1000, None) == 3
    assert f(4, 24, 16, OK_PTR, OK_PTR, OK_PTR, OK_PTR, OK_PTR, 1000, None) == 2       # N % 16


def test_noalloc_refuses_sizes_beyond_its_scratch_before_any_launch(lib):
    """The static scratch holds 32 MiB: a call whose codes would not fit is
    refused on the host (no CUDA call is made), with the limit in the message."""
    f = lib.aria_qgemm_w8a8_fused_noalloc
    assert f(4096, 16, 16384, OK_PTR, OK_PTR, OK_PTR, None, None, 0.0, None, OK_PTR, None) == 2
    assert b"scratch" in lib.aria_last_error_message()
    assert f(4, 16, 16, None, OK_PTR, OK_PTR, None, None, 0.0, None, OK_PTR, None) == 1
    assert f(4, 16, 16, ctypes.c_void_p(0x10008), OK_PTR, OK_PTR, None, None, 0.0, None, OK_PTR, None) == 3

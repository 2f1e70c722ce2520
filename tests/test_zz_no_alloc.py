"""The no-allocation variant of the fused W8A8 linear (needs a B200).

aria_qgemm_w8a8_fused_noalloc is for callers that must not allocate device
memory while they run -- a real-time audio render callback, where
cudaMalloc can block or synchronise the device, or a host that fixes the
device memory budget at load time. Its scratch is a static device array
inside the library instead of a caller workspace. Called through the C ABI
twice in a row (with different activations, so a stale scratch would show),
each output must match the workspace entry point's within the W8A8 bar of
one fp16 ulp (the same kernel: identical bytes are expected); a size beyond
the static scratch must be refused without launching anything.

This file is collected last, so that a failure here stops a run only after
every other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

import int8_int4_b200 as aq
import synthetic

pytestmark = pytest.mark.gpu


def ulp_dist(a_bits, b_bits):
    def ordered(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(ordered(a_bits) - ordered(b_bits))


def test_noalloc_matches_the_workspace_entry_point_twice():
    lib = aq.load_library()
    M, N, K = 432, 4608, 1536
    key = "gpu/noalloc"
    Wq, sw = aq.qpack("q8", synthetic.weight(f"{key}/W", N, K).cuda())
    b = synthetic.bias(key, N).cuda()
    v = synthetic.steer_vec(key, N).cuda()
    ws = aq.w8a8_workspace(M, K, device="cuda")
    stream = torch.cuda.current_stream()
    for call in range(2):
        X = synthetic.activation(f"{key}/x{call}", M, K, outlier_channel_frac=0.01).cuda()
        ref = aq.qgemm_w8a8_fused(X, Wq, sw, bias=b, steer_vec=v, alpha=0.3, workspace=ws)
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        st = lib.aria_qgemm_w8a8_fused_noalloc(M, N, K, X.data_ptr(), Wq.data_ptr(), sw.data_ptr(),
                                               b.data_ptr(), v.data_ptr(), 0.3, None, Y.data_ptr(),
                                               stream.cuda_stream)
        assert st == 0, lib.aria_last_error_message()
        torch.cuda.synchronize()
        d = ulp_dist(Y.cpu().numpy().view(np.uint16), ref.cpu().numpy().view(np.uint16))
        assert d.max() <= 1, (call, d.max())
        assert (d == 0).all(), (call, int((d != 0).sum()))
    aq.device_status()


def test_noalloc_refuses_a_size_beyond_its_scratch():
    lib = aq.load_library()
    M, N, K = 4096, 16, 16384                     # 64 MiB of codes: more than the scratch
    X = torch.zeros(16, dtype=torch.float16, device="cuda")   # never read: refused first
    Y = torch.zeros(16, dtype=torch.float16, device="cuda")
    st = lib.aria_qgemm_w8a8_fused_noalloc(M, N, K, X.data_ptr(), X.data_ptr(), X.data_ptr(), None,
                                           None, 0.0, None, Y.data_ptr(), None)
    assert st == 2
    assert b"scratch" in lib.aria_last_error_message()
    torch.cuda.synchronize()
    assert not Y.any()

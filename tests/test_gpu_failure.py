"""Failure detection on the GPU without a fault (needs a B200).

Every wait in the library's kernels is bounded. The self-test entry point
launches the W8A8 GEMM with the first pipeline stage of each CTA's first
tile withheld (a barrier that nothing completes) and a short wait limit:
the waits on it must run out, the kernel must unwind (drain its copies,
free tensor memory) and record the timeout in the device status word, the
host must read ARIA_ERR_TIMEOUT, and the context must stay usable -- the
next GEMM on the same stream matches the oracle bit for bit. No trap, no
fault, no endless loop is involved.
"""
import time

import numpy as np
import pytest
import torch

import int8_int4_b200 as aq
import oracle
import synthetic

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K", [(432, 6144, 1536),   # one tile per CTA
                                   (1, 1024, 4096)])    # split-K clusters: every rank gives up
def test_bounded_wait_times_out_and_context_survives(M, N, K):
    aq.load_library()
    key = f"gpu/failure/{M}x{N}x{K}"
    X = synthetic.activation(key, M, K, outlier_channel_frac=0.01)
    W = synthetic.weight(f"{key}/W", N, K)
    Wq, sw = aq.qpack("q8", W.cuda())
    Xq, sx = aq.act_quant(X.cuda())
    aq.device_status()                                   # a clean start
    t0 = time.perf_counter()
    aq.selftest_bounded_wait(Xq, sx, Wq, sw, wait_limit_us=50000)
    with pytest.raises(aq.AriaError) as e:
        aq.device_status()
    elapsed = time.perf_counter() - t0
    assert e.value.status == 5, e.value                   # ARIA_ERR_TIMEOUT
    assert elapsed < 3.0, elapsed                         # the short limit, not the default 4 s
    aq.device_status()                                    # reported once, then cleared
    # the context is intact: the same GEMM, run normally, is exact
    Y = aq.qgemm("w8a8", Xq, Wq, sw, sx=sx)
    rows = np.arange(min(M, 8))
    ref = oracle.w8a8(X.numpy(), Wq.cpu().numpy(), sw.cpu().numpy(), rows=rows)
    assert np.array_equal(Y.cpu().numpy().view(np.uint16)[rows], ref)
    aq.device_status()

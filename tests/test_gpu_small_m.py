"""GPU parity of the few-token weight-only GEMM (M <= 16 tokens; needs a B200).

At a handful of tokens ("Results", aria project page: the q8 / q4 / fp16
linears of the transformer) the library runs a weight-streaming kernel:
every CTA copies its weight rows to shared memory before the dependency wait
and may let its successor start early. These tests compare it with the
oracle on ragged row ranges, 1..16 tokens (one and two token blocks), K
split across clusters, bias / steering / a device-resident strength, and in
a dependent chain where each call reads the previous call's output, eager
and captured in one CUDA graph.
"""
import numpy as np
import pytest
import torch

import int8_int4_b200 as aq
import oracle
import synthetic

pytestmark = pytest.mark.gpu

WO_MAXABS = 1e-2
WO_FROB = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    aq.load_library()   # raises if the CUDA library is missing: no fallback
    yield
    aq.device_status()


def check_wo(y_gpu, y_ref):
    y = y_gpu.astype(np.float64)
    err = np.abs(y - y_ref)
    scale = np.abs(y_ref).max()
    assert err.max() <= WO_MAXABS * scale, (err.max(), scale)
    assert np.linalg.norm(y - y_ref) <= WO_FROB * np.linalg.norm(y_ref)


def _case(fmt, M, N, K, key, bias=True, steer=True):
    W = synthetic.weight(f"{key}/W", N, K, outlier_frac=0.001 if fmt == "q4" else 0.0)
    X = synthetic.activation(key, M, K)
    b = synthetic.bias(key, N) if bias else None
    v = synthetic.steer_vec(key, N) if steer else None
    if fmt == "f16":
        Wd, sc = W.cuda(), None
        ref = lambda a: oracle.f16_ref(X.numpy(), W.numpy(), None if b is None else b.numpy(),
                                       None if v is None else v.numpy(), a)
    else:
        Wd, sc = aq.qpack(fmt, W.cuda())
        rq, rs = oracle.pack_q8(W.numpy()) if fmt == "q8" else oracle.pack_q4(W.numpy())
        ref = lambda a: oracle.wo_ref(fmt, X.numpy(), rq, rs, None if b is None else b.numpy(),
                                      None if v is None else v.numpy(), a)
    return X, Wd, sc, b, v, ref


@pytest.mark.parametrize("fmt", ["q8", "q4", "f16"])
@pytest.mark.parametrize("M", [1, 3, 8, 9, 16])
@pytest.mark.parametrize("N,K", [(208, 512),       # ragged row ranges (1-2 rows per CTA)
                                 (1536, 1536),     # 10-11 rows per CTA
                                 (1024, 4096)])    # K split over a cluster
def test_few_tokens_against_oracle(fmt, M, N, K):
    key = f"gpu/smallm/{fmt}/{M}x{N}x{K}"
    X, Wd, sc, b, v, ref = _case(fmt, M, N, K, key)
    Y = aq.qgemm(fmt, X.cuda(), Wd, sc, bias=b.cuda(), steer_vec=v.cuda(), alpha=0.3)
    check_wo(Y.cpu().numpy(), ref(0.3))


@pytest.mark.parametrize("fmt,N,K", [("q8", 3072, 1024), ("q8", 4096, 1024), ("q4", 4608, 1536),
                                     ("q4", 6144, 1536), ("q4", 1536, 6144)])
@pytest.mark.parametrize("M", [1, 8, 16])
def test_few_tokens_workload_shapes(fmt, N, K, M):
    """The benchmark configurations' own shapes (q8 d=1024, q4 d=1536)."""
    key = f"gpu/smallm/shape/{fmt}/{M}x{N}x{K}"
    X, Wd, sc, b, v, ref = _case(fmt, M, N, K, key, bias=False, steer=False)
    Y = aq.qgemm(fmt, X.cuda(), Wd, sc)
    check_wo(Y.cpu().numpy(), ref(0.0))


@pytest.mark.parametrize("fmt", ["q8", "q4", "f16"])
def test_few_tokens_deterministic_and_device_alpha(fmt):
    M, N, K = 5, 1024, 4096
    key = f"gpu/smallm/det/{fmt}"
    X, Wd, sc, b, v, ref = _case(fmt, M, N, K, key)
    Xd, bd, vd = X.cuda(), b.cuda(), v.cuda()
    base = aq.qgemm(fmt, Xd, Wd, sc, bias=bd, steer_vec=vd, alpha=0.3)
    for _ in range(3):
        assert torch.equal(aq.qgemm(fmt, Xd, Wd, sc, bias=bd, steer_vec=vd, alpha=0.3).view(torch.int16),
                           base.view(torch.int16))
    sched = torch.tensor([0.3, 0.0], dtype=torch.float32, device="cuda")
    dev = aq.qgemm(fmt, Xd, Wd, sc, bias=bd, steer_vec=vd, alpha_dev=sched[0:1])
    assert torch.equal(dev.view(torch.int16), base.view(torch.int16))
    unsteered = aq.qgemm(fmt, Xd, Wd, sc, bias=bd)
    dev0 = aq.qgemm(fmt, Xd, Wd, sc, bias=bd, steer_vec=vd, alpha_dev=sched[1:2])
    assert torch.equal(dev0.view(torch.int16), unsteered.view(torch.int16))
    assert torch.equal(aq.qgemm(fmt, Xd, Wd, sc, bias=bd, steer_vec=vd, alpha=0.0).view(torch.int16),
                       unsteered.view(torch.int16))


def test_zero_activations_give_bias():
    M, N, K = 8, 1536, 1536
    b = synthetic.bias("gpu/smallm/zero", N).cuda()
    W = synthetic.weight("gpu/smallm/zero/W", N, K).cuda()
    X = torch.zeros(M, K, dtype=torch.float16, device="cuda")
    for fmt in ("q8", "q4", "f16"):
        Wq, sc = (W, None) if fmt == "f16" else aq.qpack(fmt, W)
        Y = aq.qgemm(fmt, X, Wq, sc, bias=b)
        assert torch.equal(Y.float(), b.float().expand(M, N)), fmt


@pytest.mark.parametrize("graph", [False, True])
def test_few_token_dependent_chain(graph):
    """Back-to-back few-token calls on one stream, each reading the previous
    call's output, each allowed to start (and to stream its weights) while
    its predecessor still runs: q8 1536 -> 6144, q4 6144 -> 1536, fp16
    1536 -> 1536, q4 1536 -> 4608, at M = 8, run three times with new inputs.
    Each stage is checked against the oracle on the input the GPU gave it:
    a call that read its input before the predecessor had written it would
    be computed from the previous run's values."""
    M, d, f = 8, 1536, 6144
    key = "gpu/smallm/chain"
    q1, s1 = aq.qpack("q8", synthetic.weight(f"{key}/up", f, d).cuda())
    p2, t2 = aq.qpack("q4", synthetic.weight(f"{key}/down", d, f, outlier_frac=0.001).cuda())
    W3 = synthetic.weight(f"{key}/out", d, d)
    W3d = W3.cuda()
    p4, t4 = aq.qpack("q4", synthetic.weight(f"{key}/qkv", 3 * d, d).cuda())
    b3 = synthetic.bias(key, d)
    v3 = synthetic.steer_vec(key, d)
    b3d, v3d = b3.cuda(), v3.cuda()
    alpha = torch.tensor([0.3], dtype=torch.float32, device="cuda")
    X0 = torch.empty(M, d, dtype=torch.float16, device="cuda")
    y1 = torch.empty(M, f, dtype=torch.float16, device="cuda")
    y2 = torch.empty(M, d, dtype=torch.float16, device="cuda")
    y3 = torch.empty(M, d, dtype=torch.float16, device="cuda")
    y4 = torch.empty(M, 3 * d, dtype=torch.float16, device="cuda")
    st = torch.cuda.Stream()

    def chain():
        aq.qgemm("q8", X0, q1, s1, out=y1, stream=st)
        aq.qgemm("q4", y1, p2, t2, out=y2, stream=st)
        aq.qgemm("f16", y2, W3d, None, bias=b3d, steer_vec=v3d, alpha_dev=alpha, out=y3, stream=st)
        aq.qgemm("q4", y3, p4, t4, out=y4, stream=st)

    g = None
    if graph:
        X0.zero_()
        torch.cuda.synchronize()
        with torch.cuda.stream(st):
            chain()
            st.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=st):
                chain()
        torch.cuda.synchronize()
    w1, sw1 = q1.cpu().numpy(), s1.cpu().numpy()
    w2, sw2 = p2.cpu().numpy(), t2.cpu().numpy().view(np.uint16)
    w4, sw4 = p4.cpu().numpy(), t4.cpu().numpy().view(np.uint16)
    for r in range(3):
        X0.copy_(synthetic.activation(f"{key}/x{r}", M, d).cuda())
        torch.cuda.synchronize()
        if g is not None:
            g.replay()
        else:
            chain()
        torch.cuda.synchronize()
        x0, h1, h2, h3, h4 = (t.cpu().numpy() for t in (X0, y1, y2, y3, y4))
        check_wo(h1, oracle.wo_ref("q8", x0, w1, sw1))
        check_wo(h2, oracle.wo_ref("q4", h1, w2, sw2))
        check_wo(h3, oracle.f16_ref(h2, W3.numpy(), b3.numpy(), v3.numpy(), 0.3))
        check_wo(h4, oracle.wo_ref("q4", h3, w4, sw4))
    del g
    aq.device_status()

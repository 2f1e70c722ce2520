"""GPU parity of the fp16 rung and of device-resident steering (needs a B200).

- fp16 ("Results", aria project page: the fp16 column of the precision
  table): the unquantised GEMM on fp16 tensor cores against the oracle's
  fp64 reference, at the weight-only tolerance.
- Live steering ("Live steering while streaming": steering lives inside the
  captured graph, so control changes mid-stream; "Run it": the steer spec's
  step window): the strength is read from device memory, so one captured
  graph follows an alpha schedule. Each step's output is checked against the
  oracle at that step's alpha -- W8A8 bit for bit, weight-only at the
  tolerance -- and against an eager call with the same host alpha, byte for
  byte; a step whose alpha is 0 is bit-identical to an unsteered call.
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


def sample_rows(M, k, seed=0):
    if M <= k:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, M - 1], rng.choice(M, k - 2, replace=False)]))


# ------------------------------------------------------------ fp16 rung ---

@pytest.mark.parametrize("M,N,K,bias,steer", [
    (16, 16, 16, False, False), (1, 128, 128, True, False), (64, 256, 256, True, True),
    (300, 400, 1040, True, True), (432, 1536, 1536, False, True), (8, 1536, 6144, False, False),
    (1, 1024, 4096, True, False),        # few tiles: split-K across a cluster
    (4096, 1536, 1536, False, False),    # many tiles per CTA: persistent, double-buffered
    (432, 6144, 1536, True, False)])
def test_f16_gemm(M, N, K, bias, steer):
    key = f"gpu/f16/{M}x{N}x{K}"
    W = synthetic.weight(f"{key}/W", N, K, outlier_frac=0.001)
    X = synthetic.activation(key, M, K)
    b = synthetic.bias(key, N) if bias else None
    v = synthetic.steer_vec(key, N) if steer else None
    alpha = 0.3 if steer else 0.0
    Y = aq.qgemm("f16", X.cuda(), W.cuda(), None, bias=None if b is None else b.cuda(),
                 steer_vec=None if v is None else v.cuda(), alpha=alpha)
    rows = sample_rows(M, 24)
    ref = oracle.f16_ref(X.numpy(), W.numpy(), None if b is None else b.numpy(),
                         None if v is None else v.numpy(), alpha, rows=rows)
    check_wo(Y.cpu().numpy()[rows], ref)


def test_f16_deterministic_and_alpha_zero_identity():
    M, N, K = 96, 512, 1024
    W = synthetic.weight("gpu/f16det/W", N, K).cuda()
    X = synthetic.activation("gpu/f16det", M, K).cuda()
    b = synthetic.bias("gpu/f16det", N).cuda()
    v = synthetic.steer_vec("gpu/f16det", N).cuda()
    base = aq.qgemm("f16", X, W, None, bias=b)
    for _ in range(3):
        assert torch.equal(aq.qgemm("f16", X, W, None, bias=b).view(torch.int16), base.view(torch.int16))
    assert torch.equal(aq.qgemm("f16", X, W, None, bias=b, steer_vec=v, alpha=0.0).view(torch.int16),
                       base.view(torch.int16))


# ---------------------------------------------------- device-resident alpha ---

def _operands(fmt, M, N, K, key):
    W = synthetic.weight(f"{key}/W", N, K, outlier_frac=0.001 if fmt == "q4" else 0.0)
    X = synthetic.activation(key, M, K, outlier_channel_frac=0.01 if fmt == "w8a8" else 0.0)
    kw = {}
    if fmt == "f16":
        Wq, sc = W.cuda(), None
        Xd = X.cuda()
    else:
        Wq, sc = aq.qpack("q8" if fmt == "w8a8" else fmt, W.cuda())
        Xd = X.cuda()
        if fmt == "w8a8":
            Xd, kw["sx"] = aq.act_quant(Xd)
    return X, W, Xd, Wq, sc, kw


def _oracle(fmt, X, W, Wq, sc, b, v, alpha, rows):
    bn = None if b is None else b.numpy()
    vn = None if (v is None or alpha == 0.0) else v.numpy()
    a = alpha if vn is not None else 0.0
    if fmt == "w8a8":
        return oracle.w8a8(X.numpy(), Wq.cpu().numpy(), sc.cpu().numpy(), bn, vn, a, rows=rows)
    if fmt == "f16":
        return oracle.f16_ref(X.numpy(), W.numpy(), bn, vn, a, rows=rows)
    scn = sc.cpu().numpy()
    return oracle.wo_ref(fmt, X.numpy(), Wq.cpu().numpy(), scn if fmt == "q8" else scn.view(np.uint16),
                         bn, vn, a, rows=rows)


@pytest.mark.parametrize("fmt", ["q8", "q4", "w8a8", "f16"])
@pytest.mark.parametrize("M,N,K", [(432, 1536, 1536), (1, 1024, 4096)])   # persistent / split-K
def test_device_alpha_equals_host_alpha(fmt, M, N, K):
    key = f"gpu/adev/{fmt}/{M}x{N}x{K}"
    X, W, Xd, Wq, sc, kw = _operands(fmt, M, N, K, key)
    b = synthetic.bias(key, N).cuda()
    v = synthetic.steer_vec(key, N).cuda()
    sched = torch.tensor([0.3, 0.0, -0.7], dtype=torch.float32, device="cuda")
    unsteered = aq.qgemm(fmt, Xd, Wq, sc, bias=b, **kw)
    for i, a in enumerate((0.3, 0.0, -0.7)):
        host = aq.qgemm(fmt, Xd, Wq, sc, bias=b, steer_vec=v, alpha=a, **kw)
        dev = aq.qgemm(fmt, Xd, Wq, sc, bias=b, steer_vec=v, alpha_dev=sched[i:i + 1], **kw)
        assert torch.equal(dev.view(torch.int16), host.view(torch.int16)), a
        if a == 0.0:
            assert torch.equal(dev.view(torch.int16), unsteered.view(torch.int16))
    # without a vector, a device alpha is ignored
    dev = aq.qgemm(fmt, Xd, Wq, sc, bias=b, steer_vec=None, alpha_dev=sched[0:1], **kw)
    assert torch.equal(dev.view(torch.int16), unsteered.view(torch.int16))


@pytest.mark.parametrize("fmt", ["w8a8", "q8", "q4", "f16"])
def test_captured_graph_follows_an_alpha_schedule(fmt):
    """One CUDA graph of 8 steps (the replay's steered out-projection,
    d = 1536, M = 432), step s reading schedule[s]. Replayed under the steer
    spec residual:12:v:0.3:2-5 (alpha 0.3 in steps 2..5, 0 elsewhere), then
    -- the graph unchanged, only the device schedule rewritten -- under a
    0 -> 0.5 -> 0 ramp ("Live steering while streaming")."""
    M, N, K, S = 432, 1536, 1536, 8
    key = f"gpu/graphsched/{fmt}"
    X, W, Xd, Wq, sc, kw = _operands(fmt, M, N, K, key)
    b = synthetic.bias(key, N)
    v = synthetic.steer_vec(key, N)
    bd, vd = b.cuda(), v.cuda()
    sched = torch.zeros(S, dtype=torch.float32, device="cuda")
    Y = [torch.empty(M, N, dtype=torch.float16, device="cuda") for _ in range(S)]
    st = torch.cuda.Stream()

    def steps():
        for s in range(S):
            aq.qgemm(fmt, Xd, Wq, sc, bias=bd, steer_vec=vd, alpha_dev=sched[s:s + 1], out=Y[s],
                     stream=st, **kw)

    torch.cuda.synchronize()
    with torch.cuda.stream(st):
        steps()                          # eager once: first-call set-up outside capture
        st.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            steps()
    torch.cuda.synchronize()
    rows = sample_rows(M, 12)
    window = aq.steer_schedule("residual:12:v:0.3:2-5", S)
    ramp = [0.0, 0.125, 0.25, 0.5, 0.5, 0.25, 0.125, 0.0]
    unsteered = aq.qgemm(fmt, Xd, Wq, sc, bias=bd, **kw)
    for schedule in (window, ramp):
        sched.copy_(torch.tensor(schedule, dtype=torch.float32))
        torch.cuda.synchronize()
        with torch.cuda.stream(st):
            g.replay()
        torch.cuda.synchronize()
        for s, a in enumerate(schedule):
            a32 = float(np.float32(a))
            eager = aq.qgemm(fmt, Xd, Wq, sc, bias=bd, steer_vec=vd, alpha=a32, **kw)
            assert torch.equal(Y[s].view(torch.int16), eager.view(torch.int16)), (s, a)
            if a == 0.0:
                assert torch.equal(Y[s].view(torch.int16), unsteered.view(torch.int16)), s
            ref = _oracle(fmt, X, W, Wq, sc, b, v, a32, rows)
            got = Y[s].cpu().numpy()[rows]
            if fmt == "w8a8":
                assert np.array_equal(got.view(np.uint16), ref), (s, a)
            else:
                check_wo(got, ref)
    del g
    aq.device_status()

"""GPU parity of the W8A8 linear with the activation quantisation fused into
the GEMM launch (needs a B200).

"Results" (aria project page): W8A8 runs 8-bit arithmetic on integer tensor
cores, with the activations quantised per token. aria_qgemm_w8a8_fused
quantises the fp16 activations inside the GEMM kernel (every CTA a share of
the rows, then a grid-wide barrier) instead of in a separate launch. Its
output must be the same bytes as aria_act_quant followed by
aria_qgemm(W8A8); the codes and token scales it leaves in its workspace must
equal the oracle's bit for bit; the grid barrier must leave the workspace
ready for the next call (its arrival count back to zero; the generation
word counts the calls).
"""
import numpy as np
import pytest
import torch

import int8_int4_b200 as aq
import oracle
import synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    aq.load_library()   # raises if the CUDA library is missing: no fallback
    yield
    aq.device_status()


def sample_rows(M, k, seed=0):
    if M <= k:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, M - 1], rng.choice(M, k - 2, replace=False)]))


@pytest.mark.parametrize("M,N,K", [
    (432, 6144, 1536),    # one tile per CTA
    (432, 1536, 1536),    # split-K clusters: the barrier spans every rank of every cluster
    (432, 1536, 6144),
    (4096, 4608, 1536),   # several tiles per CTA
    (1, 16, 16), (7, 256, 2064), (300, 400, 1040)])
@pytest.mark.parametrize("epi", ["none", "bias_steer"])
def test_fused_equals_separate_and_oracle(M, N, K, epi):
    key = f"gpu/fused/{M}x{N}x{K}"
    W = synthetic.weight(f"{key}/W", N, K)
    X = synthetic.activation(key, M, K, outlier_channel_frac=0.01)
    if M > 2:
        X[1] = 0                                    # an all-zero token: scale 0, codes 0
    Xd = X.cuda()
    Wq, sw = aq.qpack("q8", W.cuda())
    b = synthetic.bias(key, N) if epi != "none" else None
    v = synthetic.steer_vec(key, N) if epi != "none" else None
    alpha = 0.3 if epi != "none" else 0.0
    bd = None if b is None else b.cuda()
    vd = None if v is None else v.cuda()
    ws = aq.w8a8_workspace(M, K, device="cuda")
    Y = aq.qgemm_w8a8_fused(Xd, Wq, sw, bias=bd, steer_vec=vd, alpha=alpha, workspace=ws)
    Xq, sx = aq.act_quant(Xd)
    Ysep = aq.qgemm("w8a8", Xq, Wq, sw, sx=sx, bias=bd, steer_vec=vd, alpha=alpha)
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Ysep.view(torch.int16))
    wq, wsx = aq.workspace_codes(ws, M, K)
    rq, rs = oracle.act_quant(X.numpy())
    assert np.array_equal(wq.cpu().numpy(), rq)
    assert np.array_equal(wsx.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert not ws[:4].any(), "grid barrier arrival count not reset"
    rows = sample_rows(M, 16)
    ref = oracle.w8a8(X.numpy(), Wq.cpu().numpy(), sw.cpu().numpy(), None if b is None else b.numpy(),
                      None if v is None else v.numpy(), alpha, rows=rows)
    assert np.array_equal(Y.cpu().numpy().view(np.uint16)[rows], ref)


def test_fused_repeated_calls_and_device_alpha():
    M, N, K = 432, 4608, 1536
    key = "gpu/fused/repeat"
    Xd = synthetic.activation(key, M, K, outlier_channel_frac=0.01).cuda()
    Wq, sw = aq.qpack("q8", synthetic.weight(f"{key}/W", N, K).cuda())
    v = synthetic.steer_vec(key, N).cuda()
    ws = aq.w8a8_workspace(M, K, device="cuda")
    sched = torch.tensor([0.3, 0.0], dtype=torch.float32, device="cuda")
    base = aq.qgemm_w8a8_fused(Xd, Wq, sw, steer_vec=v, alpha=0.3, workspace=ws)
    for _ in range(10):
        assert torch.equal(aq.qgemm_w8a8_fused(Xd, Wq, sw, steer_vec=v, alpha=0.3, workspace=ws)
                           .view(torch.int16), base.view(torch.int16))
    dev = aq.qgemm_w8a8_fused(Xd, Wq, sw, steer_vec=v, alpha_dev=sched[0:1], workspace=ws)
    assert torch.equal(dev.view(torch.int16), base.view(torch.int16))
    unsteered = aq.qgemm_w8a8_fused(Xd, Wq, sw, workspace=ws)
    dev0 = aq.qgemm_w8a8_fused(Xd, Wq, sw, steer_vec=v, alpha_dev=sched[1:2], workspace=ws)
    assert torch.equal(dev0.view(torch.int16), unsteered.view(torch.int16))
    torch.cuda.synchronize()
    assert not ws[:4].any()                           # arrival count back to zero
    assert ws[4:8].view(torch.int32).item() == 14     # the generation counts the calls
    aq.device_status()


@pytest.mark.parametrize("graph", [False, True])
def test_fused_in_a_dependent_chain(graph):
    """q8 (1536 -> 6144) -> fused W8A8 (6144 -> 1536, steered) -> q4
    (1536 -> 4608) at M = 432 on one stream under programmatic dependent
    launch, eager and in one CUDA graph, three runs with new inputs; the
    fused call quantises the q8 output the GPU just wrote."""
    M, d, f = 432, 1536, 6144
    key = "gpu/fused/chain"
    q1, s1 = aq.qpack("q8", synthetic.weight(f"{key}/up", f, d).cuda())
    q2, s2 = aq.qpack("q8", synthetic.weight(f"{key}/down", d, f).cuda())
    p3, t3 = aq.qpack("q4", synthetic.weight(f"{key}/qkv", 3 * d, d, outlier_frac=0.001).cuda())
    v = synthetic.steer_vec(key, d)
    vd = v.cuda()
    ws = aq.w8a8_workspace(M, f, device="cuda")
    X0 = torch.empty(M, d, dtype=torch.float16, device="cuda")
    y1 = torch.empty(M, f, dtype=torch.float16, device="cuda")
    y2 = torch.empty(M, d, dtype=torch.float16, device="cuda")
    y3 = torch.empty(M, 3 * d, dtype=torch.float16, device="cuda")
    st = torch.cuda.Stream()

    def chain():
        aq.qgemm("q8", X0, q1, s1, out=y1, stream=st)
        aq.qgemm_w8a8_fused(y1, q2, s2, steer_vec=vd, alpha=0.3, out=y2, workspace=ws, stream=st)
        aq.qgemm("q4", y2, p3, t3, out=y3, stream=st)

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
    w2, sw2 = q2.cpu().numpy(), s2.cpu().numpy()
    w3, sw3 = p3.cpu().numpy(), t3.cpu().numpy().view(np.uint16)
    rows = sample_rows(M, 12)
    for r in range(3):
        X0.copy_(synthetic.activation(f"{key}/x{r}", M, d).cuda())
        torch.cuda.synchronize()
        if g is not None:
            g.replay()
        else:
            chain()
        torch.cuda.synchronize()
        h1, h2, h3 = (t.cpu().numpy() for t in (y1, y2, y3))
        wq, wsx = aq.workspace_codes(ws, M, f)
        rq, rs = oracle.act_quant(h1)
        assert np.array_equal(wq.cpu().numpy(), rq), r
        assert np.array_equal(wsx.cpu().numpy().view(np.uint32), rs.view(np.uint32)), r
        ref2 = oracle.w8a8(h1, w2, sw2, None, v.numpy(), 0.3, rows=rows)
        assert np.array_equal(h2.view(np.uint16)[rows], ref2), r
        y = h3[rows].astype(np.float64)
        ref3 = oracle.wo_ref("q4", h2, w3, sw3, rows=rows)
        assert np.abs(y - ref3).max() <= 1e-2 * np.abs(ref3).max()
    assert not ws[:4].any()
    del g
    aq.device_status()

"""GPU parity of the CUDA path against the CPU oracle (needs a B200).

Bars (element by element, same seeded inputs on both sides):
- packed bytes, scales, activation codes and int32 accumulators: bit-exact;
- W8A8 fp16 outputs: within 1 fp16 ulp (the fp64 epilogue is expected to be
  bit-exact; the test reports the worst distance);
- q8 / q4 weight-only fp16 outputs vs the unrounded fp64 reference:
  max |y - y_ref| <= 1e-2 * max |y_ref| and ||y - y_ref||_F <= 1e-3 * ||y_ref||_F.
Shapes span several tiles, ragged tails in M, N and K, the degenerate cases
(M = 1, zero rows, N = K = 16) and, on sampled rows, the full workload sizes.
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


def f16np(t):
    return t.detach().cpu().numpy()


def ulp_dist(a_bits, b_bits):
    """distance in fp16 ulps between bit patterns (+0 == -0)"""
    def ordered(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(ordered(a_bits) - ordered(b_bits))


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


# ------------------------------------------------------------------ packs --

@pytest.mark.parametrize("N,K", [(256, 256), (48, 48), (3072, 1024), (1024, 4096),
                                 (4608, 1536), (1536, 6144), (130, 2064)])
def test_pack_q8_bit_exact(N, K):
    W = synthetic.weight(f"gpu/pq8/{N}x{K}", N, K, outlier_frac=0.001)
    W[1] = 0                                   # an all-zero channel
    t = 2.0 ** -24                             # a channel of fp16 subnormals
    W[2] = torch.from_numpy(((np.arange(K) % 23) - 11) * t).to(torch.float16)
    Wq, s = aq.qpack("q8", W.cuda())
    rq, rs = oracle.pack_q8(W.numpy())
    assert np.array_equal(Wq.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("N,K", [(16, 64), (64, 96), (4608, 1536), (1536, 6144), (6144, 1536), (40, 256)])
def test_pack_q4_bit_exact(N, K):
    W = synthetic.weight(f"gpu/pq4/{N}x{K}", N, K, outlier_frac=0.001)
    W[0, :32] = 0                              # an all-zero group
    t = 2.0 ** -24                             # groups whose scale is an fp16 subnormal:
    W[1, :32] = 0
    W[1, 0], W[1, 3], W[1, 9] = 10 * t, -2 * t, -10 * t   # s16 = 1 step: +-10 clamp to +-7
    W[1, 32:64] = 0
    W[1, 37], W[1, 38] = 3 * t, -3 * t         # s16 rounds to 0: every code 0
    P, S = aq.qpack("q4", W.cuda())
    rp, rs = oracle.pack_q4(W.numpy())
    assert np.array_equal(P.cpu().numpy(), rp)
    assert np.array_equal(S.cpu().numpy().view(np.uint16), rs)


@pytest.mark.parametrize("M,K", [(1, 16), (432, 1536), (432, 6144), (4096, 1536), (4096, 6144),
                                 (7, 8208), (33, 2064)])
def test_act_quant_bit_exact(M, K):
    X = synthetic.activation(f"gpu/aq/{M}x{K}", M, K, outlier_channel_frac=0.01)
    if M > 2:
        X[2] = 0
    Xq, sx = aq.act_quant(X.cuda())
    rq, rs = oracle.act_quant(X.numpy())
    assert np.array_equal(Xq.cpu().numpy(), rq)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), rs.view(np.uint32))


# ------------------------------------------------------------ int8 GEMM ---

def _w8a8_inputs(M, N, K, key):
    """GPU pack and activation codes, each first checked bit for bit against
    the oracle's own (so the GEMM parity below runs pack -> GEMM end to end
    against the oracle's pack -> GEMM)."""
    W = synthetic.weight(f"{key}/W", N, K)
    X = synthetic.activation(key, M, K, outlier_channel_frac=0.01)
    Wq, sw = aq.qpack("q8", W.cuda())
    Xq, sx = aq.act_quant(X.cuda())
    rq, rs = oracle.pack_q8(W.numpy())
    assert np.array_equal(Wq.cpu().numpy(), rq) and np.array_equal(sw.cpu().numpy().view(np.uint32),
                                                                   rs.view(np.uint32))
    if M * K <= 4096 * 6144:
        xq, xs = oracle.act_quant(X.numpy())
        assert np.array_equal(Xq.cpu().numpy(), xq) and np.array_equal(sx.cpu().numpy().view(np.uint32),
                                                                       xs.view(np.uint32))
    return X, W, Xq, sx, Wq, sw


@pytest.mark.parametrize("M,N,K", [(16, 16, 16), (1, 128, 128), (64, 256, 256), (300, 400, 1040),
                                   (432, 1536, 1536), (257, 128, 4096), (2, 4608, 1536)])
def test_s32_bit_exact(M, N, K):
    X, W, Xq, sx, Wq, sw = _w8a8_inputs(M, N, K, f"gpu/s32/{M}x{N}x{K}")
    C = aq.qgemm_s32(Xq, Wq)
    ref = oracle.gemm_s32(Xq.cpu().numpy(), Wq.cpu().numpy())
    assert np.array_equal(C.cpu().numpy(), ref)


@pytest.mark.parametrize("M,N,K", [(4096, 6144, 1536), (4096, 1536, 6144), (432, 4608, 1536)])
def test_s32_full_size_sampled(M, N, K):
    X, W, Xq, sx, Wq, sw = _w8a8_inputs(M, N, K, f"gpu/s32f/{M}x{N}x{K}")
    C = aq.qgemm_s32(Xq, Wq)
    rows = sample_rows(M, 12)
    ref = oracle.gemm_s32(Xq.cpu().numpy(), Wq.cpu().numpy(), rows=rows)
    assert np.array_equal(C.cpu().numpy()[rows], ref)


@pytest.mark.parametrize("M,N,K,bias,steer", [
    (64, 256, 256, True, False), (300, 400, 1040, True, True), (432, 1536, 1536, False, True),
    (1, 16, 16, True, True), (432, 6144, 1536, False, False)])
def test_w8a8_within_one_ulp(M, N, K, bias, steer):
    key = f"gpu/w8a8/{M}x{N}x{K}"
    X, W, Xq, sx, Wq, sw = _w8a8_inputs(M, N, K, key)
    b = synthetic.bias(key, N) if bias else None
    v = synthetic.steer_vec(key, N) if steer else None
    alpha = 0.3 if steer else 0.0
    Y = aq.qgemm("w8a8", Xq, Wq, sw, sx=sx, bias=None if b is None else b.cuda(),
                 steer_vec=None if v is None else v.cuda(), alpha=alpha)
    ref = oracle.w8a8(X.numpy(), Wq.cpu().numpy(), sw.cpu().numpy(),
                      None if b is None else b.numpy(), None if v is None else v.numpy(), alpha)
    d = ulp_dist(Y.cpu().numpy().view(np.uint16), ref)
    assert d.max() <= 1, d.max()
    assert (d == 0).all(), (d != 0).sum()  # the epilogue rounds exactly


@pytest.mark.parametrize("M,N,K", [(96, 256, 512),      # 2 tiles: split-K cluster reduction
                                   (4096, 1280, 256)])  # 160 tiles: persistent epilogue
@pytest.mark.parametrize("bias,steer", [(False, False), (True, False), (True, True)])
def test_w8a8_exact_fp16_ties_round_to_even(M, N, K, bias, steer):
    """s_x = 2^-5 and s_w = 2^-11 make acc * s_x * s_w = acc * 2^-16 exact in
    binary, so every odd |acc| in [2^11, 2^12) (and many others) lands exactly
    on an fp16 rounding midpoint; the result must be the tie-to-even value."""
    rng = np.random.default_rng(11)
    xc = rng.integers(-127, 128, (M, K)); xc[:, 0] = rng.choice([-127, 127], M)
    wc = rng.integers(-127, 128, (N, K)); wc[:, 0] = rng.choice([-127, 127], N)
    X = torch.from_numpy((xc * 2.0 ** -5).astype(np.float16))     # row absmax 127 * 2^-5
    W = torch.from_numpy((wc * 2.0 ** -11).astype(np.float16))    # row absmax 127 * 2^-11
    Wq, sw = aq.qpack("q8", W.cuda())
    Xq, sx = aq.act_quant(X.cuda())
    assert (sx == 2.0 ** -5).all() and (sw == 2.0 ** -11).all()
    key = "gpu/w8a8ties"
    b = synthetic.bias(key, N) if bias else None
    v = synthetic.steer_vec(key, N) if steer else None
    alpha = 0.3 if steer else 0.0
    Y = aq.qgemm("w8a8", Xq, Wq, sw, sx=sx, bias=None if b is None else b.cuda(),
                 steer_vec=None if v is None else v.cuda(), alpha=alpha)
    rows = sample_rows(M, 48) if M > 256 else None
    ref = oracle.w8a8(X.numpy(), Wq.cpu().numpy(), sw.cpu().numpy(),
                      None if b is None else b.numpy(), None if v is None else v.numpy(), alpha, rows=rows)
    if not bias:
        acc = (xc if rows is None else xc[rows]) @ wc.T
        assert ((np.abs(acc) >= 2 ** 11) & (np.abs(acc) < 2 ** 12) & (acc % 2 == 1)).sum() > 100
    got = Y.cpu().numpy().view(np.uint16)
    if rows is not None:
        got = got[rows]
    assert np.array_equal(got, ref), (got != ref).sum()


@pytest.mark.parametrize("M,N", [(1, 16), (4096, 1280)])   # split-K and persistent epilogues
@pytest.mark.parametrize("term", ["bias", "steer"])
def test_w8a8_just_below_the_overflow_midpoint(M, N, term):
    """acc * s_x * s_w = 65520 exactly (the midpoint between 65504 and
    overflow) plus a negative bias of 2^-14 (or the same through alpha*v): in
    fp32 the sum rounds to 65520 itself, and converting that to fp16 ties up
    to infinity, but the exact value lies below the midpoint and rounds to
    65504. Rows alternate with the exact midpoint (bias / steer 0 there:
    infinity is right) to keep both sides covered."""
    K = 512
    xc = np.zeros((M, K)); wc = np.zeros((N, K))
    xc[:, :5] = 127; xc[:, 5] = -12                # s_x = 1
    wc[:, :4] = 127; wc[:, 4] = 8; wc[:, 5] = 1    # s_w = 1; acc = 4*127^2 + 127*8 - 12 = 65520
    X = torch.from_numpy(xc.astype(np.float16))
    W = torch.from_numpy(wc.astype(np.float16))
    Wq, sw = aq.qpack("q8", W.cuda())
    Xq, sx = aq.act_quant(X.cuda())
    assert (sx == 1).all() and (sw == 1).all()
    assert (aq.qgemm_s32(Xq, Wq) == 65520).all()
    small = np.where(np.arange(N) % 2 == 0, -2.0 ** -14, 0.0)
    if term == "bias":
        b, v, alpha = small.astype(np.float16), None, 0.0
    else:
        b, v, alpha = None, (small * 2.0).astype(np.float32), 0.5      # alpha*v = small, exactly
    Y = aq.qgemm("w8a8", Xq, Wq, sw, sx=sx, bias=None if b is None else torch.from_numpy(b).cuda(),
                 steer_vec=None if v is None else torch.from_numpy(v).cuda(), alpha=alpha)
    rows = sample_rows(M, 32)
    ref = oracle.w8a8(X.numpy(), Wq.cpu().numpy(), sw.cpu().numpy(), b, v, alpha, rows=rows)
    assert (ref[:, 0] == 0x7BFF).all() and (ref[:, 1] == 0x7C00).all()
    assert np.array_equal(Y.cpu().numpy().view(np.uint16)[rows], ref)


def test_w8a8_large_accumulators_take_exact_path():
    """|acc| >= 2^22 (all codes +-127 over K = 4096) and exact fp16 results
    exercise the kernel's fp64 branch; sign patterns vary per row/column."""
    M, N, K = 64, 256, 4096
    rng = np.random.default_rng(5)
    sgn_x = rng.choice([-1.0, 1.0], (M, 1)) * np.ones((1, K))
    sgn_w = rng.choice([-1.0, 1.0], (N, 1)) * np.ones((1, K))
    sgn_x[:, ::3] *= -1                        # mixed signs inside a row
    X = torch.from_numpy((sgn_x * rng.uniform(0.5, 2.0, (M, 1))).astype(np.float16))
    W = torch.from_numpy((sgn_w * 0.01).astype(np.float16))
    Wq, sw = aq.qpack("q8", W.cuda())
    Xq, sx = aq.act_quant(X.cuda())
    acc = aq.qgemm_s32(Xq, Wq).abs().max().item()
    assert acc >= 2 ** 22
    Y = aq.qgemm("w8a8", Xq, Wq, sw, sx=sx)
    ref = oracle.w8a8(X.numpy(), Wq.cpu().numpy(), sw.cpu().numpy())
    assert np.array_equal(Y.cpu().numpy().view(np.uint16), ref)


@pytest.mark.parametrize("M,N,K", [(4096, 6144, 1536), (4096, 1536, 6144), (4096, 4608, 1536),
                                   (4096, 1536, 1536)])
def test_w8a8_full_size_sampled(M, N, K):
    key = f"gpu/w8a8f/{M}x{N}x{K}"
    X, W, Xq, sx, Wq, sw = _w8a8_inputs(M, N, K, key)
    Y = aq.qgemm("w8a8", Xq, Wq, sw, sx=sx)
    rows = sample_rows(M, 8)
    ref = oracle.w8a8(X.numpy(), Wq.cpu().numpy(), sw.cpu().numpy(), rows=rows)
    d = ulp_dist(Y.cpu().numpy().view(np.uint16)[rows], ref)
    assert d.max() <= 1, d.max()
    # the exact-rounding epilogue is expected to agree bit for bit
    assert (d == 0).mean() == 1.0, (d != 0).sum()


# ------------------------------------------------------- weight-only GEMM ---

def _wo(fmt, M, N, K, key, bias=False, steer=False, rows=None, outliers=0.0):
    W = synthetic.weight(f"{key}/W", N, K, outlier_frac=outliers)
    X = synthetic.activation(key, M, K)
    b = synthetic.bias(key, N) if bias else None
    v = synthetic.steer_vec(key, N) if steer else None
    alpha = 0.3 if steer else 0.0
    Wq, sc = aq.qpack(fmt, W.cuda())
    Y = aq.qgemm(fmt, X.cuda(), Wq, sc, bias=None if b is None else b.cuda(),
                 steer_vec=None if v is None else v.cuda(), alpha=alpha)
    # the oracle's own pack: the GPU's must equal it, and the reference is
    # computed from it (pack -> GEMM end to end on both sides)
    rq, rs = oracle.pack_q8(W.numpy()) if fmt == "q8" else oracle.pack_q4(W.numpy())
    scn = sc.cpu().numpy()
    assert np.array_equal(Wq.cpu().numpy(), rq)
    assert np.array_equal(scn.view(np.uint32) if fmt == "q8" else scn.view(np.uint16),
                          rs.view(np.uint32) if fmt == "q8" else rs)
    ref = oracle.wo_ref(fmt, X.numpy(), rq, rs, None if b is None else b.numpy(),
                        None if v is None else v.numpy(), alpha, rows=rows)
    y = f16np(Y)
    return (y if rows is None else y[rows]), ref


def test_tiny_q8_config():
    """W [256,256] ~N(0,0.02^2), X [64,256] ~N(0,1), bias ~N(0,0.01^2), seed 0."""
    d = synthetic.tiny_q8()
    Wq, s = aq.qpack("q8", d["W"].cuda())
    rq, rs = oracle.pack_q8(d["W"].numpy())
    assert np.array_equal(Wq.cpu().numpy(), rq) and np.array_equal(s.cpu().numpy(), rs)
    Y = aq.qgemm("q8", d["X"].cuda(), Wq, s, bias=d["bias"].cuda())
    check_wo(f16np(Y), oracle.wo_ref("q8", d["X"].numpy(), rq, rs, d["bias"].numpy()))


@pytest.mark.parametrize("M,N,K,bias,steer", [
    (16, 16, 16, False, False), (1, 128, 128, True, False), (64, 256, 256, True, True),
    (300, 400, 1040, True, True), (17, 3072, 1024, False, False), (432, 1024, 1024, True, False),
    (5, 1024, 4096, False, True)])
def test_q8_weight_only(M, N, K, bias, steer):
    y, ref = _wo("q8", M, N, K, f"gpu/q8/{M}x{N}x{K}", bias, steer)
    check_wo(y, ref)


@pytest.mark.parametrize("name", ["qkv", "out", "up", "down"])
@pytest.mark.parametrize("M", [1, 16, 432])
def test_q8_d1024_block(name, M):
    W, X = synthetic.q8_block_d1024(name, M)
    Wq, s = aq.qpack("q8", W.cuda())
    Y = aq.qgemm("q8", X.cuda(), Wq, s)
    rows = sample_rows(M, 24)
    rq, rs = oracle.pack_q8(W.numpy())
    assert np.array_equal(Wq.cpu().numpy(), rq) and np.array_equal(s.cpu().numpy(), rs)
    ref = oracle.wo_ref("q8", X.numpy(), rq, rs, rows=rows)
    check_wo(f16np(Y)[rows], ref)


@pytest.mark.parametrize("M,N,K,bias,steer", [
    (16, 16, 256, False, False), (1, 128, 256, True, False), (64, 256, 512, True, True),
    (300, 400, 1024, True, True), (8, 1536, 6144, False, False)])
def test_q4_weight_only(M, N, K, bias, steer):
    y, ref = _wo("q4", M, N, K, f"gpu/q4/{M}x{N}x{K}", bias, steer, outliers=0.001)
    check_wo(y, ref)


@pytest.mark.parametrize("name", ["qkv", "out", "up", "down"])
@pytest.mark.parametrize("M", [1, 8, 432])
def test_q4_d1536_block(name, M):
    W, X = synthetic.q4_d1536(name, M)
    P, S = aq.qpack("q4", W.cuda())
    Y = aq.qgemm("q4", X.cuda(), P, S)
    rows = sample_rows(M, 16)
    rp, rs = oracle.pack_q4(W.numpy())
    assert np.array_equal(P.cpu().numpy(), rp) and np.array_equal(S.cpu().numpy().view(np.uint16), rs)
    ref = oracle.wo_ref("q4", X.numpy(), rp, rs, rows=rows)
    check_wo(f16np(Y)[rows], ref)


# ---------------------------------------------------------- epilogue rules --

@pytest.mark.parametrize("fmt", ["q8", "q4", "w8a8"])
def test_alpha_zero_is_bit_identical(fmt):
    M, N, K = 96, 512, 1024
    W = synthetic.weight(f"gpu/a0/{fmt}/W", N, K)
    X = synthetic.activation(f"gpu/a0/{fmt}", M, K).cuda()
    v = synthetic.steer_vec(f"gpu/a0/{fmt}", N).cuda()
    b = synthetic.bias(f"gpu/a0/{fmt}", N).cuda()
    Wq, sc = aq.qpack("q8" if fmt == "w8a8" else fmt, W.cuda())
    kw = {}
    if fmt == "w8a8":
        X, sx = aq.act_quant(X)
        kw["sx"] = sx
    base = aq.qgemm(fmt, X, Wq, sc, bias=b, **kw)
    assert torch.equal(aq.qgemm(fmt, X, Wq, sc, bias=b, steer_vec=v, alpha=0.0, **kw).view(torch.int16),
                       base.view(torch.int16))
    assert torch.equal(aq.qgemm(fmt, X, Wq, sc, bias=b, steer_vec=None, alpha=0.5, **kw).view(torch.int16),
                       base.view(torch.int16))
    steered = aq.qgemm(fmt, X, Wq, sc, bias=b, steer_vec=v, alpha=0.3, **kw)
    diff = (steered.double() - base.double()) - 0.3 * v.double()[None, :]
    assert diff.abs().max().item() < 2e-3          # y + alpha*v, up to fp16 rounding


@pytest.mark.parametrize("fmt,K", [("q8", 128), ("q4", 256), ("w8a8", 128), ("w8a8", 256)])
def test_small_k_many_tiles(fmt, K):
    """Short K with hundreds of output tiles: the producer and dequant warps
    finish their rings several tiles ahead of the MMA and then join the last
    tile's epilogue; they must wait for that tile, not an earlier one that
    shares its accumulator buffer."""
    M, N = 4096, 6144
    rows = sample_rows(M, 16)
    key = f"gpu/smallk/{fmt}/{K}"
    if fmt == "w8a8":
        X, W, Xq, sx, Wq, sw = _w8a8_inputs(M, N, K, key)
        Y = aq.qgemm("w8a8", Xq, Wq, sw, sx=sx)
        ref = oracle.w8a8(X.numpy(), Wq.cpu().numpy(), sw.cpu().numpy(), rows=rows)
        assert np.array_equal(Y.cpu().numpy().view(np.uint16)[rows], ref)
    else:
        y, ref = _wo(fmt, M, N, K, key, rows=rows)
        check_wo(y, ref)


@pytest.mark.parametrize("fmt", ["q8", "q4", "w8a8"])
def test_repeated_launches_bit_identical(fmt):
    """Persistent multi-tile launches (M = 4096: several tiles per CTA, rings
    wrapping many times) give bit-identical results run after run; a
    cross-proxy ordering race on the raw-weight ring showed up here as a few
    wrong weight rows in about one launch in three."""
    M, N, K = 4096, 6144, 1536
    key = f"gpu/repeat/{fmt}"
    W = synthetic.weight(f"{key}/W", N, K).cuda()
    X = synthetic.activation(key, M, K).cuda()
    Wq, sc = aq.qpack("q8" if fmt == "w8a8" else fmt, W)
    sx = None
    if fmt == "w8a8":
        X, sx = aq.act_quant(X)
    outs = [aq.qgemm(fmt, X, Wq, sc, sx=sx) for _ in range(12)]
    for i, Y in enumerate(outs[1:], 1):
        assert torch.equal(Y, outs[0]), (i, int((Y != outs[0]).sum()))


@pytest.mark.parametrize("fmt", ["q8", "q4", "w8a8"])
def test_deterministic_split_k(fmt):
    M, N, K = 1, 1024, 4096                        # few tiles: split-K across a cluster
    W = synthetic.weight(f"gpu/det/{fmt}/W", N, K)
    X = synthetic.activation(f"gpu/det/{fmt}", M, K).cuda()
    Wq, sc = aq.qpack("q8" if fmt == "w8a8" else fmt, W.cuda())
    kw = {}
    if fmt == "w8a8":
        X, sx = aq.act_quant(X)
        kw["sx"] = sx
    ys = [aq.qgemm(fmt, X, Wq, sc, **kw).view(torch.int16) for _ in range(3)]
    assert all(torch.equal(ys[0], y) for y in ys[1:])


def test_zero_inputs_give_bias():
    M, N, K = 8, 256, 512
    b = synthetic.bias("gpu/zero", N).cuda()
    W = synthetic.weight("gpu/zero/W", N, K).cuda()
    X = torch.zeros(M, K, dtype=torch.float16, device="cuda")
    for fmt in ("q8", "q4"):
        Wq, sc = aq.qpack(fmt, W)
        Y = aq.qgemm(fmt, X, Wq, sc, bias=b)
        assert torch.equal(Y.float(), b.float().expand(M, N))
    Wq, sw = aq.qpack("q8", W)
    Xq, sx = aq.act_quant(X)
    assert not Xq.any() and not sx.any()
    Y = aq.qgemm("w8a8", Xq, Wq, sw, sx=sx, bias=b)
    assert torch.equal(Y.float(), b.float().expand(M, N))


# --------------------------------------- the replay's launch configuration --

@pytest.mark.parametrize("graph", [False, True])
def test_dependent_chain_in_replay_launch_configuration(graph):
    """The replay's launch configuration -- back-to-back calls on one stream,
    each kernel allowed to start before its predecessor has finished
    (programmatic dependent launch), captured in one CUDA graph as bench.py
    does -- with each call reading the previous call's output: q8
    (1536 -> 6144), per-token activation quantisation of that output, W8A8
    (6144 -> 1536, steered), q4 (1536 -> 4608), at M = 432. Each stage is
    checked against the oracle on the input the GPU actually gave it, and the
    chain runs three times with new activations, so a kernel that read its
    input before its predecessor had written it would be computed from the
    previous run's values."""
    M, d, f = 432, 1536, 6144
    key = "gpu/chain"
    q1, s1 = aq.qpack("q8", synthetic.weight(f"{key}/up", f, d).cuda())
    q2, s2 = aq.qpack("q8", synthetic.weight(f"{key}/down", d, f).cuda())
    p3, t3 = aq.qpack("q4", synthetic.weight(f"{key}/qkv", 3 * d, d, outlier_frac=0.001).cuda())
    v = synthetic.steer_vec(key, d)
    vd = v.cuda()
    X0 = torch.empty(M, d, dtype=torch.float16, device="cuda")
    y1 = torch.empty(M, f, dtype=torch.float16, device="cuda")
    xq = torch.empty(M, f, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    y2 = torch.empty(M, d, dtype=torch.float16, device="cuda")
    y3 = torch.empty(M, 3 * d, dtype=torch.float16, device="cuda")
    st = torch.cuda.Stream()

    def chain():
        aq.qgemm("q8", X0, q1, s1, out=y1, stream=st)
        aq.act_quant(y1, out=(xq, sx), stream=st)
        aq.qgemm("w8a8", xq, q2, s2, sx=sx, steer_vec=vd, alpha=0.3, out=y2, stream=st)
        aq.qgemm("q4", y2, p3, t3, out=y3, stream=st)

    g = None
    if graph:
        X0.zero_()
        torch.cuda.synchronize()
        with torch.cuda.stream(st):
            chain()                      # eager once: first-call set-up outside capture
            st.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=st):
                chain()
        torch.cuda.synchronize()
    w1, sw1 = q1.cpu().numpy(), s1.cpu().numpy()
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
        x0, h1, h2, h3 = (f16np(t) for t in (X0, y1, y2, y3))
        check_wo(h1[rows], oracle.wo_ref("q8", x0, w1, sw1, rows=rows))
        rq, rs = oracle.act_quant(h1)
        assert np.array_equal(xq.cpu().numpy(), rq), r
        assert np.array_equal(sx.cpu().numpy().view(np.uint32), rs.view(np.uint32)), r
        ref2 = oracle.w8a8(h1, w2, sw2, None, v.numpy(), 0.3, rows=rows)
        assert np.array_equal(h2.view(np.uint16)[rows], ref2), r
        check_wo(h3[rows], oracle.wo_ref("q4", h2, w3, sw3, rows=rows))
    del g
    aq.device_status()


def test_bench_replay_outputs_match_oracle():
    """bench.py's own workload and launches: bench.Replay's CUDA graphs (24
    blocks x 4 linears x 8 steps per precision at M = 432, steering on block
    12's out-projection with the strength read from the device schedule),
    replayed precision by precision, from both input buffers; then sampled
    outputs of blocks 0, 12 and 23 against the oracle: q8, q4 and fp16 within
    the weight-only tolerance, W8A8 bit-exact."""
    import bench
    rep = bench.Replay(torch.device("cuda", torch.cuda.current_device()), buffers=2, fp16=True)
    rep.capture()
    rows = sample_rows(bench.M, 4)
    blocks = (0, synthetic.REPLAY_STEER_BLOCK, bench.BLOCKS - 1)
    v = rep.steer.cpu().numpy()

    def steer(b, name):
        on = b == synthetic.REPLAY_STEER_BLOCK and name == "out"
        return (v, synthetic.REPLAY_ALPHA) if on else (None, 0.0)

    def replay(buf, *kinds):
        for kind in kinds:
            prec = kind.replace("_gemm", "").replace("_fused", "")
            for key in rep.y.get(prec, {}):
                rep.y[prec][key].fill_(float("nan"))   # no stale result passes
        torch.cuda.synchronize()
        with torch.cuda.stream(rep.stream):
            for kind in kinds:
                rep.graphs[kind, buf if kind != "w8a8_gemm" else 0].replay()
        torch.cuda.synchronize()

    for buf in (0, 1):
        replay(buf, "q8")
        for b in blocks:
            for name, k, n in bench.LINEARS:
                x = rep.x_host[b, name].numpy()
                Wq, sw = (t.cpu().numpy() for t in rep.q8[b, name])
                vv, a = steer(b, name)
                check_wo(f16np(rep.y["q8"][b, name])[rows],
                         oracle.wo_ref("q8", x, Wq, sw, None, vv, a, rows=rows))
        for w8a8_kinds in (("w8a8_fused",), ("act_quant", "w8a8_gemm")):   # fused, and separate launches
            replay(buf, *w8a8_kinds)
            for b in blocks:
                for name, k, n in bench.LINEARS:
                    x = rep.x_host[b, name].numpy()
                    Wq, sw = (t.cpu().numpy() for t in rep.q8[b, name])
                    vv, a = steer(b, name)
                    ref = oracle.w8a8(x, Wq, sw, None, vv, a, rows=rows)
                    assert np.array_equal(f16np(rep.y["w8a8"][b, name]).view(np.uint16)[rows], ref), \
                        (w8a8_kinds, b, name)
        replay(buf, "q4")
        for b in blocks:
            for name, k, n in bench.LINEARS:
                x = rep.x_host[b, name].numpy()
                P, S = rep.q4[b, name]
                vv, a = steer(b, name)
                ref = oracle.wo_ref("q4", x, P.cpu().numpy(), S.cpu().numpy().view(np.uint16), None, vv, a,
                                    rows=rows)
                check_wo(f16np(rep.y["q4"][b, name])[rows], ref)
        replay(buf, "f16")
        for b in blocks:
            for name, k, n in bench.LINEARS:
                x = rep.x_host[b, name].numpy()
                vv, a = steer(b, name)
                ref = oracle.f16_ref(x, rep.w16[b, name].cpu().numpy(), None, vv, a, rows=rows)
                check_wo(f16np(rep.y["f16"][b, name])[rows], ref)
    rep.aq.device_status(rep.stream)

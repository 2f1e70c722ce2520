"""Pins for the oracle's GEMMs and fused epilogue (CPU only).

- the int32 GEMM against numpy's int64 matmul and closed-form extremes;
- the W8A8 fp16 output against the exact rational value rounded to fp16 by
  an independent Fraction-based round-half-even;
- the weight-only fp64 reference against numpy's float64 matmul;
- both against the unquantised product, within the quantisation error bound;
- bias / steering special cases ("Steering is real": removable at alpha = 0
  with bit-identical output).
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synthetic


def _i8(rng, shape):
    return rng.integers(-127, 128, shape, dtype=np.int64).astype(np.int8)


@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (3, 5, 7), (17, 33, 64), (64, 48, 256)])
def test_gemm_s32_matches_numpy(M, N, K):
    rng = np.random.default_rng(M * 1000 + N * 10 + K)
    Xq, Wq = _i8(rng, (M, K)), _i8(rng, (N, K))
    C = oracle.gemm_s32(Xq, Wq)
    assert np.array_equal(C.astype(np.int64), Xq.astype(np.int64) @ Wq.astype(np.int64).T)
    rows = rng.integers(0, M, 5)
    Cr = oracle.gemm_s32(Xq, Wq, rows=rows)
    assert np.array_equal(Cr, C[rows])


def test_gemm_s32_extremes_and_overflow():
    K = 6144
    Xq = np.full((2, K), 127, np.int8)
    Wq = np.stack([np.full(K, -127, np.int8), np.full(K, 127, np.int8)])
    C = oracle.gemm_s32(Xq, Wq)
    assert C[0, 0] == -127 * 127 * K and C[0, 1] == 127 * 127 * K
    Kbig = (2 ** 31) // (127 * 127) + 1
    with pytest.raises(OverflowError):
        oracle.gemm_s32(np.full((1, Kbig), 127, np.int8), np.full((1, Kbig), 127, np.int8))
    # below INT32_MIN as well (sum of -127 * 127 terms)
    Kneg = (2 ** 31) // (127 * 127) + 2
    with pytest.raises(OverflowError):
        oracle.gemm_s32(np.full((1, Kneg), 127, np.int8), np.full((1, Kneg), -127, np.int8))
    # and just inside the range: no error, exact value
    Kok = (2 ** 31 - 1) // (127 * 127)
    C = oracle.gemm_s32(np.full((1, Kok), -127, np.int8), np.full((1, Kok), 127, np.int8))
    assert C[0, 0] == -127 * 127 * Kok


def _half_rne_exact(x: Fraction) -> int:
    """Round an exact rational to binary16 bits, ties to even, from the
    definition: pick the binade, count units in the last place, round."""
    sign = 0x8000 if x < 0 else 0
    a = -x if x < 0 else x
    if a == 0:
        return sign
    e = -14
    while a >= Fraction(2) ** (e + 1) and e < 15:
        e += 1
    ulp = Fraction(2) ** (e - 10)
    q = a / ulp
    n = q.numerator // q.denominator
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    if e == -14 and n < 1024:                      # subnormal (or rounds up to min normal)
        return sign | n
    if n == 2048:
        n, e = 1024, e + 1
    if e > 15:
        return sign | 0x7C00
    return sign | ((e + 15) << 10) | (n - 1024)


def test_half_rne_exact_helper_agrees_with_numpy():
    rng = np.random.default_rng(3)
    for v in np.concatenate([rng.normal(0, 1, 300), rng.normal(0, 1e-6, 100), [6e-8, 65503.9]]):
        assert _half_rne_exact(Fraction(float(v))) == int(np.float16(v).view(np.uint16))


@pytest.mark.parametrize("with_bias,with_steer", [(False, False), (True, False), (True, True)])
def test_w8a8_out_exact_rational(with_bias, with_steer):
    M, N, K = 6, 40, 1536
    W = synthetic.weight("pin/w8a8/W", N, K).numpy()
    X = synthetic.activation("pin/w8a8", M, K, outlier_channel_frac=0.01).numpy()
    Wq, sw = oracle.pack_q8(W)
    Xq, sx = oracle.act_quant(X)
    C = oracle.gemm_s32(Xq, Wq)
    b = synthetic.bias("pin/w8a8", N).numpy() if with_bias else None
    v = synthetic.steer_vec("pin/w8a8", N).numpy() if with_steer else None
    alpha = 0.3 if with_steer else 0.0
    Y = oracle.w8a8_out(C, sx, sw, b, v, alpha)
    for m in range(M):
        for n in range(N):
            t = Fraction(int(C[m, n])) * Fraction(float(sx[m])) * Fraction(float(sw[n]))
            if b is not None:
                t += Fraction(float(b[n]))
            if v is not None:
                t += Fraction(float(np.float32(alpha))) * Fraction(float(v[n]))
            assert Y[m, n] == _half_rne_exact(t), (m, n)


def test_w8a8_out_single_rounding_near_midpoints():
    """Worked by hand at 2048..2052, where fp16 steps by 2: 2049 and 2051 are
    exact midpoints (ties go to the even significand: 2048, 2052); 2049 plus
    a bias of 2^-14 lies just above the midpoint and must round up to 2050.
    Rounding through fp32 first would land on 2049.0 and then tie down to
    2048, so this pins one rounding of the fp64 value."""
    C = np.array([[2049, 2051, 2049]], np.int32)
    sx = np.array([1.0], np.float32)
    sw = np.array([1.0, 1.0, 1.0], np.float32)
    b = np.array([0.0, 0.0, 2.0 ** -14], np.float16)
    Y = oracle.w8a8_out(C, sx, sw, b)
    assert list(Y[0]) == [0x6800, 0x6802, 0x6801]


def test_w8a8_rows_subset_matches_full():
    """Sampled rows (as the GPU tests use them) give the rows of the full
    result: each output row takes the token scale of its own X row."""
    M, N, K = 11, 48, 256
    W = synthetic.weight("pin/w8a8rows/W", N, K).numpy()
    X = synthetic.activation("pin/w8a8rows", M, K, outlier_channel_frac=0.01).numpy()
    X[4] *= 8                                  # token scales that differ a lot
    Wq, sw = oracle.pack_q8(W)
    full = oracle.w8a8(X, Wq, sw)
    rows = [9, 0, 4, 7]
    assert np.array_equal(oracle.w8a8(X, Wq, sw, rows=rows), full[rows])


def test_w8a8_close_to_unquantised_product():
    """|acc*sx*sw - x.w| <= sum_k (|x|*sw/2 + |w|*sx/2 + sx*sw/4) (plus fp32
    quotient slack): pins operand order, scale indexing and the int GEMM."""
    M, N, K = 8, 64, 1536
    W = synthetic.weight("pin/w8a8b/W", N, K).numpy()
    X = synthetic.activation("pin/w8a8b", M, K, outlier_channel_frac=0.01).numpy()
    Wq, sw = oracle.pack_q8(W)
    Xq, sx = oracle.act_quant(X)
    C = oracle.gemm_s32(Xq, Wq).astype(np.float64)
    y = C * sx.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :]
    x64, w64 = X.astype(np.float64), W.astype(np.float64)
    exact = x64 @ w64.T
    sxd, swd = sx.astype(np.float64)[:, None], sw.astype(np.float64)[None, :]
    h = 0.5 + 128 * 2.0 ** -24
    bound = (np.abs(x64).sum(1)[:, None] * swd * h + np.abs(w64).sum(1)[None, :] * sxd * h
             + K * sxd * swd * h * h)
    assert np.all(np.abs(y - exact) <= bound)
    # and the bound is not vacuous: the error is well below |y| typically
    assert np.median(np.abs(y - exact)) < 0.05 * np.median(np.abs(exact))


@pytest.mark.parametrize("fmt", ["q8", "q4"])
def test_wo_ref_matches_numpy_matmul(fmt):
    M, N, K = 9, 48, 512
    W = synthetic.weight(f"pin/wo/{fmt}", N, K, outlier_frac=0.001).numpy()
    X = synthetic.activation(f"pin/wo/{fmt}", M, K).numpy()
    b = synthetic.bias(f"pin/wo/{fmt}", N).numpy()
    v = synthetic.steer_vec(f"pin/wo/{fmt}", N).numpy()
    if fmt == "q8":
        Wq, sc = oracle.pack_q8(W)
        deq = oracle.dequant_q8(Wq, sc)
    else:
        Wq, sc = oracle.pack_q4(W)
        deq = oracle.dequant_q4(Wq, sc)
    Y = oracle.wo_ref(fmt, X, Wq, sc, b, v, 0.3)
    a32 = np.float64(np.float32(0.3))  # alpha crosses the boundary as fp32
    ref = X.astype(np.float64) @ deq.T + b.astype(np.float64) + a32 * v.astype(np.float64)
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)
    rows = [8, 0, 3]
    assert np.array_equal(oracle.wo_ref(fmt, X, Wq, sc, b, v, 0.3, rows=rows), Y[rows])


def test_wo_q8_close_to_unquantised_product():
    M, N, K = 5, 32, 1024
    W = synthetic.weight("pin/woq8b", N, K).numpy()
    X = synthetic.activation("pin/woq8b", M, K).numpy()
    Wq, sw = oracle.pack_q8(W)
    Y = oracle.wo_ref("q8", X, Wq, sw)
    x64 = X.astype(np.float64)
    exact = x64 @ W.astype(np.float64).T
    bound = np.abs(x64).sum(1)[:, None] * sw.astype(np.float64)[None, :] * (0.5 + 128 * 2.0 ** -24)
    assert np.all(np.abs(Y - exact) <= bound * (1 + 1e-9))


def test_epilogue_special_cases():
    N, K = 32, 256
    W = synthetic.weight("pin/epi", N, K).numpy()
    b = synthetic.bias("pin/epi", N).numpy()
    v = synthetic.steer_vec("pin/epi", N).numpy()
    Wq, sw = oracle.pack_q8(W)
    Z = np.zeros((3, K), np.float16)
    # zero activations: the output is the bias, exactly
    assert np.array_equal(oracle.wo_ref("q8", Z, Wq, sw, b), np.tile(b.astype(np.float64), (3, 1)))
    assert np.array_equal(oracle.w8a8(Z, Wq, sw, b), np.tile(b.view(np.uint16), (3, 1)))
    # alpha = 0 or no vector: bit-identical to the unsteered output
    X = synthetic.activation("pin/epi", 4, K).numpy()
    base = oracle.w8a8(X, Wq, sw, b)
    assert np.array_equal(oracle.w8a8(X, Wq, sw, b, v, 0.0), base)
    assert np.array_equal(oracle.w8a8(X, Wq, sw, b, None, 0.7), base)
    # steering is linear in alpha in the unrounded reference
    y0 = oracle.wo_ref("q8", X, Wq, sw, b)
    y1 = oracle.wo_ref("q8", X, Wq, sw, b, v, 0.3)
    assert np.allclose(y1 - y0, np.float64(np.float32(0.3)) * v.astype(np.float64), rtol=0, atol=1e-12)


# --------------------------------------------------- the unquantised rung ---
# "Results" (aria project page): the fp16 column of the precision table is
# the transformer with its weights left in fp16. Its reference is the plain
# product in fp64, unrounded.

def test_f16_ref_matches_numpy_matmul():
    M, N, K = 7, 40, 384
    W = synthetic.weight("pin/f16/W", N, K, outlier_frac=0.001).numpy()
    X = synthetic.activation("pin/f16", M, K).numpy()
    b = synthetic.bias("pin/f16", N).numpy()
    v = synthetic.steer_vec("pin/f16", N).numpy()
    Y = oracle.f16_ref(X, W, b, v, 0.3)
    a32 = np.float64(np.float32(0.3))
    ref = X.astype(np.float64) @ W.astype(np.float64).T + b.astype(np.float64) + a32 * v.astype(np.float64)
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)
    rows = [6, 0, 2]
    assert np.array_equal(oracle.f16_ref(X, W, b, v, 0.3, rows=rows), Y[rows])


def test_f16_ref_exact_on_small_integers():
    """Integer-valued operands (|x|, |w| <= 8): every product and partial sum
    is an integer far below 2^53, so the fp64 result equals numpy's int64
    matmul exactly, independent of summation order."""
    rng = np.random.default_rng(3)
    M, N, K = 5, 24, 300
    xi = rng.integers(-8, 9, (M, K))
    wi = rng.integers(-8, 9, (N, K))
    Y = oracle.f16_ref(xi.astype(np.float16), wi.astype(np.float16))
    assert np.array_equal(Y, (xi @ wi.T).astype(np.float64))


def test_f16_ref_one_hot_reads_the_layout_back():
    """X = e_k reads column k of W [N,K] (out x in), exactly: a transposed or
    shifted index gives other values."""
    N, K = 24, 40                              # N != K: a transposed read differs
    W = synthetic.weight("pin/f16onehot/W", N, K).numpy()
    X = np.zeros((K, K), np.float16)
    X[np.arange(K), np.arange(K)] = 1
    Y = oracle.f16_ref(X, W)
    assert np.array_equal(Y, W.astype(np.float64).T)


def test_f16_ref_epilogue_special_cases():
    N, K = 32, 128
    W = synthetic.weight("pin/f16epi/W", N, K).numpy()
    b = synthetic.bias("pin/f16epi", N).numpy()
    v = synthetic.steer_vec("pin/f16epi", N).numpy()
    Z = np.zeros((3, K), np.float16)
    assert np.array_equal(oracle.f16_ref(Z, W, b), np.tile(b.astype(np.float64), (3, 1)))
    X = synthetic.activation("pin/f16epi", 4, K).numpy()
    base = oracle.f16_ref(X, W, b)
    assert np.array_equal(oracle.f16_ref(X, W, b, v, 0.0), base)
    assert np.array_equal(oracle.f16_ref(X, W, b, None, 0.7), base)
    y1 = oracle.f16_ref(X, W, b, v, 0.3)
    assert np.allclose(y1 - base, np.float64(np.float32(0.3)) * v.astype(np.float64), rtol=0, atol=1e-12)

"""Pins for the oracle's quantisers (q8 pack, per-token act quant, q4 pack).

Each check ties the oracle to something other than itself: hand-derived tie
cases (tests/golden), the quantisation error bound |w - q*s| <= s/2, the
attained clamp extremes, the zero / identity matrices, and a one-hot GEMM that
reads the packed layout back column by column.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
# fp32 quotient rounding: |fl(w/s) - w/s| <= 2^-24 * 127.x, so the integer
# rounding of the stored quotient can be off the exact one by that much
SLACK8 = 128 * 2.0 ** -24
SLACK4 = 8 * 2.0 ** -24


def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split(":", 1)
            out[k.strip()] = v.split()
    return out


def _f16(vals):
    return np.array([float(v) for v in vals], np.float64).astype(np.float16)


def test_q8_golden_ties():
    g = _read_golden("q8_ties.txt")
    for r in range(3):
        W = _f16(g[f"w{r}"])[None, :]
        Wq, s = oracle.pack_q8(W)
        assert Wq[0].tolist() == [int(v) for v in g[f"q{r}"]]
        assert float(s[0]) == float(g[f"s{r}"][0])
        Xq, sx = oracle.act_quant(W)               # same rule per token row
        assert np.array_equal(Xq, Wq) and np.array_equal(sx, s)


def test_q4_golden_ties():
    g = _read_golden("q4_ties.txt")
    W = _f16(g["w"])[None, :]
    P, S = oracle.pack_q4(W)
    assert [f"{b:02x}" for b in P[0]] == g["bytes"]
    assert [f"{v:04x}" for v in S[0]] == g["scales"]
    deq = oracle.dequant_q4(P, S)[0]
    assert deq.tolist() == [float(q) * s for q, s in
                            zip([int(v) for v in g["q"]], [1.0] * 32 + [2.0] * 32)]


def _bound_q8(W16, Wq, s):
    w = W16.astype(np.float64)
    err = np.abs(w - Wq.astype(np.float64) * s.astype(np.float64)[:, None])
    lim = s.astype(np.float64)[:, None] * (0.5 + SLACK8)
    return err, lim


@pytest.mark.parametrize("N,K,std", [(64, 256, 0.02), (33, 1536, 1.0), (8, 6144, 3e-3)])
def test_q8_error_bound_and_extremes(N, K, std):
    W = synthetic.weight(f"pin/q8/{N}x{K}", N, K, std=std, outlier_frac=0.001).numpy()
    Wq, s = oracle.pack_q8(W)
    err, lim = _bound_q8(W, Wq, s)
    assert np.all(err <= lim)
    assert Wq.min() >= -127 and Wq.max() <= 127
    # the absmax element of every row lands exactly on +-127
    amax = np.abs(W.astype(np.float64)).argmax(axis=1)
    assert np.all(np.abs(Wq[np.arange(N), amax].astype(int)) == 127)
    # the scale is the absmax / 127 up to one fp32 rounding
    a = np.abs(W.astype(np.float64)).max(axis=1)
    assert np.all(np.abs(s.astype(np.float64) - a / 127) <= a / 127 * 2.0 ** -24)


def test_q8_codes_match_ieee_fp32_rule():
    """Brute force against an independent statement of the rule with numpy's
    IEEE fp32 arithmetic: s = fp32(absmax / 127), q = rint(fp32(x / s)) (half
    to even), over a million fp16 values at many scales. Codes near .5 tell a
    correctly rounded quotient from, e.g., x * (1 / s)."""
    rng = np.random.default_rng(0)
    R, K = 4000, 256
    X16 = (rng.standard_normal((R, K)) * rng.uniform(0.01, 10, (R, 1))).astype(np.float16)
    X = X16.astype(np.float32)
    a = np.abs(X).max(axis=1, keepdims=True)
    s = (a / np.float32(127)).astype(np.float32)
    q = np.clip(np.rint((X / s).astype(np.float32)), -127, 127).astype(np.int8)
    Wq, sw = oracle.pack_q8(X16)
    assert np.array_equal(sw, s[:, 0])
    assert np.array_equal(Wq, q)
    Xq, sx = oracle.act_quant(X16)
    assert np.array_equal(sx, s[:, 0]) and np.array_equal(Xq, q)


def test_q8_zero_and_identity():
    Z = np.zeros((16, 32), np.float16)
    Wq, s = oracle.pack_q8(Z)
    assert not Wq.any() and not s.any()
    I = np.eye(48, dtype=np.float16)
    Wq, s = oracle.pack_q8(I)
    assert np.array_equal(Wq, 127 * np.eye(48, dtype=np.int8))
    assert np.all(s == np.float32(1.0) / np.float32(127.0))


def test_act_quant_outlier_channels():
    X = synthetic.activation("pin/act", 40, 1536, outlier_channel_frac=0.01).numpy()
    Xq, sx = oracle.act_quant(X)
    err, lim = _bound_q8(X, Xq, sx)
    assert np.all(err <= lim)
    amax = np.abs(X.astype(np.float64)).argmax(axis=1)
    assert np.all(np.abs(Xq[np.arange(40), amax].astype(int)) == 127)


@pytest.mark.parametrize("N,K", [(16, 256), (5, 1536), (3, 6144)])
def test_q4_error_bound_and_layout(N, K):
    W = synthetic.weight(f"pin/q4/{N}x{K}", N, K, outlier_frac=0.001).numpy()
    P, S = oracle.pack_q4(W)
    assert P.shape == (N, K // 2) and S.shape == (N, K // 32)
    lo, hi = P & 0x0F, P >> 4
    assert lo.min() >= 1 and hi.min() >= 1        # offset-binary codes in [1, 15]
    deq = oracle.dequant_q4(P, S)
    sf = S.view(np.float16).astype(np.float64)
    sk = np.repeat(sf, 32, axis=1)
    w = W.astype(np.float64)
    assert np.all(sf > 2.0 ** -14)                 # normal scales for these draws
    assert np.all(np.abs(w - deq) <= sk * (0.5 + SLACK4))
    # every group's absmax element lands on +-7
    g = w.reshape(N, K // 32, 32)
    am = np.abs(g).argmax(axis=2)
    codes = np.rint(deq.reshape(N, K // 32, 32) / sf[:, :, None])
    picked = np.take_along_axis(codes, am[:, :, None], axis=2)
    assert np.all(np.abs(picked) == 7)
    # the scale is fp16_rn(absmax/7): within half an fp16 ulp of the exact quotient
    a = np.abs(g).max(axis=2)
    assert np.all(np.abs(sf - a / 7) <= np.abs(a / 7) * 2.0 ** -11 * (1 + 1e-6))


def test_q4_zero_group():
    W = np.zeros((2, 64), np.float16)
    W[1, 40] = 1.0
    P, S = oracle.pack_q4(W)
    assert np.all(P[0] == 0x88) and not S[0].any()
    assert S[1, 0] == 0 and S[1, 1] == np.float16(1 / 7).view(np.uint16)


def test_q4_subnormal_scales():
    """Groups whose scale falls in the fp16 subnormal range, worked by hand
    (2^-24 is the smallest fp16 step):
    - absmax 10 * 2^-24: absmax / 7 = 1.43 steps rounds to s16 = 1 step, so
      the quotients +-10 are clamped to codes +-7 (nibbles 15 and 1);
    - absmax 3 * 2^-24: absmax / 7 = 0.43 steps rounds to s16 = 0, and a zero
      scale gives code 0 (nibble 8) for every element, not +-7."""
    t = 2.0 ** -24
    W = np.zeros((2, 32), np.float64)
    W[0, 0], W[0, 3], W[0, 9] = 10 * t, -2 * t, -10 * t
    W[1, 5], W[1, 6] = 3 * t, -3 * t
    P, S = oracle.pack_q4(W.astype(np.float16))
    assert S[0, 0] == 0x0001 and S[1, 0] == 0x0000
    nib = np.stack([P & 0x0F, P >> 4], axis=-1).reshape(2, 32)
    expect0 = np.full(32, 8)
    expect0[0], expect0[3], expect0[9] = 15, 8 - 2, 1
    assert np.array_equal(nib[0], expect0)
    assert np.all(nib[1] == 8)


@pytest.mark.parametrize("fmt", ["q8", "q4"])
def test_one_hot_reads_layout_back(fmt):
    """X = e_k picks column k of the dequantised weights; since dequant(W) is
    within s/2 of W, a swapped nibble, transposed layout or wrong scale index
    lands far outside the bound."""
    N, K = 24, 128
    W = synthetic.weight(f"pin/onehot/{fmt}", N, K, std=1.0).numpy()
    Wq, sc = oracle.pack_q8(W) if fmt == "q8" else oracle.pack_q4(W)
    X = np.eye(K, dtype=np.float16)
    Y = oracle.wo_ref(fmt, X, Wq, sc)
    w = W.astype(np.float64)
    if fmt == "q8":
        lim = sc.astype(np.float64)[None, :] * (0.5 + SLACK8)
    else:
        lim = np.repeat(sc.view(np.float16).astype(np.float64), 32, axis=1).T * (0.5 + SLACK4)
    assert np.all(np.abs(Y - w.T) <= lim)

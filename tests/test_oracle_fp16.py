"""Pins for the oracle's own binary16 conversions (CPU only).

The oracle decodes and rounds fp16 with its own bit-level C code; these tests
tie it to two independent implementations (numpy's and torch's conversions)
and to the IEEE definition of round-to-nearest-even.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def test_half_decode_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.half_to_double(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # signed zeros survive
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_double_to_half_matches_numpy_random():
    rng = np.random.default_rng(1)
    # log-uniform magnitudes across subnormal, normal and overflow ranges
    mag = np.exp2(rng.uniform(-30, 17, 400_000))
    x = mag * rng.choice([-1.0, 1.0], mag.size)
    ours = oracle.double_to_half(x)
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


def test_double_to_half_round_trip_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16).astype(np.float64)
    ok = ~np.isnan(vals)
    assert np.array_equal(oracle.double_to_half(vals[ok]), bits[ok])


def test_double_to_half_ties_to_even():
    # exact midpoints between adjacent halves go to the even significand
    bits = np.arange(0x0000, 0x7bff, dtype=np.uint16)          # finite positive, not max
    lo = bits.view(np.float16).astype(np.float64)
    hi = (bits + 1).view(np.float16).astype(np.float64)
    mid = (lo + hi) / 2                                          # exact in fp64
    expect = np.where(bits % 2 == 0, bits, bits + 1).astype(np.uint16)
    assert np.array_equal(oracle.double_to_half(mid), expect)
    # just above / below a midpoint goes to the nearer neighbour (single rounding)
    up = np.nextafter(mid, np.inf)
    dn = np.nextafter(mid, -np.inf)
    assert np.array_equal(oracle.double_to_half(up), (bits + 1).astype(np.uint16))
    assert np.array_equal(oracle.double_to_half(dn), bits)


def test_overflow_and_specials():
    x = np.array([65504.0, 65519.999, 65520.0, 1e9, -65520.0, np.inf, -np.inf, 0.0, -0.0])
    got = oracle.double_to_half(x)
    assert list(got) == [0x7BFF, 0x7BFF, 0x7C00, 0x7C00, 0xFC00, 0x7C00, 0xFC00, 0x0000, 0x8000]
    h = int(oracle.double_to_half(np.array([np.nan]))[0])
    assert (h & 0x7C00) == 0x7C00 and (h & 0x03FF) != 0   # a NaN, not an infinity


def test_float_to_half_matches_torch():
    g = torch.Generator().manual_seed(7)
    x = torch.randn(1_000_000, generator=g) * torch.exp2(torch.randint(-20, 12, (1_000_000,), generator=g).float())
    ref = x.to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    ours = oracle.float_to_half(x.numpy())
    assert np.array_equal(ours, ref)

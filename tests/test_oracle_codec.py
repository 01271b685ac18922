"""Pins of the oracle's E4M3 codec and ExpCast byte map against things other
than the oracle itself: torch's float8_e4m3fn conversion (an independent
implementation of the format), exact rational arithmetic, and the byte
identity printed on chooseai.io news 7051 (ExpCast-FP8 section)."""
import math
import os
from fractions import Fraction

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def torch_encode(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_decode_exhaustive_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_value(codes)
    ref = torch_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert set(codes[nan]) == {0x7F, 0xFF}
    assert np.array_equal(ours[~nan], ref[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x38] == 1.0


def test_encode_random_vs_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(400_000) * 60,
        rng.standard_normal(200_000) * 0.01,  # subnormal range
        rng.uniform(-448, 448, 200_000),
    ]).astype(np.float32)
    x = np.clip(x, -448, 448)
    assert np.array_equal(oracle.e4m3_encode(x), torch_encode(x))


def test_encode_ties_go_to_even_code():
    vals = oracle.e4m3_value(np.arange(127, dtype=np.uint8))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (vals[:-1] + vals[1:]) / 2)  # exact in fp32
    ours = oracle.e4m3_encode(mids)
    assert np.array_equal(ours, torch_encode(mids))
    assert np.all(ours % 2 == 0)
    assert np.array_equal(oracle.e4m3_encode(-mids), torch_encode(-mids))


def test_encode_saturates_and_signs():
    big = np.array([448.0, 449.0, 463.9, 464.0, 1e4, 3e38], np.float32)
    assert np.all(oracle.e4m3_encode(big) == 0x7E)
    assert np.all(oracle.e4m3_encode(-big) == 0xFE)
    assert oracle.e4m3_encode(np.array([0.0], np.float32))[0] == 0x00
    assert oracle.e4m3_encode(np.array([-1e-6], np.float32))[0] == 0x80  # -0, as torch
    assert torch_encode(np.array([-1e-6], np.float32))[0] == 0x80


def test_byte_identity_golden():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e4m3_byte_identity.txt")) if l.strip() and l[0] != "#"]
    for k, byte, p in rows:
        assert int(byte) == 56 + 8 * int(k)
        assert oracle.e4m3_value(np.array([int(byte)], np.uint8))[0] == float(p) == 2.0 ** int(k)


def test_byte_identity_mitchell_bound():
    """dec(b) / 2^((b-56)/8) lies in [1, max_f (1+f)/2^f] for every normal byte."""
    b = np.arange(8, 127)
    ratio = oracle.e4m3_value(b.astype(np.uint8)) / 2.0 ** ((b - 56) / 8.0)
    f = 1.0 / math.log(2.0) - 1.0
    bound = (1.0 + f) / 2.0 ** f
    assert abs(bound - 1.0615) < 1e-4
    assert ratio.min() >= 1.0 - 1e-15
    assert ratio.max() <= bound + 1e-12
    assert np.all(ratio[(b % 8) == 0] == 1.0)


def _expcast_exact(A, s, cb):
    t = Fraction(float(A)) * Fraction(float(s)) + Fraction(float(cb))
    return min(255, max(0, round(t)))  # Python rounds a Fraction half to even


def test_expcast_matches_exact_rationals():
    rng = np.random.default_rng(1)
    n = 20000
    A = rng.uniform(0.0, 3.0, n).astype(np.float32)
    s = (rng.standard_normal(n) * 50).astype(np.float32)
    cb = rng.integers(-100, 130, n).astype(np.float32)
    ours = oracle.expcast_bytes(A, s, cb)
    ref = np.array([_expcast_exact(a, b, c) for a, b, c in zip(A, s, cb)])
    assert np.array_equal(ours, ref)


def test_expcast_ties_and_clamp():
    # A*s = m + 1/2 exactly: the result is the even integer, for odd and even cb.
    A = np.full(8, 0.5, np.float32)
    s = np.array([1, 3, 5, 7, 1, 3, 5, 7], np.float32)
    cb = np.array([0, 0, 0, 0, 1, 1, 1, 1], np.float32)
    got = oracle.expcast_bytes(A, s, cb)
    assert list(got) == [0, 2, 2, 4, 2, 2, 4, 4]
    # just below / above a half: no tie
    up = np.nextafter(np.float32(0.5), np.float32(1))
    dn = np.nextafter(np.float32(0.5), np.float32(0))
    assert list(oracle.expcast_bytes(np.array([1, 1], np.float32), np.array([up, dn], np.float32),
                                     np.array([10, 10], np.float32))) == [11, 10]
    # negative t clamps to byte 0 (probability 0)
    assert list(oracle.expcast_bytes(np.array([1, 2], np.float32), np.array([-3.2, -1e6], np.float32),
                                     np.array([2, 120], np.float32))) == [0, 0]


def test_expcast_tracks_2_to_the_z():
    """byte = round(8z + 56 + beta) decodes to 2^(z + beta/8) within the Mitchell bound and half a step."""
    beta = 64
    z = np.linspace(-14.0, 0.0, 100001)
    s = (8.0 * z).astype(np.float32)
    got = oracle.e4m3_value(oracle.expcast_bytes(np.ones_like(s), s, np.full_like(s, 56 + beta)))
    ratio = got / 2.0 ** (s.astype(np.float64) / 8.0 + beta / 8.0)
    assert ratio.min() >= 2.0 ** (-1 / 16) - 1e-12
    assert ratio.max() <= 1.0615 * 2.0 ** (1 / 16) + 1e-12
    lr = np.log2(ratio)
    assert 0.03 < lr.std() < 0.06


def test_kappa_constants():
    assert oracle.kappa(64) == float(np.float32(math.log2(math.e)))
    assert oracle.kappa(128) == float(np.float32(math.log2(math.e) / math.sqrt(2.0)))
    assert np.float32(oracle.kappa(64)).view(np.uint32) == 0x3FB8AA3B


def test_expcast_rounds_once_on_constructed_witnesses():
    """Thousands of inputs where one rounding and two disagree: the oracle's
    byte is the exact rational A*s + cb rounded once, never the byte that an
    fp32 product would give."""
    from conftest import expcast_rounding_witnesses

    A, s, cb, prod = expcast_rounding_witnesses(11, 20_000)
    assert A.size > 10_000
    got = oracle.expcast_bytes(A, s, cb)
    for i in range(0, A.size, 7):
        t = Fraction(float(A[i])) * Fraction(float(s[i])) + int(cb[i])
        assert t.denominator > 2  # never an exact tie
        assert got[i] == max(0, round(t)), (i, float(A[i]), float(s[i]), float(cb[i]))
    d32 = (A * s).astype(np.float64)  # the product rounded to fp32 first: a tie
    assert np.all(d32 - np.floor(d32) == 0.5)
    two = d32 + cb.astype(np.float64)
    two = np.where(np.floor(two) % 2 == 0, np.floor(two), np.ceil(two))
    assert np.all(got != two)


def test_expcast_rounds_once():
    """A constructed witness: A * s lies 1.7e-7 above -9.5, so A * s + 120 is
    just above the tie 110.5 and rounds once to byte 111.  Rounding the
    product to fp32 first would give exactly -9.5, whose tie goes to the even
    byte 110.  The single FMA of the method has one rounding."""
    A = np.float32(float.fromhex("0x1.1787cep+0"))
    s = np.float32(float.fromhex("-0x1.1668e2p+3"))
    exact = Fraction(float(A)) * Fraction(float(s))
    assert Fraction(-19, 2) < exact < Fraction(-19, 2) + Fraction(1, 2 ** 20)
    assert np.float32(A * s) == np.float32(-9.5)  # the product alone rounds onto the tie
    b = oracle.expcast_bytes(np.array([A]), np.array([s]), np.array([120.0], np.float32))
    assert b[0] == 111

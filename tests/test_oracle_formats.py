"""Pins for the oracle's scalar E2M1 / E4M3 encoders and decoders.

The pins come from outside the oracle: the bit-field definitions of the two
formats, hand-derived round-to-nearest-even ties, and two independent library
casts (ml_dtypes float4_e2m1fn / float8_e4m3fn and torch float8_e4m3fn).
"""
import numpy as np
import pytest
import torch

ml_dtypes = pytest.importorskip("ml_dtypes")


def e2m1_from_bits(c: int) -> float:
    """E2M1: sign bit 3, 2 exponent bits (bias 1), 1 mantissa bit; e=0 is subnormal."""
    s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
    mag = m * 0.5 if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
    return -mag if s else mag


def e4m3_from_bits(b: int) -> float:
    """E4M3 (fn): sign bit 7, 4 exponent bits (bias 7), 3 mantissa bits; S.1111.111 is NaN."""
    s, e, m = (b >> 7) & 1, (b >> 3) & 15, b & 7
    if e == 15 and m == 7:
        return float("nan")
    mag = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
    return -mag if s else mag


def test_e2m1_decode_table(orc):
    for c in range(16):
        assert orc.e2m1_decode(c) == e2m1_from_bits(c), c
    # the magnitude set the pages describe
    assert sorted({abs(e2m1_from_bits(c)) for c in range(16)}) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_e2m1_roundtrip(orc):
    for c in range(16):
        assert orc.e2m1_encode(e2m1_from_bits(c)) == c


def test_e2m1_ties_to_even(orc):
    # midpoint -> (code below, code above, code chosen at the tie), derived by hand:
    # the tie goes to the neighbour whose code is even
    ties = {0.25: (0, 1, 0), 0.75: (1, 2, 2), 1.25: (2, 3, 2), 1.75: (3, 4, 4),
            2.5: (4, 5, 4), 3.5: (5, 6, 6), 5.0: (6, 7, 6)}
    for q, (below, above, tie) in ties.items():
        assert orc.e2m1_encode(q) == tie, q
        assert orc.e2m1_encode(-q) == tie | 8, -q
        assert orc.e2m1_encode(np.nextafter(np.float32(q), np.float32(10))) == above
        assert orc.e2m1_encode(np.nextafter(np.float32(q), np.float32(-10))) == below


def test_e2m1_saturation_and_sign(orc):
    for q in (6.0, 6.5, 7.0, 100.0, 3e38, float("inf")):
        assert orc.e2m1_encode(q) == 7
        assert orc.e2m1_encode(-q) == 15
    assert orc.e2m1_encode(0.0) == 0
    assert orc.e2m1_encode(-0.0) == 8
    assert orc.e2m1_encode(-0.1) == 8  # rounds to zero, sign kept


def test_e2m1_matches_ml_dtypes_dense_sweep(orc):
    # every fp32 with |q| in [2^-4, 8) (all rounding decisions live there), both signs,
    # strided by 37 ulps, plus a random sample of all finite fp32
    lo = np.float32(2.0 ** -4).view(np.uint32)
    hi = np.float32(8.0).view(np.uint32)
    bits = np.arange(lo, hi, 37, dtype=np.uint32)
    rng = np.random.default_rng(7)
    rnd = rng.integers(0, 0x7F800000, 1 << 18, dtype=np.uint32)
    q = np.concatenate([bits, rnd]).view(np.float32)
    q = np.concatenate([q, -q])
    ours = orc.e2m1_encode_array(q)
    ref = q.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    np.testing.assert_array_equal(ours, ref)


def test_e4m3_decode_all_bytes(orc):
    lib = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for b in range(256):
        v = orc.e4m3_decode(b)
        if np.isnan(lib[b]):
            assert np.isnan(v) and np.isnan(e4m3_from_bits(b))
        else:
            assert v == lib[b] == e4m3_from_bits(b), b
    assert orc.e4m3_decode(0x7E) == 448.0
    assert orc.e4m3_decode(0x08) == 2.0 ** -6  # smallest normal, step 2^-3 relative
    assert orc.e4m3_decode(0x01) == 2.0 ** -9


def test_e4m3_roundtrip(orc):
    for b in range(0x7F):
        assert orc.e4m3_encode(e4m3_from_bits(b)) == b


def test_e4m3_matches_libraries(orc):
    rng = np.random.default_rng(11)
    # log-uniform sample over the whole useful range, plus every midpoint +-1 ulp
    x = np.exp2(rng.uniform(-14, np.log2(464.0), 1 << 18)).astype(np.float32)
    vals = np.array([e4m3_from_bits(b) for b in range(0x7F)], dtype=np.float64)
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, np.nextafter(mids, np.float32(1e9)), np.nextafter(mids, np.float32(0)),
                        np.float32([0.0, 448.0, 460.0, 464.0])])
    ours = orc.e4m3_encode_array(x)
    ref_ml = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    ref_t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, ref_ml)
    np.testing.assert_array_equal(ours, ref_t)


def test_e4m3_saturates(orc):
    # the libraries return NaN above 464; the reading is saturation to 448
    for x in (464.0, 465.0, 1000.0, 3e38, float("inf")):
        assert orc.e4m3_encode(x) == 0x7E
    assert orc.e4m3_encode(2.0 ** -10) == 0          # tie between 0 and 2^-9 -> even (0)
    assert orc.e4m3_encode(1.5 * 2.0 ** -9) == 2     # tie between 2^-9 (odd) and 2^-8 (even)

"""Pins for the MXFP4 oracle (a NEXT row: 32-element blocks, E8M0 scales).

The pages give the format (E8M0 power-of-two scales, step 2^1, 32-element
blocks: ARCQuant blog sections 2.2 and 4.2) but no scale rule; the reading
pinned here is the shared-exponent rule: scale 2^(floor(log2 amax_b) - 2)
clamped to 2^-127..2^127, 2^-127 for an all-zero block, elements rounded to
the nearest E2M1 value (ties to even) and saturated at 6.  The pins are
special cases the rule fixes, brute force on small blocks, exact reproduction
of representable blocks, power-of-two equivariance and the per-element error
bound."""
import itertools
import math

import numpy as np
import pytest

import oracle as orc

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e8m0_all_bytes():
    for b in range(255):
        assert orc.e8m0_decode(b) == 2.0 ** (b - 127)
    assert math.isnan(orc.e8m0_decode(255))


@pytest.mark.parametrize("k", [-125, -30, -2, -1, 0, 1, 2, 7, 100, 127])
def test_scale_byte_at_powers_of_two(k):
    # amax = 2^k: floor(log2) = k -> exponent k - 2; just below 2^k -> k - 3
    assert orc.mx_scale_byte(2.0 ** k) == max(0, min(254, k - 2 + 127))
    below = np.nextafter(np.float32(2.0 ** k), np.float32(0))
    if below > 0:
        assert orc.mx_scale_byte(float(below)) == max(0, min(254, k - 3 + 127))


def test_scale_byte_special_cases():
    assert orc.mx_scale_byte(0.0) == 0                      # all-zero block
    assert orc.mx_scale_byte(6.0) == 127                    # 6 = 1.5 * 2^2 -> 2^0
    assert orc.mx_scale_byte(1.0e38) == 124 + 127           # 2^126 <= 1e38 < 2^127
    assert orc.mx_scale_byte(float(np.finfo(np.float32).max)) == 125 + 127   # fp32 never reaches the clamp
    assert orc.mx_scale_byte(1.0e-44) == 0                  # subnormal: clamps at 2^-127


def _brute_code(q):
    """Nearest E2M1 code to q by enumeration (ties to the even code), saturating."""
    sign = 8 if math.copysign(1.0, q) < 0 else 0
    a = abs(q)
    if a >= 6.0:
        return sign | 7
    best = min(range(8), key=lambda c: (abs(a - E2M1[c]), c & 1))
    return sign | best


def test_brute_force_small_blocks():
    rng = np.random.default_rng(7)
    for trial in range(200):
        x = (rng.standard_normal((1, 32)) * np.exp2(rng.integers(-20, 20))).astype(np.float32)
        if trial % 7 == 0:
            x[0, rng.integers(0, 32, 5)] = 0.0
        codes, scales = orc.mx_quantize(x)
        amax = float(np.max(np.abs(x)))
        e = math.frexp(amax)[1] - 1 - 2 if amax > 0 else -127
        assert scales[0, 0] == e + 127
        for i in range(32):
            assert codes[0, i] == _brute_code(float(x[0, i]) / 2.0 ** e), (trial, i)


def test_representable_blocks_reproduce():
    rng = np.random.default_rng(3)
    for e in (-100, -9, -2, 0, 3, 60):
        for _ in range(20):
            c = rng.integers(0, 16, 32).astype(np.uint8)
            c[rng.integers(0, 32)] = rng.choice([6, 7, 14, 15])     # |v| in {4, 6} fixes the exponent
            vals = np.array([orc.e2m1_decode(int(k)) for k in c]) * 2.0 ** e
            x = vals.astype(np.float32)[None, :]
            codes, scales = orc.mx_quantize(x)
            assert scales[0, 0] == e + 127
            np.testing.assert_array_equal(orc.mx_dequant(codes, scales), vals[None, :])


def test_power_of_two_equivariance():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((4, 128)).astype(np.float32)
    c0, s0 = orc.mx_quantize(x)
    for j in (-20, -3, 5, 40):
        c1, s1 = orc.mx_quantize((x * np.float32(2.0 ** j)).astype(np.float32))
        np.testing.assert_array_equal(c1, c0)
        np.testing.assert_array_equal(s1.astype(int), s0.astype(int) + j)


def test_error_bound():
    """|x - deq| <= half the E2M1 spacing at |x|/scale (0.25, 0.5 or 1) x scale
    below 6 x scale; within (6, 8) x scale the clip error is at most 2 x scale."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((16, 256)) * np.exp2(rng.uniform(-30, 30, (16, 8)).repeat(32, axis=1)))
    x = x.astype(np.float32)
    codes, scales = orc.mx_quantize(x)
    deq = orc.mx_dequant(codes, scales)
    scale = np.exp2(scales.astype(np.float64) - 127).repeat(32, axis=1)
    q = np.abs(x.astype(np.float64)) / scale
    half = np.where(q <= 2.0, 0.25, np.where(q <= 4.0, 0.5, 1.0))
    bound = np.where(q <= 6.0, half, 2.0) * scale
    assert np.all(np.abs(x - deq) <= bound * (1 + 1e-12))
    assert np.all(q < 8.0)


def test_residue_bounds_and_gain():
    rng = np.random.default_rng(9)
    x = (0.5 * rng.standard_t(3, (8, 512))).astype(np.float32)
    (cx, sx), (cr, sr) = orc.mx_quantize_residue(x)
    r = (x - orc.mx_dequant(cx, sx).astype(np.float32)).astype(np.float32)
    np.testing.assert_array_equal(orc.mx_quantize(r)[0], cr)   # R is quantized like any tensor
    e1 = np.linalg.norm(x - orc.mx_dequant(cx, sx))
    e2 = np.linalg.norm(x - orc.mx_dequant(cx, sx) - orc.mx_dequant(cr, sr))
    assert e2 < e1 / 4


def test_gemm_is_the_plain_triple_sum():
    rng = np.random.default_rng(2)
    a = rng.standard_normal((3, 64)).astype(np.float32)
    w = rng.standard_normal((5, 64)).astype(np.float32)
    qa, qw = orc.mx_quantize(a), orc.mx_quantize(w)
    ad, wd = orc.mx_dequant(*qa), orc.mx_dequant(*qw)
    y = orc.mx_gemm(qa, qw)
    for m, n in itertools.product(range(3), range(5)):
        assert y[m, n] == pytest.approx(sum(ad[m, k] * wd[n, k] for k in range(64)), rel=1e-12)
    (qa2, qr2) = orc.mx_quantize_residue(a)
    y2 = orc.mx_gemm(qa2, qw, qr2)
    rd = orc.mx_dequant(*qr2)
    assert y2[1, 2] == pytest.approx(sum((ad[1, k] + rd[1, k]) * wd[2, k] for k in range(64)), rel=1e-12)

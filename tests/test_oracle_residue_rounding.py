"""Pins for the rounding of the oracle's residue stage, in exact rational arithmetic.

The residue is R = X - deq(Q(X)) (ResServe abstract: the FP4-quantized residue
of what quantization lost; ARCQuant blog post section 3.1: the second stage
quantizes what the first left).  The pages do not fix its fp32 operation order;
the reading taken is

    deq = fl32(fl32(v * d) * s),   R = fl32(x - deq)

with v the E2M1 value, d the E4M3 block scale and s the FP32 tensor scale.
v * d is exact in binary32, so deq is the single rounding RN32(v d s) of an
exact rational.  These tests recompute every element from Python Fractions,
rounded to binary32 by an integer routine written here, so a different order
(for instance d * s rounded first) or a dropped rounding fails element by
element.  The tensor scales used are not powers of two, where every order
would agree.  MXFP4 (a NEXT row; ARCQuant blog post sections 2.2 and 4.2):
deq = v * 2^(b - 127) is exact, so only the subtraction rounds.
"""
from fractions import Fraction

import numpy as np
import pytest

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def e4m3_value(b: int) -> Fraction:
    e, m = (b >> 3) & 15, b & 7
    v = Fraction(m, 2 ** 9) if e == 0 else Fraction(8 + m, 8) * Fraction(2) ** (e - 7)
    return -v if b & 0x80 else v


def e2m1_value(c: int) -> Fraction:
    v = Fraction(E2M1[c & 7])
    return -v if c & 8 else v


def round_f32(q: Fraction) -> float:
    """The binary32 value nearest to the rational q, ties to the even significand
    (normal and subnormal range; the inputs here never overflow)."""
    if q == 0:
        return 0.0
    neg = q < 0
    a = -q if neg else q
    # exponent e with 2^e <= a < 2^(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)                     # subnormals share the spacing 2^-149
    ulp = Fraction(2) ** (e - 23)
    n, rem = divmod(a, ulp)              # a = n * ulp + rem, 0 <= rem < ulp
    n = int(n)
    if rem * 2 > ulp or (rem * 2 == ulp and n % 2 == 1):
        n += 1
    v = float(Fraction(n) * ulp)         # n * 2^k is exact in binary64 here
    return -v if neg else v


def test_round_f32_against_numpy():
    """The helper agrees with numpy's binary64 -> binary32 cast, a single IEEE rounding,
    on rationals that binary64 holds exactly (ties and subnormals included)."""
    rng = np.random.default_rng(0)
    vals = list(rng.standard_normal(2000) * np.exp2(rng.integers(-140, 60, 2000)))
    vals += [1 + 2.0 ** -24, 1 + 3 * 2.0 ** -24, 2.0 ** -149 * 1.5, 2.0 ** -149 * 2.5, 2.0 ** -130 / 3]
    for v in vals:
        assert round_f32(Fraction(v)) == float(np.float32(v)), v


def _nvfp4_case(orc, seed, scale_mul):
    rng = np.random.default_rng(seed)
    x = (scale_mul * rng.standard_normal((6, 96))).astype(np.float32)
    x[:, 5] *= 37.0                       # an outlier channel, as in the workloads
    q = orc.quantize(x)
    s = float(q.s)
    assert np.frexp(s)[0] != 0.5, "the tensor scale must not be a power of two"
    return x, q, s


@pytest.mark.parametrize("seed,scale_mul", [(21, 1.0), (22, 0.37), (23, 1e-3)])
def test_nvfp4_residue_is_exact_rational(orc, seed, scale_mul):
    x, q, s = _nvfp4_case(orc, seed, scale_mul)
    codes = q.unpacked_codes()
    rows, cols = x.shape
    deq = np.empty_like(x)
    res = np.empty_like(x)
    wrong = np.empty_like(x)              # d * s rounded first: fl32(v * fl32(d * s))
    for r in range(rows):
        for k in range(cols):
            v = e2m1_value(int(codes[r, k]))
            d = e4m3_value(int(q.scales[r, k // 16]))
            dq = round_f32(v * d * Fraction(s))
            deq[r, k] = dq
            res[r, k] = round_f32(Fraction(float(x[r, k])) - Fraction(dq))
            wrong[r, k] = round_f32(v * Fraction(round_f32(d * Fraction(s))))
    np.testing.assert_array_equal(orc.dequant_f32(q), deq)
    np.testing.assert_array_equal(orc.residue(x, q), res)
    # the test can tell the two orders apart on these inputs
    assert np.count_nonzero(wrong != deq) > 0


def test_resserve_and_arcquant_residues_use_that_r(orc):
    """Both residue stages quantize exactly this R: ResServe under its own tensor scale,
    ARCQuant's first S reordered columns under the shared s_aug."""
    x, q, s = _nvfp4_case(orc, 24, 0.8)
    codes = q.unpacked_codes()
    rows, cols = x.shape
    res = np.empty_like(x)
    for r in range(rows):
        for k in range(cols):
            dq = round_f32(e2m1_value(int(codes[r, k])) * e4m3_value(int(q.scales[r, k // 16])) * Fraction(s))
            res[r, k] = round_f32(Fraction(float(x[r, k])) - Fraction(dq))
    _, qr = orc.quantize_residue(x)
    qr_ref = orc.quantize(res)
    np.testing.assert_array_equal(qr.codes, qr_ref.codes)
    np.testing.assert_array_equal(qr.scales, qr_ref.scales)
    assert qr.s == qr_ref.s
    S = 32
    xa = orc.rmsnorm_reorder_quantize(x, gamma=None, perm=None, S=S)
    qs = orc.quantize(res[:, :S], s)
    np.testing.assert_array_equal(xa.codes[:, cols // 2:], qs.codes)
    np.testing.assert_array_equal(xa.scales[:, cols // 16:], qs.scales)


def test_mx_residue_is_exact_rational(orc):
    rng = np.random.default_rng(25)
    x = (0.5 * rng.standard_t(3, (4, 128))).astype(np.float32)
    x[1, :32] *= 1e-30                     # a block of tiny values (small E8M0 scale)
    (cx, sx), _ = orc.mx_quantize_residue(x)
    r = orc.mx_residue(x, (cx, sx))
    rows, cols = x.shape
    for i in range(rows):
        for k in range(cols):
            deq = e2m1_value(int(cx[i, k])) * Fraction(2) ** (int(sx[i, k // 32]) - 127)
            assert r[i, k] == round_f32(Fraction(float(x[i, k])) - deq), (i, k)

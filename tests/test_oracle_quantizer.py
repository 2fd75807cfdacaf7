"""Pins for the oracle's block quantizer, residue stages and ARCQuant augmentation.

Checks come from the mathematics and the pages, never from re-running the
oracle's own steps: exactly representable inputs, exact-rational nearest-point
search, sign and power-of-two symmetries, the per-element half-spacing bound and
the two-stage bounds stated in the ARCQuant post (section 4.1-4.2).
"""
from fractions import Fraction

import numpy as np
import pytest

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def e4m3_values():
    out = []
    for b in range(0x7F):
        e, m = (b >> 3) & 15, b & 7
        out.append(m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return np.array(out)


E4M3 = e4m3_values()


def decode_block_scales(scales):
    return E4M3[scales.astype(np.int64) & 0x7F]


def test_representable_inputs_reproduce(orc):
    """x = v(c) * d * s with s a power of two, one block at d = 448 and a +-6 in every
    block: the quantizer must return exactly c, d, s and a zero residue."""
    rng = np.random.default_rng(3)
    rows, cols = 8, 256
    s = np.float32(2.0 ** -5)
    nb = cols // 16
    d_idx = rng.integers(8, 0x7F, size=(rows, nb))            # normal E4M3 scales
    d_idx[0, 0] = 0x7E                                        # d = 448 fixes amax = 2688 s
    codes = rng.integers(0, 16, size=(rows, cols))
    codes[:, ::16] = rng.choice([7, 15], size=(rows, nb))       # a +-6 in every block
    v = np.array([E2M1[c & 7] * (-1 if c & 8 else 1) for c in codes.ravel()]).reshape(rows, cols)
    d = E4M3[d_idx]
    x = (v * np.repeat(d, 16, axis=1) * float(s)).astype(np.float32)
    assert np.all(x.astype(np.float64) == v * np.repeat(d, 16, axis=1) * float(s))
    q = orc.quantize(x)
    assert q.s == s
    np.testing.assert_array_equal(q.scales, d_idx)
    got = q.unpacked_codes()
    # -0 codes stay -0 only where the input was -0: a zero value was built from code 0 or 8
    np.testing.assert_array_equal(got & 7, codes & 7)
    nz = (codes & 7) != 0
    np.testing.assert_array_equal(got[nz], codes[nz])
    r = orc.residue(x, q)
    assert np.all(r == 0)


def _nearest_e4m3_exact(ratio: Fraction):
    """All E4M3 values at minimal exact distance from ratio (saturating at 448)."""
    if ratio >= 448:
        return {0x7E}
    dists = [abs(Fraction(float(v)) - ratio) for v in E4M3]
    m = min(dists)
    return {b for b, dd in enumerate(dists) if dd == m}


def test_block_scale_is_nearest_e4m3(orc):
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((64, 512)) * np.exp2(rng.uniform(-8, 8, (64, 1)))).astype(np.float32)
    q = orc.quantize(x)
    s = Fraction(float(q.s))
    assert q.s == np.float32(np.abs(x).max() / np.float32(2688.0))
    blocks = np.abs(x).reshape(64, 32, 16).max(axis=2)
    for (r, b), a in np.ndenumerate(blocks):
        exact = Fraction(float(a)) / (6 * s)
        cand = _nearest_e4m3_exact(exact)
        got = int(q.scales[r, b])
        if len(cand) == 1 and got not in cand:
            # only a near-tie may differ (the ratio is formed in fp32)
            lo = max(v for v in E4M3 if v <= exact)
            hi = min(v for v in E4M3 if v >= exact)
            mid = (Fraction(lo) + Fraction(hi)) / 2
            assert abs(exact - mid) / exact < Fraction(1, 1 << 20), (r, b)
        else:
            assert got in cand or len(cand) > 1


def test_codes_are_nearest_grid_points(orc):
    """Each code minimises |x - v(c) d s| over all 16 codes, up to fp32 rounding of x/(d s)."""
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((32, 256)) * 3).astype(np.float32)
    x[:, 5] *= 40
    q = orc.quantize(x)
    codes = q.unpacked_codes()
    d = np.repeat(decode_block_scales(q.scales), 16, axis=1)
    ds = d * float(q.s)
    grid = np.array([E2M1[c & 7] * (-1 if c & 8 else 1) for c in range(16)])
    err_all = np.abs(x[..., None].astype(np.float64) - grid[None, None, :] * ds[..., None])
    best = err_all.min(axis=2)
    got = np.abs(x.astype(np.float64) - grid[codes] * ds)
    assert np.all(got <= best + 1e-6 * ds)


def test_sign_symmetry(orc):
    rng = np.random.default_rng(8)
    x = rng.standard_normal((16, 128)).astype(np.float32)
    a, b = orc.quantize(x), orc.quantize(-x)
    np.testing.assert_array_equal(a.scales, b.scales)
    np.testing.assert_array_equal(a.unpacked_codes() ^ 8, b.unpacked_codes())
    assert a.s == b.s


@pytest.mark.parametrize("k", [-20, -3, 1, 7])
def test_power_of_two_invariance(orc, k):
    rng = np.random.default_rng(9)
    x = rng.standard_normal((16, 128)).astype(np.float32)
    a, b = orc.quantize(x), orc.quantize(np.ldexp(x, k).astype(np.float32))
    np.testing.assert_array_equal(a.codes, b.codes)
    np.testing.assert_array_equal(a.scales, b.scales)
    assert b.s == np.float32(np.ldexp(np.float64(a.s), k))


def test_zero_block_and_zero_tensor(orc):
    x = np.zeros((2, 32), np.float32)
    q = orc.quantize(x)
    assert q.s == 0 and np.all(q.scales == 0) and np.all(q.codes == 0)
    x[0, 16:] = 1.0  # second block of row 0 non-zero, everything else zero
    q = orc.quantize(x)
    assert q.scales[0, 0] == 0 and q.scales[1, 0] == 0 and q.scales[0, 1] != 0


def _elementwise_bound(q_abs):
    """Half the E2M1 grid spacing around |q| (in units of d*s)."""
    return np.where(q_abs <= 2, 0.25, np.where(q_abs <= 4, 0.5, 1.0))


def test_per_element_error_bound(orc):
    rng = np.random.default_rng(10)
    x = (rng.standard_normal((64, 512)) * np.exp2(rng.uniform(-6, 6, (64, 1)))).astype(np.float32)
    x[:, 17] *= 50
    q = orc.quantize(x)
    d = np.repeat(decode_block_scales(q.scales), 16, axis=1)
    ds = d * float(q.s)
    deq = orc.dequant_f64(q)
    err = np.abs(x - deq)
    qa = np.abs(x) / ds
    inside = qa <= 6
    assert np.all(err[inside] <= _elementwise_bound(qa[inside]) * ds[inside] * (1 + 1e-6))
    # saturated elements: |x| > 6 d s only when d was rounded down, by at most 2^-4 relative
    sat = ~inside & (d >= 2.0 ** -6)
    assert np.all(err[sat] <= 0.4 * ds[sat] * (1 + 1e-6))


def _two_stage_check(x, deq1, deq2, scales1, scales2):
    """ARCQuant section 4: |e1| <= a1 M eps4, |e2| <= a1 a2 M eps4^2 with eps4 = 2^-2,
    a <= 1.125 (sup a1 a2 = 1.266), M the block absolute maximum; checked on blocks whose
    main and residue scales are both normal E4M3 values."""
    eps4 = 0.25
    d1 = decode_block_scales(scales1)
    d2 = decode_block_scales(scales2)
    xb = np.abs(x).reshape(x.shape[0], -1, 16)
    M = xb.max(axis=2)
    e1 = np.abs(x.astype(np.float64) - deq1).reshape(xb.shape).max(axis=2)
    e2 = np.abs(x.astype(np.float64) - deq1 - deq2).reshape(xb.shape).max(axis=2)
    ok = (d1 >= 2.0 ** -6) & (d2 >= 2.0 ** -6)
    assert ok.mean() > 0.5
    assert np.all(e1[ok] <= 1.125 * M[ok] * eps4)
    assert np.all(e2[ok] <= 1.125 ** 2 * M[ok] * eps4 ** 2)
    return e1, e2, ok


def test_resserve_residue_bound(orc):
    rng = np.random.default_rng(12)
    x = (0.5 * rng.standard_t(3, size=(64, 512))).astype(np.float32)
    q, qr = orc.quantize_residue(x)
    # the residue tensor scale is its own amax / 2688
    r = orc.residue(x, q)
    assert qr.s == np.float32(np.abs(r).max() / np.float32(2688.0))
    e1, e2, ok = _two_stage_check(x, orc.dequant_f64(q), orc.dequant_f64(qr), q.scales, qr.scales)
    # the correction must actually reduce the error on normal blocks
    assert e2[ok].sum() < 0.25 * e1[ok].sum()


def _split_aug(orc, xa, K):
    main = orc.QTensor(np.ascontiguousarray(xa.codes[:, : K // 2]),
                       np.ascontiguousarray(xa.scales[:, : K // 16]), xa.s)
    res = orc.QTensor(np.ascontiguousarray(xa.codes[:, K // 2:]),
                      np.ascontiguousarray(xa.scales[:, K // 16:]), xa.s)
    return main, res


def test_arcquant_residue_bound_shared_scale(orc):
    rng = np.random.default_rng(13)
    K, S = 256, 64
    x = rng.standard_normal((32, K)).astype(np.float32)
    x[:, :S] *= 30  # outliers first (already in channel order)
    xa = orc.rmsnorm_reorder_quantize(x, gamma=None, perm=None, S=S)
    main, res = _split_aug(orc, xa, K)
    _two_stage_check(x[:, :S], orc.dequant_f64(main)[:, :S], orc.dequant_f64(res),
                     main.scales[:, : S // 16], res.scales)


def test_arcquant_s0_is_plain_quantize_of_reordered(orc):
    rng = np.random.default_rng(14)
    x = rng.standard_normal((8, 128)).astype(np.float32)
    perm = rng.permutation(128).astype(np.int32)
    xa = orc.rmsnorm_reorder_quantize(x, gamma=None, perm=perm, S=0)
    q = orc.quantize(x[:, perm])
    np.testing.assert_array_equal(xa.codes, q.codes)
    np.testing.assert_array_equal(xa.scales, q.scales)
    assert xa.s == q.s


def test_arcquant_s_eq_k_is_full_residue_under_shared_scale(orc):
    rng = np.random.default_rng(15)
    x = (0.5 * rng.standard_t(3, size=(8, 128))).astype(np.float32)
    xa = orc.rmsnorm_reorder_quantize(x, gamma=None, perm=None, S=128)
    q = orc.quantize(x)
    qr = orc.quantize(orc.residue(x, q), q.s)   # residue under the main tensor scale
    np.testing.assert_array_equal(xa.codes, np.concatenate([q.codes, qr.codes], axis=1))
    np.testing.assert_array_equal(xa.scales, np.concatenate([q.scales, qr.scales], axis=1))


def test_residue_is_exact_difference(orc):
    """R = X - deq(Q(X)) with deq = fl32(fl32(v d) s): R + deq reproduces X (Sterbenz-exact
    where |deq| is within a factor 2 of |x|)."""
    rng = np.random.default_rng(16)
    x = rng.standard_normal((16, 128)).astype(np.float32)
    q = orc.quantize(x)
    deq32 = orc.dequant_f32(q)
    r = orc.residue(x, q)
    close = (np.abs(deq32) >= np.abs(x) / 2) & (np.abs(deq32) <= 2 * np.abs(x)) & (np.sign(deq32) == np.sign(x))
    assert close.mean() > 0.5
    np.testing.assert_array_equal((r + deq32)[close], x[close])

"""Pins for the oracle's RMSNorm and fp64 GEMM.

RMSNorm: closed forms (constant rows, +-1 rows), order independence, and the
textbook definition evaluated by torch in fp64.  GEMM: brute force in exact
rational arithmetic on tiny operands, one-hot operands (which fix every index
and the scale placement), and the ARCQuant K+S identity
Q(X)Q(W)^T + Q(R)Q(W_o)^T = [QX | QR][QW | QW_o]^T.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _e4m3(b):
    e, m = (b >> 3) & 15, b & 7
    return m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)


# ------------------------------------------------------------------ RMSNorm

@pytest.mark.parametrize("c", [1.0, 0.375, 3.0, 1e-3, 250.0])
def test_rmsnorm_constant_row(orc, c):
    eps = 1e-5
    x = np.full((1, 512), c, np.float32)
    y, rinv = orc.rmsnorm(x, None, eps, return_rinv=True)
    expect = np.float32(1.0 / np.sqrt(np.float64(np.float32(c)) ** 2 + np.float64(np.float32(eps))))
    assert rinv[0] == expect
    assert np.all(y == np.float32(np.float32(c) * expect))


def test_rmsnorm_pm_one_rows(orc):
    rng = np.random.default_rng(1)
    x = rng.choice([-1.0, 1.0], size=(4, 4096)).astype(np.float32)
    gamma = rng.uniform(0.8, 1.2, 4096).astype(np.float32)
    y, rinv = orc.rmsnorm(x, gamma, 1e-6, return_rinv=True)
    expect = np.float32(1.0 / np.sqrt(1.0 + np.float64(np.float32(1e-6))))
    assert np.all(rinv == expect)
    np.testing.assert_array_equal(y, (x * expect).astype(np.float32) * gamma)


def test_rmsnorm_order_independent(orc):
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((8, 1024)) * np.exp2(rng.uniform(-10, 10, (8, 1024)))).astype(np.float32)
    _, r0 = orc.rmsnorm(x, None, 1e-5, return_rinv=True)
    for seed in range(3):
        p = np.random.default_rng(seed).permutation(1024)
        _, r1 = orc.rmsnorm(x[:, p], None, 1e-5, return_rinv=True)
        np.testing.assert_array_equal(r0, r1)


def test_rmsnorm_matches_fp64_definition(orc):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 4096)).astype(np.float32)
    x[:, :80] *= 30
    gamma = rng.uniform(0.8, 1.2, 4096).astype(np.float32)
    y = orc.rmsnorm(x, gamma, 1e-5)
    xt = torch.from_numpy(x).double()
    ref = xt * torch.rsqrt(xt.pow(2).mean(-1, keepdim=True) + float(np.float32(1e-5))) * torch.from_numpy(gamma).double()
    rel = np.abs(y - ref.numpy()) / np.abs(ref.numpy()).clip(1e-30)
    # three fp32 roundings (rinv, x*rinv, *gamma), each at most 2^-24 relative
    assert rel.max() < 3.01 * 2.0 ** -24


def test_rmsnorm_zero_row(orc):
    x = np.zeros((2, 64), np.float32)
    y, rinv = orc.rmsnorm(x, None, 1e-5, return_rinv=True)
    assert np.all(y == 0) and rinv[0] == np.float32(1 / np.sqrt(np.float64(np.float32(1e-5))))


# --------------------------------------------------------------------- GEMM

def _rand_qtensor(orc, rng, rows, cols, s):
    codes = rng.integers(0, 256, size=(rows, cols // 2), dtype=np.uint8)
    scales = rng.integers(0, 0x7F, size=(rows, cols // 16), dtype=np.uint8)
    return orc.QTensor(codes, scales, np.float32(s))


def _exact_value(q, r, k):
    byte = int(q.codes[r, k // 2])
    c = (byte >> 4) if k & 1 else (byte & 15)
    v = Fraction(E2M1[c & 7]) * (-1 if c & 8 else 1)
    return v * Fraction(_e4m3(int(q.scales[r, k // 16]))) * Fraction(float(q.s))


def test_gemm_bruteforce_exact(orc):
    rng = np.random.default_rng(4)
    M, N, K = 3, 5, 64
    a = _rand_qtensor(orc, rng, M, K, 0.0371)
    w = _rand_qtensor(orc, rng, N, K, 1.7e-3)
    y = orc.gemm(a, w)
    for m in range(M):
        for n in range(N):
            exact = sum(_exact_value(a, m, k) * _exact_value(w, n, k) for k in range(K))
            assert abs(y[m, n] - float(exact)) <= 1e-13 * max(1e-300, abs(float(exact))) + 1e-300


def test_gemm_one_hot_fixes_indices(orc):
    M, N, K = 4, 6, 96
    for (m, n, k) in [(0, 0, 0), (3, 5, 95), (1, 2, 17), (2, 4, 48)]:
        a = orc.QTensor(np.zeros((M, K // 2), np.uint8), np.zeros((M, K // 16), np.uint8), np.float32(0.5))
        w = orc.QTensor(np.zeros((N, K // 2), np.uint8), np.zeros((N, K // 16), np.uint8), np.float32(0.25))
        a.codes[m, k // 2] = 0x7 << (4 * (k & 1))      # +6
        a.scales[m, k // 16] = 0x38                      # 1.0
        w.codes[n, k // 2] = 0xD << (4 * (k & 1))      # -3
        w.scales[n, k // 16] = 0x40                      # 2.0
        y = orc.gemm(a, w)
        expect = np.zeros((M, N))
        expect[m, n] = 6 * 1.0 * 0.5 * (-3) * 2.0 * 0.25
        np.testing.assert_array_equal(y, expect)


def test_gemm_residue_is_sum(orc):
    rng = np.random.default_rng(5)
    a = _rand_qtensor(orc, rng, 2, 32, 0.1)
    r = _rand_qtensor(orc, rng, 2, 32, 0.01)
    w = _rand_qtensor(orc, rng, 3, 32, 0.2)
    np.testing.assert_allclose(orc.gemm_residue(a, r, w), orc.gemm(a, w) + orc.gemm(r, w), rtol=0, atol=0)


def test_arcquant_k_plus_s_identity(orc):
    """One GEMM over K+S columns equals main term plus outlier-residue term (ARCQuant 3.1)."""
    rng = np.random.default_rng(6)
    M, N, K, S = 4, 8, 128, 32
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, [5, 70]] *= 40
    perm = np.argsort(-np.abs(x).max(axis=0), kind="stable").astype(np.int32)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    xa = orc.rmsnorm_reorder_quantize(x, None, perm=perm, S=S)
    wa = orc.quantize(orc.augment_weight(w, perm, S))
    y_aug = orc.gemm(xa, wa)
    # split form: Q(X')Q(W')^T + Q(R)Q(W'_o)^T, computed term by term in exact arithmetic
    xs = x[:, perm]
    qx = orc.QTensor(np.ascontiguousarray(xa.codes[:, : K // 2]), np.ascontiguousarray(xa.scales[:, : K // 16]), xa.s)
    qr = orc.QTensor(np.ascontiguousarray(xa.codes[:, K // 2:]), np.ascontiguousarray(xa.scales[:, K // 16:]), xa.s)
    qw = orc.QTensor(np.ascontiguousarray(wa.codes[:, : K // 2]), np.ascontiguousarray(wa.scales[:, : K // 16]), wa.s)
    qwo = orc.QTensor(np.ascontiguousarray(wa.codes[:, K // 2:]), np.ascontiguousarray(wa.scales[:, K // 16:]), wa.s)
    for m in range(M):
        for n in range(N):
            main = sum(_exact_value(qx, m, k) * _exact_value(qw, n, k) for k in range(K))
            res = sum(_exact_value(qr, m, k) * _exact_value(qwo, n, k) for k in range(S))
            assert abs(y_aug[m, n] - float(main + res)) <= 1e-12 * abs(float(main + res)) + 1e-300
    # and the residue term makes the outlier channels' product closer to the fp32 one
    ref = xs.astype(np.float64) @ w[:, perm].astype(np.float64).T
    y_plain = orc.gemm(qx, qw)
    assert np.linalg.norm(y_aug - ref) < np.linalg.norm(y_plain - ref)

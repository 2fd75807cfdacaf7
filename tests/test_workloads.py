"""The seeded input generators follow their stated recipes: shapes, bf16
storage, the outlier channels and their gains, the calibrated channel order,
the RMSNorm gain range, and determinism (both the CUDA path and the oracle read
their inputs from here)."""
import numpy as np

from nvfp4_block_scaled_18_b200 import workloads as wl


def _bf16_exact(x):
    return np.array_equal(wl.bf16_values(x), x)


def test_configs_match_the_workloads():
    assert wl.DECODE_M == (1, 2, 4, 8, 16)
    assert wl.DECODE_SHAPES == ((4096, 4096), (14336, 4096), (4096, 14336))
    assert wl.RESSERVE_M == (1, 4, 16, 64)
    assert wl.RESSERVE_SHAPES == ((5120, 5120), (27648, 5120), (5120, 27648))
    assert (wl.ARC_M, wl.ARC_K, wl.ARC_N, wl.ARC_S) == (2048, 4096, 11008, (128, 256, 512))
    assert wl.PREFILL_M == 8192
    assert wl.PREFILL_SHAPES == ((14336, 4096), (4096, 14336), (28672, 8192))


def test_decode_activations_recipe():
    x = wl.decode_x(64, 4096)
    assert x.shape == (64, 4096) and x.dtype == np.float32
    assert _bf16_exact(x)
    assert np.array_equal(x, wl.decode_x(64, 4096))          # seeded
    ch = wl.outlier_channels(4096, 0.01)
    assert len(ch) == 41 and len(np.unique(ch)) == 41
    rest = np.setdiff1d(np.arange(4096), ch)
    assert 40.0 < x[:, ch].std() < 60.0                      # N(0,1) x 50
    assert 0.9 < x[:, rest].std() < 1.1
    # the first rows of a larger draw are the smaller draw (one stream, row-major)
    assert np.array_equal(wl.decode_x(4, 4096), x[:4])


def test_resserve_activations_recipe():
    x = wl.resserve_x(64, 5120)
    assert x.shape == (64, 5120) and _bf16_exact(x)
    a = np.abs(x.astype(np.float64))
    # 0.5 * Student-t(3): median |t3| = 0.765, so the median |x| is near 0.38
    assert 0.33 < np.median(a) < 0.43
    # heavy tails: far more mass beyond 10 median deviations than a normal has
    assert (a > 3.8).mean() > 1e-3


def test_arcquant_inputs_recipe():
    x, gamma, perm = wl.arc_inputs(M=64)
    K = wl.ARC_K
    assert x.shape == (64, K) and _bf16_exact(x)
    assert gamma.shape == (K,) and _bf16_exact(gamma)
    assert gamma.min() >= 0.8 - 2 ** -8 and gamma.max() <= 1.2 + 2 ** -7   # U(0.8, 1.2), bf16-rounded
    assert perm.dtype == np.int32 and np.array_equal(np.sort(perm), np.arange(K))
    ch = wl.outlier_channels(K, 0.02)
    assert len(ch) == 82
    # the calibrated order puts exactly the x30 channels first
    assert np.array_equal(np.sort(perm[:82]), ch)
    rest = np.setdiff1d(np.arange(K), ch)
    assert 25.0 < x[:, ch].std() < 35.0 and 0.9 < x[:, rest].std() < 1.1
    # the order is by calibrated absmax, largest first, ties by channel index
    calib = wl.activations_normal(512, K, 0.02, 30.0, wl.SEED_CALIB, ch)
    am = np.abs(calib).max(axis=0)
    assert np.all(np.diff(am[perm]) <= 0)


def test_prefill_and_weights_recipe():
    x = wl.prefill_x(32, 4096)
    assert _bf16_exact(x) and np.array_equal(x, wl.decode_x(32, 4096))   # same recipe and seed
    w = wl.weights_normal(256, 512)
    assert w.dtype == np.float32 and 0.018 < w.std() < 0.022
    assert np.array_equal(w, wl.weights_normal(256, 512))
    perm = wl.prefill_perm(4096)
    assert np.array_equal(np.sort(perm[:41]), wl.outlier_channels(4096, 0.01))


def test_tiny_recipe():
    x, w = wl.tiny()
    assert x.shape == (4, 256) and w.shape == (256, 256)
    rng = np.random.default_rng(0)
    x0 = rng.standard_normal((4, 256)).astype(np.float32)
    assert np.array_equal(x[:, [3, 77]], x0[:, [3, 77]] * np.float32(40.0))
    keep = np.setdiff1d(np.arange(256), [3, 77])
    assert np.array_equal(x[:, keep], x0[:, keep])

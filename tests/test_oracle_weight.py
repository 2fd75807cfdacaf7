"""Pins for the oracle's offline weight preparation (ARCQuant blog post sections
3.1 and 6.3: W' = W[:, perm], W_aug = [W' | W'[:, :S]]; OSFP4 page, abstract:
a smoothing vector absorbed as W diag(sigma)), checked against exact values."""
from fractions import Fraction

import numpy as np

from test_oracle_residue_rounding import round_f32


def test_augment_is_a_column_gather(orc):
    rng = np.random.default_rng(31)
    w = rng.standard_normal((5, 64)).astype(np.float32)
    perm = rng.permutation(64).astype(np.int32)
    wa = orc.augment_weight(w, perm, 32)
    assert wa.shape == (5, 96)
    for j in range(64):
        np.testing.assert_array_equal(wa[:, j], w[:, perm[j]])
    np.testing.assert_array_equal(wa[:, 64:], wa[:, :32])


def test_sigma_is_one_rounded_product_per_element(orc):
    rng = np.random.default_rng(32)
    w = rng.standard_normal((4, 48)).astype(np.float32)
    sigma = rng.uniform(0.3, 3.0, 48).astype(np.float32)
    perm = rng.permutation(48).astype(np.int32)
    wa = orc.augment_weight(w, perm, 16, sigma)
    for r in range(4):
        for j in range(48):
            c = perm[j]
            assert wa[r, j] == round_f32(Fraction(float(w[r, c])) * Fraction(float(sigma[c])))
    # sigma = 1 is no smoothing; powers of two scale exactly
    np.testing.assert_array_equal(orc.augment_weight(w, perm, 16, np.ones(48, np.float32)),
                                  orc.augment_weight(w, perm, 16))
    p2 = np.exp2(rng.integers(-3, 4, 48)).astype(np.float32)
    np.testing.assert_array_equal(orc.augment_weight(w, perm, 0, p2), (w * p2)[:, perm])

"""The oracle reproduces the committed tiny-case fixture (tests/golden/make_golden.py)."""
import os

import numpy as np

from nvfp4_block_scaled_18_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_w4a4.npz")


def test_tiny_golden_regression(orc):
    g = np.load(GOLDEN)
    x, w = workloads.tiny()
    np.testing.assert_array_equal(x, g["x"])
    np.testing.assert_array_equal(w, g["w"])
    qx, qr = orc.quantize_residue(x)
    qw = orc.quantize(w)
    for name, q in (("x", qx), ("r", qr), ("w", qw)):
        np.testing.assert_array_equal(q.codes, g[name + "_codes"])
        np.testing.assert_array_equal(q.scales, g[name + "_scales"])
        assert q.s == g[name + "_s"]
    np.testing.assert_array_equal(orc.gemm(qx, qw), g["y"])
    np.testing.assert_array_equal(orc.gemm_residue(qx, qr, qw), g["y_res"])
    # the residue correction removes most of the activation-quantization error
    ref = x.astype(np.float64) @ orc.dequant_f64(qw).T
    assert np.linalg.norm(g["y_res"] - ref) < 0.25 * np.linalg.norm(g["y"] - ref)

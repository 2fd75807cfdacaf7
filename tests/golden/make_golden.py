"""Write tests/golden/tiny_w4a4.npz from the CPU oracle (and nothing else).

The tiny W4A4 case: X 4x256 fp32 N(0,1) with channels 3 and 77 scaled x40,
W 256x256 N(0, 0.02), one default_rng(0) drawing X then W.  Stored: the
NVFP4 codes/scales/tensor scales of X, of its ResServe residue and of W, and
the fp64 outputs Y = Q(X)Q(W)^T and Y + Q(R)Q(W)^T.  The pages print no worked
example, so these values are the oracle's; they guard the oracle (and the GPU
path) against silent drift.

Run:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from nvfp4_block_scaled_18_b200 import workloads  # noqa: E402


def main():
    x, w = workloads.tiny()
    qx, qr = oracle.quantize_residue(x)
    qw = oracle.quantize(w)
    y = oracle.gemm(qx, qw)
    y_res = oracle.gemm_residue(qx, qr, qw)
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_w4a4.npz")
    np.savez_compressed(out, x=x, w=w,
                        x_codes=qx.codes, x_scales=qx.scales, x_s=np.float32(qx.s),
                        r_codes=qr.codes, r_scales=qr.scales, r_s=np.float32(qr.s),
                        w_codes=qw.codes, w_scales=qw.scales, w_s=np.float32(qw.s),
                        y=y, y_res=y_res)
    print("wrote", out)


if __name__ == "__main__":
    main()

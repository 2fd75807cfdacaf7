"""The allocation-free fused quantizer, nvfp4_rmsnorm_reorder_quantize_noalloc,
called through the C ABI, gives the same codes, scales and tensor scale as the
regular entry point with a caller workspace, on two calls in a row.

It exists for callers that cannot allocate device memory (hosts that own
every allocation, paths that must never call the allocator); its scratch is a
device array inside the library.  This file is collected last so a failure here leaves the rest of the
suite already run."""
import ctypes

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_18_b200 as nv
from nvfp4_block_scaled_18_b200 import workloads as wl

from gpu_util import assert_same_q

pytestmark = pytest.mark.gpu


def _regular(x, gamma, perm, S, layout):
    M, K = x.shape
    xa = nv.NVFP4Tensor.empty(M, K + S, layout)
    nv.nvfp4_rmsnorm_reorder_quantize(x, xa, gamma=gamma, eps=1e-5, perm=perm, S=S, workspace=nv.Workspace(M, K))
    return xa


def _noalloc_abi(lib, x, gamma, perm, S, layout):
    M, K = x.shape
    xa = nv.NVFP4Tensor.empty(M, K + S, layout)
    xc = xa.c()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.nvfp4_rmsnorm_reorder_quantize_noalloc(
        x.data_ptr(), nv.NVFP4_BF16, M, K, x.stride(0), None if gamma is None else gamma.data_ptr(),
        ctypes.c_float(1e-5), None if perm is None else perm.data_ptr(), S, None, ctypes.byref(xc),
        st.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0, nv.status_string(rc)
    torch.cuda.synchronize()
    assert st.item() == 0
    return xa


def test_noalloc_matches_regular_entry_point_twice():
    assert torch.cuda.is_available()
    lib = nv.load_library()
    x, gamma, perm = wl.arc_inputs(M=512)
    xt, gt, pt = wl.to_bf16(x).cuda(), wl.to_bf16(gamma).cuda(), torch.from_numpy(perm).cuda()
    # second call: other rows, no normalisation, other S and layout (different scratch use)
    x2 = wl.prefill_x(300, 4096)
    x2t = wl.to_bf16(x2).cuda()
    cases = [(xt, gt, pt, 256, nv.SF_TILED), (x2t, None, pt, 128, nv.SF_ROWMAJOR)]
    for (xx, gg, pp, S, layout) in cases:
        got = _noalloc_abi(lib, xx, gg, pp, S, layout)
        ref = _regular(xx, gg, pp, S, layout)
        torch.cuda.synchronize()
        assert torch.equal(got.codes, ref.codes)
        assert torch.equal(got.scales, ref.scales)
        assert torch.equal(got.tensor_scale, ref.tensor_scale)


def test_noalloc_stream_ordered_calls_share_the_scratch(orc):
    """Four calls enqueued back to back on one stream (other M, S, gain and layout each
    time), one synchronize at the end: stream order alone separates their uses of the
    shared scratch.  Every result must equal the oracle's encoding bit for bit."""
    lib = nv.load_library()
    x, gamma, perm = wl.arc_inputs(M=256)
    K = x.shape[1]
    xt, gt, pt = wl.to_bf16(x).cuda(), wl.to_bf16(gamma).cuda(), torch.from_numpy(perm).cuda()
    x2 = wl.prefill_x(96, K)
    x2t = wl.to_bf16(x2).cuda()
    cases = [(xt, x, gt, gamma, 256, nv.SF_TILED), (x2t, x2, None, None, 128, nv.SF_ROWMAJOR),
             (xt[:17], x[:17], gt, gamma, 512, nv.SF_ROWMAJOR), (x2t, x2, gt, gamma, 0, nv.SF_TILED)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    outs, sts = [], []
    with torch.cuda.stream(s):
        for (xx, _, gg, _, S, layout) in cases:
            M = xx.shape[0]
            xa = nv.NVFP4Tensor.empty(M, K + S, layout)
            xc = xa.c()
            st = torch.zeros(1, dtype=torch.int32, device="cuda")
            rc = lib.nvfp4_rmsnorm_reorder_quantize_noalloc(
                xx.data_ptr(), nv.NVFP4_BF16, M, K, xx.stride(0), None if gg is None else gg.data_ptr(),
                ctypes.c_float(1e-5), pt.data_ptr(), S, None, ctypes.byref(xc), st.data_ptr(), s.cuda_stream)
            assert rc == 0, nv.status_string(rc)
            outs.append(xa)
            sts.append(st)
    s.synchronize()
    for (xx, xnp, gg, gnp, S, layout), xa, st in zip(cases, outs, sts):
        assert st.item() == 0
        xb = wl.bf16_values(xnp.astype(np.float32))
        gb = None if gnp is None else wl.bf16_values(gnp.astype(np.float32))
        ref = orc.rmsnorm_reorder_quantize(xb, gb, 1e-5, perm, S)
        assert_same_q(xa, ref)


def test_noalloc_rejects_rows_beyond_capacity():
    lib = nv.load_library()
    M = nv.NVFP4_NOALLOC_MAX_ROWS + 1
    xa = nv._CTensor(1 << 20, 1 << 20, 1 << 20, M, 64, 0)
    rc = lib.nvfp4_rmsnorm_reorder_quantize_noalloc(1 << 20, nv.NVFP4_BF16, M, 64, 64, None, ctypes.c_float(1e-5),
                                                    None, 0, None, ctypes.byref(xa), None, None)
    assert rc == 7  # NVFP4_ERR_WORKSPACE, before anything is enqueued

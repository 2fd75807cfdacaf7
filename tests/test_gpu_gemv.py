"""GPU parity: the decode GEMV (M <= 16) against the fp64 oracle on the same
quantized operands, relative Frobenius error <= 1e-5.

Full-size shapes are checked on a sample of output columns (W rows) that the
oracle evaluates one by one; small and ragged shapes are checked in full."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_18_b200 as nv
from nvfp4_block_scaled_18_b200 import workloads as wl

from gpu_util import REL_FRO_TOL, assert_same_q, rel_fro, run_quantize, sub_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nv.load_library()


_W = {}


def quantized_weight(orc, N, K, layout=nv.SF_ROWMAJOR):
    """W ~ N(0, 0.02) quantized on the GPU; the oracle's per-tensor scale and a
    sample of rows quantized by the oracle (bit-exact with the GPU)."""
    key = (N, K, layout)
    if key not in _W:
        w = wl.weights_normal(N, K)
        qw = run_quantize(to_dev(w, torch.float32), layout)
        s_w = orc.tensor_scale(np.abs(w).max())
        rng = np.random.default_rng(N + K)
        rows = np.unique(np.concatenate([[0, N - 1], rng.choice(N, size=min(N, 384), replace=False)]))
        ow = orc.quantize(w[rows], s_w)
        _W[key] = (qw, ow, rows)
    return _W[key]


def check_y(y_gpu, y_ref):
    err = rel_fro(y_gpu, y_ref)
    assert err <= REL_FRO_TOL, err
    return err


@pytest.mark.parametrize("N,K", wl.DECODE_SHAPES)
def test_decode_gemv_full_size(orc, N, K):
    qw, ow, rows = quantized_weight(orc, N, K)
    np.testing.assert_array_equal(qw.codes[torch.from_numpy(rows).cuda()].cpu().numpy(), ow.codes)
    for M in wl.DECODE_M:
        x = wl.decode_x(M, K)
        qx = run_quantize(to_dev(x))
        ox = orc.quantize(x)
        assert_same_q(qx, ox)
        y = torch.empty((M, N), dtype=torch.float32, device="cuda")
        nv.nvfp4_gemm(qx, qw, y)
        torch.cuda.synchronize()
        check_y(y.cpu().numpy()[:, rows], orc.gemm(ox, ow))


@pytest.mark.parametrize("N,K", wl.RESSERVE_SHAPES)
def test_resserve_gemv_full_size(orc, N, K):
    qw, ow, rows = quantized_weight(orc, N, K)
    for M in (1, 4, 16):
        x = wl.resserve_x(M, K)
        q, r = nv.NVFP4Tensor.empty(M, K), nv.NVFP4Tensor.empty(M, K)
        nv.nvfp4_quantize_residue(to_dev(x), q, r, workspace=nv.Workspace(M, K))
        y = torch.empty((M, N), dtype=torch.float32, device="cuda")
        nv.nvfp4_gemm_residue(q, r, qw, y)
        torch.cuda.synchronize()
        oq, orr = orc.quantize_residue(x)
        assert_same_q(q, oq)
        assert_same_q(r, orr)
        check_y(y.cpu().numpy()[:, rows], orc.gemm_residue(oq, orr, ow))


def test_tiny_config_gemv(orc):
    g = np.load(__import__("os").path.join(__import__("os").path.dirname(__file__), "golden", "tiny_w4a4.npz"))
    x, w = wl.tiny()
    q, r = nv.NVFP4Tensor.empty(4, 256), nv.NVFP4Tensor.empty(4, 256)
    nv.nvfp4_quantize_residue(to_dev(x, torch.float32), q, r, workspace=nv.Workspace(4, 256))
    qw = run_quantize(to_dev(w, torch.float32))
    y = torch.empty((4, 256), dtype=torch.float32, device="cuda")
    yr = torch.empty((4, 256), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(q, qw, y)
    nv.nvfp4_gemm_residue(q, r, qw, yr)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(q.codes.cpu().numpy(), g["x_codes"])
    np.testing.assert_array_equal(r.codes.cpu().numpy(), g["r_codes"])
    np.testing.assert_array_equal(qw.codes.cpu().numpy(), g["w_codes"])
    check_y(y.cpu().numpy(), g["y"])
    check_y(yr.cpu().numpy(), g["y_res"])


@pytest.mark.parametrize("M,N,K", [(1, 1, 64), (3, 100, 128), (16, 33, 192), (7, 4100, 640), (2, 31, 4096)])
def test_ragged_shapes(orc, M, N, K):
    rng = np.random.default_rng(M * 1000 + N)
    x = (rng.standard_normal((M, K)) * 2).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    qx, qw = run_quantize(to_dev(x, torch.float32)), run_quantize(to_dev(w, torch.float32))
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(qx, qw, y)
    torch.cuda.synchronize()
    check_y(y.cpu().numpy(), orc.gemm(orc.quantize(x), orc.quantize(w)))


def test_bf16_output_and_ld(orc):
    """bf16 output = RNE of the same kernel's fp32 output; the padding of the strided
    output rows is left untouched."""
    M, N, K = 4, 256, 512
    x, w = wl.decode_x(M, K), wl.weights_normal(N, K)
    qx, qw = run_quantize(to_dev(x)), run_quantize(to_dev(w, torch.float32))
    big = torch.zeros((M, N + 64), dtype=torch.bfloat16, device="cuda")
    y32 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(qx, qw, big[:, :N])
    nv.nvfp4_gemm(qx, qw, y32)
    torch.cuda.synchronize()
    check_y(y32.cpu().numpy(), orc.gemm(orc.quantize(x), orc.quantize(w)))
    assert torch.equal(big[:, :N], y32.to(torch.bfloat16))
    assert torch.count_nonzero(big[:, N:]) == 0


@pytest.mark.parametrize("M,residue", [(2, False), (4, True), (8, True)])
def test_k_split_bf16_output_and_ld(orc, M, residue):
    """Few rows of W and a long K: the M <= 4 kernel splits K over a cluster and the
    owners sum the peers' partial rows; bf16 output = RNE of the fp32 result, the
    padding of the strided output rows untouched."""
    N, K = 40, 4096
    rng = np.random.default_rng(900 + M)
    x = (rng.standard_normal((M, K)) * 1.5).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    qw = run_quantize(to_dev(w, torch.float32))
    y32 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    big = torch.zeros((M, N + 24), dtype=torch.bfloat16, device="cuda")
    if residue:
        q, r = nv.NVFP4Tensor.empty(M, K), nv.NVFP4Tensor.empty(M, K)
        nv.nvfp4_quantize_residue(to_dev(x, torch.float32), q, r, workspace=nv.Workspace(M, K))
        nv.nvfp4_gemm_residue(q, r, qw, y32)
        nv.nvfp4_gemm_residue(q, r, qw, big[:, :N])
        oq, orr = orc.quantize_residue(x)
        ref = orc.gemm_residue(oq, orr, orc.quantize(w))
    else:
        qx = run_quantize(to_dev(x, torch.float32))
        nv.nvfp4_gemm(qx, qw, y32)
        nv.nvfp4_gemm(qx, qw, big[:, :N])
        ref = orc.gemm(orc.quantize(x), orc.quantize(w))
    torch.cuda.synchronize()
    check_y(y32.cpu().numpy(), ref)
    assert torch.equal(big[:, :N], y32.to(torch.bfloat16))
    assert torch.count_nonzero(big[:, N:]) == 0


def test_exact_sums_are_exact(orc):
    """Power-of-two tensor scales, small K: every partial sum is exactly representable,
    so the GPU result must equal the exact result bit for bit."""
    M, N, K = 2, 64, 64
    rng = np.random.default_rng(77)
    codes_x = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    codes_w = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sc_x = rng.integers(0x30, 0x40, (M, K // 16), dtype=np.uint8)
    sc_w = rng.integers(0x30, 0x40, (N, K // 16), dtype=np.uint8)
    a = nv.NVFP4Tensor(torch.from_numpy(codes_x).cuda(), torch.from_numpy(sc_x.reshape(-1)).cuda(),
                       torch.tensor([0.5], device="cuda"), M, K)
    w = nv.NVFP4Tensor(torch.from_numpy(codes_w).cuda(), torch.from_numpy(sc_w.reshape(-1)).cuda(),
                       torch.tensor([0.25], device="cuda"), N, K)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(a, w, y)
    torch.cuda.synchronize()
    ref = orc.gemm(orc.QTensor(codes_x, sc_x, 0.5), orc.QTensor(codes_w, sc_w, 0.25))
    np.testing.assert_array_equal(y.cpu().numpy().astype(np.float64), ref)

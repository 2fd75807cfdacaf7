"""GPU parity: the few-row tensor-core path (M <= 128, TILED scales; W is the
128-row MMA operand, the activation rows the narrow one, K split across a
cluster) against the fp64 oracle on the same quantized operands, relative
Frobenius error <= 1e-5."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_18_b200 as nv
from nvfp4_block_scaled_18_b200 import workloads as wl

from gpu_util import REL_FRO_TOL, assert_same_q, gpu_tensor, rel_fro, run_quantize, to_dev

pytestmark = pytest.mark.gpu
T = nv.SF_TILED


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nv.load_library()


def gemm(a, w, r=None, out_dtype=torch.float32):
    y = torch.full((a.rows, w.rows), float("nan"), dtype=out_dtype, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if r is None:
        nv.nvfp4_gemm(a, w, y, dev_status=st)
    else:
        nv.nvfp4_gemm_residue(a, r, w, y, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0, nv.status_string(st.item())
    return y


_W = {}


def weight(orc, N, K):
    if (N, K) not in _W:
        w = wl.weights_normal(N, K)
        qw = run_quantize(to_dev(w, torch.float32), T)
        rng = np.random.default_rng(N * 7 + K)
        cols = np.unique(np.concatenate([[0, N - 1], rng.choice(N, min(N, 320), replace=False)]))
        _W[(N, K)] = (qw, orc.quantize(w[cols], orc.tensor_scale(np.abs(w).max())), cols)
    return _W[(N, K)]


@pytest.mark.parametrize("N,K", wl.DECODE_SHAPES)
def test_decode_shapes(orc, N, K):
    qw, ow, cols = weight(orc, N, K)
    for M in wl.DECODE_M:
        x = wl.decode_x(M, K)
        qx = run_quantize(to_dev(x), T)
        ox = orc.quantize(x)
        assert_same_q(qx, ox)
        y = gemm(qx, qw).cpu().numpy()[:, cols]
        err = rel_fro(y, orc.gemm(ox, ow))
        assert err <= REL_FRO_TOL, (M, err)


@pytest.mark.parametrize("N,K", wl.RESSERVE_SHAPES)
def test_resserve_shapes(orc, N, K):
    qw, ow, cols = weight(orc, N, K)
    for M in wl.RESSERVE_M:
        x = wl.resserve_x(M, K)
        q, r = nv.NVFP4Tensor.empty(M, K, T), nv.NVFP4Tensor.empty(M, K, T)
        nv.nvfp4_quantize_residue(to_dev(x), q, r, workspace=nv.Workspace(M, K))
        oq, orr = orc.quantize_residue(x)
        y = gemm(q, qw, r).cpu().numpy()[:, cols]
        err = rel_fro(y, orc.gemm_residue(oq, orr, ow))
        assert err <= REL_FRO_TOL, (M, err)
        y0 = gemm(q, qw).cpu().numpy()[:, cols]
        assert rel_fro(y0, orc.gemm(oq, ow)) <= REL_FRO_TOL


@pytest.mark.parametrize("M,N,K", [(1, 1, 256), (3, 100, 320), (16, 200, 4224), (17, 130, 512), (64, 300, 1024),
                                   (100, 257, 768), (128, 128, 256), (5, 1000, 27648)])
@pytest.mark.parametrize("residue", [False, True])
def test_ragged(orc, M, N, K, residue):
    rng = np.random.default_rng(M + 3 * N + K)
    x = (0.5 * rng.standard_t(3, size=(M, K))).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    qw = run_quantize(to_dev(w, torch.float32), T)
    ow = orc.quantize(w)
    if residue:
        q, r = nv.NVFP4Tensor.empty(M, K, T), nv.NVFP4Tensor.empty(M, K, T)
        nv.nvfp4_quantize_residue(to_dev(x, torch.float32), q, r, workspace=nv.Workspace(M, K))
        oq, orr = orc.quantize_residue(x)
        ref = orc.gemm_residue(oq, orr, ow)
        y = gemm(q, qw, r)
    else:
        q = run_quantize(to_dev(x, torch.float32), T)
        ref = orc.gemm(orc.quantize(x), ow)
        y = gemm(q, qw)
    err = rel_fro(y.cpu().numpy(), ref)
    assert err <= REL_FRO_TOL, err


@pytest.mark.parametrize("m,n,k", [(0, 0, 0), (3, 127, 255), (15, 64, 130), (9, 33, 200), (0, 96, 64)])
def test_one_hot_placement(orc, m, n, k):
    M, N, K = 16, 128, 256
    ca, cw = np.zeros((M, K // 2), np.uint8), np.zeros((N, K // 2), np.uint8)
    sa, sw = np.zeros((M, K // 16), np.uint8), np.zeros((N, K // 16), np.uint8)
    ca[m, k // 2] = 0x5 << (4 * (k & 1))      # +3
    cw[n, k // 2] = 0xF << (4 * (k & 1))      # -6
    sa[m, k // 16] = 0x3A                     # 1.25
    sw[n, k // 16] = 0x28                     # 0.25
    sa[m, (k // 16 + 2) % 16] = 0x7E
    sw[n, (k // 16 + 1) % 16] = 0x7E
    y = gemm(gpu_tensor(ca, sa, 0.5), gpu_tensor(cw, sw, 4.0)).cpu().numpy()
    expect = np.zeros((M, N))
    expect[m, n] = 3 * 1.25 * 0.5 * (-6) * 0.25 * 4.0
    np.testing.assert_array_equal(y, expect)
    np.testing.assert_array_equal(orc.gemm(orc.QTensor(ca, sa, 0.5), orc.QTensor(cw, sw, 4.0)), expect)


def test_exact_sums_exact(orc):
    M, N, K = 16, 256, 256
    rng = np.random.default_rng(19)
    ca, cw = rng.integers(0, 256, (M, K // 2), dtype=np.uint8), rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa = rng.integers(0x30, 0x40, (M, K // 16), dtype=np.uint8)
    sw = rng.integers(0x30, 0x40, (N, K // 16), dtype=np.uint8)
    y = gemm(gpu_tensor(ca, sa, 0.5), gpu_tensor(cw, sw, 0.25)).cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(y, orc.gemm(orc.QTensor(ca, sa, 0.5), orc.QTensor(cw, sw, 0.25)))


def test_bf16_output(orc):
    M, N, K = 8, 512, 1024
    x, w = wl.decode_x(M, K), wl.weights_normal(N, K)
    qx, qw = run_quantize(to_dev(x), T), run_quantize(to_dev(w, torch.float32), T)
    y32 = gemm(qx, qw)
    y16 = gemm(qx, qw, out_dtype=torch.bfloat16)
    assert rel_fro(y32.cpu().numpy(), orc.gemm(orc.quantize(x), orc.quantize(w))) <= REL_FRO_TOL
    assert torch.equal(y16, y32.to(torch.bfloat16))

"""GPU parity: the tcgen05 block-scaled GEMM (M > 16, TILED scales) against the
fp64 oracle on the same quantized operands, relative Frobenius error <= 1e-5.

One-hot operands pin the code/scale placement (tile rows, TMEM lane quadrants,
k-blocks inside a k-tile, both 128-row groups of a 256-wide W tile); ragged
shapes exercise the M, N and K tails; the large configurations are checked on
sampled rows and columns that the oracle evaluates."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_18_b200 as nv
from nvfp4_block_scaled_18_b200 import workloads as wl

from gpu_util import REL_FRO_TOL, assert_same_q, gpu_tensor, rel_fro, run_quantize, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nv.load_library()


def run_gemm(a, w, out_dtype=torch.float32):
    y = torch.full((a.rows, w.rows), float("nan"), dtype=out_dtype, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_gemm(a, w, y, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0, nv.status_string(st.item())
    return y


@pytest.mark.parametrize("m,n,k", [(0, 0, 0), (33, 131, 17), (77, 255, 95), (127, 128, 130), (64, 200, 255),
                                   (5, 17, 64), (96, 250, 191)])
def test_one_hot_placement(orc, m, n, k):
    M, N, K = 128, 256, 256
    ca = np.zeros((M, K // 2), np.uint8)
    cw = np.zeros((N, K // 2), np.uint8)
    sa = np.zeros((M, K // 16), np.uint8)
    sw = np.zeros((N, K // 16), np.uint8)
    ca[m, k // 2] = 0x7 << (4 * (k & 1))      # +6
    cw[n, k // 2] = 0xB << (4 * (k & 1))      # -1.5
    sa[m, k // 16] = 0x40                     # 2.0
    sw[n, k // 16] = 0x31                     # 0.5625
    # decoys: other blocks of the same rows carry different scales and zero codes
    sa[m, (k // 16 + 1) % 16] = 0x7E
    sw[n, (k // 16 + 3) % 16] = 0x7E
    a, w = gpu_tensor(ca, sa, 0.5), gpu_tensor(cw, sw, 0.25)
    y = run_gemm(a, w).cpu().numpy()
    expect = np.zeros((M, N))
    expect[m, n] = 6 * 2.0 * 0.5 * (-1.5) * 0.5625 * 0.25
    np.testing.assert_array_equal(y, expect)
    ref = orc.gemm(orc.QTensor(ca, sa, 0.5), orc.QTensor(cw, sw, 0.25))
    np.testing.assert_array_equal(ref, expect)


def _random_case(orc, M, N, K, seed, out_dtype=torch.float32):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((M, K)) * 2).astype(np.float32)
    x[:, rng.choice(K, max(1, K // 64), replace=False)] *= 30
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    qa = run_quantize(to_dev(x, torch.float32), nv.SF_TILED)
    qw = run_quantize(to_dev(w, torch.float32), nv.SF_TILED)
    y = run_gemm(qa, qw, out_dtype)
    return y, orc.gemm(orc.quantize(x), orc.quantize(w))


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (256, 512, 1024), (200, 300, 320), (129, 1000, 4224),
                                   (17, 64, 256), (1000, 130, 576), (384, 768, 2048)])
def test_random_shapes(orc, M, N, K):
    y, ref = _random_case(orc, M, N, K, M + N + K)
    err = rel_fro(y.cpu().numpy(), ref)
    assert err <= REL_FRO_TOL, err


def test_bf16_output(orc):
    """bf16 output = round-to-nearest-even of the same kernel's fp32 output, bit for bit
    (the fp32 output itself is checked against the oracle)."""
    y16, ref = _random_case(orc, 256, 512, 512, 5, torch.bfloat16)
    y32, _ = _random_case(orc, 256, 512, 512, 5, torch.float32)
    assert rel_fro(y32.cpu().numpy(), ref) <= REL_FRO_TOL
    assert torch.equal(y16, y32.to(torch.bfloat16))


def test_exact_sums_exact(orc):
    """Power-of-two tensor scales and scales in [0.5, 2): every partial sum of a
    K = 256 product is a small multiple of 2^-8, so the fp32 result must be exact."""
    M, N, K = 128, 256, 256
    rng = np.random.default_rng(9)
    ca = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    cw = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa = rng.integers(0x30, 0x40, (M, K // 16), dtype=np.uint8)
    sw = rng.integers(0x30, 0x40, (N, K // 16), dtype=np.uint8)
    y = run_gemm(gpu_tensor(ca, sa, 0.5), gpu_tensor(cw, sw, 0.25)).cpu().numpy().astype(np.float64)
    ref = orc.gemm(orc.QTensor(ca, sa, 0.5), orc.QTensor(cw, sw, 0.25))
    np.testing.assert_array_equal(y, ref)


def _sampled_check(orc, x, w, qa, qw, n_rows=96, n_cols=384, seed=0):
    """Compare Y on a sample of rows and columns, the oracle quantizing only those
    rows of X and W (under the full tensors' scales, so they are bit-identical)."""
    M, N = x.shape[0], w.shape[0]
    y = run_gemm(qa, qw)
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, n_rows, replace=False)]))
    cols = np.unique(np.concatenate([[0, N - 1], rng.choice(N, n_cols, replace=False)]))
    ox = orc.quantize(x[rows], orc.tensor_scale(np.abs(x).max()))
    ow = orc.quantize(w[cols], orc.tensor_scale(np.abs(w).max()))
    ys = y[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()].cpu().numpy()
    err = rel_fro(ys, orc.gemm(ox, ow))
    assert err <= REL_FRO_TOL, err
    return err


@pytest.mark.parametrize("N,K", wl.PREFILL_SHAPES)
def test_large_prefill_sampled(orc, N, K):
    M = wl.PREFILL_M
    x = wl.prefill_x(M, K)
    w = wl.weights_normal(N, K)
    qa = run_quantize(to_dev(x), nv.SF_TILED)
    qw = run_quantize(to_dev(w, torch.float32), nv.SF_TILED)
    _sampled_check(orc, x, w, qa, qw)


@pytest.mark.parametrize("S", [128, 256, 512])
def test_arcquant_augmented_gemm(orc, S):
    """ARCQuant: fused quantizer to X_aug (K+S) and W_aug = [W' | W'_o], one GEMM."""
    x, gamma, perm = wl.arc_inputs()
    M, K = x.shape
    N = wl.ARC_N
    w = wl.weights_normal(N, K)
    xa = nv.NVFP4Tensor.empty(M, K + S, nv.SF_TILED)
    nv.nvfp4_rmsnorm_reorder_quantize(to_dev(x), xa, gamma=to_dev(gamma), eps=1e-5,
                                      perm=torch.from_numpy(perm).cuda(), S=S, workspace=nv.Workspace(M, K))
    w_aug = orc.augment_weight(w, perm, S)
    qw = run_quantize(to_dev(w_aug, torch.float32), nv.SF_TILED)
    y = run_gemm(xa, qw)
    rng = np.random.default_rng(S)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 64, replace=False)]))
    cols = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 256, replace=False)]))
    ref_xa = orc.rmsnorm_reorder_quantize(x, gamma, 1e-5, perm, S)
    assert_same_q(xa, ref_xa)
    ox = orc.QTensor(ref_xa.codes[rows], ref_xa.scales[rows], ref_xa.s)
    ow = orc.quantize(w_aug[cols], orc.tensor_scale(np.abs(w_aug).max()))
    ys = y[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()].cpu().numpy()
    err = rel_fro(ys, orc.gemm(ox, ow))
    assert err <= REL_FRO_TOL, err


@pytest.mark.parametrize("N,K", wl.PREFILL_SHAPES)
def test_large_prefill_k_plus_s_end_to_end(orc, N, K):
    """The large prefill with the S = 256 outlier-residue extension at full size
    (ARCQuant blog post section 3.1: K -> K+S as one GEMM): the reorder quantizer
    without normalisation writes X_aug (M x (K+S)), the GEMM multiplies it by
    W_aug = [W' | W'_o].  Codes and scales are compared byte for byte on sampled
    rows, Y on sampled rows and columns."""
    S = 256
    M = wl.PREFILL_M
    x = wl.prefill_x(M, K)
    perm = wl.prefill_perm(K)
    xa = nv.NVFP4Tensor.empty(M, K + S, nv.SF_TILED)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = nv.Workspace(M, K)
    nv.nvfp4_rmsnorm_reorder_quantize(to_dev(x), xa, perm=torch.from_numpy(perm).cuda(), S=S, workspace=ws,
                                      dev_status=st)
    w_aug = orc.augment_weight(wl.weights_normal(N, K), perm, S)
    qw = run_quantize(to_dev(w_aug, torch.float32), nv.SF_TILED)
    y = run_gemm(xa, qw)
    assert st.item() == 0, nv.status_string(st.item())
    assert int(ws.buf.count_nonzero()) == 0, "workspace not left zeroed"
    rng = np.random.default_rng(K + N)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 64, replace=False)]))
    cols = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 256, replace=False)]))
    s_aug = orc.tensor_scale(np.abs(x).max())   # no normalisation: the reorder keeps amax
    ox = orc.rmsnorm_reorder_quantize(x[rows], None, perm=perm, S=S, s=s_aug)
    rows_t = torch.from_numpy(rows).cuda()
    np.testing.assert_array_equal(xa.codes[rows_t].cpu().numpy(), ox.codes, err_msg="X_aug codes")
    np.testing.assert_array_equal(xa.scales_rowmajor()[rows_t].cpu().numpy(), ox.scales, err_msg="X_aug scales")
    assert np.float32(xa.tensor_scale.item()) == s_aug
    ow = orc.quantize(w_aug[cols], orc.tensor_scale(np.abs(w_aug).max()))
    cols_t = torch.from_numpy(cols).cuda()
    np.testing.assert_array_equal(qw.codes[cols_t].cpu().numpy(), ow.codes, err_msg="W_aug codes")
    np.testing.assert_array_equal(qw.scales_rowmajor()[cols_t].cpu().numpy(), ow.scales, err_msg="W_aug scales")
    ys = y[rows_t][:, cols_t].cpu().numpy()
    err = rel_fro(ys, orc.gemm(ox, ow))
    assert err <= REL_FRO_TOL, err


# ------------------------------------------- ResServe residue on the large-M GEMM

@pytest.mark.parametrize("M,N,K", [(256, 512, 1024), (200, 300, 320), (1000, 130, 576), (129, 1000, 4224)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_residue_large_m(orc, M, N, K, out_dtype):
    """Y = s_a s_w A W^T + s_r s_w R W^T for M > 128: the residue runs as a second
    accumulation pass of the same tiles, combined before the single store."""
    rng = np.random.default_rng(M * 7 + N + K)
    x = (0.5 * rng.standard_t(3.0, (M, K))).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    q = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED)
    r = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED)
    nv.nvfp4_quantize_residue(to_dev(x, torch.float32), q, r, workspace=nv.Workspace(M, K))
    qw = run_quantize(to_dev(w, torch.float32), nv.SF_TILED)
    y = torch.full((M, N), float("nan"), dtype=out_dtype, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_gemm_residue(q, r, qw, y, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0, nv.status_string(st.item())
    oq, orr = orc.quantize_residue(x)
    assert_same_q(q, oq, "Q(X)")
    assert_same_q(r, orr, "Q(R)")
    ref = orc.gemm_residue(oq, orr, orc.quantize(w))
    yv = y.float().cpu().numpy()
    if out_dtype == torch.float32:
        assert rel_fro(yv, ref) <= REL_FRO_TOL
    else:   # bf16 rounding of each output on top of the fp32 accumulation
        atol = 1e-5 * np.sqrt(np.mean(ref ** 2))
        assert np.all(np.abs(yv - ref) <= 2.0 ** -8 * np.abs(ref) + atol)

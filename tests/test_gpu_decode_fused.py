"""GPU parity: the decode linear with online activation quantization in one
launch (nvfp4_quantize_gemm / nvfp4_quantize_residue_gemm) and the tensor-core
decode kernel on NVFP4 operands (nvfp4_gemm, M <= 16, TILED W, either
activation scale layout).  Q(X) (and Q(R)) must equal the oracle's encoding bit
for bit; Y must match the fp64 oracle on the oracle's quantized operands within
relative Frobenius 1e-5."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_18_b200 as nv
from nvfp4_block_scaled_18_b200 import workloads as wl

from gpu_util import REL_FRO_TOL, assert_same_q, rel_fro, run_quantize, to_dev

pytestmark = pytest.mark.gpu
T, RM = nv.SF_TILED, nv.SF_ROWMAJOR


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nv.load_library()


_W = {}


def weight(orc, N, K):
    """W quantized on the device (TILED) and, for a sample of rows, by the oracle."""
    if (N, K) not in _W:
        w = wl.weights_normal(N, K)
        qw = run_quantize(to_dev(w, torch.float32), T)
        rng = np.random.default_rng(N * 5 + K)
        rows = np.unique(np.concatenate([[0, N - 1], rng.choice(N, min(N, 256), replace=False)]))
        _W[(N, K)] = (qw, orc.quantize(w[rows], orc.tensor_scale(np.abs(w).max())), rows)
    return _W[(N, K)]


def fused(x_t, qw, layout=T, residue=False, scale_in=None, rscale_in=None, out_dtype=torch.float32):
    M, K = x_t.shape
    q = nv.NVFP4Tensor.empty(M, K, layout)
    r = nv.NVFP4Tensor.empty(M, K, layout) if residue else None
    y = torch.full((M, qw.rows), float("nan"), dtype=out_dtype, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    s_in = None if scale_in is None else torch.tensor([scale_in], dtype=torch.float32, device="cuda")
    sr_in = None if rscale_in is None else torch.tensor([rscale_in], dtype=torch.float32, device="cuda")
    if residue:
        nv.nvfp4_quantize_residue_gemm(x_t, q, r, qw, y, scale_in=s_in, rscale_in=sr_in, dev_status=st)
    else:
        nv.nvfp4_quantize_gemm(x_t, q, qw, y, scale_in=s_in, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0, nv.status_string(st.item())
    return q, r, y


@pytest.mark.parametrize("N,K", wl.DECODE_SHAPES)
def test_fused_decode_shapes(orc, N, K):
    qw, ow, rows = weight(orc, N, K)
    for M in wl.DECODE_M:
        x = wl.decode_x(M, K)
        q, _, y = fused(to_dev(x), qw)
        ox = orc.quantize(x)
        assert_same_q(q, ox, f"M={M}")
        err = rel_fro(y.cpu().numpy()[:, rows], orc.gemm(ox, ow))
        assert err <= REL_FRO_TOL, (M, err)


@pytest.mark.parametrize("N,K", wl.RESSERVE_SHAPES)
def test_fused_resserve_shapes(orc, N, K):
    qw, ow, rows = weight(orc, N, K)
    for M in [m for m in wl.RESSERVE_M if m <= 16]:
        x = wl.resserve_x(M, K)
        q, r, y = fused(to_dev(x), qw, residue=True)
        oq, orr = orc.quantize_residue(x)
        assert_same_q(q, oq, "main")
        assert_same_q(r, orr, "residue")
        err = rel_fro(y.cpu().numpy()[:, rows], orc.gemm_residue(oq, orr, ow))
        assert err <= REL_FRO_TOL, (M, err)


# (3, 100, 320) and (4, 300, 4160): a ragged last k-tile, so the CTAs of a
# cluster encode slices of two widths; M = 3: the last warp holding units is
# only partly filled
@pytest.mark.parametrize("M,N,K", [(1, 1, 256), (3, 100, 320), (16, 200, 4224), (5, 130, 512), (16, 4000, 1088),
                                   (2, 513, 14336), (9, 128, 27648), (4, 300, 4096), (1, 260, 16384),
                                   (4, 300, 4160)])
@pytest.mark.parametrize("residue", [False, True])
@pytest.mark.parametrize("layout", [T, RM])
def test_fused_ragged(orc, M, N, K, residue, layout):
    qw, ow, rows = weight(orc, N, K)
    x = wl.resserve_x(M, K)
    q, r, y = fused(to_dev(x), qw, layout=layout, residue=residue)
    if residue:
        oq, orr = orc.quantize_residue(x)
        assert_same_q(r, orr, "residue")
        ref = orc.gemm_residue(oq, orr, ow)
    else:
        oq = orc.quantize(x)
        ref = orc.gemm(oq, ow)
    assert_same_q(q, oq, "main")
    err = rel_fro(y.cpu().numpy()[:, rows], ref)
    assert err <= REL_FRO_TOL, err


def test_fused_fp32_input_given_scales_bf16_out(orc):
    N, K, M = 640, 2048, 7
    qw, ow, rows = weight(orc, N, K)
    x = wl.resserve_x(M, K).astype(np.float32) * np.float32(1.7)
    s, s_r = np.float32(0.004), np.float32(3e-4)
    q, r, y = fused(to_dev(x, torch.float32), qw, residue=True, scale_in=s, rscale_in=s_r,
                    out_dtype=torch.bfloat16)
    oq, orr = orc.quantize_residue(x, s, s_r)
    assert_same_q(q, oq, "main")
    assert_same_q(r, orr, "residue")
    # bf16 output = the kernel's fp32 result rounded once: compare with the fp32 run
    _, _, y32 = fused(to_dev(x, torch.float32), qw, residue=True, scale_in=s, rscale_in=s_r)
    assert torch.equal(y, y32.to(torch.bfloat16))
    assert rel_fro(y32.cpu().numpy()[:, rows], orc.gemm_residue(oq, orr, ow)) <= REL_FRO_TOL


def test_fused_register_overflow_falls_back(orc):
    """A slice too large for the fused kernel's registers runs as two launches
    with the same results."""
    N, K, M = 128, 32768, 16
    qw, ow, rows = weight(orc, N, K)
    x = wl.decode_x(M, K)
    q, _, y = fused(to_dev(x), qw)
    ox = orc.quantize(x)
    assert_same_q(q, ox)
    assert rel_fro(y.cpu().numpy()[:, rows], orc.gemm(ox, ow)) <= REL_FRO_TOL


def test_fused_one_hot_placement(orc):
    """Exact integer sums: one non-zero activation per row hits a known W column."""
    N, K, M = 384, 1024, 16
    qw, ow, rows = weight(orc, N, K)
    x = np.zeros((M, K), np.float32)
    cols = (np.arange(M) * 61 + 5) % K
    x[np.arange(M), cols] = 3.0
    q, _, y = fused(to_dev(x, torch.float32), qw)
    ox = orc.quantize(x)
    assert_same_q(q, ox)
    ref = orc.gemm(ox, ow)
    assert rel_fro(y.cpu().numpy()[:, rows], ref) <= REL_FRO_TOL


def test_fused_nonfinite_reported():
    N, K = 256, 512
    w = torch.randn(N, K, device="cuda") * 0.02
    qw = nv.NVFP4Tensor.empty(N, K, T)
    nv.nvfp4_quantize(w, qw, workspace=nv.Workspace(N, K))
    x = torch.ones((2, K), dtype=torch.bfloat16, device="cuda")
    x[1, 100] = float("inf")
    q = nv.NVFP4Tensor.empty(2, K, T)
    y = torch.empty((2, N), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_quantize_gemm(x, q, qw, y, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 5


@pytest.mark.parametrize("x_layout", [T, RM])
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 257, 14336), (4, 1000, 320)])
def test_decode_kernel_on_nvfp4_operands(orc, x_layout, M, N, K):
    """nvfp4_gemm with TILED W and M <= 16 runs the tensor-core decode kernel
    on NVFP4 activations in either scale layout (ROWMAJOR activations meet
    TILED weights here too)."""
    qw, ow, rows = weight(orc, N, K)
    x = wl.decode_x(M, K)
    ox = orc.quantize(x)
    for residue in (False, True):
        qx = run_quantize(to_dev(x), x_layout)
        y = torch.full((M, N), float("nan"), device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        if residue:
            q, r = nv.NVFP4Tensor.empty(M, K, x_layout), nv.NVFP4Tensor.empty(M, K, x_layout)
            nv.nvfp4_quantize_residue(to_dev(x), q, r, workspace=nv.Workspace(M, K))
            nv.nvfp4_gemm_residue(q, r, qw, y, dev_status=st)
            oq, orr = orc.quantize_residue(x)
            ref = orc.gemm_residue(oq, orr, ow)
        else:
            nv.nvfp4_gemm(qx, qw, y, dev_status=st)
            ref = orc.gemm(ox, ow)
        torch.cuda.synchronize()
        assert st.item() == 0
        assert rel_fro(y.cpu().numpy()[:, rows], ref) <= REL_FRO_TOL


def test_quantize_gemm_plan():
    """The launch plan names one fused launch for the small decode calls and
    at most two launches for every decode shape."""
    assert nv.nvfp4_quantize_gemm_plan(1, 4096, 4096) == 1
    for M in wl.DECODE_M:
        for (N, K) in wl.DECODE_SHAPES:
            assert nv.nvfp4_quantize_gemm_plan(M, N, K) in (1, 2)
        for (N, K) in wl.RESSERVE_SHAPES:
            assert nv.nvfp4_quantize_gemm_plan(M, N, K, residue=True) in (1, 2)
    assert nv.nvfp4_quantize_gemm_plan(17, 4096, 4096) == 0

"""GPU parity: the MXFP4 linear (nvfp4_mx_gemm, kind::mxf4 tensor-core GEMM)
against the fp64 oracle on the same quantized operands (relative Frobenius
error <= 1e-5), and the MXFP4 quantizer's TILED scale layout bit for bit."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_18_b200 as nv
from nvfp4_block_scaled_18_b200 import workloads as wl

from gpu_util import REL_FRO_TOL, rel_fro, tiled_from_rowmajor, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nv.load_library()


def pack(codes: np.ndarray) -> torch.Tensor:
    """Unpacked E2M1 codes (rows x K) -> packed device bytes (low nibble first)."""
    c = np.ascontiguousarray(codes, np.uint8)
    return torch.from_numpy((c[:, 0::2] | (c[:, 1::2] << 4)).reshape(-1).copy()).cuda()


def dev_operand(q):
    codes, scales = q
    return pack(codes), torch.from_numpy(tiled_from_rowmajor(scales)).cuda()


def run_gemm(qa, qw, out_dtype=torch.float32):
    M, N = qa[0].shape[0], qw[0].shape[0]
    ac, asc = dev_operand(qa)
    wc, wsc = dev_operand(qw)
    y = torch.full((M, N), float("nan"), dtype=out_dtype, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_mx_gemm(ac.view(M, -1), asc, wc.view(N, -1), wsc, y, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0, nv.status_string(st.item())
    return y.float().cpu().numpy()


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (200, 300, 384), (1, 256, 512), (333, 520, 1280),
                                   (256, 1024, 4096)])
def test_mx_gemm_random(orc, M, N, K):
    a = wl.resserve_x(M, K)
    w = wl.weights_normal(N, K)
    qa, qw = orc.mx_quantize(a), orc.mx_quantize(w)
    y = run_gemm(qa, qw)
    assert rel_fro(y, orc.mx_gemm(qa, qw)) <= REL_FRO_TOL


def test_mx_gemm_scale_placement(orc):
    """Every 32-block of A and W carries its own power-of-two gain, so a scale
    byte read from the wrong block, row or scale-factor slot shows at once."""
    rng = np.random.default_rng(11)
    M, N, K = 160, 272, 768
    ga = np.exp2(rng.integers(-12, 13, (M, K // 32))).repeat(32, axis=1)
    gw = np.exp2(rng.integers(-12, 13, (N, K // 32))).repeat(32, axis=1)
    a = (rng.standard_normal((M, K)) * ga).astype(np.float32)
    w = (rng.standard_normal((N, K)) * gw).astype(np.float32)
    qa, qw = orc.mx_quantize(a), orc.mx_quantize(w)
    y = run_gemm(qa, qw)
    ref = orc.mx_gemm(qa, qw)
    assert rel_fro(y, ref) <= REL_FRO_TOL
    # every row and column, not only the norm: each row's error is small too
    err = np.abs(y - ref).max(axis=1) / np.maximum(np.abs(ref).max(axis=1), 1e-300)
    assert err.max() <= 1e-4


def test_mx_gemm_one_hot(orc):
    """A single nonzero code per operand row: Y[i, j] is one exact product."""
    M, N, K = 130, 260, 512
    rng = np.random.default_rng(5)
    ca = np.zeros((M, K), np.uint8)
    cw = np.zeros((N, K), np.uint8)
    ka = rng.integers(0, K, M)
    kw = ka[rng.integers(0, M, N)]
    ca[np.arange(M), ka] = rng.integers(1, 16, M)
    cw[np.arange(N), kw] = rng.integers(1, 16, N)
    sa = rng.integers(110, 140, (M, K // 32)).astype(np.uint8)
    sw = rng.integers(110, 140, (N, K // 32)).astype(np.uint8)
    y = run_gemm((ca, sa), (cw, sw))
    np.testing.assert_array_equal(y, orc.mx_gemm((ca, sa), (cw, sw)))


def test_mx_gemm_bf16_output(orc):
    M, N, K = 192, 384, 1024
    qa, qw = orc.mx_quantize(wl.resserve_x(M, K)), orc.mx_quantize(wl.weights_normal(N, K))
    y = run_gemm(qa, qw, torch.bfloat16)
    ref = orc.mx_gemm(qa, qw)
    # bf16 rounding of each fp32 output (relative 2^-9) plus the fp32
    # accumulation error, which is absolute on the scale of the row norms
    atol = 1e-5 * np.sqrt(np.mean(ref ** 2))
    assert np.all(np.abs(y - ref) <= 2.0 ** -8 * np.abs(ref) + atol)


def test_mx_quantize_tiled_then_gemm(orc):
    """The product path end to end: X and W quantized on the device with TILED
    scales (checked bit for bit), then the MXFP4 GEMM."""
    M, N, K = 300, 512, 2048
    x, w = wl.resserve_x(M, K), wl.weights_normal(N, K)
    ops = []
    for v, rows in ((x, M), (w, N)):
        c = torch.zeros(rows * K // 2, dtype=torch.uint8, device="cuda")
        s = torch.zeros(nv.mx_scales_bytes(rows, K, nv.SF_TILED), dtype=torch.uint8, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        nv.nvfp4_mx_quantize(to_dev(v), c, s, dev_status=st, sf_layout=nv.SF_TILED)
        torch.cuda.synchronize()
        assert st.item() == 0
        oc, osc = orc.mx_quantize(wl.bf16_values(v))
        b = c.cpu().numpy().reshape(rows, K // 2)
        np.testing.assert_array_equal(b & 0xF, oc[:, 0::2])
        np.testing.assert_array_equal(b >> 4, oc[:, 1::2])
        np.testing.assert_array_equal(s.cpu().numpy(), tiled_from_rowmajor(osc))
        ops.append((c, s, (oc, osc)))
    (ac, asc, qa), (wc, wsc, qw) = ops
    y = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_mx_gemm(ac.view(M, -1), asc, wc.view(N, -1), wsc, y)
    torch.cuda.synchronize()
    assert rel_fro(y.cpu().numpy(), orc.mx_gemm(qa, qw)) <= REL_FRO_TOL


def test_mx_gemm_large_sampled(orc):
    """A prefill-sized MXFP4 linear (8192 x 4096 x 4096), checked on sampled rows."""
    M, N, K = 8192, 4096, 4096
    rng = np.random.default_rng(3)
    a = wl.prefill_x(M, K)
    w = wl.weights_normal(N, K)
    qa, qw = orc.mx_quantize(a), orc.mx_quantize(w)
    y = run_gemm(qa, qw)
    rows = np.sort(rng.choice(M, 48, replace=False))
    ref = orc.mx_gemm((qa[0][rows], qa[1][rows]), qw)
    assert rel_fro(y[rows], ref) <= REL_FRO_TOL
    assert np.isfinite(y).all()


@pytest.mark.parametrize("K", [192, 128, 320])
def test_mx_gemm_rejects_unsupported_k(K):
    M, N = 128, 256
    ac = torch.zeros((M, K // 2), dtype=torch.uint8, device="cuda")
    wc = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    asc = torch.zeros(nv.mx_scales_bytes(M, K, nv.SF_TILED), dtype=torch.uint8, device="cuda")
    wsc = torch.zeros(nv.mx_scales_bytes(N, K, nv.SF_TILED), dtype=torch.uint8, device="cuda")
    y = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    with pytest.raises(nv.NVFP4Error) as e:
        nv.nvfp4_mx_gemm(ac, asc, wc, wsc, y)
    assert e.value.status == 3


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (333, 520, 1280), (1, 256, 512), (256, 1024, 4096)])
def test_mx_gemm_residue(orc, M, N, K):
    """MXFP4 compensated linear: the residue's K-tiles continue the same accumulation."""
    qa, qr = orc.mx_quantize_residue(wl.resserve_x(M, K))
    qw = orc.mx_quantize(wl.weights_normal(N, K))
    (ac, asc), (rc, rsc), (wc, wsc) = dev_operand(qa), dev_operand(qr), dev_operand(qw)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_mx_gemm_residue(ac.view(M, -1), asc, rc.view(M, -1), rsc, wc.view(N, -1), wsc, y, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert rel_fro(y.cpu().numpy(), orc.mx_gemm(qa, qw, qr)) <= REL_FRO_TOL


def test_mx_residue_on_device_then_gemm(orc):
    """X quantized with its residue on the device (TILED scales, checked bit for
    bit), W likewise without residue, then the compensated MXFP4 linear."""
    M, N, K = 300, 512, 2048
    x, w = wl.resserve_x(M, K), wl.weights_normal(N, K)
    ns_x, ns_w = nv.mx_scales_bytes(M, K, nv.SF_TILED), nv.mx_scales_bytes(N, K, nv.SF_TILED)
    xc = torch.zeros(M * K // 2, dtype=torch.uint8, device="cuda")
    xs = torch.zeros(ns_x, dtype=torch.uint8, device="cuda")
    rc, rs = torch.zeros_like(xc), torch.zeros_like(xs)
    wc = torch.zeros(N * K // 2, dtype=torch.uint8, device="cuda")
    wsc = torch.zeros(ns_w, dtype=torch.uint8, device="cuda")
    nv.nvfp4_mx_quantize(to_dev(x), xc, xs, rc, rs, sf_layout=nv.SF_TILED)
    nv.nvfp4_mx_quantize(to_dev(w), wc, wsc, sf_layout=nv.SF_TILED)
    y = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_mx_gemm_residue(xc.view(M, -1), xs, rc.view(M, -1), rs, wc.view(N, -1), wsc, y)
    torch.cuda.synchronize()
    (oc, osc), (orc_c, ors) = orc.mx_quantize_residue(wl.bf16_values(x))
    np.testing.assert_array_equal(rs.cpu().numpy(), tiled_from_rowmajor(ors))
    b = rc.cpu().numpy().reshape(M, K // 2)
    np.testing.assert_array_equal(b & 0xF, orc_c[:, 0::2])
    np.testing.assert_array_equal(b >> 4, orc_c[:, 1::2])
    qw = orc.mx_quantize(wl.bf16_values(w))
    assert rel_fro(y.cpu().numpy(), orc.mx_gemm((oc, osc), qw, (orc_c, ors))) <= REL_FRO_TOL

"""GPU parity: the CUDA quantizers against the CPU oracle, bit-exact codes and scales."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_18_b200 as nv
from nvfp4_block_scaled_18_b200 import workloads as wl

from gpu_util import assert_same_q, run_quantize, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nv.load_library()


@pytest.mark.parametrize("layout", [nv.SF_ROWMAJOR, nv.SF_TILED])
def test_tiny_config(orc, layout):
    x, w = wl.tiny()
    for arr, dt in ((x, torch.float32), (w, torch.float32)):
        q = run_quantize(to_dev(arr, dt), layout)
        assert_same_q(q, orc.quantize(arr))


@pytest.mark.parametrize("M,K", [(1, 4096), (16, 4096), (4, 14336), (37, 48), (1, 16), (130, 272)])
def test_decode_activations_bf16(orc, M, K):
    x = wl.decode_x(M, K)
    for layout in (nv.SF_ROWMAJOR, nv.SF_TILED):
        q = run_quantize(to_dev(x), layout)
        assert_same_q(q, orc.quantize(x), f"M={M} K={K} layout={layout}")


def test_weights_fp32(orc):
    w = wl.weights_normal(512, 4096)
    assert_same_q(run_quantize(to_dev(w, torch.float32)), orc.quantize(w))


def test_wide_dynamic_range_and_subnormal_scales(orc):
    rng = np.random.default_rng(21)
    x = (rng.standard_normal((64, 512)) * np.exp2(rng.uniform(-40, 40, (64, 32)).repeat(16, axis=1)))
    x = x.astype(np.float32)
    x[3, :] = 0.0
    x[5, 16:32] = 1e-30
    assert_same_q(run_quantize(to_dev(x, torch.float32)), orc.quantize(x))


def test_strided_rows(orc):
    x = wl.decode_x(8, 512)
    big = torch.zeros((8, 640), dtype=torch.bfloat16, device="cuda")
    big[:, :512] = to_dev(x)
    q = run_quantize(big[:, :512])
    assert_same_q(q, orc.quantize(x))


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("layout", [nv.SF_TILED, nv.SF_ROWMAJOR])
def test_strided_rows_multi_launch(orc, dt, layout):
    """Rows with a pitch larger than K through the multi-launch passes (the
    strided amax loop and the block pass's row split), plain and residue."""
    M, K, pad = 600, 4160, 64
    x = wl.resserve_x(M, K)
    big = torch.zeros((M, K + pad), dtype=dt, device="cuda")
    big[:, :K] = to_dev(x, dt)
    view = big[:, :K]
    assert_same_q(run_quantize(view, layout), orc.quantize(x), "plain")
    q, r = nv.NVFP4Tensor.empty(M, K, layout), nv.NVFP4Tensor.empty(M, K, layout)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_quantize_residue(view, q, r, workspace=nv.Workspace(M, K), dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    oq, orr = orc.quantize_residue(x)
    assert_same_q(q, oq, "main")
    assert_same_q(r, orr, "residue")


@pytest.mark.parametrize("s", [0.01, 1.0 / 2688, 3.0e-7])
def test_given_tensor_scale(orc, s):
    x = wl.decode_x(16, 1024)
    q = run_quantize(to_dev(x), scale_in=np.float32(s))
    assert_same_q(q, orc.quantize(x, np.float32(s)))


def test_zero_tensor(orc):
    x = np.zeros((4, 64), np.float32)
    q = run_quantize(to_dev(x, torch.float32))
    assert_same_q(q, orc.quantize(x))


def test_nonfinite_reported():
    x = torch.ones((2, 64), dtype=torch.float32, device="cuda")
    x[1, 7] = float("nan")
    q = nv.NVFP4Tensor.empty(2, 64)
    ws = nv.Workspace(2, 64)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_quantize(x, q, workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 5
    # the workspace is left reusable: a clean call afterwards succeeds
    st.zero_()
    x[1, 7] = 1.0
    nv.nvfp4_quantize(x, q, workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0


def test_e2m1_exhaustive_through_quantizer(orc):
    """Every fp32 with |v| <= 6 (both signs) goes through the device E2M1 encoder:
    blocks [6, v1..v15] under tensor scale 1 have d = 1, so the element codes are
    E2M1_RNE(v) exactly."""
    top = int(np.float32(6.0).view(np.uint32))
    all_bits = np.arange(0, top + 1, dtype=np.uint32)
    K = 1024
    chunk = 15 * 64 * 65536
    q_scale = torch.tensor([1.0], dtype=torch.float32, device="cuda")
    for sign in (0, 0x80000000):
        for start in range(0, all_bits.size, chunk):
            v = (all_bits[start:start + chunk] | np.uint32(sign)).view(np.float32)
            nblk = -(-v.size // 15)
            vals = np.zeros(nblk * 15, np.float32)
            vals[: v.size] = v
            blocks = np.concatenate([np.full((nblk, 1), 6.0, np.float32), vals.reshape(nblk, 15)], axis=1)
            rows = -(-nblk // 64)
            x = np.zeros((rows * 64, 16), np.float32)
            x[:, 0] = 6.0
            x[:nblk] = blocks
            x = x.reshape(rows, K)
            q = nv.NVFP4Tensor.empty(rows, K)
            nv.nvfp4_quantize(to_dev(x, torch.float32), q, scale_in=q_scale)
            codes = q.codes.cpu().numpy().reshape(-1)
            scales = q.scales.cpu().numpy()
            assert np.all(scales == 0x38)
            got = np.stack([codes & 0xF, codes >> 4], axis=1).reshape(-1, 16)[:nblk, 1:].reshape(-1)
            expect = orc.e2m1_encode_array(vals)
            np.testing.assert_array_equal(got[: v.size], expect[: v.size])


def test_e4m3_exhaustive_through_quantizer(orc):
    """Every fp32 ratio in [2^-12, 470] goes through the device E4M3 encoder:
    with s = fl32(1/6), fl32(6 s) = 1 so the block scale is E4M3_RNE(amax)."""
    s = np.float32(1.0) / np.float32(6.0)
    assert np.float32(np.float32(6.0) * s) == np.float32(1.0)
    lo = int(np.float32(2.0 ** -12).view(np.uint32))
    hi = int(np.float32(470.0).view(np.uint32))
    K = 1024
    chunk = 64 * 65536
    s_t = torch.tensor([s], dtype=torch.float32, device="cuda")
    for start in range(lo, hi + 1, chunk):
        a = np.arange(start, min(start + chunk, hi + 1), dtype=np.uint32).view(np.float32)
        rows = -(-a.size // 64)
        x = np.zeros((rows * 64, 16), np.float32)
        x[: a.size, 0] = a
        x = x.reshape(rows, K)
        q = nv.NVFP4Tensor.empty(rows, K)
        nv.nvfp4_quantize(to_dev(x, torch.float32), q, scale_in=s_t)
        got = q.scales.cpu().numpy().reshape(-1)[: a.size]
        np.testing.assert_array_equal(got, orc.e4m3_encode_array(a))


# ------------------------------------------------------------------ residue

@pytest.mark.parametrize("M,K", [(1, 5120), (4, 27648), (16, 5120), (16, 27648), (64, 5120), (128, 5120), (3, 80)])
def test_resserve_residue(orc, M, K):
    x = wl.resserve_x(M, K)
    xt = to_dev(x)
    for layout in (nv.SF_ROWMAJOR, nv.SF_TILED):
        q, r = nv.NVFP4Tensor.empty(M, K, layout), nv.NVFP4Tensor.empty(M, K, layout)
        ws = nv.Workspace(M, K)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        nv.nvfp4_quantize_residue(xt, q, r, workspace=ws, dev_status=st)
        torch.cuda.synchronize()
        assert st.item() == 0 and int(ws.buf.count_nonzero()) == 0
        oq, orr = orc.quantize_residue(x)
        assert_same_q(q, oq, "main")
        assert_same_q(r, orr, "residue")


def test_resserve_residue_given_scales(orc):
    x = wl.resserve_x(16, 1024)
    s, s_r = np.float32(0.004), np.float32(3e-4)
    q, r = nv.NVFP4Tensor.empty(16, 1024), nv.NVFP4Tensor.empty(16, 1024)
    nv.nvfp4_quantize_residue(to_dev(x), q, r,
                              scale_in=torch.tensor([s], device="cuda"),
                              rscale_in=torch.tensor([s_r], device="cuda"))
    torch.cuda.synchronize()
    oq, orr = orc.quantize_residue(x, s, s_r)
    assert_same_q(q, oq, "main")
    assert_same_q(r, orr, "residue")


# --------------------------------------------------------------- ARCQuant

@pytest.fixture(scope="module")
def arc():
    return wl.arc_inputs()


@pytest.mark.parametrize("S", [128, 256, 512])
def test_arcquant_fused_quantizer(orc, arc, S):
    x, gamma, perm = arc
    M, K = x.shape
    for layout in (nv.SF_ROWMAJOR, nv.SF_TILED):
        xa = nv.NVFP4Tensor.empty(M, K + S, layout)
        ws = nv.Workspace(M, K)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        nv.nvfp4_rmsnorm_reorder_quantize(to_dev(x), xa, gamma=to_dev(gamma), eps=1e-5,
                                          perm=torch.from_numpy(perm).cuda(), S=S, workspace=ws,
                                          dev_status=st)
        torch.cuda.synchronize()
        assert st.item() == 0 and int(ws.buf[:256].count_nonzero()) == 0
        ref = orc.rmsnorm_reorder_quantize(x, gamma, 1e-5, perm, S)
        assert_same_q(xa, ref, f"S={S} layout={layout}")


def test_reorder_residue_without_norm(orc):
    """The K -> K+S extension on raw activations (no RMSNorm), as in the large prefill case."""
    M, K, S = 256, 4096, 256
    x = wl.prefill_x(M, K)
    perm = wl.calibrated_perm(np.abs(x[:64]))
    xa = nv.NVFP4Tensor.empty(M, K + S, nv.SF_TILED)
    nv.nvfp4_rmsnorm_reorder_quantize(to_dev(x), xa, perm=torch.from_numpy(perm).cuda(), S=S,
                                      workspace=nv.Workspace(M, K))
    torch.cuda.synchronize()
    assert_same_q(xa, orc.rmsnorm_reorder_quantize(x, None, perm=perm, S=S))


def test_rmsnorm_identity_perm_f32_and_ragged(orc):
    rng = np.random.default_rng(31)
    M, K, S = 37, 208, 16
    x = (rng.standard_normal((M, K)) * np.exp2(rng.uniform(-20, 20, (M, 1)))).astype(np.float32)
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float32)
    xa = nv.NVFP4Tensor.empty(M, K + S)
    nv.nvfp4_rmsnorm_reorder_quantize(to_dev(x, torch.float32), xa, gamma=to_dev(gamma, torch.float32),
                                      eps=1e-6, S=S, workspace=nv.Workspace(M, K))
    torch.cuda.synchronize()
    assert_same_q(xa, orc.rmsnorm_reorder_quantize(x, gamma, 1e-6, None, S))


# ----------------------------------------- one-launch (small) vs multi-launch path

# Inputs of at most 65536 (bf16) / 32768 (fp32) 8-element units run as one
# cluster launch; larger ones as amax + quantize launches.  Both sides of the
# boundary, plain and residue, computed and given tensor scales.
@pytest.mark.parametrize("M,K,dt", [(16, 32768, torch.bfloat16), (17, 32768, torch.bfloat16),
                                    (8, 32768, torch.float32), (9, 32768, torch.float32),
                                    (5, 2048, torch.float32)])
@pytest.mark.parametrize("given", [False, True])
def test_quantize_paths_at_threshold(orc, M, K, dt, given):
    x = wl.resserve_x(M, K)
    xt = to_dev(x, dt)
    s_in = np.float32(0.0035) if given else None
    q = run_quantize(xt, nv.SF_TILED, scale_in=s_in)
    assert_same_q(q, orc.quantize(x, s_in), f"plain M={M} K={K}")
    q, r = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED), nv.NVFP4Tensor.empty(M, K, nv.SF_TILED)
    ws = nv.Workspace(M, K)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kw = {}
    if given:
        kw = dict(scale_in=torch.tensor([s_in], device="cuda"),
                  rscale_in=torch.tensor([np.float32(4e-4)], device="cuda"))
    nv.nvfp4_quantize_residue(xt, q, r, workspace=ws, dev_status=st, **kw)
    torch.cuda.synchronize()
    assert st.item() == 0 and int(ws.buf.count_nonzero()) == 0
    oq, orr = orc.quantize_residue(x, s_in, np.float32(4e-4)) if given else orc.quantize_residue(x)
    assert_same_q(q, oq, "main")
    assert_same_q(r, orr, "residue")


def test_nonfinite_reported_multi_launch():
    x = torch.ones((600, 4096), dtype=torch.float32, device="cuda")
    x[599, 4095] = float("inf")
    q = nv.NVFP4Tensor.empty(600, 4096)
    ws = nv.Workspace(600, 4096)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_quantize(x, q, workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 5
    assert int(ws.buf.count_nonzero()) == 0


# ------------------------------- ARCQuant quantizer: one launch or two passes

# X that fits in the shared memory of one wave of CTAs is quantized by one
# cooperative launch (rows read once, one grid-wide exchange of the maximum);
# larger X by the statistics pass and the reorder pass.  Both must give the
# oracle's codes and scales bit for bit and leave the workspace header zeroed.
@pytest.mark.parametrize("M,K,norm,given", [(2048, 4096, True, False), (2048, 4096, True, True),
                                            (2048, 4096, False, False), (3000, 4096, True, False),
                                            (8192, 4096, True, False), (5, 512, True, False)])
def test_reorder_one_launch_and_two_pass(orc, M, K, norm, given):
    S = 256 if K >= 256 else 0
    ch = wl.outlier_channels(K, 0.02)
    x = wl.bf16_values(wl.activations_normal(M, K, 0.02, 30.0, wl.SEED_X, ch))
    gamma = wl.bf16_values(wl.gamma_uniform(K)) if norm else None
    perm = wl.calibrated_perm(wl.activations_normal(64, K, 0.02, 30.0, wl.SEED_CALIB, ch))
    s_given = np.float32(0.05) if given else None
    xa = nv.NVFP4Tensor.empty(M, K + S, nv.SF_TILED)
    ws = nv.Workspace(M, K)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_rmsnorm_reorder_quantize(
        to_dev(x), xa, gamma=to_dev(gamma) if norm else None, eps=1e-5, perm=torch.from_numpy(perm).cuda(), S=S,
        scale_in=torch.tensor([s_given], dtype=torch.float32, device="cuda") if given else None,
        workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0 and int(ws.buf[:256].count_nonzero()) == 0
    ref = orc.rmsnorm_reorder_quantize(x, gamma, 1e-5, perm, S, s=s_given)
    assert_same_q(xa, ref, f"M={M} K={K}")


@pytest.mark.parametrize("M", [64, 4096])   # one launch / two passes
def test_reorder_bad_perm_reported(M):
    """A permutation entry outside 0..K-1 is reported (NVFP4_ERR_INVALID_ARG) and
    never used as an index; both set-up paths (16-byte aligned and not)."""
    K, S = 4096, 256
    x = to_dev(wl.prefill_x(M, K))
    gamma = to_dev(wl.bf16_values(wl.gamma_uniform(K)))
    base = torch.arange(K + 1, dtype=torch.int32, device="cuda")
    for perm in (base[:K].clone(), base[1:]):                  # aligned copy, 4-byte offset view
        perm[7] = K + 5
        perm[100] = -3
        xa = nv.NVFP4Tensor.empty(M, K + S, nv.SF_TILED)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        nv.nvfp4_rmsnorm_reorder_quantize(x, xa, gamma=gamma, perm=perm, S=S, workspace=nv.Workspace(M, K),
                                          dev_status=st)
        torch.cuda.synchronize()
        assert st.item() == 1


def test_reorder_unaligned_perm_same_result(orc):
    """The permutation set-up reads 16-byte vectors when it can and single
    entries otherwise; both give the oracle's result."""
    x, gamma, perm = wl.arc_inputs(M=256)
    K, S = x.shape[1], 128
    big = torch.zeros(K + 1, dtype=torch.int32, device="cuda")
    big[1:] = torch.from_numpy(np.ascontiguousarray(perm, dtype=np.int32)).cuda()
    xa = nv.NVFP4Tensor.empty(256, K + S, nv.SF_TILED)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_rmsnorm_reorder_quantize(to_dev(x), xa, gamma=to_dev(gamma), eps=1e-5, perm=big[1:], S=S,
                                      workspace=nv.Workspace(256, K), dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert_same_q(xa, orc.rmsnorm_reorder_quantize(x, gamma, 1e-5, perm, S))


@pytest.mark.parametrize("M,K", [(24, 512), (8192, 4096)])   # one launch / two passes
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_rmsnorm_mean_square_extremes(orc, M, K, dtype):
    """The exact mean square at its edges: rows of subnormal values only, rows
    where one large element pushes the others' squares below the 2^-34 grain,
    all-zero rows and ordinary rows, with gamma, both launch forms."""
    S = 64
    rng = np.random.default_rng(M + (dtype == torch.float32))
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[0::4] *= np.float32(2.0 ** -130)          # fp32 subnormals (bf16: flush to the smallest normals' grain)
    x[1::4] *= np.float32(2.0 ** -30)
    x[1::4, 7] = np.float32(3.0e4)              # one large element per row
    x[2::4] = 0.0
    if dtype == torch.bfloat16:
        x = wl.bf16_values(x)
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float32)
    if dtype == torch.bfloat16:
        gamma = wl.bf16_values(gamma)
    xa = nv.NVFP4Tensor.empty(M, K + S, nv.SF_TILED)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_rmsnorm_reorder_quantize(to_dev(x, dtype), xa, gamma=to_dev(gamma, dtype), eps=1e-5, S=S,
                                      workspace=nv.Workspace(M, K), dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0, nv.status_string(st.item())
    assert_same_q(xa, orc.rmsnorm_reorder_quantize(x, gamma, 1e-5, None, S))

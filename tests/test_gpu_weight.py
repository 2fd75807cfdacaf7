"""GPU parity: the offline weight preparation (nvfp4_quantize_weight) against the
oracle, and the smoothing fold end to end.

ARCQuant blog post sections 3.1 and 6.3: the weight takes the activations'
channel order and repeats its S outlier columns, W_aug = [W' | W'[:, :S]], so
that one GEMM over K+S columns multiplies X_aug.  OSFP4 page, abstract: a
per-channel smoothing vector sigma is absorbed at inference time, 1/sigma in
the RMSNorm gain and W diag(sigma) in the weight."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_18_b200 as nv
from nvfp4_block_scaled_18_b200 import workloads as wl

from gpu_util import REL_FRO_TOL, assert_same_q, rel_fro, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nv.load_library()


def _prep(w_t, K, S, sigma=None, perm=None, layout=nv.SF_TILED):
    N = w_t.shape[0]
    q = nv.NVFP4Tensor.empty(N, K + S, layout)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = nv.Workspace(N, K)
    nv.nvfp4_quantize_weight(w_t, q, sigma=sigma, perm=perm, S=S, workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    return q, st.item(), ws


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("S", [0, 64, 256])
@pytest.mark.parametrize("smooth", [False, True])
@pytest.mark.parametrize("layout", [nv.SF_ROWMAJOR, nv.SF_TILED])
def test_weight_prep_matches_oracle(orc, dtype, S, smooth, layout):
    N, K = 200, 512
    rng = np.random.default_rng(S + 7 * smooth + 3 * layout)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[:, rng.choice(K, 5, replace=False)] *= 20
    if dtype == torch.bfloat16:
        w = wl.bf16_values(w)
    perm = rng.permutation(K).astype(np.int32)
    sigma = rng.uniform(0.5, 2.0, K).astype(np.float32) if smooth else None
    q, st, ws = _prep(to_dev(w, dtype), K, S, None if sigma is None else torch.from_numpy(sigma).cuda(),
                      torch.from_numpy(perm).cuda(), layout)
    assert st == 0, nv.status_string(st)
    assert int(ws.buf.count_nonzero()) == 0, "workspace not left zeroed"
    assert_same_q(q, orc.quantize(orc.augment_weight(w, perm, S, sigma)), "W_aug")


def test_weight_prep_identity_and_given_scale(orc):
    """No permutation and no smoothing is nvfp4_quantize; a given tensor scale is used
    and written to the output tensor."""
    N, K = 64, 256
    w = wl.weights_normal(N, K)
    q, st, _ = _prep(to_dev(w, torch.float32), K, 0)
    assert st == 0
    assert_same_q(q, orc.quantize(w), "W")
    s_in = torch.tensor([1e-5], dtype=torch.float32, device="cuda")
    q2 = nv.NVFP4Tensor.empty(N, K + 32, nv.SF_TILED)
    nv.nvfp4_quantize_weight(to_dev(w, torch.float32), q2, S=32, scale_in=s_in)
    torch.cuda.synchronize()
    assert_same_q(q2, orc.quantize(orc.augment_weight(w, np.arange(K), 32), np.float32(1e-5)), "W given s")


def test_weight_prep_reports_bad_permutation():
    N, K = 16, 64
    perm = torch.arange(K, dtype=torch.int32, device="cuda")
    perm[5] = K + 3
    _, st, _ = _prep(torch.ones((N, K), device="cuda"), K, 16, perm=perm)
    assert st == 1, nv.status_string(st)   # NVFP4_ERR_INVALID_ARG


def test_smoothing_fold_end_to_end(orc):
    """sigma folded into the gain (gamma / sigma, in the activations' bf16) and into
    the weight (W diag(sigma)) before quantization: the fused quantizer, the weight
    preparation and the K+S GEMM give the oracle's Y on the same folded operands,
    and that Y stays close to the unquantized product of the unsmoothed layer."""
    M, K, N, S = 96, 1024, 384, 128
    ch = wl.outlier_channels(K, 0.02)
    x = wl.bf16_values(wl.activations_normal(M, K, 0.02, 30.0, wl.SEED_X, ch))
    gamma = wl.gamma_uniform(K)
    w = wl.weights_normal(N, K)
    w[:, ch] *= 0.2
    # a smoothing vector that moves magnitude from the activation outliers to W
    act = np.abs(x).max(axis=0) + 1e-3
    wmax = np.abs(w).max(axis=0) + 1e-6
    sigma = np.sqrt(act / wmax).astype(np.float32)
    sigma /= np.float32(np.median(sigma))
    gamma_s = wl.bf16_values((gamma / sigma).astype(np.float32))     # folded gain, rounded to bf16
    perm = wl.calibrated_perm(wl.activations_normal(512, K, 0.02, 30.0, wl.SEED_CALIB, ch) / sigma)
    xa = nv.NVFP4Tensor.empty(M, K + S, nv.SF_TILED)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_rmsnorm_reorder_quantize(to_dev(x), xa, gamma=to_dev(gamma_s), eps=1e-5,
                                      perm=torch.from_numpy(perm).cuda(), S=S, workspace=nv.Workspace(M, K),
                                      dev_status=st)
    qw, st_w, _ = _prep(to_dev(w, torch.float32), K, S, torch.from_numpy(sigma).cuda(),
                        torch.from_numpy(perm).cuda())
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(xa, qw, y, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0 and st_w == 0
    ox = orc.rmsnorm_reorder_quantize(x, gamma_s, 1e-5, perm, S)
    ow = orc.quantize(orc.augment_weight(w, perm, S, sigma))
    assert_same_q(xa, ox, "X_aug")
    assert_same_q(qw, ow, "W_aug")
    yv = y.cpu().numpy()
    assert rel_fro(yv, orc.gemm(ox, ow)) <= REL_FRO_TOL
    # the fold is an identity of the unquantized layer RMSNorm(x) gamma W^T: the
    # folded W4A4 result is as close to it as the unfolded W4A4 result (the oracle's)
    xn = orc.rmsnorm(x, None, 1e-5).astype(np.float64) * gamma.astype(np.float64)
    y_exact = xn @ w.astype(np.float64).T
    perm0 = wl.calibrated_perm(wl.activations_normal(512, K, 0.02, 30.0, wl.SEED_CALIB, ch))
    y0 = orc.gemm(orc.rmsnorm_reorder_quantize(x, wl.bf16_values(gamma), 1e-5, perm0, S),
                  orc.quantize(orc.augment_weight(w, perm0, S)))
    err_fold, err_plain = rel_fro(yv, y_exact), rel_fro(y0, y_exact)
    assert err_fold < 0.25 and err_fold <= 1.5 * err_plain + 0.01, (err_fold, err_plain)

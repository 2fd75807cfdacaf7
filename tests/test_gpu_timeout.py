"""GPU: the bounded device-side waits of the tensor-core kernels give up, report
NVFP4_ERR_TIMEOUT through dev_status and leave the context usable.

A wait is made to run out without any fault: with nvfp4_test_wait_fault the
load issuers of the next launches skip their weight tiles, so the roles that
wait for those tiles reach the (shortened) limit.  No bulk copy is in flight
then; every CTA still completes the exchanges its cluster peers count on,
waits for its own MMAs, frees its tensor memory and exits.  The call after
the reset must give the same output as before, matching the oracle.
The pages have no counterpart: this is failure detection around the method.
"""
import time

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_18_b200 as nv

from gpu_util import REL_FRO_TOL, rel_fro, run_quantize, to_dev

pytestmark = pytest.mark.gpu

ERR_TIMEOUT = 6
LIMIT_NS = 20_000_000   # 20 ms


@pytest.fixture(autouse=True)
def _reset_hook():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nv.load_library()
    nv.nvfp4_test_wait_fault(0, False)
    yield
    nv.nvfp4_test_wait_fault(0, False)


def _timed_out_then_recovers(run, ref):
    """run(st) launches one call writing its output; ref: the oracle's output."""
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    good = run(st).clone()
    torch.cuda.synchronize()
    assert st.item() == 0, nv.status_string(st.item())
    assert rel_fro(good.float().cpu().numpy(), ref) <= REL_FRO_TOL

    nv.nvfp4_test_wait_fault(LIMIT_NS, True)
    try:
        t0 = time.perf_counter()
        run(st)
        torch.cuda.synchronize()
        dt = time.perf_counter() - t0
    finally:
        nv.nvfp4_test_wait_fault(0, False)
    assert st.item() == ERR_TIMEOUT, nv.status_string(st.item())
    assert dt < 2.0, f"the timed-out launch took {dt:.3f} s"

    st.zero_()
    again = run(st)
    torch.cuda.synchronize()
    assert st.item() == 0, nv.status_string(st.item())
    assert torch.equal(again, good)


def _operands(orc, M, N, K, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    return x, w


@pytest.mark.parametrize("M", [8, 64, 256])
def test_gemm_wait_times_out_and_recovers(orc, M):
    """M = 8: tensor-core decode kernel (cluster split of K); 64: few-row kernel;
    256: large-M GEMM.  (M <= 4 runs on CUDA cores, which have no such waits.)"""
    N, K = 384, 1024
    x, w = _operands(orc, M, N, K, M)
    qa = run_quantize(to_dev(x, torch.float32), nv.SF_TILED)
    qw = run_quantize(to_dev(w, torch.float32), nv.SF_TILED)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")

    def run(st):
        nv.nvfp4_gemm(qa, qw, y, dev_status=st)
        return y
    _timed_out_then_recovers(run, orc.gemm(orc.quantize(x), orc.quantize(w)))


@pytest.mark.parametrize("M", [8, 64, 256])
def test_residue_gemm_wait_times_out_and_recovers(orc, M):
    N, K = 256, 512
    x, w = _operands(orc, M, N, K, 100 + M)
    q = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED)
    r = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED)
    nv.nvfp4_quantize_residue(to_dev(x, torch.float32), q, r, workspace=nv.Workspace(M, K))
    qw = run_quantize(to_dev(w, torch.float32), nv.SF_TILED)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")

    def run(st):
        nv.nvfp4_gemm_residue(q, r, qw, y, dev_status=st)
        return y
    oq, orr = orc.quantize_residue(x)
    _timed_out_then_recovers(run, orc.gemm_residue(oq, orr, orc.quantize(w)))


@pytest.mark.parametrize("residue", [False, True])
@pytest.mark.parametrize("M,K", [(8, 2048), (16, 2048)])
def test_fused_decode_wait_times_out_and_recovers(orc, residue, M, K):
    """The fused quantize + GEMM decode kernel: its CTAs still exchange the tensor
    maxima and their partial rows with their cluster peers while timing out
    (M = 8: X and R share one 16-row operand; M = 16: a 32-row operand)."""
    N = 512   # the tensor-core decode kernel (M <= 4 runs on CUDA cores)
    assert nv.nvfp4_quantize_gemm_plan(M, N, K, x_dtype=torch.float32, residue=residue) == 1
    x, w = _operands(orc, M, N, K, 7)
    xt = to_dev(x, torch.float32)
    qw = run_quantize(to_dev(w, torch.float32), nv.SF_TILED)
    q = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED)
    r = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED) if residue else None
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")

    def run(st):
        if residue:
            nv.nvfp4_quantize_residue_gemm(xt, q, r, qw, y, dev_status=st)
        else:
            nv.nvfp4_quantize_gemm(xt, q, qw, y, dev_status=st)
        return y
    if residue:
        oq, orr = orc.quantize_residue(x)
        ref = orc.gemm_residue(oq, orr, orc.quantize(w))
    else:
        ref = orc.gemm(orc.quantize(x), orc.quantize(w))
    _timed_out_then_recovers(run, ref)


def test_mx_gemm_wait_times_out_and_recovers(orc):
    M, N, K = 256, 256, 512
    x, w = _operands(orc, M, N, K, 11)
    ops = []
    for v in (x, w):
        rows = v.shape[0]
        c = torch.empty((rows, K // 2), dtype=torch.uint8, device="cuda")
        sc = torch.empty(nv.mx_scales_bytes(rows, K, nv.SF_TILED), dtype=torch.uint8, device="cuda")
        nv.nvfp4_mx_quantize(to_dev(v, torch.float32), c.view(-1), sc, sf_layout=nv.SF_TILED)
        ops.append((c, sc))
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")

    def run(st):
        nv.nvfp4_mx_gemm(ops[0][0], ops[0][1], ops[1][0], ops[1][1], y, dev_status=st)
        return y
    _timed_out_then_recovers(run, orc.mx_gemm(orc.mx_quantize(x), orc.mx_quantize(w)))


def test_short_limit_without_withholding_changes_nothing(orc):
    """A 50 ms limit is far above any wait of a normal call: results are unchanged."""
    M, N, K = 256, 512, 1024
    x, w = _operands(orc, M, N, K, 13)
    qa = run_quantize(to_dev(x, torch.float32), nv.SF_TILED)
    qw = run_quantize(to_dev(w, torch.float32), nv.SF_TILED)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_test_wait_fault(50_000_000, False)
    nv.nvfp4_gemm(qa, qw, y, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0, nv.status_string(st.item())
    assert rel_fro(y.cpu().numpy(), orc.gemm(orc.quantize(x), orc.quantize(w))) <= REL_FRO_TOL

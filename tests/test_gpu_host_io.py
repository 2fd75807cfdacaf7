"""GPU: nvfp4_quantize_gemm_host, the decode linear between host buffers.  The
activations are copied from host memory, quantized and multiplied on the device,
and Y is copied back, all on one stream.  Q(X) must equal the oracle's encoding
bit for bit, Y must match the fp64 oracle within relative Frobenius 1e-5, and
the host result must equal the device-buffer call on the same inputs."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_18_b200 as nv
from nvfp4_block_scaled_18_b200 import workloads as wl

from gpu_util import REL_FRO_TOL, assert_same_q, rel_fro, run_quantize, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nv.load_library()


@pytest.mark.parametrize("M,N,K,pinned", [(1, 512, 1024, True), (4, 4096, 4096, True), (16, 384, 2048, False),
                                          (3, 200, 320, True)])
def test_host_buffers_match_device_call_and_oracle(orc, M, N, K, pinned):
    x = wl.decode_x(M, K)
    w = wl.weights_normal(N, K)
    qw = run_quantize(to_dev(w, torch.float32), nv.SF_TILED)
    x_host = torch.from_numpy(x).to(torch.bfloat16)
    y_host = torch.full((M, N), float("nan"), dtype=torch.float32)
    if pinned:
        x_host, y_host = x_host.pin_memory(), y_host.pin_memory()
    x_dev = torch.empty((M, K + 64), dtype=torch.bfloat16, device="cuda")[:, :K]   # strided device rows
    y_dev = torch.empty((M, N + 32), dtype=torch.float32, device="cuda")[:, :N]
    q = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED)
    nv.nvfp4_quantize_gemm_host(x_host, x_dev, q, qw, y_dev, y_host)
    torch.cuda.current_stream().synchronize()

    ox = orc.quantize(x_host.float().numpy())
    assert_same_q(q, ox)
    assert torch.equal(x_dev.cpu(), x_host)
    ow = orc.quantize(w)
    assert rel_fro(y_host.numpy(), orc.gemm(ox, ow)) <= REL_FRO_TOL

    y_ref = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_quantize_gemm(to_dev(x), nv.NVFP4Tensor.empty(M, K, nv.SF_TILED), qw, y_ref)
    torch.cuda.synchronize()
    assert torch.equal(y_host, y_ref.cpu())


def test_host_buffers_in_a_graph(orc):
    """Pinned buffers: the copies and the kernel replay from a CUDA graph; new host
    inputs written between replays give new outputs."""
    M, N, K = 2, 1024, 2048
    w = wl.weights_normal(N, K)
    qw = run_quantize(to_dev(w, torch.float32), nv.SF_TILED)
    x_host = torch.empty((M, K), dtype=torch.bfloat16).pin_memory()
    y_host = torch.empty((M, N), dtype=torch.float32).pin_memory()
    x_dev = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    y_dev = torch.empty((M, N), dtype=torch.float32, device="cuda")
    q = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED)
    x_host.copy_(torch.from_numpy(wl.decode_x(M, K)).to(torch.bfloat16))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        nv.nvfp4_quantize_gemm_host(x_host, x_dev, q, qw, y_dev, y_host)   # warm-up (kernel attributes)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        nv.nvfp4_quantize_gemm_host(x_host, x_dev, q, qw, y_dev, y_host)
    ow = orc.quantize(w)
    for seed in (5, 6):
        xs = (np.random.default_rng(seed).standard_normal((M, K)) * 3).astype(np.float32)
        x_host.copy_(torch.from_numpy(xs).to(torch.bfloat16))
        g.replay()
        torch.cuda.synchronize()
        ox = orc.quantize(x_host.float().numpy())
        assert rel_fro(y_host.numpy(), orc.gemm(ox, ow)) <= REL_FRO_TOL

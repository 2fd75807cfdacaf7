"""GPU parity: the MXFP4 quantizer (nvfp4_mx_quantize) against the oracle, bit
for bit on codes and E8M0 scales, with and without the residue."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_18_b200 as nv
from nvfp4_block_scaled_18_b200 import workloads as wl

from gpu_util import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nv.load_library()


def unpack(codes: torch.Tensor, M: int, K: int) -> np.ndarray:
    b = codes.cpu().numpy().reshape(M, K // 2)
    out = np.empty((M, K), np.uint8)
    out[:, 0::2] = b & 0xF
    out[:, 1::2] = b >> 4
    return out


def run_mx(x_t, residue=False):
    M, K = x_t.shape
    c = torch.zeros(M * K // 2, dtype=torch.uint8, device="cuda")
    s = torch.zeros(M * K // 32, dtype=torch.uint8, device="cuda")
    rc = torch.zeros_like(c) if residue else None
    rs = torch.zeros_like(s) if residue else None
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_mx_quantize(x_t, c, s, rc, rs, dev_status=st)
    torch.cuda.synchronize()
    return c, s, rc, rs, st.item()


def check(orc, x, x_t, residue):
    M, K = x.shape
    c, s, rc, rs, st = run_mx(x_t, residue)
    assert st == 0
    if residue:
        (oc, osc), (orc_, ors) = orc.mx_quantize_residue(x)
        np.testing.assert_array_equal(unpack(rc, M, K), orc_)
        np.testing.assert_array_equal(rs.cpu().numpy().reshape(M, K // 32), ors)
    else:
        oc, osc = orc.mx_quantize(x)
    np.testing.assert_array_equal(unpack(c, M, K), oc)
    np.testing.assert_array_equal(s.cpu().numpy().reshape(M, K // 32), osc)


@pytest.mark.parametrize("residue", [False, True])
@pytest.mark.parametrize("M,K", [(4, 256), (16, 5120), (64, 5120), (600, 4160)])
def test_mx_bf16(orc, M, K, residue):
    x = wl.resserve_x(M, K)
    check(orc, x, to_dev(x), residue)


@pytest.mark.parametrize("residue", [False, True])
def test_mx_fp32_wide_range_zeros_subnormals(orc, residue):
    rng = np.random.default_rng(4)
    M, K = 32, 512
    x = rng.standard_normal((M, K)) * np.exp2(rng.uniform(-140, 120, (M, K // 32)).repeat(32, axis=1))
    x = x.astype(np.float32)
    x[3, :] = 0.0
    x[5, 32:64] = 1e-42
    x[7, 64:96] = np.float32(3.4e38)
    check(orc, x, to_dev(x, torch.float32), residue)


def test_mx_strided_rows(orc):
    M, K = 48, 1024
    x = wl.decode_x(M, K)
    big = torch.zeros((M, K + 96), dtype=torch.bfloat16, device="cuda")
    big[:, :K] = to_dev(x)
    check(orc, x, big[:, :K], True)


def test_mx_nonfinite_reported():
    x = torch.ones((4, 256), dtype=torch.float32, device="cuda")
    x[2, 77] = float("nan")
    assert run_mx(x)[4] == 5


def test_mx_rejects_bad_arguments():
    x = torch.ones((4, 48), dtype=torch.bfloat16, device="cuda")     # K % 32 != 0
    c = torch.zeros(4 * 24, dtype=torch.uint8, device="cuda")
    s = torch.zeros(6, dtype=torch.uint8, device="cuda")
    with pytest.raises(nv.NVFP4Error):
        nv.nvfp4_mx_quantize(x, c, s)

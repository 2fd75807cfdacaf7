"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare with the CPU oracle (which never sees CUDA-path values as inputs)."""
import numpy as np
import torch

import nvfp4_block_scaled_18_b200 as nv

REL_FRO_TOL = 1e-5   # GEMM outputs vs the fp64 oracle on the same quantized operands


def to_dev(x: np.ndarray, dtype=torch.bfloat16) -> torch.Tensor:
    """Upload fp32 values (already representable in dtype) to the GPU."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(dtype).cuda()


def run_quantize(x_t, layout=nv.SF_ROWMAJOR, scale_in=None):
    M, K = x_t.shape
    q = nv.NVFP4Tensor.empty(M, K, layout)
    ws = nv.Workspace(M, K)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    s_in = None if scale_in is None else torch.tensor([scale_in], dtype=torch.float32, device="cuda")
    nv.nvfp4_quantize(x_t, q, scale_in=s_in, workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0, nv.status_string(st.item())
    assert int(ws.buf.count_nonzero()) == 0, "workspace not left zeroed"
    return q


def assert_same_q(q_gpu, q_orc, what=""):
    np.testing.assert_array_equal(q_gpu.codes.cpu().numpy(), q_orc.codes, err_msg=what + " codes")
    np.testing.assert_array_equal(q_gpu.scales_rowmajor().cpu().numpy(), q_orc.scales,
                                  err_msg=what + " scales")
    assert np.float32(q_gpu.tensor_scale.item()) == np.float32(q_orc.s), what + " tensor scale"


def rel_fro(y, ref) -> float:
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300))


def sub_rows(orc, q_full_codes, q_full_scales, s, rows):
    """An oracle QTensor of selected rows (slicing only)."""
    return orc.QTensor(np.ascontiguousarray(q_full_codes[rows]), np.ascontiguousarray(q_full_scales[rows]), s)


def tiled_from_rowmajor(scales: np.ndarray) -> np.ndarray:
    """Place row-major block scales (rows x nb) into the TILED atom layout (layout only)."""
    rows, nb = scales.shape
    katoms = (nb + 3) // 4
    out = np.zeros(((rows + 127) // 128) * katoms * 512, np.uint8)
    r = np.arange(rows)[:, None]
    b = np.arange(nb)[None, :]
    off = ((r // 128) * katoms + b // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (b % 4)
    out[off] = scales
    return out


def gpu_tensor(codes, scales_rowmajor, s, layout=nv.SF_TILED):
    rows, cols = codes.shape[0], codes.shape[1] * 2
    sc = tiled_from_rowmajor(scales_rowmajor) if layout == nv.SF_TILED else scales_rowmajor.reshape(-1)
    return nv.NVFP4Tensor(torch.from_numpy(np.ascontiguousarray(codes)).cuda(), torch.from_numpy(sc).cuda(),
                          torch.tensor([s], dtype=torch.float32, device="cuda"), rows, cols, layout)

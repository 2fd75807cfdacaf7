"""Python binding of the NVFP4 B200 library (include/nvfp4.h).

Argument marshalling only: every step of the hot path runs in the CUDA kernels
of libnvfp4.so; torch supplies device memory and streams.  The functions keep
the C names.  There is no CPU fallback: importing works anywhere, but any
compute call raises if the CUDA library or a CUDA device is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4.so")

NVFP4_OK = 0
STATUS_NAMES = {0: "NVFP4_OK", 1: "NVFP4_ERR_INVALID_ARG", 2: "NVFP4_ERR_ALIGNMENT",
                3: "NVFP4_ERR_UNSUPPORTED", 4: "NVFP4_ERR_CUDA", 5: "NVFP4_ERR_NONFINITE",
                6: "NVFP4_ERR_TIMEOUT", 7: "NVFP4_ERR_WORKSPACE"}
NVFP4_F32, NVFP4_BF16 = 0, 1
SF_ROWMAJOR, SF_TILED = 0, 1

EXPORTED_SYMBOLS = ("nvfp4_scales_bytes", "nvfp4_workspace_size", "nvfp4_quantize",
                    "nvfp4_quantize_residue", "nvfp4_rmsnorm_reorder_quantize", "nvfp4_gemm",
                    "nvfp4_gemm_residue", "nvfp4_quantize_gemm", "nvfp4_quantize_residue_gemm",
                    "nvfp4_quantize_gemm_plan", "nvfp4_quantize_gemm_host",
                    "nvfp4_rmsnorm_reorder_quantize_noalloc", "nvfp4_mx_quantize",
                    "nvfp4_mx_scales_bytes", "nvfp4_mx_gemm", "nvfp4_mx_gemm_residue", "nvfp4_quantize_weight",
                    "nvfp4_test_wait_fault", "nvfp4_status_string", "nvfp4_version")
NVFP4_NOALLOC_MAX_ROWS = 65536


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({status_string(status)})")


class _CTensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("sf_layout", ctypes.c_int)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libnvfp4.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"CUDA library not built: {path} (run python -m nvfp4_block_scaled_18_b200.build)")
        lib = ctypes.CDLL(path)
        P, I64, SZ, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
        T = ctypes.POINTER(_CTensor)
        lib.nvfp4_scales_bytes.argtypes = [I64, I64, ctypes.c_int]
        lib.nvfp4_scales_bytes.restype = SZ
        lib.nvfp4_workspace_size.argtypes = [I64, I64]
        lib.nvfp4_workspace_size.restype = SZ
        lib.nvfp4_quantize.argtypes = [P, ctypes.c_int, I64, I64, I64, P, T, P, SZ, P, P]
        lib.nvfp4_quantize_residue.argtypes = [P, ctypes.c_int, I64, I64, I64, P, P, T, T, P, SZ, P, P]
        lib.nvfp4_rmsnorm_reorder_quantize.argtypes = [P, ctypes.c_int, I64, I64, I64, P, F, P, I64, P, T,
                                                       P, SZ, P, P]
        lib.nvfp4_rmsnorm_reorder_quantize_noalloc.argtypes = [P, ctypes.c_int, I64, I64, I64, P, F, P, I64, P,
                                                               T, P, P]
        lib.nvfp4_gemm.argtypes = [T, T, P, ctypes.c_int, I64, P, P]
        lib.nvfp4_gemm_residue.argtypes = [T, T, T, P, ctypes.c_int, I64, P, P]
        lib.nvfp4_quantize_gemm.argtypes = [P, ctypes.c_int, I64, I64, I64, P, T, T, P, ctypes.c_int, I64, P, P]
        lib.nvfp4_quantize_gemm_host.argtypes = [P, P, ctypes.c_int, I64, I64, I64, P, T, T, P, P, ctypes.c_int,
                                                 I64, P, P]
        lib.nvfp4_quantize_gemm_plan.argtypes = [I64, I64, I64, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.nvfp4_quantize_gemm_plan.restype = ctypes.c_int
        lib.nvfp4_quantize_residue_gemm.argtypes = [P, ctypes.c_int, I64, I64, I64, P, P, T, T, T, P,
                                                    ctypes.c_int, I64, P, P]
        lib.nvfp4_mx_quantize.argtypes = [P, ctypes.c_int, I64, I64, I64, P, P, P, P, ctypes.c_int, P, P]
        lib.nvfp4_mx_scales_bytes.argtypes = [I64, I64, ctypes.c_int]
        lib.nvfp4_mx_scales_bytes.restype = SZ
        lib.nvfp4_mx_gemm.argtypes = [P, P, P, P, I64, I64, I64, P, ctypes.c_int, I64, P, P]
        lib.nvfp4_mx_gemm_residue.argtypes = [P, P, P, P, P, P, I64, I64, I64, P, ctypes.c_int, I64, P, P]
        for fn in ("nvfp4_quantize", "nvfp4_quantize_residue", "nvfp4_rmsnorm_reorder_quantize",
                   "nvfp4_rmsnorm_reorder_quantize_noalloc", "nvfp4_gemm", "nvfp4_gemm_residue",
                   "nvfp4_mx_quantize", "nvfp4_mx_gemm", "nvfp4_mx_gemm_residue"):
            getattr(lib, fn).restype = ctypes.c_int
        lib.nvfp4_quantize_weight.argtypes = [P, ctypes.c_int, I64, I64, I64, P, P, I64, P, T, P, SZ, P, P]
        lib.nvfp4_quantize_weight.restype = ctypes.c_int
        lib.nvfp4_test_wait_fault.argtypes = [ctypes.c_uint64, ctypes.c_int]
        lib.nvfp4_test_wait_fault.restype = None
        lib.nvfp4_status_string.argtypes = [ctypes.c_int]
        lib.nvfp4_status_string.restype = ctypes.c_char_p
        lib.nvfp4_version.restype = ctypes.c_char_p
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    try:
        return load_library().nvfp4_status_string(int(status)).decode()
    except RuntimeError:
        return STATUS_NAMES.get(status, "unknown")


def nvfp4_test_wait_fault(limit_ns: int = 0, withhold: bool = False) -> None:
    """Test support: bound every device-side wait of the tensor-core kernels by
    limit_ns (0 = the default 4 s); withhold=True makes the following launches
    skip their weight-tile loads so that the waits run out (NVFP4_ERR_TIMEOUT
    in dev_status).  Process wide; for tests only."""
    load_library().nvfp4_test_wait_fault(int(limit_ns), 1 if withhold else 0)


def nvfp4_version() -> str:
    return load_library().nvfp4_version().decode()


def nvfp4_scales_bytes(rows: int, cols: int, sf_layout: int = SF_ROWMAJOR) -> int:
    return int(load_library().nvfp4_scales_bytes(rows, cols, sf_layout))


def nvfp4_workspace_size(M: int, K: int) -> int:
    return int(load_library().nvfp4_workspace_size(M, K))


class NVFP4Tensor:
    """An NVFP4 matrix held in torch device memory (see nvfp4_tensor in nvfp4.h)."""

    def __init__(self, codes: torch.Tensor, scales: torch.Tensor, tensor_scale: torch.Tensor,
                 rows: int, cols: int, sf_layout: int = SF_ROWMAJOR):
        self.codes, self.scales, self.tensor_scale = codes, scales, tensor_scale
        self.rows, self.cols, self.sf_layout = int(rows), int(cols), int(sf_layout)

    @classmethod
    def empty(cls, rows: int, cols: int, sf_layout: int = SF_ROWMAJOR, device="cuda") -> "NVFP4Tensor":
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
        scales = torch.zeros(nvfp4_scales_bytes(rows, cols, sf_layout), dtype=torch.uint8, device=device)
        ts = torch.zeros(1, dtype=torch.float32, device=device)
        return cls(codes, scales, ts, rows, cols, sf_layout)

    def c(self) -> _CTensor:
        return _CTensor(self.codes.data_ptr(), self.scales.data_ptr(), self.tensor_scale.data_ptr(),
                        self.rows, self.cols, self.sf_layout)

    def scales_rowmajor(self) -> torch.Tensor:
        """Block scales as a rows x cols/16 tensor (a view for ROWMAJOR; a gather for TILED)."""
        nb = self.cols // 16
        if self.sf_layout == SF_ROWMAJOR:
            return self.scales.view(self.rows, nb)
        r = torch.arange(self.rows, device=self.scales.device).view(-1, 1)
        b = torch.arange(nb, device=self.scales.device).view(1, -1)
        katoms = (nb + 3) // 4
        off = ((r // 128) * katoms + b // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (b % 4)
        return self.scales[off]


class Workspace:
    """Zero-filled device workspace reused across quantizer calls (nvfp4_workspace_size)."""

    def __init__(self, M: int, K: int, device="cuda"):
        self.nbytes = nvfp4_workspace_size(M, K)
        self.buf = torch.zeros(self.nbytes, dtype=torch.uint8, device=device)

    def ptr(self) -> int:
        return self.buf.data_ptr()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return NVFP4_BF16
    if t.dtype == torch.float32:
        return NVFP4_F32
    raise TypeError(f"unsupported input dtype {t.dtype}")


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check(status: int, where: str) -> None:
    if status != NVFP4_OK:
        raise NVFP4Error(status, where)


def _ldx(x: torch.Tensor) -> int:
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D row-major tensor")
    return x.stride(0)


def nvfp4_quantize(x: torch.Tensor, q: NVFP4Tensor, scale_in: Optional[torch.Tensor] = None,
                   workspace: Optional[Workspace] = None, dev_status: Optional[torch.Tensor] = None,
                   stream=None) -> None:
    lib = load_library()
    M, K = x.shape
    qc = q.c()
    ws_ptr, ws_n = (workspace.ptr(), workspace.nbytes) if workspace is not None else (None, 0)
    _check(lib.nvfp4_quantize(x.data_ptr(), _dtype_code(x), M, K, _ldx(x), _ptr(scale_in),
                              ctypes.byref(qc), ws_ptr, ws_n, _ptr(dev_status), _stream(stream)),
           "nvfp4_quantize")


def mx_scales_bytes(rows: int, cols: int, layout: int = SF_ROWMAJOR) -> int:
    """Bytes of an MXFP4 scale buffer (one E8M0 byte per 32 elements)."""
    return int(load_library().nvfp4_mx_scales_bytes(rows, cols, layout))


def nvfp4_mx_quantize(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
                      r_codes: Optional[torch.Tensor] = None, r_scales: Optional[torch.Tensor] = None,
                      dev_status: Optional[torch.Tensor] = None, stream=None,
                      sf_layout: int = SF_ROWMAJOR) -> None:
    """MXFP4: codes uint8 [M, K/2] (packed, row-major), scales uint8 (E8M0;
    M x K/32 row-major, or the TILED atom layout), and optionally the
    residue's codes and scales in the same layouts; all on the device."""
    lib = load_library()
    M, K = x.shape
    ns = mx_scales_bytes(M, K, sf_layout) if K % 32 == 0 else M * K // 32
    for t, n in ((codes, M * K // 2), (scales, ns), (r_codes, M * K // 2), (r_scales, ns)):
        if t is not None and (t.dtype != torch.uint8 or t.numel() != n or not t.is_contiguous()):
            raise ValueError("nvfp4_mx_quantize: output buffers must be contiguous uint8 of the MXFP4 sizes")
    _check(lib.nvfp4_mx_quantize(x.data_ptr(), _dtype_code(x), M, K, _ldx(x), codes.data_ptr(), scales.data_ptr(),
                                 _ptr(r_codes), _ptr(r_scales), sf_layout, _ptr(dev_status), _stream(stream)),
           "nvfp4_mx_quantize")


def _mx_gemm_checks(a_codes, a_scales, w_codes, w_scales, y, where, r_codes=None, r_scales=None):
    M, N, K = a_codes.shape[0], w_codes.shape[0], 2 * a_codes.shape[1]
    if w_codes.shape[1] * 2 != K or tuple(y.shape) != (M, N):
        raise ValueError(f"{where}: shapes do not match")
    ops = [(a_codes, M * K // 2), (w_codes, N * K // 2),
           (a_scales, mx_scales_bytes(M, K, SF_TILED)), (w_scales, mx_scales_bytes(N, K, SF_TILED))]
    if r_codes is not None:
        ops += [(r_codes, M * K // 2), (r_scales, mx_scales_bytes(M, K, SF_TILED))]
    for t, n in ops:
        if t.dtype != torch.uint8 or t.numel() != n or not t.is_contiguous():
            raise ValueError(f"{where}: operands must be contiguous uint8 of the MXFP4 sizes")
    return M, N, K


def nvfp4_mx_gemm(a_codes: torch.Tensor, a_scales: torch.Tensor, w_codes: torch.Tensor,
                  w_scales: torch.Tensor, y: torch.Tensor,
                  dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """MXFP4 linear y = deq(A) deq(W)^T: a_codes uint8 [M, K/2], w_codes uint8
    [N, K/2], both scale buffers in the TILED layout; y [M, N] fp32 or bf16."""
    lib = load_library()
    M, N, K = _mx_gemm_checks(a_codes, a_scales, w_codes, w_scales, y, "nvfp4_mx_gemm")
    _check(lib.nvfp4_mx_gemm(a_codes.data_ptr(), a_scales.data_ptr(), w_codes.data_ptr(), w_scales.data_ptr(),
                             M, N, K, y.data_ptr(), _out_dtype(y), _ldx(y), _ptr(dev_status), _stream(stream)),
           "nvfp4_mx_gemm")


def nvfp4_mx_gemm_residue(a_codes: torch.Tensor, a_scales: torch.Tensor, r_codes: torch.Tensor,
                          r_scales: torch.Tensor, w_codes: torch.Tensor, w_scales: torch.Tensor, y: torch.Tensor,
                          dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """MXFP4 compensated linear y = deq(A) deq(W)^T + deq(R) deq(W)^T (TILED scales)."""
    lib = load_library()
    if r_codes is None or r_scales is None:
        raise ValueError("nvfp4_mx_gemm_residue: the residue operand is required")
    M, N, K = _mx_gemm_checks(a_codes, a_scales, w_codes, w_scales, y, "nvfp4_mx_gemm_residue", r_codes, r_scales)
    _check(lib.nvfp4_mx_gemm_residue(a_codes.data_ptr(), a_scales.data_ptr(), r_codes.data_ptr(),
                                     r_scales.data_ptr(), w_codes.data_ptr(), w_scales.data_ptr(), M, N, K,
                                     y.data_ptr(), _out_dtype(y), _ldx(y), _ptr(dev_status), _stream(stream)),
           "nvfp4_mx_gemm_residue")


def nvfp4_quantize_residue(x: torch.Tensor, q: NVFP4Tensor, r: NVFP4Tensor,
                           scale_in: Optional[torch.Tensor] = None,
                           rscale_in: Optional[torch.Tensor] = None,
                           workspace: Optional[Workspace] = None,
                           dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    lib = load_library()
    M, K = x.shape
    qc, rc = q.c(), r.c()
    ws_ptr, ws_n = (workspace.ptr(), workspace.nbytes) if workspace is not None else (None, 0)
    _check(lib.nvfp4_quantize_residue(x.data_ptr(), _dtype_code(x), M, K, _ldx(x), _ptr(scale_in),
                                      _ptr(rscale_in), ctypes.byref(qc), ctypes.byref(rc), ws_ptr, ws_n,
                                      _ptr(dev_status), _stream(stream)),
           "nvfp4_quantize_residue")


def nvfp4_rmsnorm_reorder_quantize(x: torch.Tensor, x_aug: NVFP4Tensor,
                                   gamma: Optional[torch.Tensor] = None, eps: float = 1e-5,
                                   perm: Optional[torch.Tensor] = None, S: int = 0,
                                   scale_in: Optional[torch.Tensor] = None,
                                   workspace: Optional[Workspace] = None,
                                   dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    lib = load_library()
    M, K = x.shape
    if gamma is not None and gamma.dtype != x.dtype:
        raise TypeError("gamma must have the dtype of x")
    if perm is not None and perm.dtype != torch.int32:
        raise TypeError("perm must be int32")
    xc = x_aug.c()
    ws_ptr, ws_n = (workspace.ptr(), workspace.nbytes) if workspace is not None else (None, 0)
    _check(lib.nvfp4_rmsnorm_reorder_quantize(x.data_ptr(), _dtype_code(x), M, K, _ldx(x), _ptr(gamma),
                                              ctypes.c_float(eps), _ptr(perm), S, _ptr(scale_in),
                                              ctypes.byref(xc), ws_ptr, ws_n, _ptr(dev_status),
                                              _stream(stream)),
           "nvfp4_rmsnorm_reorder_quantize")


def nvfp4_quantize_weight(w: torch.Tensor, w_aug: NVFP4Tensor, sigma: Optional[torch.Tensor] = None,
                          perm: Optional[torch.Tensor] = None, S: int = 0,
                          scale_in: Optional[torch.Tensor] = None, workspace: Optional[Workspace] = None,
                          dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Offline weight preparation: w_aug = Q([W' | W'[:, :S]]), W'[:, j] = W[:, perm[j]] * sigma[perm[j]]."""
    lib = load_library()
    N, K = w.shape
    if sigma is not None and sigma.dtype != torch.float32:
        raise TypeError("sigma must be float32")
    if perm is not None and perm.dtype != torch.int32:
        raise TypeError("perm must be int32")
    wc = w_aug.c()
    ws_ptr, ws_n = (workspace.ptr(), workspace.nbytes) if workspace is not None else (None, 0)
    _check(lib.nvfp4_quantize_weight(w.data_ptr(), _dtype_code(w), N, K, _ldx(w), _ptr(sigma), _ptr(perm), S,
                                     _ptr(scale_in), ctypes.byref(wc), ws_ptr, ws_n, _ptr(dev_status),
                                     _stream(stream)),
           "nvfp4_quantize_weight")


def nvfp4_rmsnorm_reorder_quantize_noalloc(x: torch.Tensor, x_aug: NVFP4Tensor,
                                           gamma: Optional[torch.Tensor] = None, eps: float = 1e-5,
                                           perm: Optional[torch.Tensor] = None, S: int = 0,
                                           scale_in: Optional[torch.Tensor] = None,
                                           dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """As nvfp4_rmsnorm_reorder_quantize, with the library's built-in scratch
    instead of a caller workspace (for callers that cannot allocate)."""
    lib = load_library()
    M, K = x.shape
    xc = x_aug.c()
    _check(lib.nvfp4_rmsnorm_reorder_quantize_noalloc(x.data_ptr(), _dtype_code(x), M, K, _ldx(x), _ptr(gamma),
                                                      ctypes.c_float(eps), _ptr(perm), S, _ptr(scale_in),
                                                      ctypes.byref(xc), _ptr(dev_status), _stream(stream)),
           "nvfp4_rmsnorm_reorder_quantize_noalloc")


def _out_dtype(y: torch.Tensor) -> int:
    return _dtype_code(y)


def nvfp4_gemm(a: NVFP4Tensor, w: NVFP4Tensor, y: torch.Tensor,
               dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    lib = load_library()
    ac, wc = a.c(), w.c()
    _check(lib.nvfp4_gemm(ctypes.byref(ac), ctypes.byref(wc), y.data_ptr(), _out_dtype(y), _ldx(y),
                          _ptr(dev_status), _stream(stream)),
           "nvfp4_gemm")


def nvfp4_gemm_residue(a: NVFP4Tensor, r: NVFP4Tensor, w: NVFP4Tensor, y: torch.Tensor,
                       dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    lib = load_library()
    ac, rc, wc = a.c(), r.c(), w.c()
    _check(lib.nvfp4_gemm_residue(ctypes.byref(ac), ctypes.byref(rc), ctypes.byref(wc), y.data_ptr(),
                                  _out_dtype(y), _ldx(y), _ptr(dev_status), _stream(stream)),
           "nvfp4_gemm_residue")


def nvfp4_quantize_gemm(x: torch.Tensor, q: NVFP4Tensor, w: NVFP4Tensor, y: torch.Tensor,
                        scale_in: Optional[torch.Tensor] = None,
                        dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Decode linear with online activation quantization in one launch:
    q <- Q(x), y <- s_x s_w Q(x) W^T (M <= 16, W with TILED scales)."""
    lib = load_library()
    M, K = x.shape
    qc, wc = q.c(), w.c()
    _check(lib.nvfp4_quantize_gemm(x.data_ptr(), _dtype_code(x), M, K, _ldx(x), _ptr(scale_in),
                                   ctypes.byref(qc), ctypes.byref(wc), y.data_ptr(), _out_dtype(y), _ldx(y),
                                   _ptr(dev_status), _stream(stream)),
           "nvfp4_quantize_gemm")


def nvfp4_quantize_gemm_host(x_host: torch.Tensor, x_dev: torch.Tensor, q: NVFP4Tensor, w: NVFP4Tensor,
                             y_dev: torch.Tensor, y_host: torch.Tensor, scale_in: Optional[torch.Tensor] = None,
                             dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """nvfp4_quantize_gemm between host buffers: x_host (CPU, M x K, dense) is copied
    into x_dev, the decode linear runs on the device, y_dev is copied into y_host
    (CPU, M x N, dense); all on the stream.  Pinned host tensors keep it asynchronous."""
    lib = load_library()
    M, K = x_dev.shape
    N = w.rows
    if x_host.device.type != "cpu" or y_host.device.type != "cpu":
        raise ValueError("x_host and y_host must be CPU tensors")
    if tuple(x_host.shape) != (M, K) or x_host.dtype != x_dev.dtype or not x_host.is_contiguous():
        raise ValueError("x_host must be a dense M x K tensor of x_dev's dtype")
    if tuple(y_host.shape) != (M, N) or y_host.dtype != y_dev.dtype or not y_host.is_contiguous():
        raise ValueError("y_host must be a dense M x N tensor of y_dev's dtype")
    qc, wc = q.c(), w.c()
    _check(lib.nvfp4_quantize_gemm_host(x_host.data_ptr(), x_dev.data_ptr(), _dtype_code(x_dev), M, K,
                                        _ldx(x_dev), _ptr(scale_in), ctypes.byref(qc), ctypes.byref(wc),
                                        y_dev.data_ptr(), y_host.data_ptr(), _out_dtype(y_dev), _ldx(y_dev),
                                        _ptr(dev_status), _stream(stream)),
           "nvfp4_quantize_gemm_host")


def nvfp4_quantize_residue_gemm(x: torch.Tensor, q: NVFP4Tensor, r: Optional[NVFP4Tensor], w: NVFP4Tensor,
                                y: torch.Tensor, scale_in: Optional[torch.Tensor] = None,
                                rscale_in: Optional[torch.Tensor] = None,
                                dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """ResServe compensated decode linear in one launch: (q, r) <- Q(x), Q(x - deq Q(x));
    y <- s_x s_w Q(x) W^T + s_r s_w Q(r) W^T."""
    lib = load_library()
    M, K = x.shape
    qc, wc = q.c(), w.c()
    rc = r.c() if r is not None else None
    _check(lib.nvfp4_quantize_residue_gemm(x.data_ptr(), _dtype_code(x), M, K, _ldx(x), _ptr(scale_in),
                                           _ptr(rscale_in), ctypes.byref(qc),
                                           ctypes.byref(rc) if rc is not None else None, ctypes.byref(wc),
                                           y.data_ptr(), _out_dtype(y), _ldx(y), _ptr(dev_status),
                                           _stream(stream)),
           "nvfp4_quantize_residue_gemm")


def nvfp4_quantize_gemm_plan(M: int, N: int, K: int, x_dtype=torch.bfloat16, residue: bool = False,
                             out_dtype=torch.float32) -> int:
    """Kernel launches one nvfp4_quantize[_residue]_gemm call makes for these sizes
    (1 fused, 2 quantize-then-GEMM, 0 unsupported).  Host-only."""
    lib = load_library()
    code = lambda d: NVFP4_BF16 if d == torch.bfloat16 else NVFP4_F32
    return lib.nvfp4_quantize_gemm_plan(M, N, K, code(x_dtype), 1 if residue else 0, code(out_dtype))

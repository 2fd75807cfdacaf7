"""NVFP4 reference oracle -- TEST INFRASTRUCTURE ONLY.

Plain, slow and obviously-correct CPU definitions of what the NVFP4 hot path
computes.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import this module; the product package never does, and it
shares no code with the CUDA library.

The scalar encoders, the block quantizer and the RMSNorm live in
``nvfp4_oracle.c`` (plain C, IEEE round-to-nearest-even, no fused multiply-add);
this module composes them, numpy doing only array bookkeeping and the fp64
matrix product.

Page citations (page title, section):
  [RC]  "Replay the Curvature: Accurate and Scalable NVFP4 Quantization for
        Large Language Model Inference", abstract -- 16 E2M1 values share one
        E4M3 block scale.
  [ARC] ARCQuant blog post (zizhi168.cn), section 1 (format), section 3.1
        (augmented residual channel, two-stage quantization, X_aug of K+S
        columns, Y = Q(X)Q(W)^T + Q(R)Q(W_o)^T), section 3.2 (fused
        reorder + RMSNorm + main + residue quantizer), section 4 (error bounds).
  [RS]  "ResServe: Accurate and Efficient FP4 LLM Inference with Residue
        Compensation", abstract -- FP4 activation base plus FP4-quantized
        residue, both contributions combined on-chip.

Parity status: every function below is pinned by tests/test_oracle_*.py
(exhaustive code tables, library cross-checks, brute force, closed forms and
the pages' error bounds); the rounding of the residue stages (dequant_f32,
residue, mx_residue) by exact-rational recomputation in
tests/test_oracle_residue_rounding.py; the MXFP4 functions at the end by
tests/test_oracle_mx.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libnvfp4_oracle.so")
_lib = None
_lock = threading.Lock()

E2M1_MAX = 6.0
E4M3_MAX = 448.0


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, -O2, no fused multiply-add) in place."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
               "-fopenmp", _SRC, "-o", _LIB_PATH + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def _L():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u8p = ctypes.POINTER(ctypes.c_uint8)
            f32p = ctypes.POINTER(ctypes.c_float)
            f64p = ctypes.POINTER(ctypes.c_double)
            i64 = ctypes.c_int64
            lib.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
            lib.orc_e2m1_decode.restype = ctypes.c_double
            lib.orc_e2m1_encode.argtypes = [ctypes.c_float]
            lib.orc_e2m1_encode.restype = ctypes.c_uint8
            lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.orc_e4m3_decode.restype = ctypes.c_double
            lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
            lib.orc_e4m3_encode.restype = ctypes.c_uint8
            lib.orc_e2m1_encode_array.argtypes = [f32p, i64, u8p]
            lib.orc_e4m3_encode_array.argtypes = [f32p, i64, u8p]
            lib.orc_amax.argtypes = [f32p, i64, i64, i64]
            lib.orc_amax.restype = ctypes.c_float
            lib.orc_tensor_scale.argtypes = [ctypes.c_float]
            lib.orc_tensor_scale.restype = ctypes.c_float
            lib.orc_quantize.argtypes = [f32p, i64, i64, i64, ctypes.c_float, u8p, u8p]
            lib.orc_dequant_f32.argtypes = [u8p, u8p, ctypes.c_float, i64, i64, f32p]
            lib.orc_residue.argtypes = [f32p, i64, i64, i64, u8p, u8p, ctypes.c_float, f32p]
            lib.orc_rmsnorm.argtypes = [f32p, i64, i64, i64, f32p, ctypes.c_float, f32p, f32p]
            lib.orc_dequant_f64.argtypes = [u8p, u8p, ctypes.c_float, i64, i64, f64p]
            lib.orc_e8m0_decode.argtypes = [ctypes.c_uint8]
            lib.orc_e8m0_decode.restype = ctypes.c_double
            lib.orc_mx_scale_byte.argtypes = [ctypes.c_float]
            lib.orc_mx_scale_byte.restype = ctypes.c_uint8
            lib.orc_mx_quantize.argtypes = [f32p, i64, i64, i64, u8p, u8p]
            lib.orc_mx_dequant_f64.argtypes = [u8p, u8p, i64, i64, f64p]
            _lib = lib
    return _lib


def _p(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


# ----------------------------------------------------------------- scalars

def e2m1_decode(code: int) -> float:
    """[ARC] s1: E2M1 value of a 4-bit code (bit 3 = sign)."""
    return _L().orc_e2m1_decode(int(code) & 0xF)


def e2m1_encode(q: float) -> int:
    """[ARC] s1 round-to-nearest onto the E2M1 grid; ties to even, saturating at 6."""
    return _L().orc_e2m1_encode(float(q))


def e4m3_decode(b: int) -> float:
    """[RC] abstract: the E4M3 block-scale format (bias 7, max 448, 0x7F = NaN)."""
    return _L().orc_e4m3_decode(int(b) & 0xFF)


def e4m3_encode(x: float) -> int:
    """Round-to-nearest-even onto finite E4M3, saturating at 448."""
    return _L().orc_e4m3_encode(float(x))


def e2m1_encode_array(q) -> np.ndarray:
    q = _f32(q).ravel()
    out = np.empty(q.size, np.uint8)
    _L().orc_e2m1_encode_array(_p(q, ctypes.c_float), q.size, _p(out, ctypes.c_uint8))
    return out


def e4m3_encode_array(x) -> np.ndarray:
    x = _f32(x).ravel()
    out = np.empty(x.size, np.uint8)
    _L().orc_e4m3_encode_array(_p(x, ctypes.c_float), x.size, _p(out, ctypes.c_uint8))
    return out


def e4m3_decode_array(b) -> np.ndarray:
    table = np.array([e4m3_decode(i) for i in range(256)], dtype=np.float64)
    return table[np.asarray(b, dtype=np.uint8)]


def e2m1_decode_array(c) -> np.ndarray:
    table = np.array([e2m1_decode(i) for i in range(16)], dtype=np.float64)
    return table[np.asarray(c, dtype=np.uint8)]


# ---------------------------------------------------------- NVFP4 tensors

class QTensor:
    """An NVFP4 tensor: packed codes (rows x cols/2, element 2j in the low
    nibble), row-major E4M3 block scales (rows x cols/16), FP32 tensor scale."""

    __slots__ = ("codes", "scales", "s")

    def __init__(self, codes: np.ndarray, scales: np.ndarray, s: float):
        self.codes = codes
        self.scales = scales
        self.s = np.float32(s)

    @property
    def rows(self) -> int:
        return self.codes.shape[0]

    @property
    def cols(self) -> int:
        return self.codes.shape[1] * 2

    def unpacked_codes(self) -> np.ndarray:
        lo = self.codes & 0xF
        hi = self.codes >> 4
        return np.stack([lo, hi], axis=-1).reshape(self.rows, self.cols)


def amax(x) -> np.float32:
    x = _f32(x)
    return np.float32(_L().orc_amax(_p(x, ctypes.c_float), x.shape[0], x.shape[1], x.shape[1]))


def tensor_scale(amax_value) -> np.float32:
    """Per-tensor FP32 scale s = fl32(amax / (6 * 448)) (ARCQuant s3.1 s_aug)."""
    return np.float32(_L().orc_tensor_scale(float(np.float32(amax_value))))


def quantize(x, s=None) -> QTensor:
    """NVFP4-quantize a rows x cols fp32 matrix ([RC] abstract, [ARC] s1).

    s=None computes the per-tensor scale from amax(x) first."""
    x = _f32(x)
    rows, cols = x.shape
    assert cols % 16 == 0
    if s is None:
        s = tensor_scale(amax(x))
    s = np.float32(s)
    codes = np.empty((rows, cols // 2), np.uint8)
    scales = np.empty((rows, cols // 16), np.uint8)
    _L().orc_quantize(_p(x, ctypes.c_float), rows, cols, cols, float(s),
                      _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8))
    return QTensor(codes, scales, s)


def dequant_f32(q: QTensor) -> np.ndarray:
    """fp32 dequantization fl32(fl32(v * d) * s), as the residue stage uses it."""
    out = np.empty((q.rows, q.cols), np.float32)
    codes = np.ascontiguousarray(q.codes)
    scales = np.ascontiguousarray(q.scales)
    _L().orc_dequant_f32(_p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8), float(q.s),
                         q.rows, q.cols, _p(out, ctypes.c_float))
    return out


def dequant_f64(q: QTensor) -> np.ndarray:
    """Exact binary64 dequantization v(c) * d * s."""
    out = np.empty((q.rows, q.cols), np.float64)
    codes = np.ascontiguousarray(q.codes)
    scales = np.ascontiguousarray(q.scales)
    _L().orc_dequant_f64(_p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8), float(q.s),
                         q.rows, q.cols, _p(out, ctypes.c_double))
    return out


def residue(x, q: QTensor) -> np.ndarray:
    """R = X - deq(Q(X)) in fp32 ([RS] abstract: the information lost by quantization;
    [ARC] s3.1 residue stage)."""
    x = _f32(x)
    out = np.empty(x.shape, np.float32)
    codes = np.ascontiguousarray(q.codes)
    scales = np.ascontiguousarray(q.scales)
    _L().orc_residue(_p(x, ctypes.c_float), x.shape[0], x.shape[1], x.shape[1],
                     _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8), float(q.s),
                     _p(out, ctypes.c_float))
    return out


def quantize_residue(x, s=None, s_r=None):
    """ResServe-style full residue ([RS] abstract): Q(X) with its tensor scale,
    then R = X - deq(Q(X)) quantized to NVFP4 with its own tensor scale."""
    q = quantize(x, s)
    r = residue(x, q)
    qr = quantize(r, s_r)
    return q, qr


def rmsnorm(x, gamma=None, eps: float = 1e-5, return_rinv: bool = False):
    """Row RMSNorm of the fused quantizer ([ARC] s3.2); exact mean square, see C source."""
    x = _f32(x)
    rows, cols = x.shape
    y = np.empty((rows, cols), np.float32)
    rinv = np.empty(rows, np.float32)
    g = None if gamma is None else _f32(gamma)
    _L().orc_rmsnorm(_p(x, ctypes.c_float), rows, cols, cols,
                     None if g is None else _p(g, ctypes.c_float), ctypes.c_float(eps),
                     _p(y, ctypes.c_float), _p(rinv, ctypes.c_float))
    return (y, rinv) if return_rinv else y


def rmsnorm_reorder_quantize(x, gamma=None, eps: float = 1e-5, perm=None, S: int = 0, s=None):
    """ARCQuant fused quantizer ([ARC] s3.1-3.2).

    y = RMSNorm(x) * gamma, or y = x when gamma is None (no normalisation);
    y' = y[:, perm] (outlier channels first); s_aug = amax(y') / 2688 unless s is
    given; main stage quantizes all K columns of y'; the residue of the first S
    columns, R = y'[:, :S] - deq(Q(y'))[:, :S], is quantized under the same s_aug
    and appended as columns K..K+S-1 of X_aug."""
    x = _f32(x)
    rows, K = x.shape
    assert K % 16 == 0 and S % 16 == 0 and 0 <= S <= K
    y = rmsnorm(x, gamma, eps) if gamma is not None else x.copy()
    if perm is not None:
        y = np.ascontiguousarray(y[:, np.asarray(perm, dtype=np.int64)])
    if s is None:
        s = tensor_scale(amax(y))
    qm = quantize(y, s)
    codes = np.empty((rows, (K + S) // 2), np.uint8)
    scales = np.empty((rows, (K + S) // 16), np.uint8)
    codes[:, : K // 2] = qm.codes
    scales[:, : K // 16] = qm.scales
    if S:
        r = residue(y, qm)[:, :S]
        qr = quantize(r, s)
        codes[:, K // 2:] = qr.codes
        scales[:, K // 16:] = qr.scales
    return QTensor(codes, scales, s)


def augment_weight(w_fp32, perm, S: int, sigma=None):
    """W_aug = [W' | W'[:, :S]] with W' = W[:, perm] in fp32 ([ARC] s3.1 and s6.3:
    the weight uses the same channel order as the activation).  sigma: a
    per-channel smoothing vector absorbed as W diag(sigma) (OSFP4 page, abstract),
    W'[:, j] = fl32(W[:, perm[j]] * sigma[perm[j]])."""
    w = _f32(w_fp32)
    if sigma is not None:
        w = (w * _f32(sigma)[None, :]).astype(np.float32)   # one IEEE binary32 product per element
    wp = w[:, np.asarray(perm, dtype=np.int64)]
    return np.ascontiguousarray(np.concatenate([wp, wp[:, :S]], axis=1))


# --------------------------------------------------------------------- GEMM

def gemm(a: QTensor, w: QTensor, rows=None) -> np.ndarray:
    """Y = deq(A) deq(W)^T in binary64 ([ARC] s3.1 as one GEMM over K or K+S).

    rows: optional index array selecting output rows (for sampled checks)."""
    da = dequant_f64(a)
    if rows is not None:
        da = da[np.asarray(rows)]
    return da @ dequant_f64(w).T


def gemm_residue(a: QTensor, r: QTensor, w: QTensor, rows=None) -> np.ndarray:
    """Y = deq(Q(X)) deq(W)^T + deq(Q(R)) deq(W)^T ([RS] abstract)."""
    return gemm(a, w, rows) + gemm(r, w, rows)


# ------------------------------------------------------------------ MXFP4
# A NEXT row: 32-element blocks of E2M1 values under one E8M0 (power-of-two)
# scale and no tensor scale ([ARC] sections 2.2 and 4.2: MX formats use E8M0
# scales, step 2^1, and 32-element blocks).  Scale rule (a reading; the pages
# do not give one): the shared exponent floor(log2 amax_b) - 2, clamped to
# [-127, 127], with 2^-127 for an all-zero block; elements E2M1_RNE(x / scale),
# saturating at 6.  Pinned by tests/test_oracle_mx.py.

MX_BLOCK = 32


def e8m0_decode(b: int) -> float:
    """Value of an E8M0 byte: 2^(b - 127); 255 is NaN."""
    return _L().orc_e8m0_decode(int(b) & 0xFF)


def mx_scale_byte(amax: float) -> int:
    """E8M0 byte of a block whose largest magnitude is amax (the reading above)."""
    return _L().orc_mx_scale_byte(float(amax))


def mx_quantize(x):
    """MXFP4 quantization of an [M x K] array (K a multiple of 32).
    Returns (codes uint8 [M x K] unpacked, scales uint8 [M x K/32] E8M0)."""
    x = _f32(x)
    M, K = x.shape
    if K % MX_BLOCK:
        raise ValueError("K must be a multiple of 32")
    codes = np.empty((M, K), np.uint8)
    scales = np.empty((M, K // MX_BLOCK), np.uint8)
    _L().orc_mx_quantize(_p(x, ctypes.c_float), M, K, K, _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8))
    return codes, scales


def mx_dequant(codes, scales) -> np.ndarray:
    """Exact binary64 values v(code) * 2^(b - 127)."""
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    M, K = codes.shape
    out = np.empty((M, K), np.float64)
    _L().orc_mx_dequant_f64(_p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8), M, K,
                            _p(out, ctypes.c_double))
    return out


def mx_residue(x, qx) -> np.ndarray:
    """R = fl32(x - deq(Q(x))) in MXFP4 ([RS] abstract: what quantization lost).
    deq = v(code) * 2^(b - 127) is exact in binary32, so only the subtraction rounds."""
    x = _f32(x)
    return (x - mx_dequant(*qx).astype(np.float32)).astype(np.float32)


def mx_quantize_residue(x):
    """ResServe's residue in MXFP4 ([RS] abstract: FP4 base plus FP4 residue):
    R = fl32(x - deq(Q(x))), quantized with its own block scales.
    Returns ((codes, scales) of X, (codes, scales) of R)."""
    x = _f32(x)
    qx = mx_quantize(x)
    return qx, mx_quantize(mx_residue(x, qx))


def mx_gemm(qa, qw, qr=None) -> np.ndarray:
    """Y = deq(Q(A)) deq(Q(W))^T (+ deq(Q(R)) deq(Q(W))^T), in binary64."""
    wd = mx_dequant(*qw)
    y = mx_dequant(*qa) @ wd.T
    if qr is not None:
        y = y + mx_dequant(*qr) @ wd.T
    return y

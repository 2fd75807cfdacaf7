"""The C-ABI library loads and exports every function include/nvfp4.h declares;
host-side validation answers without touching a GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest
import torch

import nvfp4_block_scaled_18_b200 as nv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "nvfp4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from nvfp4_block_scaled_18_b200 import build
    build.build()
    return nv.load_library()


def test_exports_every_declared_symbol(lib):
    names = header_functions()
    assert len(names) >= 9
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(nv.EXPORTED_SYMBOLS)


def test_host_only_queries(lib):
    assert nv.nvfp4_version().startswith("nvfp4")
    assert nv.nvfp4_scales_bytes(4, 256, nv.SF_ROWMAJOR) == 64
    assert nv.nvfp4_scales_bytes(4, 256, nv.SF_TILED) == 4 * 512        # 1 row-atom x 4 k-atoms
    assert nv.nvfp4_scales_bytes(129, 80, nv.SF_TILED) == 2 * 2 * 512
    assert nv.nvfp4_workspace_size(1, 4096) >= 256
    assert nv.nvfp4_workspace_size(2048, 4096) >= 256 + 4 * 2048
    for code, name in nv.STATUS_NAMES.items():
        assert isinstance(nv.status_string(code), str) and nv.status_string(code)


def _tensor(rows, cols, codes=16, scales=16, ts=16, layout=0):
    return nv._CTensor(codes, scales, ts, rows, cols, layout)


def test_validation_before_launch(lib):
    # fake, never-dereferenced device addresses: validation must reject before any CUDA call
    good = 1 << 20
    q = _tensor(4, 64, good, good, good)
    f = lib.nvfp4_quantize
    assert f(None, 1, 4, 64, 64, good, ctypes.byref(q), None, 0, None, None) == 1      # null x
    assert f(good + 2, 1, 4, 64, 64, good, ctypes.byref(q), None, 0, None, None) == 2  # misaligned x
    assert f(good, 1, 4, 60, 64, good, ctypes.byref(q), None, 0, None, None) == 1      # K % 16
    assert f(good, 1, 4, 64, 68, good, ctypes.byref(q), None, 0, None, None) == 2      # ldx*2 % 16
    assert f(good, 7, 4, 64, 64, good, ctypes.byref(q), None, 0, None, None) == 1      # bad dtype
    bad_rows = _tensor(5, 64, good, good, good)
    assert f(good, 1, 4, 64, 64, good, ctypes.byref(bad_rows), None, 0, None, None) == 1
    assert f(good, 1, 4, 64, 64, None, ctypes.byref(q), None, 0, None, None) == 7      # no workspace
    xa = _tensor(4, 64 + 16, good, good, good)
    g = lib.nvfp4_rmsnorm_reorder_quantize
    assert g(good, 1, 4, 64, 64, None, ctypes.c_float(1e-5), None, 8, good, ctypes.byref(xa), None, 0,
             None, None) == 1                                                           # S % 16
    a, w = _tensor(4, 64, good, good, good), _tensor(32, 64, good, good, good)
    assert lib.nvfp4_gemm(ctypes.byref(a), ctypes.byref(w), None, 0, 32, None, None) == 1
    w_bad = _tensor(32, 128, good, good, good)
    assert lib.nvfp4_gemm(ctypes.byref(a), ctypes.byref(w_bad), good, 0, 32, None, None) == 1
    assert lib.nvfp4_gemm(ctypes.byref(a), ctypes.byref(w), good, 0, 30, None, None) == 1  # ldy < N
    a_tiled = _tensor(4, 64, good, good, good, layout=1)
    assert lib.nvfp4_gemm(ctypes.byref(a_tiled), ctypes.byref(w), good, 0, 32, None, None) == 3
    assert lib.nvfp4_gemm_residue(ctypes.byref(a), None, ctypes.byref(w), good, 0, 32, None, None) == 1


def test_fused_decode_validation_before_launch(lib):
    good = 1 << 20
    f = lib.nvfp4_quantize_residue_gemm
    g = lib.nvfp4_quantize_gemm

    def call(M=4, K=512, N=256, dt=1, wl=1, ql=1, x=good, y=good, r=True, ldx=None):
        q = _tensor(M, K, good, good, good, layout=ql)
        rr = _tensor(M, K, good, good, good, layout=ql)
        w = _tensor(N, K, good, good, good, layout=wl)
        return f(x, dt, M, K, K if ldx is None else ldx, None, None, ctypes.byref(q),
                 ctypes.byref(rr) if r else None, ctypes.byref(w), y, 0, N, None, None)

    assert call(x=None) == 1                      # null x
    assert call(y=None) == 1                      # null y
    assert call(x=good + 4) == 2                  # misaligned x
    assert call(M=17) == 3                        # decode sizes only
    assert call(wl=0) == 3                        # W must have TILED scales
    assert call(K=192) == 3                       # K >= 256
    assert call(K=320 + 16) == 3                  # K % 64
    assert call(M=16, K=65536) == 3               # beyond the one-launch quantizer
    assert call(M=16, K=32768, dt=0) == 3         # fp32: half the units
    q = _tensor(4, 512, good, good, good, layout=1)
    r_other = _tensor(4, 512, good, good, good, layout=0)
    w = _tensor(256, 512, good, good, good, layout=1)
    assert f(good, 1, 4, 512, 512, None, None, ctypes.byref(q), ctypes.byref(r_other), ctypes.byref(w), good,
             0, 256, None, None) == 3             # r layout differs from q
    w_bad = _tensor(256, 256, good, good, good, layout=1)
    assert g(good, 1, 4, 512, 512, None, ctypes.byref(q), ctypes.byref(w_bad), good, 0, 256, None, None) == 1
    assert g(good, 1, 4, 512, 512, None, None, ctypes.byref(w), good, 0, 256, None, None) == 1


def test_quantize_gemm_plan_rejects_without_device(lib):
    # unsupported sizes answer 0 before any CUDA call
    assert nv.nvfp4_quantize_gemm_plan(17, 4096, 4096) == 0
    assert nv.nvfp4_quantize_gemm_plan(4, 4096, 192) == 0
    assert nv.nvfp4_quantize_gemm_plan(4, 4096, 320 + 16) == 0
    assert nv.nvfp4_quantize_gemm_plan(16, 128, 65536) == 0
    assert nv.nvfp4_quantize_gemm_plan(16, 128, 32768, x_dtype=torch.float32) == 0


def test_mx_host_queries(lib):
    # one E8M0 byte per 32 elements; TILED atoms hold 128 rows x 4 blocks (K = 128)
    assert nv.mx_scales_bytes(4, 256, nv.SF_ROWMAJOR) == 4 * 8
    assert nv.mx_scales_bytes(4, 256, nv.SF_TILED) == 2 * 512
    assert nv.mx_scales_bytes(129, 160, nv.SF_TILED) == 2 * 2 * 512
    assert nv.mx_scales_bytes(0, 256, nv.SF_TILED) == 0


def test_mx_validation_before_launch(lib):
    good = 1 << 20
    q = lib.nvfp4_mx_quantize
    assert q(good, 1, 4, 48, 48, good, good, None, None, 0, None, None) == 1          # K % 32
    assert q(good, 1, 4, 64, 64, good, good, None, None, 5, None, None) == 1          # bad layout
    assert q(good, 1, 4, 64, 64, good, good, good, None, 0, None, None) == 1          # residue half given
    assert q(good, 1, 4, 64, 64, good + 8, good, None, None, 0, None, None) == 2      # misaligned codes
    assert q(good, 1, 4, 64, 64, None, good, None, None, 0, None, None) == 1          # no codes
    g = lib.nvfp4_mx_gemm
    assert g(None, good, good, good, 128, 256, 256, good, 0, 256, None, None) == 1    # null operand
    assert g(good, good, good, good, 128, 256, 192, good, 0, 256, None, None) == 3    # K % 128
    assert g(good, good, good, good, 128, 256, 128, good, 0, 256, None, None) == 3    # K < 256
    assert g(good, good, good, good, 128, 256, 256, good, 0, 200, None, None) == 1    # ldy < N
    assert g(good, good + 4, good, good, 128, 256, 256, good, 0, 256, None, None) == 2  # misaligned scales
    assert g(good, good, good, good, 128, 256, 256, good + 2, 0, 256, None, None) == 2  # misaligned fp32 y
    assert g(good, good, good, good, 128, 256, 256, good, 7, 256, None, None) == 1    # bad out dtype
    assert g(good, good, good, good, 0, 256, 256, good, 0, 256, None, None) == 1      # empty M


def test_mx_binding_checks_shapes(lib):
    ac = torch.zeros((128, 128), dtype=torch.uint8)
    wc = torch.zeros((256, 64), dtype=torch.uint8)                  # K mismatch
    s = torch.zeros(1024, dtype=torch.uint8)
    y = torch.zeros((128, 256))
    with pytest.raises(ValueError):
        nv.nvfp4_mx_gemm(ac, s, wc, s, y)
    with pytest.raises(ValueError):                                 # scales of the wrong size
        nv.nvfp4_mx_gemm(ac, s, torch.zeros((256, 128), dtype=torch.uint8), s, y)


def test_sizes_beyond_32_bits_rejected(lib):
    good = 1 << 20
    a, w = _tensor(4, 64, good, good, good), _tensor(1 << 31, 64, good, good, good)
    assert lib.nvfp4_gemm(ctypes.byref(a), ctypes.byref(w), good, 0, 1 << 31, None, None) == 3
    assert lib.nvfp4_quantize_gemm_plan(1, 1 << 31, 4096, 1, 0, 0) == 0
    assert lib.nvfp4_mx_gemm(good, good, good, good, 1 << 31, 256, 256, good, 0, 256, None, None) == 1


def test_mx_residue_validation_before_launch(lib):
    good = 1 << 20
    g = lib.nvfp4_mx_gemm_residue
    assert g(good, good, None, good, good, good, 128, 256, 256, good, 0, 256, None, None) == 1   # no residue
    assert g(good, good, good, None, good, good, 128, 256, 256, good, 0, 256, None, None) == 1
    assert g(good, good, good + 4, good, good, good, 128, 256, 256, good, 0, 256, None, None) == 2
    assert g(good, good, good, good, good, good, 128, 256, 192, good, 0, 256, None, None) == 3


def test_host_io_validation_before_copies(lib):
    """nvfp4_quantize_gemm_host checks every argument before it issues a copy."""
    good = 1 << 20
    q, w = _tensor(4, 1024, good, good, good), _tensor(512, 1024, good, good, good, layout=1)
    f = lib.nvfp4_quantize_gemm_host
    assert f(None, good, 1, 4, 1024, 1024, None, ctypes.byref(q), ctypes.byref(w), good, good, 0, 512,
             None, None) == 1                                                           # null x_host
    assert f(good, good, 1, 4, 1024, 1024, None, ctypes.byref(q), ctypes.byref(w), good, None, 0, 512,
             None, None) == 1                                                           # null y_host
    assert f(good, good + 2, 1, 4, 1024, 1024, None, ctypes.byref(q), ctypes.byref(w), good, good, 0, 512,
             None, None) == 2                                                           # misaligned x_dev
    assert f(good, good, 1, 4, 1024, 1024, None, ctypes.byref(q), ctypes.byref(w), good, good, 0, 256,
             None, None) == 1                                                           # ldy < N
    q17 = _tensor(17, 1024, good, good, good)
    assert f(good, good, 1, 17, 1024, 1024, None, ctypes.byref(q17), ctypes.byref(w), good, good, 0, 512,
             None, None) == 3                                                           # M > 16


def test_weight_residue_noalloc_validation_before_launch(lib):
    """nvfp4_quantize_weight, nvfp4_quantize_residue and the allocation-free fused
    quantizer reject bad arguments on the host, before any CUDA call."""
    good = 1 << 20
    N, K, S = 32, 256, 32
    wa = _tensor(N, K + S, good, good, good)
    f = lib.nvfp4_quantize_weight

    def weight(w=good, K=K, S=S, sigma=None, perm=good, t=wa, ws=good, dt=1):
        return f(w, dt, N, K, K, sigma, perm, S, None, ctypes.byref(t), ws, 1 << 20, None, None)

    assert weight(w=None) == 1                                    # null W
    assert weight(K=250) == 1                                     # K % 16
    assert weight(S=24) == 1                                      # S % 16
    assert weight(S=K + 16) == 1                                  # S > K
    assert weight(sigma=good + 2) == 2                            # misaligned sigma
    assert weight(perm=good + 2) == 2                             # misaligned perm
    assert weight(t=_tensor(N, K, good, good, good)) == 1         # W_aug must have K + S columns
    assert weight(ws=None) == 7                                   # computed scale needs a workspace
    assert weight(dt=9) == 1                                      # bad dtype

    M = 4
    q, r = _tensor(M, K, good, good, good), _tensor(M, K, good, good, good)
    g = lib.nvfp4_quantize_residue
    assert g(good, 1, M, K, K, None, None, ctypes.byref(q), None, good, 1 << 20, None, None) == 1   # no r
    r_bad = _tensor(M + 1, K, good, good, good)
    assert g(good, 1, M, K, K, None, None, ctypes.byref(q), ctypes.byref(r_bad), good, 1 << 20, None,
             None) == 1                                           # r of another shape
    assert g(good, 1, M, K, K, None, None, ctypes.byref(q), ctypes.byref(r), None, 0, None, None) == 7

    h = lib.nvfp4_rmsnorm_reorder_quantize_noalloc
    xa = _tensor(M, K + S, good, good, good)

    def noalloc(x=good, M=M, t=xa, gamma=None, eps=1e-5, ldx=K):
        return h(x, 1, M, K, ldx, gamma, ctypes.c_float(eps), None, S, None, ctypes.byref(t), None, None)

    big = _tensor(65537, K + S, good, good, good)
    assert noalloc(M=65537, t=big) == 7                           # beyond the built-in scratch
    assert noalloc(x=None) == 1
    assert noalloc(x=good + 8) == 2                               # x not 16-byte aligned
    assert noalloc(ldx=K + 4) == 2                                # row stride not 16-byte aligned
    assert noalloc(t=_tensor(M, K, good, good, good)) == 1        # X_aug must have K + S columns
    assert noalloc(gamma=good, eps=-1.0) == 1                     # negative eps

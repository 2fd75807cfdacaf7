"""Seeded synthetic inputs for the NVFP4 linear-layer workloads.

This module only draws random numbers and rounds them to the storage dtype; it
holds none of the quantization arithmetic, so both the CUDA path and the CPU
oracle take their inputs from here.

Recipes (numpy ``default_rng``; fp32 draws, cast to bf16 round-to-nearest-even
where bf16 is specified; outlier channels chosen with ``rng.choice(K, n,
replace=False)``):
  seed 0 activations, seed 1 calibration rows, seed 2 outlier channels,
  seed 3 weights, seed 4 RMSNorm gain.  The tiny case draws X then W from one
  ``default_rng(0)``.

Workload shapes follow the pages' problem statement (ARCQuant section 3: X of
N tokens x K channels, K -> K+S; ResServe abstract: few-row decode linears).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

SEED_X, SEED_CALIB, SEED_OUTLIER, SEED_W, SEED_GAMMA = 0, 1, 2, 3, 4


def to_bf16(x: np.ndarray) -> torch.Tensor:
    """fp32 -> bf16 with round-to-nearest-even (CPU torch tensor)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def bf16_values(x: np.ndarray) -> np.ndarray:
    """The fp32 values of the bf16 rounding of x."""
    return to_bf16(x).to(torch.float32).numpy()


def outlier_channels(K: int, frac: float, seed: int = SEED_OUTLIER) -> np.ndarray:
    n = int(round(frac * K))
    return np.sort(np.random.default_rng(seed).choice(K, n, replace=False))


def activations_normal(M: int, K: int, outlier_frac: float, outlier_gain: float,
                       seed: int = SEED_X, channels: Optional[np.ndarray] = None) -> np.ndarray:
    """fp32 N(0,1) rows with a fixed set of channels scaled by outlier_gain."""
    x = np.random.default_rng(seed).standard_normal((M, K), dtype=np.float32)
    ch = outlier_channels(K, outlier_frac) if channels is None else channels
    x[:, ch] *= np.float32(outlier_gain)
    return x


def activations_student_t(M: int, K: int, nu: float = 3.0, scale: float = 0.5,
                          seed: int = SEED_X) -> np.ndarray:
    """fp32 scale * Student-t(nu) values."""
    rng = np.random.default_rng(seed)
    return (np.float32(scale) * rng.standard_t(nu, size=(M, K))).astype(np.float32)


def weights_normal(N: int, K: int, std: float = 0.02, seed: int = SEED_W) -> np.ndarray:
    return np.random.default_rng(seed).normal(0.0, std, size=(N, K)).astype(np.float32)


def gamma_uniform(K: int, lo: float = 0.8, hi: float = 1.2, seed: int = SEED_GAMMA) -> np.ndarray:
    return np.random.default_rng(seed).uniform(lo, hi, size=K).astype(np.float32)


def calibrated_perm(calib: np.ndarray) -> np.ndarray:
    """Channel order by calibrated per-channel absolute maximum, largest first,
    ties by channel index (ARCQuant section 3.1: sort channels by absmax over
    calibration data, the first S are the outliers).  Offline input preparation."""
    absmax = np.abs(calib).max(axis=0)
    return np.argsort(-absmax, kind="stable").astype(np.int32)


# ------------------------------------------------------------------ configs

def tiny() -> Tuple[np.ndarray, np.ndarray]:
    """Tiny W4A4 linear: X 4x256 fp32 N(0,1) with channels 3 and 77 x40,
    W 256x256 N(0, 0.02); one rng(0) draws X then W."""
    rng = np.random.default_rng(0)
    x = rng.standard_normal((4, 256)).astype(np.float32)
    x[:, [3, 77]] *= np.float32(40.0)
    w = rng.normal(0.0, 0.02, size=(256, 256)).astype(np.float32)
    return x, w


DECODE_M = (1, 2, 4, 8, 16)
DECODE_SHAPES = ((4096, 4096), (14336, 4096), (4096, 14336))

RESSERVE_M = (1, 4, 16, 64)
RESSERVE_SHAPES = ((5120, 5120), (27648, 5120), (5120, 27648))

ARC_M, ARC_K, ARC_N = 2048, 4096, 11008
ARC_S = (128, 256, 512)

PREFILL_M = 8192
PREFILL_SHAPES = ((14336, 4096), (4096, 14336), (28672, 8192))


def decode_x(M: int, K: int) -> np.ndarray:
    """Decode activations: bf16 N(0,1), 1% of channels x50 (values as fp32)."""
    return bf16_values(activations_normal(M, K, 0.01, 50.0))


def resserve_x(M: int, K: int) -> np.ndarray:
    """ResServe decode activations: bf16 0.5 * Student-t(3) (values as fp32)."""
    return bf16_values(activations_student_t(M, K))


def arc_inputs(M: int = ARC_M, K: int = ARC_K, n_calib: int = 512):
    """ARCQuant prefill: X bf16 N(0,1) with 2% channels x30, gamma bf16 U(0.8,1.2),
    perm from n_calib calibration rows of the same distribution."""
    ch = outlier_channels(K, 0.02)
    x = bf16_values(activations_normal(M, K, 0.02, 30.0, SEED_X, ch))
    calib = activations_normal(n_calib, K, 0.02, 30.0, SEED_CALIB, ch)
    gamma = bf16_values(gamma_uniform(K))
    return x, gamma, calibrated_perm(calib)


def prefill_x(M: int, K: int) -> np.ndarray:
    """Large prefill activations: bf16 N(0,1), 1% channels x50."""
    return bf16_values(activations_normal(M, K, 0.01, 50.0))


def prefill_perm(K: int, n_calib: int = 512) -> np.ndarray:
    """Channel order for the large prefill's S-column extension, from n_calib
    calibration rows (seed 1) of the prefill distribution (same outlier channels)."""
    return calibrated_perm(activations_normal(n_calib, K, 0.01, 50.0, SEED_CALIB))

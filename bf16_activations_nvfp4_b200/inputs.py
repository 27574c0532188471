"""Seeded synthetic inputs for mm_bf16_fp4.

This module only draws random numbers; it holds none of the method's arithmetic (no
quantisation, no dequantisation, no matmul). Both the CUDA path and the CPU oracle are fed
from it.

Recipe (the decode shapes of PR #4038's performance tables, with the value distributions
this library is specified against):
  * activations A [m, k]: standard normal fp32, rounded to bf16 (round to nearest even);
    optionally 1% of the entries (Bernoulli mask) multiplied by 50 before the rounding;
  * weights W [n, k]: normal(0, 0.02) fp32; optionally each row j multiplied by a
    per-row factor drawn from U(0.5, 2).

Independent generators are keyed by (seed, stream id) so that row r of A is the same
for every m (needed for batch-invariance checks) and W does not depend on m.
"""
from __future__ import annotations

import numpy as np
import torch

_A_STREAM, _W_STREAM, _OUTLIER_STREAM, _JITTER_STREAM = 0, 1, 2, 3


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(stream)])


def activations_f32(m: int, k: int, seed: int = 0, outliers: bool = False) -> np.ndarray:
    """fp32 activations [m, k] before the bf16 rounding."""
    a = _rng(seed, _A_STREAM).standard_normal((m, k), dtype=np.float32)
    if outliers:
        mask = _rng(seed, _OUTLIER_STREAM).random((m, k)) < 0.01
        a = np.where(mask, a * np.float32(50.0), a).astype(np.float32)
    return a


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even (torch's CPU cast)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def activations(m: int, k: int, seed: int = 0, outliers: bool = False) -> np.ndarray:
    """bf16 activations [m, k] as uint16 bit patterns."""
    return to_bf16_bits(activations_f32(m, k, seed, outliers))


def weights(n: int, k: int, seed: int = 0, jitter: bool = False) -> np.ndarray:
    """fp32 weights [n, k] ~ N(0, 0.02), optionally with U(0.5, 2) per-row jitter."""
    w = _rng(seed, _W_STREAM).standard_normal((n, k), dtype=np.float32)
    w *= np.float32(0.02)
    if jitter:
        f = _rng(seed, _JITTER_STREAM).uniform(0.5, 2.0, n).astype(np.float32)
        w *= f[:, None]
    return w


# The workloads the library is specified and measured on (sizes m, n, k).
TINY = dict(m=1, n=512, k=2048)
SERVING_DECODE = [(2048, 7168), (4096, 4096), (4096, 14336), (14336, 4096), (10304, 2688)]
NARROW_N = [(n, k) for n in (512, 1024, 2048) for k in (2048, 4096)]
SMALL_BATCH_M = [1, 2, 4, 8, 16, 32]
SMALL_BATCH_NK = (4096, 14336)
LM_HEAD_NK = (152064, 5120)
LM_HEAD_M = [1, 64, 256]
# second workload: the Qwen3.6-27B-shaped decode GEMMs at m = 1 of PR #4038's table of them
# (fused gate/up 34816 x 5120, down 5120 x 17408, lm_head 248320 x 5120); synthetic weights
QWEN36_27B_DECODE = [(34816, 5120), (5120, 17408), (248320, 5120)]

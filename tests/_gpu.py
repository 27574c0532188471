"""Shared helpers for the GPU parity tests: seeded inputs on device, cached oracle packs."""
import functools

import numpy as np
import torch

import oracle
from bf16_activations_nvfp4_b200 import inputs

# Tolerance stated for the bf16 outputs: |out - ref| <= RTOL*|ref| + RRMS*rms(ref row).
RTOL = 1e-2
RRMS = 1e-2


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@functools.lru_cache(maxsize=16)
def weights(n: int, k: int, seed: int = 0, jitter: bool = False):
    """(W fp32 host, oracle pack (Wq, Ws, g)) for a seeded weight tensor."""
    W = inputs.weights(n, k, seed, jitter)
    return W, oracle.pack(W)


@functools.lru_cache(maxsize=16)
def device_weights(n: int, k: int, seed: int = 0, jitter: bool = False):
    """GPU-packed weights (Wq, Ws, g) on cuda for the same seeded tensor."""
    import bf16_activations_nvfp4_b200 as fi
    W, _ = weights(n, k, seed, jitter)
    return fi.pack_weights(torch.from_numpy(W).cuda())


def assert_within_tolerance(out_bits: np.ndarray, ref: np.ndarray, what: str = ""):
    out = bits_to_f64(out_bits)
    ok = oracle.within_tolerance(out, ref, RTOL, RRMS)
    if not ok.all():
        bad = np.argwhere(~ok)
        r, c = bad[0]
        raise AssertionError(f"{what}: {len(bad)} of {ok.size} outside tolerance; first at {tuple(bad[0])}: "
                             f"out={out[r, c]!r} ref={ref[r, c]!r}")

"""GPU weight packing (fi_nvfp4_pack_weights) is bit-exact with the oracle."""
import numpy as np
import pytest
import torch

import bf16_activations_nvfp4_b200 as fi
import oracle
from bf16_activations_nvfp4_b200 import inputs
from tests import _gpu

pytestmark = pytest.mark.gpu


def _gpu_pack(W: np.ndarray):
    Wq, Ws, g = fi.pack_weights(torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda())
    torch.cuda.synchronize()
    return Wq.cpu().numpy(), Ws.cpu().numpy(), g.cpu().numpy()[0]


def _assert_same(W):
    q, s, g = _gpu_pack(W)
    oq, os_, og = oracle.pack(W)
    assert np.float32(g).tobytes() == np.float32(og).tobytes()
    assert np.array_equal(s, os_), np.argwhere(s != os_)[:5]
    assert np.array_equal(q, oq), np.argwhere(q != oq)[:5]


@pytest.mark.parametrize("n,k,seed,jitter", [
    (512, 2048, 0, False),        # tiny correctness workload
    (37, 48, 1, False),           # ragged: n odd, k not a multiple of 32
    (1000, 2688, 2, True),        # scale rows only 8-byte aligned
    (2048, 7168, 0, False),
    (4096, 14336, 0, False),
    (14336, 4096, 0, False),
    (10304, 2688, 0, False),
])
def test_pack_bit_exact(n, k, seed, jitter):
    W, _ = _gpu.weights(n, k, seed, jitter)
    _assert_same(W)


@pytest.mark.slow
def test_pack_bit_exact_lm_head():
    W, _ = _gpu.weights(152064, 5120, 0, True)
    _assert_same(W)


def test_pack_special_values():
    """Exact E2M1 midpoints, saturation, signed zeros, zero blocks, tiny blocks whose
    scale underflows, and a block at exactly the tensor maximum."""
    rng = np.random.default_rng(5)
    W = inputs.weights(64, 256, seed=5)
    W[0, :16] = np.float32(5.25) * np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, 6, -0.25, -0.75,
                                             -1.25, -1.75, -2.5, -3.5, -5, -6], np.float32) / 6
    W[1, :16] = 0.0
    W[1, 16:32] = -0.0
    W[2, :16] = 1e-9  # scale underflows to 0 -> zero codes
    W[3, 0] = np.float32(np.abs(W).max() * 1.5)  # new tensor maximum
    W[4, :] = rng.choice([-1, 1], 256).astype(np.float32) * np.float32(1e-3)
    _assert_same(W)


def test_pack_exact_on_representable():
    """Representable weights (power-of-two global scale) come back unchanged."""
    E2M1 = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    rng = np.random.default_rng(6)
    n, k = 16, 128
    W = np.zeros((n, k), np.float32)
    for j in range(n):
        for b in range(k // 16):
            sf = float(torch.tensor([int(rng.integers(0x20, 0x7E))], dtype=torch.uint8)
                       .view(torch.float8_e4m3fn).float())
            vals = np.array([E2M1[i] for i in rng.integers(0, 8, 16)], np.float32)
            vals[0] = 6.0
            W[j, b * 16:(b + 1) * 16] = vals * rng.choice([-1, 1], 16) * sf * 2.0 ** -9
    W[0, :16] = np.float32(6 * 448 * 2.0 ** -9) * np.sign(W[0, :16] + 1e-30)
    q, s, g = _gpu_pack(W)
    assert g == np.float32(2.0 ** -9)
    assert np.array_equal(oracle.dequant(q, s, g), W.astype(np.float64))


def test_pack_empty():
    g = torch.full((1,), 7.0, device="cuda")
    W = torch.empty((0, 64), device="cuda")
    fi.pack_weights(W, out=(torch.empty((0, 32), dtype=torch.uint8, device="cuda"),
                            torch.empty((0, 4), dtype=torch.uint8, device="cuda"), g))
    assert g.item() == 0.0

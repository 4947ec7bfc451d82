"""Pins of the oracle's gated activation + 1x128 re-quantization.

The activation is checked against scipy's logistic function (a library
routine) and closed forms; the quantization half against the already pinned
row-wise quantizer, to which it reduces exactly when silu(g) is a power of two
and u is a bf16 value; the tile invariant (largest magnitude -> +-448) as for
every 1x128 tile.
"""

import math

import numpy as np
import pytest
import torch
from scipy.special import expit


def test_activation_is_gate_silu_times_up(oracle):
    rng = np.random.default_rng(7100 + 1)
    R, I = 5, 256
    G = rng.standard_normal((R, I)) * 6.0
    U = rng.standard_normal((R, I)) * 3.0
    h, _, _ = oracle.swiglu_quantize(G, U)
    want = G * expit(G) * U
    np.testing.assert_allclose(h, want, rtol=1e-14, atol=0)
    # the gate and up operands are not interchangeable
    h_swapped, _, _ = oracle.swiglu_quantize(U, G)
    assert np.max(np.abs(h_swapped - want)) > 1.0


def test_activation_closed_forms(oracle):
    I = 128
    G = np.zeros((1, I))
    U = np.ones((1, I))
    G[0, 1] = 1.0                    # silu(1) = 1 / (1 + 1/e)
    G[0, 2] = 50.0                   # 1 + exp(-50) == 1 in fp64: silu = g
    G[0, 3] = -800.0                 # exp(800) overflows: silu -> -0
    U[0, 4] = -7.0                   # g = 0: h = 0 whatever u is
    h, hq, sh = oracle.swiglu_quantize(G, U)
    assert h[0, 0] == 0.0 and h[0, 4] == 0.0
    assert h[0, 1] == 1.0 / (1.0 + math.exp(-1.0))
    assert h[0, 2] == 50.0
    assert h[0, 3] == 0.0
    assert sh[0, 0] == np.float32(50.0) / np.float32(448.0)
    assert hq[0, 2] == 0x7E          # the tile maximum maps to 448


def test_quantization_reduces_to_rowwise_quantizer(oracle):
    # silu(64) == 64 exactly in fp64 (exp(-64) < 2^-53), so h = 64 u is the bf16
    # value 64 u and its tiles must quantize exactly as the row-wise quantizer
    # quantizes that bf16 matrix (rows, blocks and the [I/128][R] scale layout).
    rng = np.random.default_rng(7100 + 2)
    R, I = 3, 384
    u32 = torch.from_numpy(rng.standard_normal((R, I)).astype(np.float32)).to(torch.bfloat16)
    u32[1, 128:256] = 0.0            # an all-zero tile: scale 1
    U = u32.to(torch.float64).numpy()
    G = np.full((R, I), 64.0)
    h, hq, sh = oracle.swiglu_quantize(G, U)
    np.testing.assert_array_equal(h, 64.0 * U)
    x_bits = (u32.to(torch.float32) * 64.0).to(torch.bfloat16).view(torch.int16).numpy()
    ref = oracle.quantize_act(x_bits.view(np.uint16), None, 1)
    np.testing.assert_array_equal(hq, ref["xq"])
    np.testing.assert_array_equal(sh.view(np.uint32), ref["sa"].view(np.uint32))
    assert sh[1, 1] == 1.0 and not hq[1, 128:256].any()


@pytest.mark.parametrize("seed", [3, 4])
def test_every_tile_maximum_maps_to_448(oracle, seed):
    rng = np.random.default_rng(7100 + seed)
    R, I = 7, 512
    G = rng.standard_normal((R, I)) * 4.0
    U = rng.standard_normal((R, I))
    h, hq, sh = oracle.swiglu_quantize(G, U)
    dq = oracle.e4m3_decode_table()
    for r in range(R):
        for c in range(I // 128):
            t = h[r, 128 * c:128 * (c + 1)].astype(np.float32)
            j = int(np.argmax(np.abs(t)))
            assert abs(dq[hq[r, 128 * c + j]]) == 448.0
            assert sh[c, r] == np.float32(np.abs(t).max()) / np.float32(448.0)
            # dequantized values within half an E4M3 step (relative 2^-4) or
            # half the subnormal step 2^-10 in scaled units
            deq = dq[hq[r, 128 * c:128 * (c + 1)]] * np.float64(sh[c, r])
            lim = np.maximum(2.0 ** -4 * np.abs(t), 2.0 ** -10 * np.float64(sh[c, r]))
            assert np.all(np.abs(deq - t) <= lim * (1 + 1e-12))

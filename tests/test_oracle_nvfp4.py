"""Pins for the oracle's NVFP4 quantizer.

The pages print one number about the format: about 4.5 bits per value and 3.6x
fewer bits than BF16 (aicoder.com 'Background'; goldendata.cloud 'Signal 02').
The rest is pinned by closed forms, invariants and brute force.
"""
import json
import os

import numpy as np
import pytest

from precision_moe_numerics_quantize_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _x(rows, cols, seed=0, std=1.0):
    return synth.bf16_bits_to_f32(synth.rows_np(seed, synth.TAG_X, 0, rows, cols, std))


def test_storage_cost_matches_pages(orc):
    rows, cols = 64, 256
    codes, scales, ts = orc.nvfp4_quantize(_x(rows, cols))
    bits = (codes.nbytes + scales.nbytes) * 8
    bpv = bits / (rows * cols)
    assert bpv == GOLD["nvfp4_bits_per_value"]["value"]
    assert round(16 / bpv, 1) == GOLD["nvfp4_fewer_bits_than_bf16"]["value"]


def test_hand_worked_block(orc):
    # amax 6 -> S_enc = 2688/6 = 448, block scale RNE(1 * 448) = 448 (E4M3 0x7E),
    # element encode factor 448/448 = 1: the codes are the grid points themselves.
    x = np.array([[6, -4, 3, -2, 1.5, 1, 0.5, 0, -0.5, -1, -1.5, 2, -3, 4, -6, 0.25]], np.float32)
    codes, scales, ts = orc.nvfp4_quantize(x)
    assert scales[0, 0] == 0x7E
    assert ts == np.float32(6.0 / 2688.0)
    nib = np.stack([codes[0] & 15, codes[0] >> 4], axis=1).ravel()
    assert list(nib) == [7, 14, 5, 12, 3, 2, 1, 0, 9, 10, 11, 4, 13, 6, 15, 0]
    deq = orc.nvfp4_dequantize(codes, scales, ts, 1, 16)
    # exact values times 448 * ts = 448 * 6/2688 = 1 up to one fp32 rounding of ts
    assert np.allclose(deq[0, :15], x[0, :15], rtol=1e-6, atol=0)


def test_zero_tensor(orc):
    codes, scales, ts = orc.nvfp4_quantize(np.zeros((2, 32), np.float32))
    assert ts == 1.0 and not codes.any() and not scales.any()


def test_on_grid_roundtrip_is_exact(orc):
    """Values that are a grid point times a power-of-two block scale, with the
    tensor amax fixed so that S_enc is a power of two, come back exactly."""
    rng = np.random.default_rng(3)
    rows, cols = 8, 64
    nib = rng.integers(0, 16, (rows, cols))
    mag = E2M1[nib & 7] * np.where(nib & 8, -1, 1)
    mag[:, ::16] = 6.0  # every block holds a 6 so its scale is its own amax / 6
    pw = 2.0 ** rng.integers(-6, 5, (rows, cols // 16))
    x = (mag * np.repeat(pw, 16, axis=1)).astype(np.float32)
    amax = np.float32(2688.0 * 2.0 ** -4)  # S_enc = 16: every block scale 16 * pw is exact in E4M3
    codes, scales, ts = orc.nvfp4_quantize(x, amax_in=amax)
    deq = orc.nvfp4_dequantize(codes, scales, ts, rows, cols)
    assert np.array_equal(deq, x)


def test_nearest_code_and_scale_bound(orc):
    """Each element's code is the nearest grid point to x * S_enc / s_b (ties
    even), and amax_b <= 6 * s_b / S_enc * (1 + 2^-4) unless the scale saturated
    at 448 or flushed to zero."""
    rows, cols = 32, 512
    x = _x(rows, cols, seed=4) * np.float32(3.0)
    x[3, 17] = 250.0
    codes, scales, ts = orc.nvfp4_quantize(x)
    amax = np.abs(x).max()
    S_enc = np.float32(np.float32(2688.0) / amax)
    sf = np.array([[orc.e4m3_decode(s) for s in r] for r in scales])
    nib = np.stack([codes & 15, codes >> 4], axis=2).reshape(rows, cols)
    for r in range(rows):
        for b in range(cols // 16):
            blk = x[r, b * 16:(b + 1) * 16].astype(np.float64)
            s = sf[r, b]
            if s == 0:
                assert not nib[r, b * 16:(b + 1) * 16].any()
                continue
            enc = np.float32(S_enc / np.float32(s))
            v = np.abs((blk.astype(np.float32) * enc).astype(np.float64))
            d = np.abs(v[:, None] - E2M1[None, :])
            got = nib[r, b * 16:(b + 1) * 16] & 7
            assert np.all(d[np.arange(16), got] == d.min(axis=1))
            amax_b = np.abs(blk).max()
            if s < 448:
                assert amax_b <= 6 * s / S_enc * (1 + 2 ** -4) * (1 + 1e-6)


def test_power_of_two_scale_invariance(orc):
    x = _x(16, 128, seed=5)
    c0, s0, t0 = orc.nvfp4_quantize(x)
    c1, s1, t1 = orc.nvfp4_quantize(x * np.float32(2.0 ** 7))
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1)
    assert t1 == t0 * np.float32(2.0 ** 7)


def test_error_bound(orc):
    """|x - x_hat| is at most half a grid step of the block (0.5 * s_b * ts for
    the finest step ... 1 * s_b * ts for the coarsest) plus the clipping of a
    saturated block."""
    x = _x(64, 256, seed=6)
    codes, scales, ts = orc.nvfp4_quantize(x)
    deq = orc.nvfp4_dequantize(codes, scales, ts, 64, 256)
    sf = np.array([[orc.e4m3_decode(s) for s in r] for r in scales])
    step = np.repeat(sf, 16, axis=1) * float(ts)
    err = np.abs(deq.astype(np.float64) - x)
    amax_b = np.repeat(np.abs(x).reshape(64, 16, 16).max(axis=2), 16, axis=1)
    clip = np.maximum(amax_b - 6 * step, 0)
    assert np.all(err <= 1.0 * step * (1 + 1e-6) + clip + 1e-30)

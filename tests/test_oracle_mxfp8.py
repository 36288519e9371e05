"""Pins for the oracle's MXFP8 quantizer and its Philox4x32-10 stream.

The pages tie stochastic rounding to the MXFP8 backward pass (news.t0001.com
'训练数值格式分工清单'; aicoder.com 'Key Takeaways'). Pins: Philox known-answer
vectors, torch's float8_e4m3fn conversion (round-to-nearest mode), the scale
definition, exact unbiasedness of stochastic rounding over 10^6 draws, and
layout identities.
"""
import os

import numpy as np
import torch

from precision_moe_numerics_quantize_b200 import synth

KAT = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def test_philox_known_answers(orc):
    n = 0
    for line in open(KAT):
        if line.startswith("#") or not line.strip():
            continue
        v = [int(t, 16) for t in line.split()]
        assert orc.philox4x32_10(v[:4], v[4:6]).tolist() == v[6:]
        n += 1
    assert n == 3


def test_philox_uniformity(orc):
    words = np.array([orc.philox_word(7, 3, i) for i in range(40000)], dtype=np.uint64)
    hist = np.bincount((words >> 28).astype(np.int64), minlength=16)
    chi2 = ((hist - 2500.0) ** 2 / 2500.0).sum()
    assert chi2 < 37.7  # 15 degrees of freedom, p = 0.001
    assert len(np.unique(words)) > 39990


def _x(rows, cols, seed, std=1.0):
    return synth.bf16_bits_to_f32(synth.rows_np(seed, synth.TAG_DY, 0, rows, cols, std))


def test_scale_is_smallest_unclipped_power_of_two(orc):
    x = _x(16, 256, 1) * np.float32(3e-3)
    x[2, 5] = 448.0 * 2 ** -10
    x[5, 40] = 0.0
    x[7, 64:96] = 0.0
    codes, scales = orc.mxfp8_quantize(x, axis=0)
    for r in range(16):
        for b in range(8):
            amax = np.abs(x[r, b * 32:(b + 1) * 32]).max()
            k = int(scales[r, b]) - 127
            assert amax <= 448.0 * 2.0 ** k
            assert k == -127 or amax > 448.0 * 2.0 ** (k - 1)
    assert scales[7, 2] == 0  # all-zero block -> k = -127


def test_rne_mode_matches_torch(orc):
    x = _x(32, 256, 2) * np.float32(0.05)
    codes, scales = orc.mxfp8_quantize(x, axis=0, rounding=0)
    k = np.repeat(scales.astype(np.int64) - 127, 32, axis=1)
    v = (x.astype(np.float64) * 2.0 ** (-k)).astype(np.float32)  # exact
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)


def test_storage_cost(orc):
    codes, scales = orc.mxfp8_quantize(_x(4, 256, 3), axis=0)
    assert (codes.nbytes + scales.nbytes) * 8 / (4 * 256) == 8.25


def test_stochastic_rounding_is_unbiased(orc):
    """Over 31 test values x 32768 draws (about 10^6), the mean of the rounded
    values equals the input within 4 standard errors of the Bernoulli draw."""
    vals = np.array([0.3, 1.1, 3.3, 7.9, 13.0, 100.5, 300.0, 431.0, 447.0, 2.0 ** -8, 3 * 2.0 ** -10,
                     0.0171, 5.55, 1.0001, 0.999, 250.7, 60.1, 19.3, 0.7, 0.07, 2.2, 9.9, 33.3,
                     77.7, 123.4, 222.2, 333.3, 401.0, 6.75, 0.5625, 0.2], np.float64)
    n = 32768
    row = np.concatenate([[448.0], vals]).astype(np.float32)  # 448 fixes k = 0
    x = np.tile(row, (n, 1))
    x[1::2, 1:] *= -1  # half of the draws on negative values
    codes, scales = orc.mxfp8_quantize(x, axis=0, seed=12345, offset=9, rounding=1)
    assert np.all(scales == 127)
    deq = orc.mxfp8_dequantize(codes, scales).astype(np.float64)
    est = np.abs(deq[:, 1:]).mean(axis=0)
    for j, v in enumerate(row[1:].astype(np.float64)):
        lo = max([g for g in _e4m3_grid() if g <= v])
        hi = min([g for g in _e4m3_grid() if g >= v])
        if hi == lo:
            assert est[j] == v
            continue
        p = (v - lo) / (hi - lo)
        se = (hi - lo) * np.sqrt(p * (1 - p) / n)
        assert abs(est[j] - v) <= 4 * se + 1e-12, (v, est[j], se)


def _e4m3_grid():
    return sorted({abs(float(t)) for t in torch.arange(127, dtype=torch.uint8)
                   .view(torch.float8_e4m3fn).float().numpy()})


def test_stochastic_rounding_determinism_and_neighbours(orc):
    x = _x(8, 128, 4) * np.float32(0.01)
    a = orc.mxfp8_quantize(x, seed=7, offset=0, rounding=1)
    b = orc.mxfp8_quantize(x, seed=7, offset=0, rounding=1)
    c = orc.mxfp8_quantize(x, seed=8, offset=0, rounding=1)
    r = orc.mxfp8_quantize(x, rounding=0)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert not np.array_equal(a[0], c[0])
    assert np.array_equal(a[1], r[1])  # the scale does not depend on rounding
    # SR results are one of the two E4M3 neighbours of the scaled value
    k = np.repeat(a[1].astype(np.int64) - 127, 32, axis=1)
    v = np.abs(x.astype(np.float64) * 2.0 ** (-k))
    g = np.array(_e4m3_grid())
    got = np.abs(orc.mxfp8_dequantize(a[0], a[1]).astype(np.float64) * 2.0 ** (-k))
    lo = g[np.searchsorted(g, v, side="right") - 1]
    hi = g[np.minimum(np.searchsorted(g, v, side="left"), len(g) - 1)]
    assert np.all((got == lo) | (got == hi))


def test_axis1_is_axis0_of_transpose(orc):
    x = _x(64, 96, 5)
    c1, s1 = orc.mxfp8_quantize(x, axis=1, rounding=0)
    c0, s0 = orc.mxfp8_quantize(np.ascontiguousarray(x.T), axis=0, rounding=0)
    assert np.array_equal(c1, c0) and np.array_equal(s1, s0)


def test_axis1_segments_pad_with_zeros(orc):
    x = _x(70, 64, 6)
    seg = np.array([0, 20, 20, 70], np.int32)  # includes an empty segment
    c, s = orc.mxfp8_quantize(x, axis=1, seg_off=seg, rounding=0)
    assert c.shape == (64, 32 + 0 + 64)
    assert not c[:, 20:32].any() and not c[:, 32 + 50:].any()
    # first segment alone, padded to 32 rows of zeros
    xa = np.zeros((32, 64), np.float32)
    xa[:20] = x[:20]
    ca, sa = orc.mxfp8_quantize(xa, axis=1, rounding=0)
    assert np.array_equal(c[:, :32], ca) and np.array_equal(s[:, :1], sa)


def test_row_offset_keeps_the_source_element_index(orc):
    """A slice of rows quantized with row0 = its first row's index gives the
    whole tensor's codes for those rows, and each stochastic decision follows
    the Philox word of the element's row-major index in the whole tensor."""
    rows, cols, r0, r1 = 96, 64, 32, 80
    x = _x(rows, cols, 8) * np.float32(0.05)
    full = orc.mxfp8_quantize(x, seed=7, offset=2, rounding=1)
    part = orc.mxfp8_quantize(x[r0:r1], seed=7, offset=2, rounding=1, row0=r0)
    assert np.array_equal(part[0], full[0][r0:r1]) and np.array_equal(part[1], full[1][r0:r1])
    # axis 1: the 32-row blocks of rows 32..95 are columns 32..95 of the whole
    full1 = orc.mxfp8_quantize(x, axis=1, seed=7, offset=3, rounding=1)
    part1 = orc.mxfp8_quantize(x[32:96], axis=1, seed=7, offset=3, rounding=1, row0=32)
    assert np.array_equal(part1[0], full1[0][:, 32:96])
    # explicit decisions: round up iff (word >> 8) * 2^-24 < the fraction of
    # the way from the lower E4M3 neighbour to the upper one
    k = np.repeat(part[1].astype(np.int64) - 127, 32, axis=1)
    v = np.abs(x[r0:r1].astype(np.float64) * 2.0 ** (-k))
    g = np.array(_e4m3_grid())
    lo = g[np.searchsorted(g, v, side="right") - 1]
    hi = g[np.minimum(np.searchsorted(g, v, side="left"), len(g) - 1)]
    got = np.abs(orc.mxfp8_dequantize(part[0], part[1]).astype(np.float64) * 2.0 ** (-k))
    for r in range(r1 - r0):
        for c in range(cols):
            if lo[r, c] == hi[r, c]:
                continue
            wd = orc.philox_word(7, 2, (r0 + r) * cols + c)
            up = (wd >> 8) * 2.0 ** -24 < (v[r, c] - lo[r, c]) / (hi[r, c] - lo[r, c])
            assert got[r, c] == (hi[r, c] if up else lo[r, c]), (r, c)

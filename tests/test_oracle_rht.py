"""Pins for the oracle's 32-point random Hadamard transform and the quantized
combine payload (aicoder.com 'Key Takeaways' and 'Architecture highlights':
a 32-dimensional random Hadamard transform before the combine traffic is
quantized into a block-scaled format).

Pins: scipy's Sylvester Hadamard matrix (library), H32 H32^T = 32 I in
integers, the exact fp64 round trip, Parseval, and the fp32 evaluation within
its rounding bound.
"""
import json
import os

import numpy as np
import scipy.linalg

from precision_moe_numerics_quantize_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))


def _matrix(orc, signs, inverse=False):
    eye = np.eye(32)
    return np.stack([orc.rht32_f64(eye[i], signs, inverse) for i in range(32)], axis=1)


def test_dimension_from_pages():
    assert GOLD["rht_dimension"]["value"] == 32


def test_transform_is_scaled_sylvester_hadamard(orc):
    M = _matrix(orc, 0)
    H = np.rint(M * np.sqrt(32.0)).astype(np.int64)
    assert np.array_equal(H, scipy.linalg.hadamard(32))
    assert np.array_equal(H @ H.T, 32 * np.eye(32, dtype=np.int64))
    assert np.abs(M * np.sqrt(32.0) - H).max() < 1e-14


def test_signs_and_diagonal(orc):
    s = orc.rht_signs(11)
    D = np.diag([-1.0 if (s >> i) & 1 else 1.0 for i in range(32)])
    M = _matrix(orc, s)
    assert np.allclose(M, scipy.linalg.hadamard(32) @ D / np.sqrt(32.0), atol=1e-15)
    # the signs are word 0 of Philox4x32-10(key = seed, counter = 0): the first
    # known-answer vector (key 0, counter 0) gives 0x6627e8d5
    assert orc.rht_signs(0) == 0x6627E8D5


def test_fp64_roundtrip_and_parseval(orc):
    rng = np.random.default_rng(0)
    s = orc.rht_signs(11)
    for _ in range(50):
        x = rng.standard_normal(32) * 10.0 ** rng.uniform(-3, 3)
        v = orc.rht32_f64(x, s)
        y = orc.rht32_f64(v, s, inverse=True)
        assert np.abs(y - x).max() <= 1e-15 * np.abs(x).max() * 32
        assert abs(np.linalg.norm(v) - np.linalg.norm(x)) <= 1e-14 * np.linalg.norm(x)


def test_fp32_forward_within_rounding_bound(orc):
    s = orc.rht_signs(3)
    x = synth.bf16_bits_to_f32(synth.payload_rows_np(5, 0, 64, 32, np.array([3, 17])))
    for row in x:
        v32 = orc.rht32_forward_f32(row, s).astype(np.float64)
        v64 = orc.rht32_f64(row.astype(np.float64), s)
        assert np.abs(v32 - v64).max() <= 7 * 2.0 ** -24 * np.abs(row).sum()
        back = orc.rht32_inverse_f32(v32.astype(np.float32), s).astype(np.float64)
        assert np.abs(back - row).max() <= 14 * 2.0 ** -24 * np.abs(row).sum()


def test_payload_roundtrip_error_is_the_quantization_error(orc):
    """The transform is orthonormal, so the round-trip error measured on x equals
    the quantization error measured on the transformed values v (Parseval), up
    to fp32 rounding. Checked for the NVFP4 and the MXFP8 payload."""
    chans = synth.outlier_channels(5, 256, 4)
    x = synth.bf16_bits_to_f32(synth.payload_rows_np(5, 0, 64, 256, chans))
    s = orc.rht_signs(11)
    v = np.stack([np.concatenate([orc.rht32_forward_f32(r[b * 32:(b + 1) * 32], s)
                                  for b in range(8)]) for r in x]).astype(np.float64)
    for fmt in (0, 1):
        c, sc, ts = orc.rht32_quantize(x, 11, fmt)
        back = orc.rht32_dequantize(c, sc, ts, 64, 256, 11, fmt).astype(np.float64)
        if fmt == 0:
            vhat = orc.nvfp4_dequantize(c, sc, ts, 64, 256).astype(np.float64)
        else:
            vhat = orc.mxfp8_dequantize(c, sc).astype(np.float64)
        ex = np.sqrt(np.sum((back - x) ** 2, axis=1))
        ev = np.sqrt(np.sum((vhat - v) ** 2, axis=1))
        assert np.all(np.abs(ex - ev) <= 1e-5 * np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=1)))


def test_nvfp4_payload_amax_is_over_transformed_values(orc):
    x = synth.bf16_bits_to_f32(synth.payload_rows_np(5, 0, 8, 64, np.array([1])))
    s = orc.rht_signs(11)
    v = np.concatenate([np.concatenate([orc.rht32_forward_f32(r[b * 32:(b + 1) * 32], s)
                                        for b in range(2)]) for r in x]).reshape(8, 64)
    c, sc, ts = orc.rht32_quantize(x, 11, 0)
    assert ts == np.float32(np.float32(np.abs(v).max()) / np.float32(2688.0))
    c2, sc2, ts2 = orc.nvfp4_quantize(v)
    assert np.array_equal(c, c2) and np.array_equal(sc, sc2)


# -- combine straight from the quantized payload --------------------------------

E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]  # the E2M1 grid, from the format


def _decode_payload(codes, scales, ts, fmt, d):
    """Dequantized payload rows in fp64, written out from the format
    definitions (E2M1 grid above, E4M3 through torch's float8_e4m3fn, E8M0 as
    a power of two), independent of the oracle's decoders."""
    import torch
    rows = codes.shape[0]
    if fmt == 0:
        lo, hi = codes & 15, codes >> 4
        nib = np.stack([lo, hi], axis=2).reshape(rows, d)
        mag = np.array(E2M1_VALUES)[nib & 7]
        val = np.where(nib & 8, -mag, mag)
        sf = torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
        return val * np.repeat(sf, 16, axis=1) * float(ts)
    e4 = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return e4 * np.repeat(np.exp2(scales.astype(np.float64) - 127.0), 32, axis=1)


def _combine_case(orc, fmt, T=6, k=3, d=128, seed=3):
    R = T * k
    x = synth.bf16_bits_to_f32(synth.payload_rows_np(seed, 0, R, d, synth.outlier_channels(seed, d, 2)))
    codes, scales, ts = orc.rht32_quantize(x, 11, fmt)
    rng = np.random.default_rng(seed)
    pos = rng.permutation(R).astype(np.int32).reshape(T, k)
    w = rng.random((T, k))
    w /= w.sum(axis=1, keepdims=True)
    return codes, scales, ts, pos, w


def test_combine_rht_equals_explicit_hadamard_arithmetic(orc):
    """oracle_combine_rht = s * (H32 @ sum_j w_j v_j) / sqrt(32) per 32-block,
    with H32 from scipy and the payload decoded from the format definitions."""
    import torch
    H = scipy.linalg.hadamard(32).astype(np.float64)
    s = orc.rht_signs(11)
    sv = np.array([-1.0 if (s >> i) & 1 else 1.0 for i in range(32)])
    for fmt in (0, 1):
        d = 128
        codes, scales, ts, pos, w = _combine_case(orc, fmt, d=d)
        v = _decode_payload(codes, scales, ts, fmt, d)
        T, k = pos.shape
        ref = np.zeros((T, d))
        for t in range(T):
            acc = sum(w[t, j] * v[pos[t, j]] for j in range(k))
            for b in range(d // 32):
                ref[t, b * 32:(b + 1) * 32] = sv * (H @ acc[b * 32:(b + 1) * 32]) / np.sqrt(32.0)
        got = orc.combine_rht(codes, scales, ts, fmt, 11, pos, w, f64=True)
        scale = np.abs(ref).max()
        assert np.abs(got - ref).max() <= 1e-12 * scale
        bits = orc.combine_rht(codes, scales, ts, fmt, 11, pos, w)
        tb = torch.from_numpy(ref).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
        # bit-equal away from exact cancellation (there fp64 rounding order
        # decides the sign of a ~1e-15 value)
        big = np.abs(ref) > 1e-9 * scale
        assert np.array_equal(bits[big], tb[big])


def test_combine_rht_is_the_combine_of_the_inverted_rows(orc):
    """Linearity: transforming once after the weighted sum equals combining the
    per-row inverse transforms (oracle_rht32_dequantize in fp32, then
    oracle_combine_f32) up to the fp32 rounding of those rows."""
    for fmt in (0, 1):
        d = 128
        codes, scales, ts, pos, w = _combine_case(orc, fmt, d=d, seed=5)
        R = pos.size
        rows = orc.rht32_dequantize(codes, scales, ts, R, d, 11, fmt)
        via_rows = synth.bf16_bits_to_f32(orc.combine_f32(rows, pos, w)).astype(np.float64)
        once = synth.bf16_bits_to_f32(orc.combine_rht(codes, scales, ts, fmt, 11, pos, w)).astype(np.float64)
        mag = np.abs(once).max()
        assert np.abs(via_rows - once).max() <= 2 ** -8 * mag
        # and the two agree to the last bit on most elements
        assert np.mean(via_rows == once) > 0.9


def test_rht32_amax_is_max_of_the_transform(orc):
    """The payload amax helper equals max |v| of the transform written out with
    scipy's Hadamard matrix in fp64, to the fp32 evaluation's rounding bound,
    and the NVFP4 payload's tensor scale is that amax / 2688."""
    x = synth.bf16_bits_to_f32(synth.payload_rows_np(5, 0, 16, 128, synth.outlier_channels(5, 128, 4)))
    s = orc.rht_signs(11)
    D = np.array([-1.0 if (s >> i) & 1 else 1.0 for i in range(32)])
    H = scipy.linalg.hadamard(32).astype(np.float64) / np.sqrt(32.0)
    v = (x.astype(np.float64).reshape(16, 4, 32) * D) @ H.T
    am = orc.rht32_amax(x, 11)
    ref = np.abs(v).max()
    bound = 5 * 2.0 ** -24 * np.abs(x.astype(np.float64).reshape(16, 4, 32)).sum(axis=2).max()
    assert abs(float(am) - ref) <= bound
    _, _, ts = orc.rht32_quantize(x, 11, 0)
    assert ts == np.float32(am / np.float32(2688.0))

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

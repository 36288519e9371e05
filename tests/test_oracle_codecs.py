"""Pins for the oracle's element codecs (E2M1, E4M3, E8M0, bf16).

E2M1 and E4M3 follow the OCP Microscaling formats that NVFP4 and MXFP8 are
built from; the pins are the formats' closed-form values, a library conversion
(torch's float8_e4m3fn) and brute-force nearest-value properties.
"""
import numpy as np
import pytest
import torch

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decode_grid(orc):
    assert [orc.e2m1_decode(m) for m in range(8)] == E2M1
    assert [orc.e2m1_decode(8 + m) for m in range(8)] == [-v for v in E2M1]


@pytest.mark.parametrize("v,code", [
    (0.25, 0), (0.2500001, 1), (0.75, 2), (0.7499999, 1), (1.25, 2), (1.2500001, 3),
    (1.75, 4), (2.5, 4), (2.5000002, 5), (3.5, 6), (3.4999998, 5), (5.0, 6), (5.0000005, 7),
    (6.0, 7), (7.0, 7), (1e30, 7), (0.0, 0), (-0.0, 8), (-0.1, 8), (-5.0, 14), (-100.0, 15),
])
def test_e2m1_ties_and_saturation(orc, v, code):
    assert orc.e2m1_encode(np.float32(v)) == code


def test_e2m1_nearest_over_all_bf16(orc):
    """Every finite bf16 value encodes to a nearest grid point, ties to the even
    code, with the sign of the input."""
    bits = np.arange(65536, dtype=np.uint32)
    vals = (bits << 16).view(np.float32)
    vals = vals[np.isfinite(vals)]
    grid = np.array(E2M1)
    enc = np.array([orc.e2m1_encode(v) for v in vals])
    dec_mag = grid[enc & 7]
    dist = np.abs(np.abs(vals.astype(np.float64))[:, None] - grid[None, :])
    best = dist.min(axis=1)
    assert np.all(np.abs(np.abs(vals) - dec_mag) == best)
    ties = (dist == best[:, None]).sum(axis=1) == 2
    assert np.all((enc[ties] & 1) == 0)
    assert np.all(((enc & 8) != 0) == np.signbit(vals))


def test_e4m3_closed_forms(orc):
    assert orc.e4m3_decode(0x7E) == 448.0
    assert orc.e4m3_decode(0x01) == 2.0 ** -9
    assert orc.e4m3_decode(0x07) == 7 * 2.0 ** -9
    assert orc.e4m3_decode(0x08) == 2.0 ** -6
    assert orc.e4m3_decode(0x38) == 1.0
    assert orc.e4m3_decode(0xFE) == -448.0
    assert np.isnan(orc.e4m3_decode(0x7F)) and np.isnan(orc.e4m3_decode(0xFF))


def test_e4m3_decode_matches_torch_all_codes(orc):
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    for c in range(256):
        a = orc.e4m3_decode(c)
        b = float(codes[c])
        assert (np.isnan(a) and np.isnan(b)) or a == b


def test_e4m3_roundtrip_all_codes(orc):
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        assert orc.e4m3_encode(np.float32(orc.e4m3_decode(c))) == c


def test_e4m3_encode_matches_torch(orc):
    rng = np.random.default_rng(1)
    v = np.concatenate([
        rng.uniform(-448, 448, 4000), rng.standard_normal(4000) * 2.0 ** rng.integers(-12, 8, 4000),
        (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)[::7],
    ]).astype(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) <= 448)]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_encode(x) for x in v], dtype=np.uint8)
    # torch keeps the sign of values that round to zero too
    assert np.array_equal(got, ref)


def test_e4m3_saturates(orc):
    for v in [448.0, 449.0, 464.0, 465.0, 1e6, 3e38]:
        assert orc.e4m3_encode(np.float32(v)) == 0x7E
        assert orc.e4m3_encode(np.float32(-v)) == 0xFE


def test_e8m0(orc):
    assert orc.e8m0_decode(127) == 1.0
    assert orc.e8m0_decode(0) == 2.0 ** -127
    assert orc.e8m0_decode(254) == 2.0 ** 127
    assert np.isnan(orc.e8m0_decode(255))


def test_bf16_rounding_matches_torch(orc):
    rng = np.random.default_rng(2)
    v = (rng.standard_normal(20000) * 2.0 ** rng.integers(-130, 120, 20000)).astype(np.float32)
    # exact halfway cases and their neighbours
    base = (rng.integers(0, 2 ** 15, 2000).astype(np.uint32) << 16) | 0x8000
    v = np.concatenate([v, base.view(np.float32), (base + 1).view(np.float32),
                        (base - 1).view(np.float32)])
    v = v[np.isfinite(v)]
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = orc.bf16_from_f64(v.astype(np.float64))
    assert np.array_equal(got, ref)

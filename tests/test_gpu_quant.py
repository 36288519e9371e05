"""GPU parity of the quantizers against the oracle: codes and scales bit-exact,
including stochastic rounding with the same Philox stream; dequantized values
bit-exact; both scale layouts; ragged and degenerate shapes."""
import numpy as np
import pytest
import torch

from precision_moe_numerics_quantize_b200 import synth
from tests.gpu_helpers import (dev_bf16, dev_f32, dev_u8, host_u8, mma_to_rowmajor,
                               rowmajor_to_mma, sync)

pytestmark = pytest.mark.gpu


def _bits(rows, cols, seed=0, std=1.0, tag=synth.TAG_X):
    return synth.rows_np(seed, tag, 0, rows, cols, std)


def _f32(bits):
    return synth.bf16_bits_to_f32(bits)


def test_amax(dev, lib):
    bits = _bits(300, 520, seed=3)
    full = np.zeros((300, 528), np.uint16)  # ld > cols: the padding must be ignored
    full[:, :520] = bits
    full[7, 523] = synth.f32_to_bf16_bits(np.array([1e4], np.float32))[0]
    x = dev_bf16(full, dev)
    out = torch.empty(1, device=dev)
    lib.nvfp4moe_amax_bf16(x, out, cols=520, ld=528)
    sync()
    assert out.item() == np.abs(_f32(bits)).max()


@pytest.mark.parametrize("rows,cols,layout,given_amax", [
    (300, 320, 0, False), (384, 512, 1, False), (128, 64, 1, True), (1, 64, 0, False),
    (257, 1024, 0, True),
])
def test_nvfp4_quantize_bitexact(dev, lib, orc, rows, cols, layout, given_amax):
    bits = _bits(rows, cols, seed=rows + cols)
    x = _f32(bits)
    amax = None
    if given_amax:
        amax = np.float32(np.abs(x).max() * 0.5)  # forces saturated scales and codes
    rc, rs, rts = orc.nvfp4_quantize(x, amax_in=amax)
    xd = dev_bf16(bits, dev)
    codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(rows * cols // 16, dtype=torch.uint8, device=dev)
    ts = torch.empty(1, device=dev)
    am = dev_f32([amax], dev) if given_amax else None
    lib.nvfp4_quantize(xd, codes, scales, ts, amax_in=am, layout=layout)
    sync()
    assert np.array_equal(host_u8(codes), rc)
    gs = host_u8(scales)
    gs = gs.reshape(rows, cols // 16) if layout == 0 else mma_to_rowmajor(gs, rows, cols // 16)
    assert np.array_equal(gs, rs)
    assert ts.item() == rts


def test_nvfp4_special_values(dev, lib, orc):
    rows, cols = 4, 64
    x = np.zeros((rows, cols), np.float32)
    x[1] = np.linspace(-3e-38, 3e-38, cols)            # subnormal-range values
    x[2, :16] = [6, -0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -5, 0.1, -0.0, 0, 4, 2, 1, 0.5]
    x[3] = 2.0 ** np.arange(-40, 24, dtype=np.float64)  # 64 binades
    bits = synth.f32_to_bf16_bits(x)
    xf = _f32(bits)
    for amax_in in (None, np.float32(6.0)):
        rc, rs, rts = orc.nvfp4_quantize(xf, amax_in=amax_in)
        codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev)
        scales = torch.empty(rows, cols // 16, dtype=torch.uint8, device=dev)
        ts = torch.empty(1, device=dev)
        lib.nvfp4_quantize(dev_bf16(bits, dev), codes, scales, ts,
                           amax_in=None if amax_in is None else dev_f32([amax_in], dev))
        sync()
        assert np.array_equal(host_u8(codes), rc)
        assert np.array_equal(host_u8(scales), rs)
        assert ts.item() == rts
    # all-zero tensor: ts = 1 and zero codes
    z = torch.zeros(2, 64, dtype=torch.bfloat16, device=dev)
    codes = torch.full((2, 32), 7, dtype=torch.uint8, device=dev)
    scales = torch.full((2, 4), 7, dtype=torch.uint8, device=dev)
    ts = torch.empty(1, device=dev)
    lib.nvfp4_quantize(z, codes, scales, ts)
    sync()
    assert ts.item() == 1.0 and not codes.any() and not scales.any()


@pytest.mark.parametrize("layout", [0, 1])
def test_nvfp4_dequantize_bitexact(dev, lib, orc, layout):
    rows, cols = 256, 192
    x = _f32(_bits(rows, cols, seed=9))
    rc, rs, rts = orc.nvfp4_quantize(x)
    ref = orc.nvfp4_dequantize(rc, rs, rts, rows, cols)
    sc = rs if layout == 0 else rowmajor_to_mma(rs)
    out = torch.empty(rows, cols, device=dev)
    lib.nvfp4_dequantize(dev_u8(rc, dev), dev_u8(sc, dev), dev_f32([rts], dev), rows, cols, out,
                         layout=layout)
    sync()
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("axis,rounding,layout,rows,cols", [
    (0, 0, 0, 96, 320), (0, 1, 0, 96, 320), (0, 1, 1, 256, 384), (0, 0, 1, 128, 128),
    (1, 0, 0, 96, 192), (1, 1, 0, 96, 192), (1, 1, 1, 384, 256), (1, 0, 1, 128, 128),
    (0, 1, 0, 1, 32),
])
def test_mxfp8_bitexact(dev, lib, orc, axis, rounding, layout, rows, cols):
    bits = synth.grad_rows_np(7, 0, rows, cols, synth.outlier_channels(7, cols, 2))
    x = _f32(bits)
    seed, offset = 7, 3 + axis
    rc, rs = orc.mxfp8_quantize(x, axis=axis, seed=seed, offset=offset, rounding=rounding)
    n_rows, n_cols = rc.shape
    codes = torch.empty(n_rows, n_cols, dtype=torch.uint8, device=dev)
    scales = torch.empty(n_rows * n_cols // 32, dtype=torch.uint8, device=dev)
    lib.mxfp8_quantize_sr(dev_bf16(bits, dev), codes, scales, axis=axis, seed=seed, offset=offset,
                          rounding=rounding, layout=layout)
    sync()
    assert np.array_equal(host_u8(codes), rc)
    gs = host_u8(scales)
    gs = gs.reshape(n_rows, n_cols // 32) if layout == 0 else mma_to_rowmajor(gs, n_rows,
                                                                                n_cols // 32)
    assert np.array_equal(gs, rs)


def test_mxfp8_sr_extreme_magnitudes(dev, lib, orc):
    rows, cols = 8, 128
    x = np.zeros((rows, cols), np.float32)
    x[0] = 2.0 ** np.linspace(-133, -120, cols)   # fp32 subnormal / tiny bf16 values
    x[1] = 2.0 ** np.linspace(100, 127, cols)     # near the top of the range
    x[2, ::3] = 447.0
    x[3] = np.linspace(-1, 1, cols)
    bits = synth.f32_to_bf16_bits(x)
    xf = _f32(bits)
    for rounding in (0, 1):
        rc, rs = orc.mxfp8_quantize(xf, axis=0, seed=11, offset=1, rounding=rounding)
        codes = torch.empty(rows, cols, dtype=torch.uint8, device=dev)
        scales = torch.empty(rows, cols // 32, dtype=torch.uint8, device=dev)
        lib.mxfp8_quantize_sr(dev_bf16(bits, dev), codes, scales, axis=0, seed=11, offset=1,
                              rounding=rounding)
        sync()
        assert np.array_equal(host_u8(codes), rc)
        assert np.array_equal(host_u8(scales), rs)


def test_mxfp8_dequantize_bitexact(dev, lib, orc):
    x = _f32(_bits(64, 256, seed=5)) * np.float32(1e-3)
    rc, rs = orc.mxfp8_quantize(x, axis=0, rounding=1, seed=1)
    ref = orc.mxfp8_dequantize(rc, rs)
    for layout in (0, 1):
        sc = rs if layout == 0 else rowmajor_to_mma(np.pad(rs, ((0, 64), (0, 0))))
        codes = np.pad(rc, ((0, 64 if layout else 0), (0, 0)))
        out = torch.empty(codes.shape, device=dev)
        lib.mxfp8_dequantize(dev_u8(codes, dev), dev_u8(sc, dev), out, layout=layout)
        sync()
        assert np.array_equal(out.cpu().numpy()[:64].view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("fmt,rows,cols,given", [(0, 100, 256, False), (1, 100, 256, False),
                                                 (0, 33, 4096, True), (1, 1, 32, False)])
def test_rht32_quantize_bitexact(dev, lib, orc, fmt, rows, cols, given):
    chans = synth.outlier_channels(5, cols, min(16, cols // 2))
    bits = synth.payload_rows_np(5, 0, rows, cols, chans)
    x = _f32(bits)
    amax = np.float32(300.0) if given else None
    rc, rs, rts = orc.rht32_quantize(x, 11, fmt, amax_in=amax)
    codes = torch.empty(rc.shape, dtype=torch.uint8, device=dev)
    scales = torch.empty(rs.shape, dtype=torch.uint8, device=dev)
    ts = torch.empty(1, device=dev)
    lib.rht32_quantize(dev_bf16(bits, dev), 11, fmt, codes, scales,
                       ts_out=ts if fmt == 0 else None,
                       amax_in=dev_f32([amax], dev) if (given and fmt == 0) else None)
    sync()
    assert np.array_equal(host_u8(codes), rc)
    assert np.array_equal(host_u8(scales), rs)
    if fmt == 0:
        assert ts.item() == rts


@pytest.mark.parametrize("fmt", [0, 1])
def test_rht32_dequantize_bitexact(dev, lib, orc, fmt):
    rows, cols = 64, 512
    bits = synth.payload_rows_np(5, 0, rows, cols, synth.outlier_channels(5, cols, 8))
    rc, rs, rts = orc.rht32_quantize(_f32(bits), 11, fmt)
    ref = orc.rht32_dequantize(rc, rs, rts, rows, cols, 11, fmt)
    out = torch.empty(rows, cols, device=dev)
    lib.rht32_dequantize(dev_u8(rc, dev), dev_u8(rs, dev), dev_f32([rts or 0.0], dev), rows, cols,
                         11, fmt, out)
    sync()
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_empty_inputs(dev, lib):
    x = torch.empty(0, 64, dtype=torch.bfloat16, device=dev)
    codes = torch.empty(0, dtype=torch.uint8, device=dev)
    ts = torch.empty(1, device=dev)
    lib.nvfp4_quantize(x, codes, codes, ts, rows=0, cols=64)
    sync()
    assert ts.item() == 1.0


@pytest.mark.parametrize("rounding,layout", [(1, 0), (0, 0), (1, 1)])
def test_mxfp8_cols_unaligned_segments(dev, lib, orc, rounding, layout):
    """Column-wise MXFP8 over segments that do not start on 32-row boundaries
    (one of them empty): each segment cut into 32-row blocks, the last one
    zero-padded, blocks packed in order; bit-exact against the oracle, which
    pads each segment the same way. Columns past the packed blocks are zero."""
    rows, cols = 200, 128
    seg = np.array([0, 20, 20, 75, 150, 200], np.int32)
    bits = synth.grad_rows_np(9, 0, rows, cols, synth.outlier_channels(9, cols, 2))
    x = _f32(bits)
    rc, rs = orc.mxfp8_quantize(x, axis=1, seg_off=seg, seed=7, offset=1, rounding=rounding)
    P = lib.mxfp8_seg_rows(rows, len(seg) - 1)
    assert P % 32 == 0 and P >= rc.shape[1]
    codes = torch.full((cols, P), 0x5A, dtype=torch.uint8, device=dev)
    scales = torch.full((cols * P // 32,), 0x5A, dtype=torch.uint8, device=dev)
    lib.mxfp8_quantize_sr(dev_bf16(bits, dev), codes, scales, axis=1, seed=7, offset=1,
                          rounding=rounding, layout=layout, seg_off=torch.tensor(seg, device=dev))
    sync()
    used = rc.shape[1]
    gc = host_u8(codes)
    gs = host_u8(scales)
    gs = gs.reshape(cols, P // 32) if layout == 0 else mma_to_rowmajor(gs, cols, P // 32)
    assert np.array_equal(gc[:, :used], rc)
    assert np.array_equal(gs[:, :used // 32], rs)
    assert not gc[:, used:].any() and not gs[:, used // 32:].any()
    st, code = lib.device_error()
    assert st == 0 and code == 0


def test_mxfp8_cols_bad_segments_are_reported(dev, lib):
    """Decreasing offsets are caught by the kernel before any load: the output
    is all zeros and the device error word says so."""
    rows, cols = 64, 64
    x = torch.ones(rows, cols, dtype=torch.bfloat16, device=dev)
    seg = torch.tensor([0, 40, 30, 64], dtype=torch.int32, device=dev)
    P = lib.mxfp8_seg_rows(rows, 3)
    codes = torch.full((cols, P), 7, dtype=torch.uint8, device=dev)
    scales = torch.full((cols * P // 32,), 7, dtype=torch.uint8, device=dev)
    lib.mxfp8_quantize_sr(x, codes, scales, axis=1, seg_off=seg)
    sync()
    st, code = lib.device_error()
    assert code == 16  # NVFP4MOE_DEVERR_SEGMENTS
    assert st == 1  # NVFP4MOE_ERR_INVALID_ARG
    assert not codes.any() and not scales.any()

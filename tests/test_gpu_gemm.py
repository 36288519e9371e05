"""GPU parity of the tcgen05 block-scaled grouped GEMMs against the oracle.

Operands are quantized by the oracle and uploaded; the fp32 accumulators must
agree with the oracle's fp64 GEMM of the dequantized operands within
1e-5 * sum_k |a_k * b_k| per element, bf16 outputs within one bf16 ulp on top.
"""
import numpy as np
import pytest
import torch

from precision_moe_numerics_quantize_b200 import synth
from tests.gpu_helpers import dev_bf16, dev_f32, dev_u8, host_bits, host_u8, rowmajor_to_mma, sync

pytestmark = pytest.mark.gpu


def _f32(bits):
    return synth.bf16_bits_to_f32(bits)


def _check_f32(got, ref, mag, rel=1e-5):
    err = np.abs(got.astype(np.float64) - ref)
    bad = err > rel * mag + 1e-30
    assert not bad.any(), (int(bad.sum()), err[bad][:4], ref[bad][:4], mag[bad][:4])


def _check_bf16(got_bits, ref, mag, rel=1e-5):
    got = _f32(got_bits).astype(np.float64)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-38))) - 7)
    err = np.abs(got - ref)
    bad = err > ulp + rel * mag + 1e-30
    assert not bad.any(), (int(bad.sum()), got[bad][:4], ref[bad][:4])


def _quant(orc, x):
    c, s, t = orc.nvfp4_quantize(x)
    return c, s, t


def test_single_group_nvfp4_gemm(dev, lib, orc):
    """A [128 x 256] ~ N(0,1), W [256 x 256] ~ N(0, 0.02): one 128 x 256 tile, one K stage."""
    A = _f32(synth.rows_np(0, synth.TAG_A, 0, 128, 256, 1.0))
    W = _f32(synth.rows_np(0, synth.TAG_W, 0, 256, 256, 0.02))
    ac, as_, at = _quant(orc, A)
    wc, ws, wt = _quant(orc, W)
    Ad = orc.nvfp4_to_f64(ac, as_, at, 128, 256)
    Wd = orc.nvfp4_to_f64(wc, ws, wt, 256, 256)
    ref = orc.gemm_f64(Ad, Wd)
    mag = orc.gemm_f64(np.abs(Ad), np.abs(Wd))
    off = torch.tensor([0, 128], dtype=torch.int32, device=dev)
    for out_dtype in (lib.OUT_F32, lib.OUT_BF16):
        c = torch.empty(128, 256, dtype=torch.float32 if out_dtype else torch.bfloat16, device=dev)
        lib.nvfp4_grouped_gemm(dev_u8(ac, dev), dev_u8(rowmajor_to_mma(as_), dev),
                               dev_f32([at], dev), 0, dev_u8(wc, dev),
                               dev_u8(rowmajor_to_mma(ws), dev), dev_f32([wt], dev), off, 1, 128,
                               256, 256, c, out_dtype=out_dtype)
        sync()
        if out_dtype == lib.OUT_F32:
            _check_f32(c.cpu().numpy(), ref, mag)
        else:
            _check_bf16(host_bits(c), ref, mag)


def test_single_group_end_to_end_quantize_then_gemm(dev, lib, orc):
    """The whole single-GEMM workload on the GPU (quantize both operands, GEMM,
    bf16 out) against the oracle's quantize + fp64 GEMM."""
    a_bits = synth.rows_np(0, synth.TAG_A, 0, 128, 256, 1.0)
    w_bits = synth.rows_np(0, synth.TAG_W, 0, 256, 256, 0.02)
    ac, as_, at = _quant(orc, _f32(a_bits))
    wc, ws, wt = _quant(orc, _f32(w_bits))
    Ad = orc.nvfp4_to_f64(ac, as_, at, 128, 256)
    Wd = orc.nvfp4_to_f64(wc, ws, wt, 256, 256)
    ref = orc.gemm_f64(Ad, Wd)
    mag = orc.gemm_f64(np.abs(Ad), np.abs(Wd))
    ga = torch.empty(128, 128, dtype=torch.uint8, device=dev)
    gas = torch.empty(128 * 16, dtype=torch.uint8, device=dev)
    gat = torch.empty(1, device=dev)
    gw = torch.empty(256, 128, dtype=torch.uint8, device=dev)
    gws = torch.empty(256 * 16, dtype=torch.uint8, device=dev)
    gwt = torch.empty(1, device=dev)
    lib.nvfp4_quantize(dev_bf16(a_bits, dev), ga, gas, gat, layout=lib.LAYOUT_MMA)
    lib.nvfp4_quantize(dev_bf16(w_bits, dev), gw, gws, gwt, layout=lib.LAYOUT_MMA)
    c = torch.empty(128, 256, dtype=torch.bfloat16, device=dev)
    off = torch.tensor([0, 128], dtype=torch.int32, device=dev)
    lib.nvfp4_grouped_gemm(ga, gas, gat, 0, gw, gws, gwt, off, 1, 128, 256, 256, c)
    sync()
    assert np.array_equal(host_u8(ga), ac) and np.array_equal(host_u8(gw), wc)
    _check_bf16(host_bits(c), ref, mag)


def test_grouped_nvfp4_gemm_ragged_groups(dev, lib, orc):
    """Four groups with 128, 0, 256 and 384 rows, K = 1024 (4 stages), N = 512."""
    rows = [128, 0, 256, 384]
    off = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    R, K, N, G = int(off[-1]), 1024, 512, 4
    A = _f32(synth.rows_np(1, synth.TAG_A, 0, R, K, 1.0))
    a_parts, a_sc, a_ts, Ad = [], [], [], np.zeros((R, K))
    for g in range(G):
        if rows[g] == 0:
            a_ts.append(np.float32(1.0))
            continue
        c, s, t = _quant(orc, A[off[g]:off[g + 1]])
        a_parts.append(c); a_sc.append(s); a_ts.append(t)
        Ad[off[g]:off[g + 1]] = orc.nvfp4_to_f64(c, s, t, rows[g], K)
    ac = np.concatenate(a_parts); asc = np.concatenate(a_sc)
    b_parts, b_sc, b_ts, Bd = [], [], [], []
    for g in range(G):
        W = _f32(synth.expert_weight_np(2, synth.TAG_W, g, N, K))
        c, s, t = _quant(orc, W)
        b_parts.append(c); b_sc.append(s); b_ts.append(t)
        Bd.append(orc.nvfp4_to_f64(c, s, t, N, K))
    bc = np.concatenate(b_parts); bsc = np.concatenate(b_sc)
    c = torch.full((R, N), float("nan"), dtype=torch.float32, device=dev)
    lib.nvfp4_grouped_gemm(dev_u8(ac, dev), dev_u8(rowmajor_to_mma(asc), dev), dev_f32(a_ts, dev),
                           1, dev_u8(bc, dev), dev_u8(rowmajor_to_mma(bsc), dev),
                           dev_f32(b_ts, dev), torch.tensor(off, device=dev), G, R, N, K, c,
                           out_dtype=lib.OUT_F32)
    sync()
    got = c.cpu().numpy()
    for g in range(G):
        if rows[g] == 0:
            continue
        sl = slice(off[g], off[g + 1])
        ref = orc.gemm_f64(Ad[sl], Bd[g])
        mag = orc.gemm_f64(np.abs(Ad[sl]), np.abs(Bd[g]))
        _check_f32(got[sl], ref, mag)


def test_grouped_nvfp4_gemm_tile_shapes(dev, lib, orc):
    """Groups of 640, 128, 512, 896, 384, 1152 and 768 rows: token tiles of
    384 (MMAs of N = 256 and 128 on one W stage), 320 (256 + 64), 256 and 128
    rows, tiles that start 64 rows into a 128-row scale block and span four
    scale chunk rows, and K = 768 (three 128-byte k-blocks: the third reuses
    the TMEM scale slot of the first); bf16 out."""
    rows = [640, 128, 512, 896, 384, 1152, 768]
    off = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    R, K, N, G = int(off[-1]), 768, 256, len(rows)
    A = _f32(synth.rows_np(7, synth.TAG_A, 0, R, K, 1.0))
    a_parts, a_sc, a_ts, Ad = [], [], [], np.zeros((R, K))
    for g in range(G):
        c, s, t = _quant(orc, A[off[g]:off[g + 1]])
        a_parts.append(c); a_sc.append(s); a_ts.append(t)
        Ad[off[g]:off[g + 1]] = orc.nvfp4_to_f64(c, s, t, rows[g], K)
    b_parts, b_sc, b_ts, Bd = [], [], [], []
    for g in range(G):
        W = _f32(synth.expert_weight_np(8, synth.TAG_W, g, N, K))
        c, s, t = _quant(orc, W)
        b_parts.append(c); b_sc.append(s); b_ts.append(t)
        Bd.append(orc.nvfp4_to_f64(c, s, t, N, K))
    c = torch.empty(R, N, dtype=torch.bfloat16, device=dev)
    lib.nvfp4_grouped_gemm(dev_u8(np.concatenate(a_parts), dev),
                           dev_u8(rowmajor_to_mma(np.concatenate(a_sc)), dev), dev_f32(a_ts, dev), 1,
                           dev_u8(np.concatenate(b_parts), dev),
                           dev_u8(rowmajor_to_mma(np.concatenate(b_sc)), dev), dev_f32(b_ts, dev),
                           torch.tensor(off, device=dev), G, R, N, K, c)
    sync()
    got = host_bits(c)
    for g in range(G):
        sl = slice(off[g], off[g + 1])
        _check_bf16(got[sl], orc.gemm_f64(Ad[sl], Bd[g]), orc.gemm_f64(np.abs(Ad[sl]), np.abs(Bd[g])))


def _mx(orc, x, axis=0):
    c, s = orc.mxfp8_quantize(x, axis=axis, rounding=0)
    return c, s


def test_mxfp8_gemm_group_m(dev, lib, orc):
    rows = [256, 128]
    off = np.array([0, 256, 384], np.int32)
    R, K, N, G = 384, 512, 256, 2
    A = _f32(synth.grad_rows_np(3, 0, R, K, synth.outlier_channels(3, K, 2)))
    ac, asc = _mx(orc, A)
    Ad = orc.mxfp8_dequantize(ac, asc).astype(np.float64)
    bcs, bscs, Bd = [], [], []
    for g in range(G):
        W = _f32(synth.expert_weight_np(4, synth.TAG_W, g, N, K))
        c, s = _mx(orc, W)
        bcs.append(c); bscs.append(s); Bd.append(orc.mxfp8_dequantize(c, s).astype(np.float64))
    c = torch.full((R, N), float("nan"), dtype=torch.float32, device=dev)
    lib.mxfp8_grouped_gemm(dev_u8(ac, dev), dev_u8(rowmajor_to_mma(asc), dev),
                           dev_u8(np.concatenate(bcs), dev),
                           dev_u8(rowmajor_to_mma(np.concatenate(bscs)), dev),
                           torch.tensor(off, device=dev), G, lib.GROUP_M, R, N, K, c)
    sync()
    got = c.cpu().numpy()
    for g in range(G):
        sl = slice(off[g], off[g + 1])
        _check_f32(got[sl], orc.gemm_f64(Ad[sl], Bd[g]), orc.gemm_f64(np.abs(Ad[sl]), np.abs(Bd[g])))


@pytest.mark.parametrize("M", [256, 384, 640])
def test_mxfp8_gemm_group_k(dev, lib, orc, M):
    """Weight-gradient shape: C_g = A[:, off_g:off_g+1] . B[:, off_g:off_g+1]^T with an empty
    group; M = 384 output rows make one token-side tile of two MMAs (N = 256 and 128),
    M = 640 two tiles of 320 rows, the second starting 64 rows into a scale block."""
    seg = [256, 0, 128, 384]
    off = np.concatenate([[0], np.cumsum(seg)]).astype(np.int32)
    N, Kt, G = 256, int(off[-1]), 4
    A = _f32(synth.grad_rows_np(5, 0, M, Kt, synth.outlier_channels(5, Kt, 2)))
    Bm = _f32(synth.rows_np(6, synth.TAG_ACT, 0, N, Kt, 0.3))
    ac, asc = _mx(orc, A)
    bc, bsc = _mx(orc, Bm)
    Ad = orc.mxfp8_dequantize(ac, asc).astype(np.float64)
    Bd = orc.mxfp8_dequantize(bc, bsc).astype(np.float64)
    c = torch.full((G, M, N), float("nan"), dtype=torch.float32, device=dev)
    lib.mxfp8_grouped_gemm(dev_u8(ac, dev), dev_u8(rowmajor_to_mma(asc), dev), dev_u8(bc, dev),
                           dev_u8(rowmajor_to_mma(bsc), dev), torch.tensor(off, device=dev), G,
                           lib.GROUP_K, M, N, Kt, c)
    sync()
    got = c.cpu().numpy()
    for g in range(G):
        if seg[g] == 0:
            assert not got[g].any()
            continue
        sl = slice(off[g], off[g + 1])
        _check_f32(got[g], orc.gemm_f64(Ad[:, sl], Bd[:, sl]),
                   orc.gemm_f64(np.abs(Ad[:, sl]), np.abs(Bd[:, sl])))


def test_bounded_wait_gives_up_and_the_context_survives(dev, lib, orc):
    """The failure path of the GEMM pipeline, without a fault: with the test
    hook set, the producers issue no load at all (nothing is in flight), so
    the MMA thread's and the scale warps' bounded waits run out after 10 ms;
    every role winds down, the launch ends, and the device error word holds
    the id of the wait that gave up first (the MMA thread's wait on `full`
    or a scale warp's wait on its scales). The same GEMM then runs normally
    on the same context and matches the oracle."""
    A = _f32(synth.rows_np(0, synth.TAG_A, 0, 128, 256, 1.0))
    W = _f32(synth.rows_np(0, synth.TAG_W, 0, 256, 256, 0.02))
    ac, as_, at = _quant(orc, A)
    wc, ws, wt = _quant(orc, W)
    args = [dev_u8(ac, dev), dev_u8(rowmajor_to_mma(as_), dev), dev_f32([at], dev), 0,
            dev_u8(wc, dev), dev_u8(rowmajor_to_mma(ws), dev), dev_f32([wt], dev),
            torch.tensor([0, 128], dtype=torch.int32, device=dev), 1, 128, 256, 256]
    c = torch.zeros(128, 256, dtype=torch.float32, device=dev)
    assert lib.device_error() == (0, 0)
    lib.debug_gemm(lib.DEBUG_WITHHOLD_LOADS, 10_000_000)
    try:
        lib.nvfp4_grouped_gemm(*args, c, out_dtype=lib.OUT_F32)
        sync()
    finally:
        lib.debug_gemm(0)
    st, code = lib.device_error()
    assert st == 6 and code in (1, 6), (st, code)  # NVFP4MOE_ERR_TIMEOUT; WAIT_GEMM_FULL / _SF_SLOT
    assert lib.device_error() == (0, 0)  # read and cleared
    lib.nvfp4_grouped_gemm(*args, c, out_dtype=lib.OUT_F32)
    sync()
    Ad = orc.nvfp4_to_f64(ac, as_, at, 128, 256)
    Wd = orc.nvfp4_to_f64(wc, ws, wt, 256, 256)
    _check_f32(c.cpu().numpy(), orc.gemm_f64(Ad, Wd), orc.gemm_f64(np.abs(Ad), np.abs(Wd)))
    assert lib.device_error() == (0, 0)

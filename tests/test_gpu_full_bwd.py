"""Full-size parity of the MXFP8 backward operands and GEMMs (the 16384-token,
384-expert, top-8 layer with d = 4096, f = 2560, uniform router), in the
launch configuration the benchmark times.

dY [R_p x d] ~ N(0, 1e-3) with 0.1% outlier channels x 100 (seed 7), zero on
padding rows, is quantized on the GPU along rows (dgrad operand) and along
rows-within-experts (wgrad operand), both with Philox stochastic rounding
(seed 7, offsets 0 and 1); the saved activation A [R_p x f] ~ N(0, 0.3) and
each expert's W2 (transposed, blocks along d) with round-to-nearest-even.
For three experts (the lightest, the median and the heaviest) the oracle
quantizes the same rows with the same Philox draws (row0 = the expert's first
row): codes and scales bit-exact. Then dgrad dA_e = dY_e . W2_e (bf16) and
wgrad dW2_e = dY_e^T . A_e (fp32, contraction over the expert's rows) are
compared with the fp64 product of the oracle's dequantized operands: fp32
within 1e-5 * sum |a b|, bf16 within one ulp on top.
"""
import numpy as np
import pytest
import torch

from precision_moe_numerics_quantize_b200 import synth
from tests.gpu_helpers import host_bits, host_u8, mma_rows_to_rowmajor, sync

pytestmark = pytest.mark.gpu

SHAPE = synth.SHAPES["full_moe"]


def _f32(bits):
    return synth.bf16_bits_to_f32(bits)


def _ulp(v):
    return np.exp2(np.floor(np.log2(np.maximum(np.abs(v), 1e-38))) - 7)


@pytest.fixture(scope="module")
def bwd(dev, lib, orc):
    T, d, f, E, k = SHAPE.T, SHAPE.d, SHAPE.f, SHAPE.E, SHAPE.k
    idx, _ = orc.route(synth.logits_uniform_np(2, T, E), k)
    off, pos, tok = orc.permute(idx, E)
    Rp = int(off[-1])
    pad = torch.from_numpy(tok[:Rp] < 0).to(dev)
    dchans = synth.outlier_channels(7, d, max(1, d // 1000))
    dy = synth.grad_rows_torch(7, 0, Rp, d, dchans, dev)
    dy[pad] = 0
    act = synth.rows_torch(8, synth.TAG_ACT, 0, Rp, f, 0.3, dev)
    act[pad] = 0
    g = {"off": off, "tok": tok, "Rp": Rp, "dchans": dchans}
    g["dyc0"] = torch.empty(Rp, d, dtype=torch.uint8, device=dev)
    g["dys0"] = torch.empty(Rp * d // 32, dtype=torch.uint8, device=dev)
    g["dyc1"] = torch.empty(d, Rp, dtype=torch.uint8, device=dev)
    g["dys1"] = torch.empty(d * Rp // 32, dtype=torch.uint8, device=dev)
    g["ac1"] = torch.empty(f, Rp, dtype=torch.uint8, device=dev)
    g["as1"] = torch.empty(f * Rp // 32, dtype=torch.uint8, device=dev)
    lib.mxfp8_quantize_sr(dy, g["dyc0"], g["dys0"], axis=0, seed=7, offset=0, layout=lib.LAYOUT_MMA)
    lib.mxfp8_quantize_sr(dy, g["dyc1"], g["dys1"], axis=1, seed=7, offset=1, layout=lib.LAYOUT_MMA)
    lib.mxfp8_quantize_sr(act, g["ac1"], g["as1"], axis=1, rounding=lib.ROUND_RNE,
                          layout=lib.LAYOUT_MMA)
    g["w2c"] = torch.empty(E * f, d, dtype=torch.uint8, device=dev)
    g["w2s"] = torch.empty(E * f * d // 32, dtype=torch.uint8, device=dev)
    for e in range(E):
        wb = synth.expert_weight_torch(1, synth.TAG_W2, e, d, f, dev)
        lib.mxfp8_quantize_sr(wb, g["w2c"][e * f:(e + 1) * f],
                              g["w2s"][e * f * d // 32:(e + 1) * f * d // 32], axis=1,
                              rounding=lib.ROUND_RNE, layout=lib.LAYOUT_MMA)
    del dy, act
    off_d = torch.tensor(off, device=dev)
    g["dA"] = torch.zeros(Rp, f, dtype=torch.bfloat16, device=dev)
    lib.mxfp8_grouped_gemm(g["dyc0"], g["dys0"], g["w2c"], g["w2s"], off_d, E, lib.GROUP_M, Rp, f,
                           d, g["dA"], out_dtype=lib.OUT_BF16)
    g["dW"] = torch.empty(E, d, f, dtype=torch.float32, device=dev)
    lib.mxfp8_grouped_gemm(g["dyc1"], g["dys1"], g["ac1"], g["as1"], off_d, E, lib.GROUP_K, d, f,
                           Rp, g["dW"], out_dtype=lib.OUT_F32)
    sync()
    real_cnt = np.array([int(np.sum(tok[off[e]:off[e + 1]] >= 0)) for e in range(E)])
    order = np.argsort(real_cnt, kind="stable")
    g["experts"] = [int(order[0]), int(order[E // 2]), int(order[-1])]
    yield g
    del g
    torch.cuda.empty_cache()


def _expert_operands(orc, g, e):
    """The oracle's own quantization of expert e's rows of dY and A."""
    d, f = SHAPE.d, SHAPE.f
    off, tok = g["off"], g["tok"]
    r0, r1 = int(off[e]), int(off[e + 1])
    n = r1 - r0
    padrow = tok[r0:r1] < 0
    dy = _f32(synth.grad_rows_np(7, r0, n, d, g["dchans"]))
    dy[padrow] = 0
    a = _f32(synth.rows_np(8, synth.TAG_ACT, r0, n, f, 0.3))
    a[padrow] = 0
    rc, rs = orc.mxfp8_quantize(dy, axis=0, seed=7, offset=0, rounding=1, row0=r0)
    cc, cs = orc.mxfp8_quantize(dy, axis=1, seed=7, offset=1, rounding=1, row0=r0)
    ac, as_ = orc.mxfp8_quantize(a, axis=1, rounding=0, row0=r0)
    return r0, r1, (rc, rs), (cc, cs), (ac, as_)


def test_full_mxfp8_sr_operands_bitexact(bwd, orc):
    g = bwd
    d, f, Rp = SHAPE.d, SHAPE.f, g["Rp"]
    gs0 = host_u8(g["dys0"])
    gs1 = host_u8(g["dys1"])
    ga1 = host_u8(g["as1"])
    for e in g["experts"]:
        r0, r1, (rc, rs), (cc, cs), (ac, as_) = _expert_operands(orc, g, e)
        rows = np.arange(r0, r1)
        # rows: blocks of 32 along d
        assert np.array_equal(host_u8(g["dyc0"][r0:r1]), rc), e
        assert np.array_equal(mma_rows_to_rowmajor(gs0, rows, d // 32), rs), e
        # columns: blocks of 32 rows inside the expert (its rows start at a
        # multiple of 128, so no block crosses an expert)
        assert np.array_equal(host_u8(g["dyc1"][:, r0:r1]), cc), e
        sc1 = mma_rows_to_rowmajor(gs1, np.arange(d), Rp // 32)[:, r0 // 32:r1 // 32]
        assert np.array_equal(sc1, cs), e
        assert np.array_equal(host_u8(g["ac1"][:, r0:r1]), ac), e
        sa1 = mma_rows_to_rowmajor(ga1, np.arange(f), Rp // 32)[:, r0 // 32:r1 // 32]
        assert np.array_equal(sa1, as_), e


def test_full_mxfp8_dgrad_wgrad(bwd, dev, orc):
    g = bwd
    d, f = SHAPE.d, SHAPE.f
    ws_all = host_u8(g["w2s"])
    for e in g["experts"]:
        r0, r1, (rc, rs), (cc, cs), (ac, as_) = _expert_operands(orc, g, e)
        W2 = _f32(host_bits(synth.expert_weight_torch(1, synth.TAG_W2, e, d, f, dev)))
        wc, wsc = orc.mxfp8_quantize(W2, axis=1, rounding=0)  # [f x d], blocks along d
        assert np.array_equal(host_u8(g["w2c"][e * f:(e + 1) * f]), wc), e
        assert np.array_equal(mma_rows_to_rowmajor(ws_all, np.arange(e * f, (e + 1) * f), d // 32),
                              wsc), e
        Wd = orc.mxfp8_dequantize(wc, wsc).astype(np.float64)
        # dgrad: dA_e = dY_e . W2_e, contraction over d
        Dr = orc.mxfp8_dequantize(rc, rs).astype(np.float64)
        ref = orc.gemm_f64(Dr, Wd)
        mag = orc.gemm_f64(np.abs(Dr), np.abs(Wd))
        got = _f32(host_bits(g["dA"][r0:r1])).astype(np.float64)
        assert np.isfinite(got).all(), e
        bad = np.abs(got - ref) > _ulp(np.maximum(np.abs(ref), np.abs(got))) + 1e-5 * mag + 1e-30
        assert not bad.any(), (e, int(bad.sum()))
        # wgrad: dW2_e = dY_e^T . A_e, contraction over the expert's rows
        Dc = orc.mxfp8_dequantize(cc, cs).astype(np.float64)
        Ac = orc.mxfp8_dequantize(ac, as_).astype(np.float64)
        ref = orc.gemm_f64(Dc, Ac)
        mag = orc.gemm_f64(np.abs(Dc), np.abs(Ac))
        got = g["dW"][e].cpu().numpy().astype(np.float64)
        bad = np.abs(got - ref) > 1e-5 * mag + 1e-30
        assert not bad.any(), (e, int(bad.sum()))

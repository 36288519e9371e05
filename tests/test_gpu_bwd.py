"""GPU parity of the SwiGLU backward against the oracle.

The kernel works in fp32 (IEEE division, expf) and rounds once to bf16; the
oracle works in fp64. Every output is within one bf16 ulp of the oracle's,
and almost all are bit-identical (the two differ only where the exact value
lies within the fp32 error of a bf16 rounding boundary).
"""
import numpy as np
import pytest
import torch

from precision_moe_numerics_quantize_b200 import synth
from tests.gpu_helpers import dev_bf16, host_bits, sync

pytestmark = pytest.mark.gpu


def _ulp(v):
    return np.exp2(np.floor(np.log2(np.maximum(np.abs(v), 1e-38))) - 7)


@pytest.mark.parametrize("rows,f", [(1000, 2560), (37, 8), (128, 512)])
def test_swiglu_bwd_matches_oracle(dev, lib, orc, rows, f):
    gu_bits = synth.rows_np(4, synth.TAG_ACT, 0, rows, 2 * f, 2.0)
    gu_bits[0, :8] = synth.f32_to_bf16_bits(np.array([-100, -30, -8, 0, 8, 30, 100, 1e-3],
                                                     np.float32))
    dh_bits = synth.rows_np(5, synth.TAG_ACT, 0, rows, f, 0.5)
    dh_bits[1, :] = 0
    out = torch.full((rows, 2 * f), -1.0, dtype=torch.bfloat16, device=dev)
    lib.swiglu_bwd(dev_bf16(gu_bits, dev), dev_bf16(dh_bits, dev), out)
    sync()
    got_bits = host_bits(out)
    ref_bits = orc.swiglu_bwd(gu_bits, dh_bits)
    got = synth.bf16_bits_to_f32(got_bits).astype(np.float64)
    ref = synth.bf16_bits_to_f32(ref_bits).astype(np.float64)
    assert np.all(np.abs(got - ref) <= _ulp(ref) + 1e-38)
    same = np.mean((got_bits == ref_bits) | ((got == 0) & (ref == 0)))
    assert same >= 0.99, same


def test_swiglu_bwd_no_rows(dev, lib):
    e = torch.empty(0, 64, dtype=torch.bfloat16, device=dev)
    lib.swiglu_bwd(torch.empty(0, 128, dtype=torch.bfloat16, device=dev), e,
                   torch.empty(0, 128, dtype=torch.bfloat16, device=dev))
    sync()


def test_expert_bwd_gemm1_matches_oracle(dev, lib, orc):
    """GEMM1 backward (dgrad and wgrad) on a Zipf-routed layer of 4 experts,
    d = 256, f = 128. The stochastically rounded gradient operands are
    bit-exact against the oracle's; dX and dW1 agree with the oracle's chain
    to the fp32 accumulation bound (1e-5 of sum |a b|) plus one rounding."""
    from tests.gpu_helpers import dev_u8, host_u8, mma_to_rowmajor
    T, E, k, d, f = 512, 4, 2, 256, 128
    f2 = 2 * f
    idx, _ = orc.route(synth.logits_zipf_np(3, T, E), k)
    off, pos, tok = orc.permute(idx, E)
    R = lib.max_rows(T, k, E)
    used = int(off[-1])
    pad = np.ones(R, bool)
    pad[:used] = tok[:used] < 0
    dgu = synth.rows_np(14, synth.TAG_ACT, 0, R, f2, 0.01)
    x = synth.rows_np(15, synth.TAG_X, 0, R, d, 1.0)
    dgu[pad] = 0
    x[pad] = 0
    W1 = np.stack([synth.expert_weight_np(16, synth.TAG_W1, e, f2, d) for e in range(E)])
    w1t = torch.empty(E * d, f2, dtype=torch.uint8, device=dev)
    w1t_sc = torch.empty(E * d * f2 // 32, dtype=torch.uint8, device=dev)
    per = d * f2 // 32
    for e in range(E):
        lib.mxfp8_quantize_sr(dev_bf16(W1[e], dev), w1t[e * d:(e + 1) * d], w1t_sc[e * per:(e + 1) * per],
                              axis=1, rounding=lib.ROUND_RNE, layout=lib.LAYOUT_MMA)
    u8 = lambda *shape: torch.empty(*shape, dtype=torch.uint8, device=dev)
    gq, gq_sc = u8(R, f2), u8(R * f2 // 32)
    gt, gt_sc = u8(f2, R), u8(f2 * R // 32)
    xt, xt_sc = u8(d, R), u8(d * R // 32)
    dx = torch.empty(R, d, dtype=torch.bfloat16, device=dev)
    dw1 = torch.full((E, f2, d), float("nan"), device=dev)
    lib.moe_expert_bwd_gemm1(dev_bf16(dgu, dev), dev_bf16(x, dev), torch.tensor(off, device=dev), E,
                             d, f, w1t, w1t_sc, 7, 2, gq, gq_sc, gt, gt_sc, xt, xt_sc, dx, dw1, R)
    sync()
    ref = orc.expert_bwd_gemm1(dgu[:used], x[:used], W1, expert_off=off, seed=7, offset=2)
    dgf = synth.bf16_bits_to_f32(dgu[:used])
    xf = synth.bf16_bits_to_f32(x[:used])
    # the gradient operands, bit for bit
    oc, osc = orc.mxfp8_quantize(dgf, axis=0, seed=7, offset=2, rounding=1)
    assert np.array_equal(host_u8(gq)[:used], oc)
    assert np.array_equal(mma_to_rowmajor(host_u8(gq_sc), R, f2 // 32)[:used], osc)
    tc, tsc = orc.mxfp8_quantize(dgf, axis=1, seg_off=off, seed=7, offset=3, rounding=1)
    assert np.array_equal(host_u8(gt)[:, :used], tc)
    assert np.array_equal(mma_to_rowmajor(host_u8(gt_sc), f2, R // 32)[:, :used // 32], tsc)
    # dX and dW1 against the oracle chain
    Gd = orc.mxfp8_dequantize(oc, osc).astype(np.float64)
    Td = orc.mxfp8_dequantize(tc, tsc).astype(np.float64)
    xc, xsc = orc.mxfp8_quantize(xf, axis=1, seg_off=off, rounding=0)
    Xd = orc.mxfp8_dequantize(xc, xsc).astype(np.float64)
    got_dx = synth.bf16_bits_to_f32(host_bits(dx)[:used]).astype(np.float64)
    ref_dx = synth.bf16_bits_to_f32(ref["dx"]).astype(np.float64)
    got_dw = dw1.cpu().numpy().astype(np.float64)
    for e in range(E):
        s = slice(off[e], off[e + 1])
        wc, ws = orc.mxfp8_quantize(synth.bf16_bits_to_f32(W1[e]), axis=1, rounding=0)
        mag = orc.gemm_f64(np.abs(Gd[s]), np.abs(orc.mxfp8_dequantize(wc, ws).astype(np.float64)))
        # one bf16 ulp (at the larger magnitude) on top of the accumulator bound
        ulp = _ulp(np.maximum(np.abs(ref_dx[s]), np.abs(got_dx[s])))
        assert np.all(np.abs(got_dx[s] - ref_dx[s]) <= ulp + 1e-5 * mag + 1e-30), e
        magw = orc.gemm_f64(np.abs(Td[:, s]), np.abs(Xd[:, s]))
        refw = ref["dw1"][e].astype(np.float64)
        assert np.all(np.abs(got_dw[e] - refw) <= 1e-5 * magw + 2.0 ** -23 * np.abs(refw) + 1e-30), e

"""Pins of the oracle's GEMM1 backward chain (MXFP8 dgrad and wgrad), each
against something other than the chain itself:
  on the grid   inputs whose every 32-block holds 448 and only E4M3 values:
                every block scale is 2^0, both roundings are exact, and the
                chain must equal plain fp64 products bit for bit;
  powers of two scaling the inputs by powers of two scales the outputs
                exactly (the stochastic draws depend on position only);
  padding       n not a multiple of 32 gives the same result as the same rows
                padded with zero rows.
"""
import numpy as np
import torch

from precision_moe_numerics_quantize_b200 import synth


def _bits(a):
    return synth.f32_to_bf16_bits(np.asarray(a, np.float32))


def _on_grid(rng, rows, cols):
    """E4M3 values (scale 2^0) with 448 wherever row = column (mod 32), so
    every 32-block along rows and along columns holds 448."""
    codes = rng.integers(0, 256, size=(rows, cols)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0  # no NaN codes
    v = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    i, j = np.indices((rows, cols))
    v[(i - j) % 32 == 0] = 448.0
    return v


def test_chain_is_exact_on_the_grid(orc):
    rng = np.random.default_rng(3)
    n, f2, d = 64, 64, 96
    dgu, x, w1 = _on_grid(rng, n, f2), _on_grid(rng, n, d), _on_grid(rng, f2, d)
    r = orc.expert_bwd_gemm1(_bits(dgu), _bits(x), _bits(w1), seed=5, offset=2)
    dx = dgu.astype(np.float64) @ w1.astype(np.float64)  # exact: few-bit dyadic values
    dw = dgu.astype(np.float64).T @ x.astype(np.float64)
    ref_dx = torch.from_numpy(dx).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(r["dx"], ref_dx)
    assert np.array_equal(r["dw1"], dw.astype(np.float32))


def test_chain_scales_exactly_with_powers_of_two(orc):
    n, f2, d = 64, 64, 64
    dgu = synth.bf16_bits_to_f32(synth.rows_np(6, synth.TAG_ACT, 0, n, f2, 0.01))
    x = synth.bf16_bits_to_f32(synth.rows_np(7, synth.TAG_X, 0, n, d, 1.0))
    w1 = synth.bf16_bits_to_f32(synth.expert_weight_np(8, synth.TAG_W1, 0, f2, d))
    r = orc.expert_bwd_gemm1(_bits(dgu), _bits(x), _bits(w1), seed=9, offset=0)
    s = orc.expert_bwd_gemm1(_bits(dgu * 32.0), _bits(x / 8.0), _bits(w1 * 4.0), seed=9, offset=0)
    dx = synth.bf16_bits_to_f32(r["dx"]).astype(np.float64)
    dx_s = synth.bf16_bits_to_f32(s["dx"]).astype(np.float64)
    assert np.array_equal(dx_s, dx * 128.0)
    assert np.array_equal(s["dw1"].astype(np.float64), r["dw1"].astype(np.float64) * 4.0)
    # and the draws matter: another seed changes some stochastically rounded result
    t = orc.expert_bwd_gemm1(_bits(dgu), _bits(x), _bits(w1), seed=10, offset=0)
    assert not np.array_equal(t["dx"], r["dx"])


def test_ragged_rows_equal_zero_padded_rows(orc):
    n, npad, f2, d = 40, 64, 64, 32
    dgu = synth.rows_np(11, synth.TAG_ACT, 0, n, f2, 0.01)
    x = synth.rows_np(12, synth.TAG_X, 0, n, d, 1.0)
    w1 = synth.expert_weight_np(13, synth.TAG_W1, 0, f2, d)
    pad = lambda a: np.concatenate([a, np.zeros((npad - n, a.shape[1]), np.uint16)])
    r = orc.expert_bwd_gemm1(dgu, x, w1, seed=1, offset=4)
    p = orc.expert_bwd_gemm1(pad(dgu), pad(x), w1, seed=1, offset=4)
    assert np.array_equal(r["dx"], p["dx"][:n])
    assert np.array_equal(r["dw1"], p["dw1"])


def _blocking_case():
    rng = np.random.default_rng(21)
    n, f2, d = 32, 64, 64
    dgu, x, w1 = _on_grid(rng, n, f2), _on_grid(rng, n, d), _on_grid(rng, f2, d)
    small = np.array([0.5, -0.75, 1.0, -0.25], np.float32)
    w1[1:32, 0] = small[np.arange(31) % 4]
    w1[0, 0] = 2.0 ** 18
    w_expect = w1.astype(np.float64)
    w_expect[1:32, 0] = 0.0
    dx = dgu.astype(np.float64) @ w_expect
    ref_dx = torch.from_numpy(dx).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return dgu, x, w1, ref_dx


def test_weight_blocks_run_along_the_contraction(orc):
    """W1's 32-blocks run along 2f (the dgrad contraction). Column 0 rows 0..31
    hold 2^18 and values of magnitude <= 1: that block's scale is 2^10, so
    the small values fall below half the smallest E4M3 step and vanish, while
    every other block keeps its on-grid values exactly. Blocks along d would
    flush row 0 instead."""
    dgu, x, w1, ref_dx = _blocking_case()
    r = orc.expert_bwd_gemm1(_bits(dgu), _bits(x), _bits(w1), seed=2, offset=0)
    assert np.array_equal(r["dx"], ref_dx)


def test_blocking_pin_rejects_weights_blocked_along_d(orc):
    """The same check fails on a planted copy of the dgrad that blocks W1
    along d (its rows) instead of along 2f."""
    dgu, x, w1, ref_dx = _blocking_case()
    gc, gs = orc.mxfp8_quantize(dgu, axis=0, seed=2, offset=0, rounding=1)
    wc, ws = orc.mxfp8_quantize(w1, axis=0, rounding=0)  # planted: blocks along d
    planted = orc.bf16_from_f64(orc.gemm_f64(orc.mxfp8_dequantize(gc, gs),
                                             orc.mxfp8_dequantize(wc, ws).T.copy()))
    assert not np.array_equal(planted, ref_dx)


def test_grouped_chain_is_per_expert_on_the_grid(orc):
    """Three experts of 64, 0 and 96 rows: on the grid every expert's dX rows
    and dW1 are its own fp64 products, and the empty expert's dW1 is zero."""
    rng = np.random.default_rng(30)
    off = np.array([0, 64, 64, 160], np.int32)
    R, f2, d = 160, 64, 96
    dgu, x = _on_grid(rng, R, f2), _on_grid(rng, R, d)
    w1 = np.stack([_on_grid(rng, f2, d) for _ in range(3)])
    r = orc.expert_bwd_gemm1(_bits(dgu), _bits(x), _bits(w1), expert_off=off, seed=3, offset=6)
    for e in range(3):
        s = slice(off[e], off[e + 1])
        dx = dgu[s].astype(np.float64) @ w1[e].astype(np.float64)
        ref = torch.from_numpy(dx).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(r["dx"][s], ref), e
        dw = dgu[s].astype(np.float64).T @ x[s].astype(np.float64)
        assert np.array_equal(r["dw1"][e], dw.astype(np.float32)), e
    assert not r["dw1"][1].any()

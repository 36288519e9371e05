"""Pins for the oracle's routing, permutation, GEMM, SwiGLU and combine.

Pins: scipy's softmax and numpy's stable sort (library routines), numpy's
matmul of the dequantized operands (library), torch's silu (library), the
E = 1 / k = 1 special case (a dense NVFP4 MLP), one-hot combine payloads, and
the model shape the pages print (10100.com 'PART 01': 384 experts, top-8).
"""
import json
import os

import numpy as np
import scipy.special
import torch

from precision_moe_numerics_quantize_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))


def test_full_size_shape_matches_pages():
    s = synth.SHAPES["full_moe"]
    assert s.E == GOLD["experts"]["value"] and s.k == GOLD["top_k"]["value"]
    # last 16.6% of 48 layers -> the last 8 layers stay in MXFP8
    assert int(np.ceil(GOLD["mxfp8_tail_layer_fraction_percent"]["value"] / 100 *
                       GOLD["layers"]["value"])) == 8


def test_route_matches_library(orc):
    logits = synth.logits_uniform_np(2, 64, 32)
    logits[5, 3] = logits[5, 9] = logits[5].max() + 1.0  # a tie: lower id first
    idx, w = orc.route(logits, 4, renorm=0)
    p = scipy.special.softmax(logits.astype(np.float64), axis=1)
    order = np.argsort(-logits, axis=1, kind="stable")[:, :4]
    assert np.array_equal(idx, order)
    assert idx[5, 0] == 3 and idx[5, 1] == 9
    assert np.allclose(w, np.take_along_axis(p, order, 1), rtol=1e-14, atol=0)
    idx2, w2 = orc.route(logits, 4, renorm=1)
    assert np.array_equal(idx2, idx)
    assert np.allclose(w2.sum(1), 1.0, rtol=1e-14)
    assert np.allclose(w2, w / w.sum(1, keepdims=True), rtol=1e-14)


def test_permute_invariants(orc):
    logits = synth.logits_zipf_np(3, 300, 16)
    idx, _ = orc.route(logits, 3)
    off, pos, tok = orc.permute(idx, 16)
    cnt = np.bincount(idx.ravel(), minlength=16)
    assert np.all(off % 128 == 0)
    assert np.array_equal(np.diff(off), (cnt + 127) // 128 * 128)
    flat = pos.ravel()
    assert len(np.unique(flat)) == flat.size
    assert np.array_equal(tok[flat], np.repeat(np.arange(300), 3))
    assert (tok >= 0).sum() == 900
    # rows of each expert in ascending (token, slot) order == a stable sort by expert
    order = np.argsort(idx.ravel(), kind="stable")
    rows = np.concatenate([off[e] + np.arange(cnt[e]) for e in range(16)])
    assert np.array_equal(flat[order], rows)


def test_gemm_matches_numpy(orc):
    rng = np.random.default_rng(0)
    A = rng.standard_normal((7, 33))
    B = rng.standard_normal((5, 33))
    assert np.allclose(orc.gemm_f64(A, B), A @ B.T, rtol=1e-13, atol=1e-13)


def test_swiglu_matches_torch(orc):
    g = np.linspace(-30, 30, 301)
    u = np.linspace(2, -3, 301)
    ref = (torch.nn.functional.silu(torch.from_numpy(g)) * torch.from_numpy(u)).numpy()
    got = np.array([orc.swiglu(a, b) for a, b in zip(g, u)])
    assert np.allclose(got, ref, rtol=1e-14, atol=1e-300)


def _quant_weights(orc, seed, tag, e, rows, cols):
    w = synth.bf16_bits_to_f32(synth.expert_weight_np(seed, tag, e, rows, cols))
    return orc.nvfp4_quantize(w)


def test_expert_ffn_matches_dense_reference(orc):
    """One expert at a tiny size against numpy: dequantize the operands, matmul,
    SwiGLU, bf16 rounding, requantize, matmul."""
    n, d, f = 16, 64, 32
    x = synth.bf16_bits_to_f32(synth.rows_np(0, synth.TAG_X, 0, n, d, 1.0))
    xq, xs, xts = orc.nvfp4_quantize(x)
    w1q, w1s, w1t = _quant_weights(orc, 1, synth.TAG_W1, 0, 2 * f, d)
    w2q, w2s, w2t = _quant_weights(orc, 1, synth.TAG_W2, 0, d, f)
    r = orc.expert_ffn(xq, xs, xts, w1q, w1s, w1t, w2q, w2s, w2t)
    A = orc.nvfp4_to_f64(xq, xs, xts, n, d)
    W1 = orc.nvfp4_to_f64(w1q, w1s, w1t, 2 * f, d)
    gu = A @ W1.T
    g, u = gu[:, :f], gu[:, f:]
    h = (torch.nn.functional.silu(torch.from_numpy(g)) * torch.from_numpy(u)).numpy()
    # h is rounded once from fp64 to bf16 (half an ulp, 2^-9 relative); the two
    # fp64 sums differ only in summation order (1e-12 of sum |a b|)
    mag1 = np.abs(A) @ np.abs(W1).T
    hv = synth.bf16_bits_to_f32(r["h"]).astype(np.float64)
    slack = 1e-12 * (mag1[:, :f] * np.abs(u) + mag1[:, f:] * np.abs(g))
    assert np.all(np.abs(hv - h) <= np.abs(h) * 2.0 ** -8 + slack + 1e-30)
    hq, hs, hts = orc.nvfp4_quantize(synth.bf16_bits_to_f32(r["h"]))
    assert np.array_equal(hq, r["hq"]) and np.array_equal(hs, r["hq_sc"]) and hts == r["h_ts"]
    H = orc.nvfp4_to_f64(hq, hs, hts, n, f)
    W2 = orc.nvfp4_to_f64(w2q, w2s, w2t, d, f)
    y = H @ W2.T
    yv = synth.bf16_bits_to_f32(r["y"]).astype(np.float64)
    slack = 1e-12 * (np.abs(H) @ np.abs(W2).T)
    assert np.all(np.abs(yv - y) <= np.abs(y) * 2.0 ** -8 + slack + 1e-30)


def _mx_decode_torch(codes, scales):
    """MXFP8 decoded with torch's float8_e4m3fn and numpy powers of two."""
    v = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return v * np.repeat(np.ldexp(1.0, scales.astype(np.int64) - 127), 32, axis=1)


def _mx_quantize_torch(x):
    """MXFP8 with round-to-nearest-even along rows: the smallest k with
    amax <= 448 * 2^k per 32-block, codes by torch's float8_e4m3fn cast."""
    rows, cols = x.shape
    blocks = x.astype(np.float64).reshape(rows, cols // 32, 32)
    amax = np.abs(blocks).max(axis=2)
    with np.errstate(divide="ignore"):
        k = np.where(amax > 0, np.ceil(np.log2(amax / 448.0)), -127.0)
    k = np.clip(k, -127, 127).astype(np.int64)
    v = blocks * np.ldexp(1.0, -k)[:, :, None]
    codes = torch.from_numpy(v.reshape(rows, cols)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, (k + 127).astype(np.uint8)


def test_expert_ffn_mxfp8_matches_dense_reference(orc):
    """The MXFP8 expert forward at a tiny size against an independent dense
    reference: operands decoded with torch's float8_e4m3fn, numpy matmul, torch
    SwiGLU, h requantized by a torch cast, matmul."""
    n, d, f = 16, 64, 64
    x = synth.bf16_bits_to_f32(synth.rows_np(0, synth.TAG_X, 0, n, d, 1.0))
    xq, xs = orc.mxfp8_quantize(x, axis=0, rounding=0)
    W1 = synth.bf16_bits_to_f32(synth.expert_weight_np(1, synth.TAG_W1, 0, 2 * f, d))
    W2 = synth.bf16_bits_to_f32(synth.expert_weight_np(1, synth.TAG_W2, 0, d, f))
    w1q, w1s = orc.mxfp8_quantize(W1, axis=0, rounding=0)
    w2q, w2s = orc.mxfp8_quantize(W2, axis=0, rounding=0)
    r = orc.expert_ffn_mxfp8(xq, xs, w1q, w1s, w2q, w2s)
    A = _mx_decode_torch(xq, xs)
    B1 = _mx_decode_torch(w1q, w1s)
    gu = A @ B1.T
    g, u = gu[:, :f], gu[:, f:]
    h = (torch.nn.functional.silu(torch.from_numpy(g)) * torch.from_numpy(u)).numpy()
    mag1 = np.abs(A) @ np.abs(B1).T
    hv = synth.bf16_bits_to_f32(r["h"]).astype(np.float64)
    slack = 1e-12 * (mag1[:, :f] * np.abs(u) + mag1[:, f:] * np.abs(g))
    assert np.all(np.abs(hv - h) <= np.abs(h) * 2.0 ** -8 + slack + 1e-30)
    hq, hs = _mx_quantize_torch(synth.bf16_bits_to_f32(r["h"]))
    assert np.array_equal(hq, r["hq"]) and np.array_equal(hs, r["hq_sc"])
    H = _mx_decode_torch(hq, hs)
    B2 = _mx_decode_torch(w2q, w2s)
    y = H @ B2.T
    yv = synth.bf16_bits_to_f32(r["y"]).astype(np.float64)
    slack = 1e-12 * (np.abs(H) @ np.abs(B2).T)
    assert np.all(np.abs(yv - y) <= np.abs(y) * 2.0 ** -8 + slack + 1e-30)
    # y rows requested one by one equal the full result
    sel = np.array([3, 0, 11], np.int32)
    assert np.array_equal(orc.expert_ffn_mxfp8(xq, xs, w1q, w1s, w2q, w2s, rows_out=sel)["y"],
                          r["y"][sel])


def test_single_expert_top1_is_dense_mlp(orc):
    """E = 1, k = 1, renormalized weights: the layer reduces to out = MLP(x)."""
    T, d, f = 24, 64, 32
    logits = np.zeros((T, 1), np.float32)
    idx, w = orc.route(logits, 1)
    assert np.all(idx == 0) and np.all(w == 1.0)
    off, pos, tok = orc.permute(idx, 1)
    assert np.array_equal(pos.ravel(), np.arange(T))
    x = synth.bf16_bits_to_f32(synth.rows_np(0, synth.TAG_X, 0, T, d, 1.0))
    xq, xs, xts = orc.nvfp4_quantize(x)
    w1q, w1s, w1t = _quant_weights(orc, 1, synth.TAG_W1, 0, 2 * f, d)
    w2q, w2s, w2t = _quant_weights(orc, 1, synth.TAG_W2, 0, d, f)
    r = orc.expert_ffn(xq, xs, xts, w1q, w1s, w1t, w2q, w2s, w2t)
    out = orc.combine(r["y"], pos, w)
    assert np.array_equal(out, r["y"])


def test_combine_one_hot(orc):
    T, k, d = 6, 3, 32
    rows = T * k + 5
    y = np.zeros((rows, d), np.uint16)
    pos = np.arange(T * k, dtype=np.int32).reshape(T, k)[:, ::-1].copy()
    w = np.full((T, k), 0.0)
    for t in range(T):
        for j in range(k):
            y[pos[t, j], (t + j) % d] = synth.f32_to_bf16_bits(np.array([1.0 + j], np.float32))[0]
            w[t, j] = 2.0 ** -j
    out = synth.bf16_bits_to_f32(orc.combine(y, pos, w))
    for t in range(T):
        for j in range(k):
            assert out[t, (t + j) % d] == (1.0 + j) * 2.0 ** -j
    assert np.count_nonzero(out) == T * k


def test_swiglu_bwd_matches_autograd(orc):
    """The SwiGLU backward against torch autograd of silu(g) * u in fp64, both
    rounded once to bf16 by torch; inputs include large |g| where s(g)
    saturates, and dh = 0."""
    rows, f = 64, 96
    gu_bits = synth.rows_np(4, synth.TAG_ACT, 0, rows, 2 * f, 2.0)
    gu_bits[0, :8] = synth.f32_to_bf16_bits(np.array([-100, -30, -8, 0, 8, 30, 100, 1e-3],
                                                     np.float32))
    dh_bits = synth.rows_np(5, synth.TAG_ACT, 0, rows, f, 0.5)
    dh_bits[1, :] = 0
    got = orc.swiglu_bwd(gu_bits, dh_bits)
    gu = torch.from_numpy(synth.bf16_bits_to_f32(gu_bits).astype(np.float64))
    g = gu[:, :f].clone().requires_grad_(True)
    u = gu[:, f:].clone().requires_grad_(True)
    dh = torch.from_numpy(synth.bf16_bits_to_f32(dh_bits).astype(np.float64))
    (torch.nn.functional.silu(g) * u).backward(dh)
    ref = torch.cat([g.grad, u.grad], dim=1).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
    assert not synth.bf16_bits_to_f32(got[1]).any()

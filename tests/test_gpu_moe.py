"""GPU parity of routing, dispatch (with fused NVFP4 quantization), the expert
FFN and the combine against the oracle.

Integer outputs (top-k ids, expert offsets, slot positions, token map, codes,
scales) are bit-exact. Router weights agree to 4e-6 relative (fp32 exp vs fp64).
The expert FFN is checked stage by stage against the oracle run on the
oracle's own inputs:
  h    within one bf16 ulp plus the propagated accumulator tolerance
       (1e-5 * sum |a b| on g and u, through dh/dg and dh/du);
  h_amax equal to max |h| of the GPU's own h (the fused reduction);
  hq   every 16-element block whose h is bit-identical to the oracle's, in an
       expert whose tensor scale matches, has the oracle's codes and scale;
       codes differ from the oracle's in under 1e-3 of all positions;
  y    within one bf16 ulp plus 1e-5 * sum |a b| on rows whose hq agrees; the
       number of experts and rows this covers is asserted, not skipped.
An fp32 accumulator rounded once to bf16 and an fp64 value rounded once to
bf16 differ by at most one bf16 ulp (of the larger magnitude) plus the
accumulator's own error, which is the bound used for h and y.
"""
import numpy as np
import pytest
import torch

from precision_moe_numerics_quantize_b200 import synth
from tests.gpu_helpers import (dev_bf16, dev_f32, dev_u8, host_bits, host_u8, mma_to_rowmajor,
                               rowmajor_to_mma, sync)

pytestmark = pytest.mark.gpu


def _f32(bits):
    return synth.bf16_bits_to_f32(bits)


def _run_route(dev, lib, logits, x_bits, k, renorm=1):
    T, E = logits.shape
    d = x_bits.shape[1]
    R = lib.max_rows(T, k, E)
    o = {
        "idx": torch.empty(T, k, dtype=torch.int32, device=dev),
        "w": torch.empty(T, k, dtype=torch.float32, device=dev),
        "off": torch.empty(E + 1, dtype=torch.int32, device=dev),
        "pos": torch.empty(T, k, dtype=torch.int32, device=dev),
        "tok": torch.empty(R, dtype=torch.int32, device=dev),
        "xq": torch.full((R, d // 2), 0xAB, dtype=torch.uint8, device=dev),
        "xq_sc": torch.full((R * d // 16,), 0xAB, dtype=torch.uint8, device=dev),
        "x_ts": torch.empty(1, device=dev),
    }
    ws = torch.empty(lib.moe_route_permute_workspace_size(T, E, k), dtype=torch.uint8, device=dev)
    lib.moe_route_permute(dev_f32(logits, dev), dev_bf16(x_bits, dev), k, renorm, o["idx"], o["w"],
                          o["off"], o["pos"], o["tok"], o["xq"], o["xq_sc"], o["x_ts"], ws)
    sync()
    return o, R


def _oracle_dispatch(orc, logits, x_bits, k, renorm=1):
    T, E = logits.shape
    idx, w = orc.route(logits, k, renorm)
    off, pos, tok = orc.permute(idx, E)
    xc, xs, xts = orc.nvfp4_quantize(_f32(x_bits))
    return idx, w, off, pos, tok, xc, xs, xts


@pytest.mark.parametrize("router,T,E,k,d,renorm", [
    ("uniform", 2048, 32, 4, 1024, 1), ("zipf", 2048, 32, 4, 1024, 1),
    ("zipf", 300, 64, 8, 256, 0), ("uniform", 5, 3, 3, 64, 1), ("uniform", 64, 1, 1, 128, 1),
    ("zipf", 1000, 384, 8, 128, 1),
])
def test_route_permute_bitexact(dev, lib, orc, router, T, E, k, d, renorm):
    logits = (synth.logits_uniform_np(2, T, E) if router == "uniform"
              else synth.logits_zipf_np(2, T, E))
    if T > 3 and E > 3:
        logits[3, :3] = logits[3].max() + 1.0  # three-way tie at the top: lower ids first
    x_bits = synth.rows_np(0, synth.TAG_X, 0, T, d, 1.0)
    o, R = _run_route(dev, lib, logits, x_bits, k, renorm)
    idx, w, off, pos, tok, xc, xs, xts = _oracle_dispatch(orc, logits, x_bits, k, renorm)
    assert np.array_equal(o["idx"].cpu().numpy(), idx)
    assert np.allclose(o["w"].cpu().numpy(), w, rtol=4e-6, atol=1e-30)
    assert np.array_equal(o["off"].cpu().numpy(), off)
    assert np.array_equal(o["pos"].cpu().numpy(), pos)
    assert np.array_equal(o["tok"].cpu().numpy(), tok)
    assert o["x_ts"].item() == xts
    used = int(off[-1])
    gq = host_u8(o["xq"])[:used]
    gs = mma_to_rowmajor(host_u8(o["xq_sc"]), R, d // 16)[:used]
    rows_tok = tok[:used]
    real = rows_tok >= 0
    assert np.array_equal(gq[real], xc[rows_tok[real]])
    assert np.array_equal(gs[real], xs[rows_tok[real]])
    assert not gq[~real].any() and not gs[~real].any()


def test_route_permute_no_tokens(dev, lib):
    logits = np.zeros((0, 8), np.float32)
    x_bits = np.zeros((0, 64), np.uint16)
    T, E, k, d = 0, 8, 2, 64
    R = lib.max_rows(T, k, E)
    off = torch.full((E + 1,), -5, dtype=torch.int32, device=dev)
    tok = torch.empty(R, dtype=torch.int32, device=dev)
    xq = torch.empty(R, d // 2, dtype=torch.uint8, device=dev)
    xs = torch.empty(R * d // 16, dtype=torch.uint8, device=dev)
    ts = torch.empty(1, device=dev)
    ws = torch.empty(max(16, lib.moe_route_permute_workspace_size(T, E, k)), dtype=torch.uint8,
                     device=dev)
    e = torch.empty(0, dtype=torch.int32, device=dev)
    lib.moe_route_permute(torch.empty(0, 8, device=dev), torch.empty(0, 64, dtype=torch.bfloat16,
                                                                     device=dev),
                          k, 1, e, torch.empty(0, device=dev), off, e, tok, xq, xs, ts, ws)
    sync()
    assert not off.any() and (tok == -1).all() and ts.item() == 1.0


def test_combine(dev, lib, orc):
    T, E, k, d = 512, 16, 4, 512
    logits = synth.logits_zipf_np(4, T, E)
    idx, w = orc.route(logits, k)
    off, pos, tok = orc.permute(idx, E)
    R = len(tok)
    y = synth.rows_np(8, synth.TAG_ACT, 0, R, d, 0.5)
    wf = w.astype(np.float32)
    out = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    lib.moe_combine(dev_bf16(y, dev), torch.tensor(pos, device=dev), dev_f32(wf, dev), out)
    sync()
    ref = orc.combine(y, pos, wf.astype(np.float64))
    got = _f32(host_bits(out)).astype(np.float64)
    refv = _f32(ref).astype(np.float64)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(refv), 1e-38))) - 7)
    # fp32 slot-order accumulation: k roundings of at most 2^-24 of the
    # running magnitude, then one bf16 rounding
    mag = np.einsum("tj,tjd->td", np.abs(wf.astype(np.float64)), np.abs(_f32(y)[pos].astype(np.float64)))
    assert np.all(np.abs(got - refv) <= ulp + 2 * k * 2.0 ** -24 * mag)


def _quant_experts(orc, seed, tag, E, rows, cols):
    cs, ss, ts, dq = [], [], [], []
    for e in range(E):
        W = _f32(synth.expert_weight_np(seed, tag, e, rows, cols))
        c, s, t = orc.nvfp4_quantize(W)
        cs.append(c); ss.append(s); ts.append(t)
    return np.concatenate(cs), np.concatenate(ss), np.array(ts, np.float32)


def _ulp(v):
    return np.exp2(np.floor(np.log2(np.maximum(np.abs(v), 1e-38))) - 7)


def _ulp2(a, b):
    """One bf16 ulp at the larger of two magnitudes."""
    return _ulp(np.maximum(np.abs(a), np.abs(b)))


def _blocks_same(a, b, n, blk):
    """Per (row, block of blk elements): all elements equal."""
    return np.all((a == b).reshape(n, -1, blk), axis=2)


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("router", ["uniform", "zipf"])
def test_expert_fwd_small_layer(dev, lib, orc, router, fused):
    """2048 tokens, d = 1024, f = 512, 32 experts, top-4; the default entry
    point and the one with the requantization fused into GEMM1."""
    sh = synth.SHAPES["small_moe"]
    T, d, f, E, k = sh.T, sh.d, sh.f, sh.E, sh.k
    logits = (synth.logits_uniform_np(2, T, E) if router == "uniform"
              else synth.logits_zipf_np(2, T, E))
    x_bits = synth.rows_np(0, synth.TAG_X, 0, T, d, 1.0)
    idx, w, off, pos, tok, xc, xs, xts = _oracle_dispatch(orc, logits, x_bits, k)
    R = lib.max_rows(T, k, E)
    xq = np.zeros((R, d // 2), np.uint8)
    xsc = np.zeros((R, d // 16), np.uint8)
    real = np.where(tok >= 0)[0]
    xq[real] = xc[tok[real]]
    xsc[real] = xs[tok[real]]
    w1c, w1s, w1t = _quant_experts(orc, 1, synth.TAG_W1, E, 2 * f, d)
    w2c, w2s, w2t = _quant_experts(orc, 1, synth.TAG_W2, E, d, f)
    # rows past the last expert are never written: zero-filled so that the
    # host copies below convert cleanly
    h = torch.zeros(R, f, dtype=torch.bfloat16, device=dev)
    hq = torch.empty(R, f // 2, dtype=torch.uint8, device=dev)
    hq_sc = torch.empty(R * f // 16, dtype=torch.uint8, device=dev)
    h_amax = torch.empty(E, device=dev)
    h_ts = torch.empty(E, device=dev)
    y = torch.zeros(R, d, dtype=torch.bfloat16, device=dev)
    args = [dev_u8(xq, dev), dev_u8(rowmajor_to_mma(xsc), dev), dev_f32([xts], dev),
            torch.tensor(off, device=dev), E, d, f, dev_u8(w1c, dev),
            dev_u8(rowmajor_to_mma(w1s), dev), dev_f32(w1t, dev), dev_u8(w2c, dev),
            dev_u8(rowmajor_to_mma(w2s), dev), dev_f32(w2t, dev), h, hq, hq_sc, h_amax, h_ts, y, R]
    if fused:
        ws = torch.empty(lib.moe_expert_fwd_fused_requant_workspace_size(E), dtype=torch.uint8,
                         device=dev)
        lib.moe_expert_fwd_fused_requant(*args, ws)
    else:
        lib.moe_expert_fwd(*args)
    sync()
    gh = _f32(host_bits(h)).astype(np.float64)
    ghq = host_u8(hq)
    ghs = mma_to_rowmajor(host_u8(hq_sc), R, f // 16)
    gy = _f32(host_bits(y)).astype(np.float64)
    gam = h_amax.cpu().numpy()
    gts = h_ts.cpu().numpy()
    ghb = host_bits(h)
    flips = total = 0
    experts_used = experts_y = rows_used = rows_y = blocks = total_blocks = 0
    for e in range(E):
        rows = np.arange(off[e], off[e + 1])
        rows_real = rows[tok[rows] >= 0]
        if len(rows_real) == 0:
            assert gam[e] == 0.0
            continue
        n = len(rows_real)
        experts_used += 1
        rows_used += n
        assert np.isfinite(gh[rows_real]).all() and np.isfinite(gy[rows_real]).all(), e
        r = orc.expert_ffn(xq[rows_real], xsc[rows_real], xts, w1c[e * 2 * f:(e + 1) * 2 * f],
                           w1s[e * 2 * f:(e + 1) * 2 * f], w1t[e], w2c[e * d:(e + 1) * d],
                           w2s[e * d:(e + 1) * d], w2t[e])
        # h: one bf16 ulp + accumulator tolerance propagated through SwiGLU
        A = orc.nvfp4_to_f64(xq[rows_real], xsc[rows_real], xts, n, d)
        W1 = orc.nvfp4_to_f64(w1c[e * 2 * f:(e + 1) * 2 * f], w1s[e * 2 * f:(e + 1) * 2 * f],
                              w1t[e], 2 * f, d)
        gu = orc.gemm_f64(A, W1)
        mag = orc.gemm_f64(np.abs(A), np.abs(W1)) * 1e-5
        g, u = gu[:, :f], gu[:, f:]
        sig = 1.0 / (1.0 + np.exp(-g))
        dh_dg = np.abs((sig * (1 + g * (1 - sig))) * u)
        dh_du = np.abs(g * sig)
        href = _f32(r["h"]).astype(np.float64)
        tol = _ulp2(href, gh[rows_real]) + dh_dg * mag[:, :f] + dh_du * mag[:, f:] + 1e-30
        assert np.all(np.abs(gh[rows_real] - href) <= tol), e
        # fused amax equals the max of the GPU's own h; padding rows are zero
        assert gam[e] == np.abs(gh[rows]).max()
        assert not gh[rows[tok[rows] < 0]].any()
        assert gts[e] == np.float32(np.float32(gam[e]) / np.float32(2688.0))
        flips += int(np.sum(ghq[rows_real] != r["hq"]))
        total += r["hq"].size
        if gts[e] != r["h_ts"]:
            continue  # the expert's tensor scale moved: no code is comparable
        # requantized codes: every 16-block whose h is bit-identical has the
        # oracle's codes (8 bytes) and scale
        hb_same = _blocks_same(ghb[rows_real], r["h"], n, 16)
        codes_same = _blocks_same(ghq[rows_real], r["hq"], n, 8)
        sc_same = ghs[rows_real] == r["hq_sc"]
        assert np.all(codes_same[hb_same] & sc_same[hb_same]), e
        blocks += int(hb_same.sum())
        total_blocks += hb_same.size
        # y on rows whose hq agrees
        same = np.all(ghq[rows_real] == r["hq"], axis=1) & np.all(ghs[rows_real] == r["hq_sc"],
                                                                   axis=1)
        H = orc.nvfp4_to_f64(r["hq"], r["hq_sc"], r["h_ts"], n, f)
        W2 = orc.nvfp4_to_f64(w2c[e * d:(e + 1) * d], w2s[e * d:(e + 1) * d], w2t[e], d, f)
        ymag = orc.gemm_f64(np.abs(H), np.abs(W2)) * 1e-5
        yref = _f32(r["y"]).astype(np.float64)
        ok = np.abs(gy[rows_real] - yref) <= _ulp2(yref, gy[rows_real]) + ymag + 1e-30
        assert np.all(ok[same]), e
        assert not gy[rows[tok[rows] < 0]].any()
        experts_y += 1
        rows_y += int(same.sum())
    assert flips <= 1e-3 * total, (flips, total)
    # h agrees bit for bit in almost every block, and y was compared on
    # nearly every expert and row (a tensor-scale mismatch is rare: it needs
    # the expert's largest |h| to be one of the values one ulp apart)
    assert blocks >= 0.99 * total_blocks, (blocks, total_blocks)
    assert experts_y >= 0.9 * experts_used, (experts_y, experts_used)
    assert rows_y >= 0.9 * rows_used, (rows_y, rows_used)


def _mx_experts(orc, seed, tag, E, rows, cols):
    cs, ss = [], []
    for e in range(E):
        W = _f32(synth.expert_weight_np(seed, tag, e, rows, cols))
        c, s = orc.mxfp8_quantize(W, axis=0, rounding=0)
        cs.append(c); ss.append(s)
    return np.concatenate(cs), np.concatenate(ss)


def _mx_f64(orc, codes, scales):
    return orc.mxfp8_dequantize(codes, scales).astype(np.float64)


@pytest.mark.parametrize("router", ["uniform", "zipf"])
def test_expert_fwd_mxfp8_small_layer(dev, lib, orc, router):
    """MXFP8 expert forward, 2048 tokens, d = 1024, f = 512, 32 experts, top-4.
    h within one bf16 ulp plus the accumulator tolerance through SwiGLU; the
    fused h_amax equals max|h|; every 32-block of hq whose h block agrees with
    the oracle's has the oracle's codes and scale; y on rows whose hq agrees."""
    sh = synth.SHAPES["small_moe"]
    T, d, f, E, k = sh.T, sh.d, sh.f, sh.E, sh.k
    logits = (synth.logits_uniform_np(2, T, E) if router == "uniform"
              else synth.logits_zipf_np(2, T, E))
    x = _f32(synth.rows_np(0, synth.TAG_X, 0, T, d, 1.0))
    idx, _ = orc.route(logits, k)
    off, pos, tok = orc.permute(idx, E)
    xc_t, xs_t = orc.mxfp8_quantize(x, axis=0, rounding=0)
    R = lib.max_rows(T, k, E)
    xq = np.zeros((R, d), np.uint8)
    xsc = np.zeros((R, d // 32), np.uint8)
    real = np.where(tok >= 0)[0]
    xq[real] = xc_t[tok[real]]
    xsc[real] = xs_t[tok[real]]
    w1c, w1s = _mx_experts(orc, 1, synth.TAG_W1, E, 2 * f, d)
    w2c, w2s = _mx_experts(orc, 1, synth.TAG_W2, E, d, f)
    h = torch.zeros(R, f, dtype=torch.bfloat16, device=dev)
    h_amax = torch.empty(E, device=dev)
    hq = torch.empty(R, f, dtype=torch.uint8, device=dev)
    hq_sc = torch.empty(R * f // 32, dtype=torch.uint8, device=dev)
    y = torch.zeros(R, d, dtype=torch.bfloat16, device=dev)
    lib.moe_expert_fwd_mxfp8(dev_u8(xq, dev), dev_u8(rowmajor_to_mma(xsc), dev),
                             torch.tensor(off, device=dev), E, d, f, dev_u8(w1c, dev),
                             dev_u8(rowmajor_to_mma(w1s), dev), dev_u8(w2c, dev),
                             dev_u8(rowmajor_to_mma(w2s), dev), h, h_amax, hq, hq_sc, y, R)
    sync()
    gh = _f32(host_bits(h)).astype(np.float64)
    ghb = host_bits(h)
    ghq = host_u8(hq)
    ghs = mma_to_rowmajor(host_u8(hq_sc), R, f // 32)
    gy = _f32(host_bits(y)).astype(np.float64)
    gam = h_amax.cpu().numpy()
    blocks = total_blocks = rows_y = rows_used = 0
    for e in range(E):
        rows = np.arange(off[e], off[e + 1])
        rows_real = rows[tok[rows] >= 0]
        if len(rows_real) == 0:
            assert gam[e] == 0.0
            continue
        n = len(rows_real)
        assert np.isfinite(gh[rows_real]).all() and np.isfinite(gy[rows_real]).all(), e
        W1 = slice(e * 2 * f, (e + 1) * 2 * f)
        W2 = slice(e * d, (e + 1) * d)
        r = orc.expert_ffn_mxfp8(xq[rows_real], xsc[rows_real], w1c[W1], w1s[W1], w2c[W2],
                                 w2s[W2])
        A = _mx_f64(orc, xq[rows_real], xsc[rows_real])
        B1 = _mx_f64(orc, w1c[W1], w1s[W1])
        gu = orc.gemm_f64(A, B1)
        mag = orc.gemm_f64(np.abs(A), np.abs(B1)) * 1e-5
        g, u = gu[:, :f], gu[:, f:]
        sig = 1.0 / (1.0 + np.exp(-g))
        href = _f32(r["h"]).astype(np.float64)
        tol = (_ulp2(href, gh[rows_real]) + np.abs(sig * (1 + g * (1 - sig)) * u) * mag[:, :f]
               + np.abs(g * sig) * mag[:, f:] + 1e-30)
        assert np.all(np.abs(gh[rows_real] - href) <= tol), e
        assert gam[e] == np.abs(gh[rows]).max()
        assert not gh[rows[tok[rows] < 0]].any()
        # hq per 32-block: where the block of h is bit-identical, so are the
        # block's codes and scale
        hb_same = np.all((ghb[rows_real] == r["h"]).reshape(n, f // 32, 32), axis=2)
        codes_same = np.all((ghq[rows_real] == r["hq"]).reshape(n, f // 32, 32), axis=2)
        sc_same = ghs[rows_real] == r["hq_sc"]
        assert np.all(codes_same[hb_same] & sc_same[hb_same]), e
        blocks += int(hb_same.sum())
        total_blocks += hb_same.size
        # y on rows whose hq agrees
        same = np.all(ghq[rows_real] == r["hq"], axis=1) & np.all(ghs[rows_real] == r["hq_sc"], axis=1)
        H = _mx_f64(orc, r["hq"], r["hq_sc"])
        B2 = _mx_f64(orc, w2c[W2], w2s[W2])
        ymag = orc.gemm_f64(np.abs(H), np.abs(B2)) * 1e-5
        yref = _f32(r["y"]).astype(np.float64)
        ok = np.abs(gy[rows_real] - yref) <= _ulp2(yref, gy[rows_real]) + ymag + 1e-30
        assert np.all(ok[same]), e
        assert not gy[rows[tok[rows] < 0]].any()
        rows_y += int(same.sum())
        rows_used += n
    assert rows_y >= 0.9 * rows_used, (rows_y, rows_used)
    # h itself agrees bit for bit in almost every block
    assert blocks >= 0.99 * total_blocks, (blocks, total_blocks)

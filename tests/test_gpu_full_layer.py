"""Full-size parity: the 16384-token, 384-expert, top-8 layer (d = 4096,
f = 2560, SwiGLU) built by the benchmark's own set-up and run with its launch
sequence (route/permute + quantize, expert FFN, combine), for the uniform and
the Zipf router.

The oracle cannot run the whole layer in seconds, so it checks what it can
compute one piece at a time:
  routing     top-k ids, offsets, slot positions and token map over all
              16384 tokens, bit-exact; router weights to 4e-6 relative;
  dispatch    the global tensor scale, and the NVFP4 codes and scales of every
              routed row of the sampled experts, bit-exact; padding rows zero;
  weights     the sampled experts' W1 and W2 codes and scales, bit-exact;
  expert FFN  three experts per router (for Zipf the lightest, a middle one and
              the heaviest, about 14000 rows): the oracle runs each expert's
              GEMM1 over all its rows (the expert's tensor scale needs every
              h), then h on sampled rows to one bf16 ulp plus the accumulator
              tolerance, h_amax, h_ts, the requantized codes block by block
              over all rows, and y on the sampled rows to one bf16 ulp plus the
              accumulator tolerance; every expert's y is compared;
  combine     256 sampled tokens of a full-size combine of a seeded y;
  repeat      a second pass of the layer gives bit-identical outputs.
The inputs (logits, x, bf16 weights) are the seeded synthetic tensors that
both sides read; nothing the oracle consumes comes from the CUDA kernels.
"""
import numpy as np
import pytest
import torch

import bench
from precision_moe_numerics_quantize_b200 import synth
from tests.gpu_helpers import host_bits, host_u8, mma_rows_to_rowmajor, mma_to_rowmajor, sync

pytestmark = pytest.mark.gpu

SHAPE = synth.SHAPES["full_moe"]
SAMPLE_ROWS = 48


def _f32(bits):
    return synth.bf16_bits_to_f32(bits)


def _ulp(v):
    return np.exp2(np.floor(np.log2(np.maximum(np.abs(v), 1e-38))) - 7)


def _ulp2(a, b):
    """One bf16 ulp at the larger of two magnitudes."""
    return _ulp(np.maximum(np.abs(a), np.abs(b)))


@pytest.fixture(scope="module", params=["uniform", "zipf"])
def layer(request, dev, lib, orc):
    router = request.param
    L = bench.setup_layer(lib, synth, torch, dev, SHAPE, router)
    for _, fn in bench.layer_calls(lib, L):
        fn()
    sync()
    T, E, k = SHAPE.T, SHAPE.E, SHAPE.k
    logits = L["logits_host"].numpy()
    idx, w = orc.route(logits, k)
    off, pos, tok = orc.permute(idx, E)
    x = _f32(host_bits(L["x_host"]))
    ref = {"idx": idx, "w": w, "off": off, "pos": pos, "tok": tok, "x": x,
           "x_amax": orc.amax(x)}
    cnt = np.diff(off)
    real_cnt = np.array([int(np.sum(tok[off[e]:off[e + 1]] >= 0)) for e in range(E)])
    if router == "uniform":
        experts = [0, E // 2 - 1, E - 1]
    else:
        order = np.argsort(real_cnt, kind="stable")
        experts = [int(order[0]), int(order[E // 2]), int(order[-1])]
    yield {"router": router, "L": L, "ref": ref, "experts": experts, "real_cnt": real_cnt,
           "cnt": cnt}
    del L
    torch.cuda.empty_cache()


def _oracle_weights(orc, dev, tag, e, rows, cols):
    wb = synth.expert_weight_torch(1, tag, e, rows, cols, dev)
    return orc.nvfp4_quantize(_f32(host_bits(wb)))


def _gpu_weights(q, e, rows, cols):
    c, s, t = q
    codes = host_u8(c[e * rows:(e + 1) * rows])
    per = rows * cols // 16
    sc = mma_to_rowmajor(host_u8(s[e * per:(e + 1) * per]), rows, cols // 16)
    return codes, sc, np.float32(t[e].item())


def test_full_route_and_dispatch(layer, orc):
    L, ref = layer["L"], layer["ref"]
    d = SHAPE.d
    assert np.array_equal(L["idx"].cpu().numpy(), ref["idx"])
    assert np.allclose(L["w"].cpu().numpy(), ref["w"], rtol=4e-6, atol=1e-30)
    assert np.array_equal(L["off"].cpu().numpy(), ref["off"])
    assert np.array_equal(L["pos"].cpu().numpy(), ref["pos"])
    assert np.array_equal(L["tok"].cpu().numpy(), ref["tok"])
    off, tok = ref["off"], ref["tok"]
    _, _, xts = orc.nvfp4_quantize(ref["x"][:1], amax_in=ref["x_amax"])
    assert L["x_ts"].item() == xts
    gsc_all = host_u8(L["xq_sc"])
    for e in layer["experts"]:
        rows = np.arange(off[e], off[e + 1])
        real = rows[tok[rows] >= 0]
        pad = rows[tok[rows] < 0]
        xc, xs, _ = orc.nvfp4_quantize(ref["x"][tok[real]], amax_in=ref["x_amax"])
        gq = host_u8(L["xq"][int(off[e]):int(off[e + 1])])
        gs = mma_rows_to_rowmajor(gsc_all, rows, d // 16)
        assert np.array_equal(gq[real - off[e]], xc), e
        assert np.array_equal(gs[real - off[e]], xs), e
        assert not gq[pad - off[e]].any() and not gs[pad - off[e]].any(), e
    # every padding row of the whole dispatch is zero
    used = int(off[-1])
    pad_rows = torch.from_numpy(np.where(tok[:used] < 0)[0]).to(L["xq"].device)
    assert not L["xq"][pad_rows].any().item()


def test_full_expert_ffn(layer, dev, orc):
    L, ref = layer["L"], layer["ref"]
    d, f = SHAPE.d, SHAPE.f
    off, tok = ref["off"], ref["tok"]
    gam = L["h_amax"].cpu().numpy()
    gts = L["h_ts"].cpu().numpy()
    ghs_all = host_u8(L["hq_sc"])
    rng = np.random.default_rng(11)
    for e in layer["experts"]:
        rows = np.arange(off[e], off[e + 1])
        real = rows[tok[rows] >= 0]
        n = len(real)
        assert n > 0
        # weights: the device quantizer's codes equal the oracle's
        w1c, w1s, w1t = _oracle_weights(orc, dev, synth.TAG_W1, e, 2 * f, d)
        w2c, w2s, w2t = _oracle_weights(orc, dev, synth.TAG_W2, e, d, f)
        g1 = _gpu_weights(L["w1"], e, 2 * f, d)
        g2 = _gpu_weights(L["w2"], e, d, f)
        assert np.array_equal(g1[0], w1c) and np.array_equal(g1[1], w1s) and g1[2] == w1t
        assert np.array_equal(g2[0], w2c) and np.array_equal(g2[1], w2s) and g2[2] == w2t
        xc, xs, xts = orc.nvfp4_quantize(ref["x"][tok[real]], amax_in=ref["x_amax"])
        S = np.sort(rng.choice(n, size=min(SAMPLE_ROWS, n), replace=False))
        # all rows through GEMM1 (the tensor scale of h needs them), y on S
        r = orc.expert_ffn(xc, xs, xts, w1c, w1s, w1t, w2c, w2s, w2t, rows_out=S)
        href_s = _f32(r["h"][S]).astype(np.float64)
        ghb = host_bits(L["h"][int(off[e]):int(off[e + 1])])
        gh = _f32(ghb).astype(np.float64)
        gh_real = gh[real - off[e]]
        assert np.isfinite(gh_real).all(), e
        # h on the sampled rows: one bf16 ulp + accumulator tolerance through SwiGLU
        A = orc.nvfp4_to_f64(xc[S], xs[S], xts, len(S), d)
        W1 = orc.nvfp4_to_f64(w1c, w1s, w1t, 2 * f, d)
        gu = orc.gemm_f64(A, W1)
        mag = orc.gemm_f64(np.abs(A), np.abs(W1)) * 1e-5
        g, u = gu[:, :f], gu[:, f:]
        sig = 1.0 / (1.0 + np.exp(-g))
        tol = (_ulp2(href_s, gh_real[S]) + np.abs(sig * (1 + g * (1 - sig)) * u) * mag[:, :f]
               + np.abs(g * sig) * mag[:, f:] + 1e-30)
        assert np.all(np.abs(gh_real[S] - href_s) <= tol), e
        # fused amax and tensor scale; padding rows of h and y are zero
        assert gam[e] == np.abs(gh).max(), e
        assert gts[e] == np.float32(np.float32(gam[e]) / np.float32(2688.0)), e
        assert not gh[tok[rows] < 0].any(), e
        gy = _f32(host_bits(L["y"][int(off[e]):int(off[e + 1])])).astype(np.float64)
        assert not gy[tok[rows] < 0].any(), e
        # the expert's tensor scale of h: equal to the oracle's (it is the
        # largest |h| over all rows, and h agrees to one ulp)
        assert gts[e] == r["h_ts"], (e, gts[e], r["h_ts"])
        # requantized codes over all rows: every 16-block whose h is
        # bit-identical has the oracle's codes and scale
        ghq = host_u8(L["hq"][int(off[e]):int(off[e + 1])])[real - off[e]]
        ghs = mma_rows_to_rowmajor(ghs_all, real, f // 16)
        flips = int(np.sum(ghq != r["hq"]))
        assert flips <= 1e-3 * r["hq"].size, (e, flips)
        hb_same = np.all((ghb[real - off[e]] == r["h"]).reshape(n, f // 16, 16), axis=2)
        codes_same = np.all((ghq == r["hq"]).reshape(n, f // 16, 8), axis=2)
        assert np.all(codes_same[hb_same] & (ghs == r["hq_sc"])[hb_same]), e
        assert hb_same.sum() >= 0.99 * hb_same.size, (e, int(hb_same.sum()), hb_same.size)
        same = np.all(ghq == r["hq"], axis=1) & np.all(ghs == r["hq_sc"], axis=1)
        # y on the sampled rows whose hq agrees
        H = orc.nvfp4_to_f64(r["hq"][S], r["hq_sc"][S], r["h_ts"], len(S), f)
        W2 = orc.nvfp4_to_f64(w2c, w2s, w2t, d, f)
        ymag = orc.gemm_f64(np.abs(H), np.abs(W2)) * 1e-5
        yref = _f32(r["y"]).astype(np.float64)
        gys = gy[real - off[e]][S]
        assert np.isfinite(gys).all(), e
        ok = np.abs(gys - yref) <= _ulp2(yref, gys) + ymag + 1e-30
        assert np.all(ok[same[S]]), e
        assert same[S].sum() >= 0.75 * len(S), (e, int(same[S].sum()), len(S))


def test_full_layer_repeats_bit_identically(layer, lib):
    L = layer["L"]

    def bits(t):
        return t.view(torch.int16) if t.dtype == torch.bfloat16 else t

    keep = {n: bits(L[n]).clone() for n in ("out", "y", "h", "hq", "hq_sc", "h_amax", "h_ts",
                                            "xq", "xq_sc", "pos", "w")}
    for _, fn in bench.layer_calls(lib, L):
        fn()
    sync()
    for n, t in keep.items():
        assert torch.equal(bits(L[n]), t), n


def test_full_combine(dev, lib, orc):
    T, d, E, k = SHAPE.T, SHAPE.d, SHAPE.E, SHAPE.k
    idx, w = orc.route(synth.logits_uniform_np(2, T, E), k)
    off, pos, tok = orc.permute(idx, E)
    R = lib.max_rows(T, k, E)
    assert R == len(tok)
    y = synth.rows_torch(8, synth.TAG_ACT, 0, R, d, 0.5, dev)
    wf = w.astype(np.float32)
    out = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    lib.moe_combine(y, torch.tensor(pos, device=dev), torch.from_numpy(wf).to(dev), out)
    sync()
    sample = np.sort(np.random.default_rng(5).choice(T, size=256, replace=False))
    sp = pos[sample]
    used = np.unique(sp)
    y_rows = host_bits(y[torch.from_numpy(used).to(dev)])
    local = np.searchsorted(used, sp).astype(np.int32)
    wl = wf[sample].astype(np.float64)
    refv = _f32(orc.combine(y_rows, local, wl)).astype(np.float64)
    got = _f32(host_bits(out[torch.from_numpy(sample).to(dev)])).astype(np.float64)
    # fp32 slot-order accumulation: k roundings of at most 2^-24 of the
    # running magnitude, then one bf16 rounding
    yv = _f32(y_rows).astype(np.float64)
    mag = np.einsum("tj,tjd->td", np.abs(wl), np.abs(yv[local]))
    assert np.all(np.abs(got - refv) <= _ulp(refv) + 2 * k * 2.0 ** -24 * mag)

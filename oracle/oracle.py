"""numpy front end of the C oracle. TEST INFRASTRUCTURE ONLY.

Every function takes and returns numpy arrays. bf16 tensors travel as uint16
bit patterns; fp32 views of them are exact. The arithmetic lives in
``nvfp4moe_oracle.c``; this file only marshals arguments.
"""
import ctypes as C

import numpy as np

from .build import build

__all__ = [
    "lib", "bf16_to_f32", "bf16_from_f64", "e2m1_decode", "e2m1_encode", "e4m3_decode",
    "e4m3_encode", "e8m0_decode", "amax", "nvfp4_quantize", "nvfp4_dequantize",
    "nvfp4_to_f64", "philox4x32_10", "philox_word", "mxfp8_quantize", "mxfp8_dequantize",
    "rht_signs", "rht32_forward_f32", "rht32_inverse_f32", "rht32_f64", "rht32_quantize",
    "rht32_dequantize", "route", "permute", "gemm_f64", "swiglu", "expert_ffn", "combine",
    "combine_f32", "combine_rht", "mxfp8_rpad", "expert_ffn_mxfp8", "swiglu_bwd",
    "expert_bwd_gemm1", "set_threads", "max_threads", "rht32_amax",
]

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _declare(_lib)
    return _lib


_P = C.c_void_p
_I64 = C.c_int64
_I32 = C.c_int32
_U64 = C.c_uint64


def _declare(L):
    sig = {
        "oracle_set_threads": (None, [C.c_int]),
        "oracle_max_threads": (C.c_int, []),
        "oracle_bf16_to_f32": (C.c_float, [C.c_uint16]),
        "oracle_bf16_from_f64": (C.c_uint16, [C.c_double]),
        "oracle_e2m1_decode": (C.c_double, [C.c_uint8]),
        "oracle_e2m1_encode": (C.c_uint8, [C.c_float]),
        "oracle_e4m3_decode": (C.c_double, [C.c_uint8]),
        "oracle_e4m3_encode": (C.c_uint8, [C.c_float]),
        "oracle_e8m0_decode": (C.c_double, [C.c_uint8]),
        "oracle_amax": (C.c_float, [_P, _I64]),
        "oracle_nvfp4_quantize": (None, [_P, _I64, _I64, _P, _P, _P, _P]),
        "oracle_nvfp4_dequantize": (None, [_P, _P, C.c_float, _I64, _I64, _P]),
        "oracle_nvfp4_to_f64": (None, [_P, _P, C.c_float, _I64, _I64, _P]),
        "oracle_philox4x32_10": (None, [_P, _P, _P]),
        "oracle_philox_word": (C.c_uint32, [_U64, _U64, _U64]),
        "oracle_mxfp8_quantize": (None, [_P, _I64, _I64, C.c_int, _P, _I32, _U64, _U64, C.c_int,
                                         _P, _P]),
        "oracle_mxfp8_quantize_at": (None, [_P, _I64, _I64, _I64, C.c_int, _P, _I32, _U64, _U64,
                                            C.c_int, _P, _P]),
        "oracle_rht32_amax": (C.c_float, [_P, _I64, _I64, _U64]),
        "oracle_mxfp8_dequantize": (None, [_P, _P, _I64, _I64, _P]),
        "oracle_rht_signs": (C.c_uint32, [_U64]),
        "oracle_rht32_forward_f32": (None, [_P, C.c_uint32, _P]),
        "oracle_rht32_inverse_f32": (None, [_P, C.c_uint32, _P]),
        "oracle_rht32_f64": (None, [_P, C.c_uint32, C.c_int, _P]),
        "oracle_rht32_quantize": (None, [_P, _I64, _I64, _U64, C.c_int, _P, _P, _P, _P]),
        "oracle_rht32_dequantize": (None, [_P, _P, C.c_float, _I64, _I64, _U64, C.c_int, _P]),
        "oracle_route": (None, [_P, _I64, _I32, _I32, C.c_int, _P, _P]),
        "oracle_permute": (None, [_P, _I64, _I32, _I32, _I64, _P, _P, _P]),
        "oracle_gemm_f64": (None, [_P, _P, _I64, _I64, _I64, _P]),
        "oracle_swiglu": (C.c_double, [C.c_double, C.c_double]),
        "oracle_expert_ffn": (None, [_P, _P, C.c_float, _I64, _I64, _I64, _P, _P, C.c_float, _P,
                                     _P, C.c_float, _P, _I64, _P, _P, _P, _P, _P]),
        "oracle_expert_ffn_mxfp8": (None, [_P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _I64,
                                           _P, _P, _P, _P]),
        "oracle_swiglu_bwd": (None, [_P, _P, _I64, _I64, _P]),
        "oracle_combine": (None, [_P, _P, _P, _I64, _I32, _I64, _P]),
        "oracle_combine_f32": (None, [_P, _P, _P, _I64, _I32, _I64, _P]),
        "oracle_combine_rht": (None, [_P, _P, C.c_float, C.c_int, _U64, _P, _P, _I64, _I32,
                                      _I64, _P]),
        "oracle_combine_rht_f64": (None, [_P, _P, C.c_float, C.c_int, _U64, _P, _P, _I64,
                                          _I32, _I64, _P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# -- scalar codecs -----------------------------------------------------------

def bf16_to_f32(bits):
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def bf16_from_f64(v):
    v = np.asarray(v, dtype=np.float64)
    f = lib().oracle_bf16_from_f64
    return np.array([f(float(x)) for x in v.ravel()], dtype=np.uint16).reshape(v.shape)


def e2m1_decode(n):
    return lib().oracle_e2m1_decode(int(n))


def e2m1_encode(v):
    return lib().oracle_e2m1_encode(float(v))


def e4m3_decode(c):
    return lib().oracle_e4m3_decode(int(c))


def e4m3_encode(v):
    return lib().oracle_e4m3_encode(float(v))


def e8m0_decode(c):
    return lib().oracle_e8m0_decode(int(c))


def amax(x):
    x = _c(x, np.float32)
    return lib().oracle_amax(_p(x), x.size)


# -- NVFP4 -------------------------------------------------------------------

def nvfp4_quantize(x, amax_in=None):
    """x: [rows, cols] fp32. Returns (codes u8 [rows, cols/2], scales u8 [rows, cols/16], ts)."""
    x = _c(x, np.float32)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    ts = np.zeros(1, np.float32)
    a = None if amax_in is None else np.array([amax_in], np.float32)
    lib().oracle_nvfp4_quantize(_p(x), rows, cols, _p(a), _p(codes), _p(scales), _p(ts))
    return codes, scales, np.float32(ts[0])


def nvfp4_dequantize(codes, scales, ts, rows, cols):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    out = np.zeros((rows, cols), np.float32)
    lib().oracle_nvfp4_dequantize(_p(codes), _p(scales), float(ts), rows, cols, _p(out))
    return out


def nvfp4_to_f64(codes, scales, ts, rows, cols):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    out = np.zeros((rows, cols), np.float64)
    lib().oracle_nvfp4_to_f64(_p(codes), _p(scales), float(ts), rows, cols, _p(out))
    return out


# -- Philox / MXFP8 ------------------------------------------------------------

def philox4x32_10(ctr, key):
    c = np.array(ctr, np.uint32)
    k = np.array(key, np.uint32)
    out = np.zeros(4, np.uint32)
    lib().oracle_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def philox_word(seed, offset, i):
    return lib().oracle_philox_word(seed, offset, i)


def mxfp8_rpad(seg_off, rows):
    if seg_off is None:
        return (rows + 31) // 32 * 32
    s = np.asarray(seg_off, np.int64)
    return int(sum((int(s[i + 1] - s[i]) + 31) // 32 * 32 for i in range(len(s) - 1)))


def mxfp8_quantize(x, axis=0, seg_off=None, seed=0, offset=0, rounding=0, row0=0):
    """Returns (codes, scales). axis 0: [rows, cols], [rows, cols/32].
    axis 1: transposed [cols, Rpad], [cols, Rpad/32]. row0: the first row's
    index in the source tensor (the stochastic draws follow the source's
    row-major element index)."""
    x = _c(x, np.float32)
    rows, cols = x.shape
    if axis == 0:
        codes = np.zeros((rows, cols), np.uint8)
        scales = np.zeros((rows, cols // 32), np.uint8)
        so, ns = None, 0
    else:
        rp = mxfp8_rpad(seg_off, rows)
        codes = np.zeros((cols, rp), np.uint8)
        scales = np.zeros((cols, rp // 32), np.uint8)
        so = None if seg_off is None else _c(seg_off, np.int32)
        ns = 0 if seg_off is None else len(seg_off) - 1
    lib().oracle_mxfp8_quantize_at(_p(x), rows, cols, int(row0), axis, _p(so), ns, seed, offset,
                                   rounding, _p(codes), _p(scales))
    return codes, scales


def mxfp8_dequantize(codes, scales):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    n_rows, n_cols = codes.shape
    out = np.zeros((n_rows, n_cols), np.float32)
    lib().oracle_mxfp8_dequantize(_p(codes), _p(scales), n_rows, n_cols, _p(out))
    return out


# -- RHT32 -------------------------------------------------------------------

def rht_signs(sign_seed):
    return lib().oracle_rht_signs(sign_seed)


def rht32_forward_f32(x, signs):
    x = _c(x, np.float32)
    v = np.zeros(32, np.float32)
    lib().oracle_rht32_forward_f32(_p(x), signs, _p(v))
    return v


def rht32_inverse_f32(v, signs):
    v = _c(v, np.float32)
    x = np.zeros(32, np.float32)
    lib().oracle_rht32_inverse_f32(_p(v), signs, _p(x))
    return x


def rht32_f64(x, signs, inverse=False):
    x = _c(x, np.float64)
    y = np.zeros(32, np.float64)
    lib().oracle_rht32_f64(_p(x), signs, int(inverse), _p(y))
    return y


def rht32_quantize(x, sign_seed, fmt, amax_in=None):
    """fmt 0 = NVFP4 -> (codes [r, c/2], scales [r, c/16], ts); 1 = MXFP8 -> (codes, scales, None)."""
    x = _c(x, np.float32)
    rows, cols = x.shape
    if fmt == 0:
        codes = np.zeros((rows, cols // 2), np.uint8)
        scales = np.zeros((rows, cols // 16), np.uint8)
    else:
        codes = np.zeros((rows, cols), np.uint8)
        scales = np.zeros((rows, cols // 32), np.uint8)
    ts = np.zeros(1, np.float32)
    a = None if amax_in is None else np.array([amax_in], np.float32)
    lib().oracle_rht32_quantize(_p(x), rows, cols, sign_seed, fmt, _p(a), _p(codes), _p(scales),
                                _p(ts))
    return codes, scales, (np.float32(ts[0]) if fmt == 0 else None)


def rht32_dequantize(codes, scales, ts, rows, cols, sign_seed, fmt):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    out = np.zeros((rows, cols), np.float32)
    lib().oracle_rht32_dequantize(_p(codes), _p(scales), float(ts or 0.0), rows, cols, sign_seed,
                                  fmt, _p(out))
    return out


def combine_rht(codes, scales, ts, fmt, sign_seed, pos, w, f64=False):
    """Combine straight from an RHT32-quantized payload (rows x d, ROWMAJOR
    scales): bf16 bits [T, d], or the fp64 values before rounding."""
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    pos = _c(pos, np.int32)
    w = _c(w, np.float64)
    T, k = pos.shape
    d = scales.shape[1] * (16 if fmt == 0 else 32)
    if f64:
        out = np.zeros((T, d), np.float64)
        lib().oracle_combine_rht_f64(_p(codes), _p(scales), float(ts or 0.0), fmt, sign_seed,
                                     _p(pos), _p(w), T, k, d, _p(out))
    else:
        out = np.zeros((T, d), np.uint16)
        lib().oracle_combine_rht(_p(codes), _p(scales), float(ts or 0.0), fmt, sign_seed,
                                 _p(pos), _p(w), T, k, d, _p(out))
    return out


# -- routing / permutation -----------------------------------------------------

def route(logits, k, renorm=1):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    lib().oracle_route(_p(logits), T, E, k, renorm, _p(idx), _p(w))
    return idx, w


def rp_max(T, k, E):
    return (T * k + E * 127 + 127) // 128 * 128


def permute(topk_idx, E):
    topk_idx = _c(topk_idx, np.int32)
    T, k = topk_idx.shape
    rp = rp_max(T, k, E)
    off = np.zeros(E + 1, np.int32)
    pos = np.zeros((T, k), np.int32)
    tok = np.zeros(rp, np.int32)
    lib().oracle_permute(_p(topk_idx), T, E, k, rp, _p(off), _p(pos), _p(tok))
    return off, pos, tok


# -- GEMM / FFN / combine ------------------------------------------------------

def gemm_f64(A, B):
    A = _c(A, np.float64)
    B = _c(B, np.float64)
    M, K = A.shape
    N = B.shape[0]
    Cm = np.zeros((M, N), np.float64)
    lib().oracle_gemm_f64(_p(A), _p(B), M, N, K, _p(Cm))
    return Cm


def swiglu(g, u):
    return lib().oracle_swiglu(float(g), float(u))


def expert_ffn(xq, xq_sc, x_ts, w1, w1_sc, w1_ts, w2, w2_sc, w2_ts, rows_out=None):
    """One expert's forward. xq [n, d/2], W1 [2f, d/2], W2 [d, f/2] codes (+ row-major scales).
    Returns dict with h (bf16 bits [n, f]), hq, hq_sc, h_ts, y (bf16 bits [len(rows_out) or n, d])."""
    xq = _c(xq, np.uint8); xq_sc = _c(xq_sc, np.uint8)
    w1 = _c(w1, np.uint8); w1_sc = _c(w1_sc, np.uint8)
    w2 = _c(w2, np.uint8); w2_sc = _c(w2_sc, np.uint8)
    n = xq.shape[0]
    d = xq.shape[1] * 2
    f = w2.shape[1] * 2
    ro = None if rows_out is None else _c(rows_out, np.int32)
    cnt = n if ro is None else len(ro)
    h = np.zeros((n, f), np.uint16)
    hq = np.zeros((n, f // 2), np.uint8)
    hq_sc = np.zeros((n, f // 16), np.uint8)
    h_ts = np.zeros(1, np.float32)
    y = np.zeros((cnt, d), np.uint16)
    lib().oracle_expert_ffn(_p(xq), _p(xq_sc), float(x_ts), n, d, f, _p(w1), _p(w1_sc),
                            float(w1_ts), _p(w2), _p(w2_sc), float(w2_ts), _p(ro),
                            0 if ro is None else len(ro), _p(h), _p(hq), _p(hq_sc), _p(h_ts),
                            _p(y))
    return {"h": h, "hq": hq, "hq_sc": hq_sc, "h_ts": np.float32(h_ts[0]), "y": y}


def expert_ffn_mxfp8(xq, xq_sc, w1, w1_sc, w2, w2_sc, rows_out=None):
    """One expert's forward with MXFP8 operands. xq [n, d] E4M3 codes with row-major E8M0
    scales [n, d/32], W1 [2f, d], W2 [d, f] likewise. Returns dict with h (bf16 bits [n, f]),
    hq [n, f], hq_sc [n, f/32], y (bf16 bits [len(rows_out) or n, d])."""
    xq = _c(xq, np.uint8); xq_sc = _c(xq_sc, np.uint8)
    w1 = _c(w1, np.uint8); w1_sc = _c(w1_sc, np.uint8)
    w2 = _c(w2, np.uint8); w2_sc = _c(w2_sc, np.uint8)
    n, d = xq.shape
    f = w2.shape[1]
    ro = None if rows_out is None else _c(rows_out, np.int32)
    cnt = n if ro is None else len(ro)
    h = np.zeros((n, f), np.uint16)
    hq = np.zeros((n, f), np.uint8)
    hq_sc = np.zeros((n, f // 32), np.uint8)
    y = np.zeros((cnt, d), np.uint16)
    lib().oracle_expert_ffn_mxfp8(_p(xq), _p(xq_sc), n, d, f, _p(w1), _p(w1_sc), _p(w2),
                                  _p(w2_sc), _p(ro), 0 if ro is None else len(ro), _p(h), _p(hq),
                                  _p(hq_sc), _p(y))
    return {"h": h, "hq": hq, "hq_sc": hq_sc, "y": y}


def swiglu_bwd(gu_bits, dh_bits):
    """SwiGLU backward: gu bf16 bits [rows, 2f] (g | u), dh [rows, f] -> dg | du bf16 bits
    [rows, 2f], fp64 arithmetic rounded once."""
    gu_bits = _c(gu_bits, np.uint16)
    dh_bits = _c(dh_bits, np.uint16)
    rows, f = dh_bits.shape
    out = np.zeros((rows, 2 * f), np.uint16)
    lib().oracle_swiglu_bwd(_p(gu_bits), _p(dh_bits), rows, f, _p(out))
    return out


def expert_bwd_gemm1(dgu_bits, x_bits, w1_bits, expert_off=None, seed=0, offset=0):
    """GEMM1's backward in MXFP8 for a grouped layer ([P1] "训练数值格式分工清单" and
    [P2] "Architecture highlights": the backward pass runs in MXFP8, the
    gradients with stochastic rounding). dgu [R, 2f] is the gradient of g | u
    and x [R, d] the experts' input rows (bf16 bits), expert e owning rows
    expert_off[e] .. expert_off[e+1] (None: one expert, all rows); W1 [E, 2f, d].
      dX_e  = dq(SR(dgu) along 2f)_e . dq(RNE(W1_e) along 2f)    -> bf16 [R, d]
      dW1_e = dq(SR(dgu) along rows)_e^T . dq(RNE(x) along rows)_e -> fp32 [E, 2f, d]
    The stochastic draws follow each element's row-major index in the whole
    [R, 2f] tensor: row-wise from (seed, offset), column-wise from
    (seed, offset + 1). Column blocks run within each expert's rows, padded to
    32 with zero rows. Products are summed in fp64 and rounded once."""
    dgu = bf16_to_f32(_c(dgu_bits, np.uint16))
    x = bf16_to_f32(_c(x_bits, np.uint16))
    w1 = bf16_to_f32(_c(w1_bits, np.uint16))
    if w1.ndim == 2:
        w1 = w1[None]
    R, f2 = dgu.shape
    off = np.array([0, R], np.int32) if expert_off is None else _c(expert_off, np.int32)
    E = len(off) - 1
    # dgrad: contraction over 2f
    gc, gs = mxfp8_quantize(dgu, axis=0, seed=seed, offset=offset, rounding=1)
    G = mxfp8_dequantize(gc, gs)
    # wgrad: contraction over each expert's rows; the padded segments follow
    # one another in the transposed outputs
    tc, ts = mxfp8_quantize(dgu, axis=1, seg_off=off, seed=seed, offset=offset + 1, rounding=1)
    xc, xs = mxfp8_quantize(x, axis=1, seg_off=off, rounding=0)
    Tq, Xq = mxfp8_dequantize(tc, ts), mxfp8_dequantize(xc, xs)
    dx = np.zeros((R, x.shape[1]), np.float64)
    dw = np.zeros((E, f2, x.shape[1]), np.float32)
    p0 = 0
    for e in range(E):
        r0, r1 = int(off[e]), int(off[e + 1])
        plen = (r1 - r0 + 31) // 32 * 32
        if r1 > r0:
            wc, ws = mxfp8_quantize(w1[e], axis=1, rounding=0)  # [d, 2f]
            dx[r0:r1] = gemm_f64(G[r0:r1], mxfp8_dequantize(wc, ws))
            dw[e] = gemm_f64(Tq[:, p0:p0 + plen], Xq[:, p0:p0 + plen]).astype(np.float32)
        p0 += plen
    return {"dx": bf16_from_f64(dx), "dw1": dw if expert_off is not None else dw[0]}


def combine(y_bits, pos, w):
    y_bits = _c(y_bits, np.uint16)
    pos = _c(pos, np.int32)
    w = _c(w, np.float64)
    T, k = pos.shape
    d = y_bits.shape[1]
    out = np.zeros((T, d), np.uint16)
    lib().oracle_combine(_p(y_bits), _p(pos), _p(w), T, k, d, _p(out))
    return out


def combine_f32(y, pos, w):
    y = _c(y, np.float32)
    pos = _c(pos, np.int32)
    w = _c(w, np.float64)
    T, k = pos.shape
    d = y.shape[1]
    out = np.zeros((T, d), np.uint16)
    lib().oracle_combine_f32(_p(y), _p(pos), _p(w), T, k, d, _p(out))
    return out


def set_threads(n):
    """Threads of the oracle's parallel loops (results do not depend on it)."""
    lib().oracle_set_threads(int(n))


def max_threads():
    return int(lib().oracle_max_threads())


def rht32_amax(x, sign_seed):
    """max |v| of the RHT32 transform of x [rows, cols] (fp32 values)."""
    x = _c(x, np.float32)
    rows, cols = x.shape
    return np.float32(lib().oracle_rht32_amax(_p(x), rows, cols, sign_seed))

"""Thin Python binding of the nvfp4moe C ABI (include/nvfp4moe.h).

Argument marshalling only: every function takes torch tensors that already
live on the GPU, passes their device pointers, the sizes and the current CUDA
stream to the entry point of the same name, and raises NvFp4MoeError on a
non-zero status. Nothing is computed here. If libnvfp4moe.so is missing or
cannot be loaded, every call raises: there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4moe.so")

LAYOUT_ROWMAJOR, LAYOUT_MMA = 0, 1
ROUND_RNE, ROUND_SR = 0, 1
FMT_NVFP4, FMT_MXFP8 = 0, 1
OUT_BF16, OUT_F32 = 0, 1
GROUP_M, GROUP_K = 0, 1

STATUS = {0: "OK", 1: "ERR_INVALID_ARG", 2: "ERR_SHAPE", 3: "ERR_ALIGN", 4: "ERR_WORKSPACE",
          5: "ERR_CUDA", 6: "ERR_TIMEOUT", 7: "ERR_UNSUPPORTED"}


class NvFp4MoeError(RuntimeError):
    def __init__(self, fn, status, text):
        super().__init__(f"{fn} -> {STATUS.get(status, status)}: {text}")
        self.status = status


_lib = None

_P, _I64, _I32, _U64, _I, _SZ = (C.c_void_p, C.c_int64, C.c_int32, C.c_uint64, C.c_int,
                                 C.c_size_t)

_SIGS = {
    "nvfp4moe_version": (C.c_int, []),
    "nvfp4moe_last_error": (C.c_char_p, []),
    "nvfp4moe_device_error": (C.c_int, [_P]),
    "nvfp4moe_debug_gemm": (C.c_int, [C.c_uint32, _U64]),
    "nvfp4moe_max_rows": (_I64, [_I64, _I32, _I32]),
    "nvfp4moe_selftest": (C.c_int, [_I, _P, _P]),
    "nvfp4moe_amax_bf16": (C.c_int, [_P, _I64, _I64, _I64, _P, _P]),
    "nvfp4_quantize": (C.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _I, _P]),
    "nvfp4_dequantize": (C.c_int, [_P, _P, _P, _I64, _I64, _I, _P, _P]),
    "mxfp8_quantize_sr": (C.c_int, [_P, _I64, _I64, _I64, _I, _P, _I32, _U64, _U64, _I, _P, _P, _I,
                                    _P]),
    "nvfp4moe_mxfp8_seg_rows": (C.c_int64, [_I64, _I32]),
    "mxfp8_dequantize": (C.c_int, [_P, _P, _I64, _I64, _I, _P, _P]),
    "rht32_quantize": (C.c_int, [_P, _I64, _I64, _I64, _U64, _I, _P, _P, _P, _P, _I, _P]),
    "rht32_dequantize": (C.c_int, [_P, _P, _P, _I64, _I64, _U64, _I, _I, _P, _P]),
    "moe_route_permute_workspace_size": (_SZ, [_I64, _I32, _I32]),
    "moe_route_permute": (C.c_int, [_P, _P, _I64, _I32, _I32, _I64, _I, _P, _P, _P, _P, _P, _P,
                                    _P, _P, _P, _P, _SZ, _P]),
    "moe_route_permute_noalloc": (C.c_int, [_P, _P, _I64, _I32, _I32, _I64, _I, _P, _P, _P, _P,
                                            _P, _P, _P, _P, _P, _P]),
    "moe_expert_fwd": (C.c_int, [_P, _P, _P, _P, _I32, _I64, _I64, _P, _P, _P, _P, _P, _P, _P,
                                 _P, _P, _P, _P, _P, _I64, _P]),
    "moe_expert_fwd_fused_requant_workspace_size": (_SZ, [_I32]),
    "moe_expert_fwd_fused_requant": (C.c_int, [_P, _P, _P, _P, _I32, _I64, _I64, _P, _P, _P, _P,
                                               _P, _P, _P, _P, _P, _P, _P, _P, _I64, _P, _SZ,
                                               _P]),
    "moe_expert_fwd_mxfp8": (C.c_int, [_P, _P, _P, _I32, _I64, _I64, _P, _P, _P, _P, _P, _P, _P,
                                       _P, _P, _I64, _P]),
    "swiglu_bwd": (C.c_int, [_P, _P, _I64, _I64, _P, _P]),
    "moe_expert_bwd_gemm1": (C.c_int, [_P, _P, _P, _I32, _I64, _I64, _P, _P, _U64, _U64, _P, _P,
                                       _P, _P, _P, _P, _P, _P, _I64, _P]),
    "moe_combine": (C.c_int, [_P, _P, _P, _I64, _I32, _I64, _P, _P]),
    "moe_combine_rht": (C.c_int, [_P, _P, _P, _I, _U64, _P, _P, _I64, _I32, _I64, _P, _P]),
    "nvfp4_grouped_gemm": (C.c_int, [_P, _P, _P, _I32, _P, _P, _P, _P, _I32, _I64, _I64, _I64, _P,
                                     _I, _P]),
    "mxfp8_grouped_gemm": (C.c_int, [_P, _P, _P, _P, _P, _I32, _I, _I64, _I64, _I64, _P, _I, _P]),
}

EXPORTED = tuple(_SIGS)


def lib():
    """Load libnvfp4moe.so (raises if it is missing: no CPU fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with "
                "`python -m precision_moe_numerics_quantize_b200.build`")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("nvfp4moe works on CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(fn, st):
    if st != 0:
        raise NvFp4MoeError(fn, st, lib().nvfp4moe_last_error().decode())


def version():
    return lib().nvfp4moe_version()


def debug_gemm(flags, wait_ns=0):
    """Test hook of the GEMMs' failure path (see include/nvfp4moe.h)."""
    _check("nvfp4moe_debug_gemm", lib().nvfp4moe_debug_gemm(flags, wait_ns))


DEBUG_WITHHOLD_LOADS = 1


def device_error():
    code = C.c_int32(0)
    st = lib().nvfp4moe_device_error(C.byref(code))
    return st, code.value


def selftest(which, mismatches, stream=None):
    """Exhaustive hardware-conversion check; mismatch count in mismatches (int64 [1])."""
    _check("nvfp4moe_selftest", lib().nvfp4moe_selftest(which, _ptr(mismatches), _stream(stream)))


def max_rows(T, k, E):
    return lib().nvfp4moe_max_rows(T, k, E)


def nvfp4moe_amax_bf16(x, amax, cols=None, ld=None, stream=None):
    rows = x.shape[0]
    cols = x.shape[1] if cols is None else cols
    _check("nvfp4moe_amax_bf16", lib().nvfp4moe_amax_bf16(
        _ptr(x), rows, cols, ld or cols, _ptr(amax), _stream(stream)))


def nvfp4_quantize(x, codes, scales, ts_out, amax_in=None, layout=LAYOUT_ROWMAJOR, rows=None,
                   cols=None, ld=None, stream=None):
    rows = x.shape[0] if rows is None else rows
    cols = x.shape[-1] if cols is None else cols
    _check("nvfp4_quantize", lib().nvfp4_quantize(
        _ptr(x), rows, cols, ld or cols, _ptr(amax_in), _ptr(codes), _ptr(scales), _ptr(ts_out),
        layout, _stream(stream)))


def nvfp4_dequantize(codes, scales, ts, rows, cols, out, layout=LAYOUT_ROWMAJOR, stream=None):
    _check("nvfp4_dequantize", lib().nvfp4_dequantize(
        _ptr(codes), _ptr(scales), _ptr(ts), rows, cols, layout, _ptr(out), _stream(stream)))


def mxfp8_quantize_sr(x, codes, scales, axis=0, seed=0, offset=0, rounding=ROUND_SR,
                      layout=LAYOUT_ROWMAJOR, ld=None, seg_off=None, stream=None):
    """seg_off: device int32 [nseg + 1] (axis 1 only); codes then have
    mxfp8_seg_rows(rows, nseg) columns."""
    rows, cols = x.shape
    nseg = 0 if seg_off is None else seg_off.numel() - 1
    _check("mxfp8_quantize_sr", lib().mxfp8_quantize_sr(
        _ptr(x), rows, cols, ld or cols, axis, _ptr(seg_off), nseg, seed, offset, rounding,
        _ptr(codes), _ptr(scales), layout, _stream(stream)))


def mxfp8_seg_rows(rows, nseg):
    return lib().nvfp4moe_mxfp8_seg_rows(rows, nseg)


def mxfp8_dequantize(codes, scales, out, layout=LAYOUT_ROWMAJOR, stream=None):
    n_rows, n_cols = codes.shape
    _check("mxfp8_dequantize", lib().mxfp8_dequantize(
        _ptr(codes), _ptr(scales), n_rows, n_cols, layout, _ptr(out), _stream(stream)))


def rht32_quantize(x, sign_seed, fmt, codes, scales, ts_out=None, amax_in=None, ld=None,
                   stream=None):
    rows, cols = x.shape
    _check("rht32_quantize", lib().rht32_quantize(
        _ptr(x), rows, cols, ld or cols, sign_seed, fmt, _ptr(amax_in), _ptr(codes), _ptr(scales),
        _ptr(ts_out), LAYOUT_ROWMAJOR, _stream(stream)))


def rht32_dequantize(codes, scales, ts, rows, cols, sign_seed, fmt, out, stream=None):
    _check("rht32_dequantize", lib().rht32_dequantize(
        _ptr(codes), _ptr(scales), _ptr(ts), rows, cols, sign_seed, fmt, LAYOUT_ROWMAJOR,
        _ptr(out), _stream(stream)))


def moe_route_permute_workspace_size(T, E, k):
    return lib().moe_route_permute_workspace_size(T, E, k)


def moe_route_permute(logits, x, k, renorm, topk_idx, topk_w, expert_off, pos, token_of, xq,
                      xq_sc, x_ts, ws, x_amax_in=None, stream=None):
    T, E = logits.shape
    d = x.shape[1]
    _check("moe_route_permute", lib().moe_route_permute(
        _ptr(logits), _ptr(x), T, E, k, d, renorm, _ptr(x_amax_in), _ptr(topk_idx), _ptr(topk_w),
        _ptr(expert_off), _ptr(pos), _ptr(token_of), _ptr(xq), _ptr(xq_sc), _ptr(x_ts), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def moe_route_permute_noalloc(logits, x, k, renorm, topk_idx, topk_w, expert_off, pos, token_of,
                              xq, xq_sc, x_ts, x_amax_in=None, stream=None):
    """moe_route_permute with the library's built-in scratch instead of a workspace."""
    T, E = logits.shape
    d = x.shape[1]
    _check("moe_route_permute_noalloc", lib().moe_route_permute_noalloc(
        _ptr(logits), _ptr(x), T, E, k, d, renorm, _ptr(x_amax_in), _ptr(topk_idx), _ptr(topk_w),
        _ptr(expert_off), _ptr(pos), _ptr(token_of), _ptr(xq), _ptr(xq_sc), _ptr(x_ts),
        _stream(stream)))


def moe_expert_fwd(xq, xq_sc, x_ts, expert_off, E, d, f, w1, w1_sc, w1_ts, w2, w2_sc, w2_ts, h,
                   hq, hq_sc, h_amax, h_ts, y, rows_alloc, stream=None):
    _check("moe_expert_fwd", lib().moe_expert_fwd(
        _ptr(xq), _ptr(xq_sc), _ptr(x_ts), _ptr(expert_off), E, d, f, _ptr(w1), _ptr(w1_sc),
        _ptr(w1_ts), _ptr(w2), _ptr(w2_sc), _ptr(w2_ts), _ptr(h), _ptr(hq), _ptr(hq_sc),
        _ptr(h_amax), _ptr(h_ts), _ptr(y), rows_alloc, _stream(stream)))


def moe_expert_fwd_fused_requant_workspace_size(E):
    return lib().moe_expert_fwd_fused_requant_workspace_size(E)


def moe_expert_fwd_fused_requant(xq, xq_sc, x_ts, expert_off, E, d, f, w1, w1_sc, w1_ts, w2,
                                 w2_sc, w2_ts, h, hq, hq_sc, h_amax, h_ts, y, rows_alloc, ws,
                                 stream=None):
    """moe_expert_fwd with the requantization of h fused into GEMM1; ws: device
    workspace of moe_expert_fwd_fused_requant_workspace_size(E) bytes."""
    _check("moe_expert_fwd_fused_requant", lib().moe_expert_fwd_fused_requant(
        _ptr(xq), _ptr(xq_sc), _ptr(x_ts), _ptr(expert_off), E, d, f, _ptr(w1), _ptr(w1_sc),
        _ptr(w1_ts), _ptr(w2), _ptr(w2_sc), _ptr(w2_ts), _ptr(h), _ptr(hq), _ptr(hq_sc),
        _ptr(h_amax), _ptr(h_ts), _ptr(y), rows_alloc, _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_expert_fwd_mxfp8(xq, xq_sc, expert_off, E, d, f, w1, w1_sc, w2, w2_sc, h, h_amax, hq,
                         hq_sc, y, rows_alloc, stream=None):
    """Expert FFN forward with MXFP8 operands (see include/nvfp4moe.h)."""
    _check("moe_expert_fwd_mxfp8", lib().moe_expert_fwd_mxfp8(
        _ptr(xq), _ptr(xq_sc), _ptr(expert_off), E, d, f, _ptr(w1), _ptr(w1_sc), _ptr(w2),
        _ptr(w2_sc), _ptr(h), _ptr(h_amax), _ptr(hq), _ptr(hq_sc), _ptr(y), rows_alloc,
        _stream(stream)))


def swiglu_bwd(gu, dh, dgu, stream=None):
    """SwiGLU backward: gu [rows, 2f] (g | u), dh [rows, f] -> dgu [rows, 2f] (dg | du), bf16."""
    rows, f = dh.shape
    _check("swiglu_bwd", lib().swiglu_bwd(_ptr(gu), _ptr(dh), rows, f, _ptr(dgu), _stream(stream)))


def moe_expert_bwd_gemm1(dgu, x, expert_off, E, d, f, w1t, w1t_sc, seed, offset, gq, gq_sc, gt,
                         gt_sc, xt, xt_sc, dx, dw1, rows_alloc, stream=None):
    """GEMM1 backward in MXFP8: dX and dW1 from dgu and x (see include/nvfp4moe.h)."""
    _check("moe_expert_bwd_gemm1", lib().moe_expert_bwd_gemm1(
        _ptr(dgu), _ptr(x), _ptr(expert_off), E, d, f, _ptr(w1t), _ptr(w1t_sc), seed, offset,
        _ptr(gq), _ptr(gq_sc), _ptr(gt), _ptr(gt_sc), _ptr(xt), _ptr(xt_sc), _ptr(dx), _ptr(dw1),
        rows_alloc, _stream(stream)))


def moe_combine(y, pos, topk_w, out, stream=None):
    T, k = pos.shape
    d = out.shape[1]
    _check("moe_combine", lib().moe_combine(
        _ptr(y), _ptr(pos), _ptr(topk_w), T, k, d, _ptr(out), _stream(stream)))


def moe_combine_rht(codes, scales, ts, fmt, sign_seed, pos, topk_w, out, stream=None):
    """Combine from an RHT32-quantized payload (as written by rht32_quantize)."""
    T, k = pos.shape
    d = out.shape[1]
    _check("moe_combine_rht", lib().moe_combine_rht(
        _ptr(codes), _ptr(scales), _ptr(ts), fmt, sign_seed, _ptr(pos), _ptr(topk_w), T, k, d,
        _ptr(out), _stream(stream)))


def nvfp4_grouped_gemm(a, a_sc, a_ts, a_ts_stride, b, b_sc, b_ts, group_off, G, R, N, K, c,
                       out_dtype=OUT_BF16, stream=None):
    _check("nvfp4_grouped_gemm", lib().nvfp4_grouped_gemm(
        _ptr(a), _ptr(a_sc), _ptr(a_ts), a_ts_stride, _ptr(b), _ptr(b_sc), _ptr(b_ts),
        _ptr(group_off), G, R, N, K, _ptr(c), out_dtype, _stream(stream)))


def mxfp8_grouped_gemm(a, a_sc, b, b_sc, group_off, G, group_axis, M, N, K, c,
                       out_dtype=OUT_F32, stream=None):
    _check("mxfp8_grouped_gemm", lib().mxfp8_grouped_gemm(
        _ptr(a), _ptr(a_sc), _ptr(b), _ptr(b_sc), _ptr(group_off), G, group_axis, M, N, K,
        _ptr(c), out_dtype, _stream(stream)))

// The C ABI of nvfp4moe: argument validation (before any launch), status
// codes, the thread-local error text, and the orchestration of the
// multi-kernel entry points. Every computation runs in the kernels of
// quant.cu, route.cu and gemm.cu.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "quant.cuh"

namespace nvfp4moe {

static thread_local char g_last_error[512] = "";

void set_last_error(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
}

nvfp4moe_status cuda_status(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return NVFP4MOE_OK;
    set_last_error("%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
    return NVFP4MOE_ERR_CUDA;
}

// The current driver context (nullptr if the driver entry point is missing).
// A __device__ variable's address belongs to the module loaded in one
// context: a reset device, or another context made current on the same
// device, loads the module again and the variable can move.
static void *current_context() {
    typedef CUresult (*GetCurrentFn)(CUcontext *);
    static GetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &ptr, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<GetCurrentFn>(ptr);
    });
    CUcontext c = nullptr;
    if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
    return c;
}

cudaError_t cached_symbol_address(SymbolAddressCache &cache, const void *symbol, void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    void *ctx = current_context();
    std::lock_guard<std::mutex> lock(cache.mu);
    for (int i = 0; i < cache.n; ++i)
        if (cache.entry[i].dev == dev && cache.entry[i].ctx == ctx) {
            *out = cache.entry[i].addr;
            return cudaSuccess;
        }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, symbol);
    if (e != cudaSuccess) return e;
    // a full table is recycled from the start: a miss only costs a lookup
    const int slot = cache.n < SymbolAddressCache::kEntries ? cache.n++ : (cache.next++ % cache.n);
    cache.entry[slot] = {dev, ctx, p};
    *out = p;
    return cudaSuccess;
}

}  // namespace nvfp4moe

using namespace nvfp4moe;

#define FAIL(code, ...)                 \
    do {                                \
        set_last_error(__VA_ARGS__);    \
        return code;                    \
    } while (0)

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define NEED_PTR(p)                                                                    \
    do {                                                                               \
        if (!(p)) FAIL(NVFP4MOE_ERR_INVALID_ARG, "%s: %s is NULL", __func__, #p);      \
        if (!aligned16(p)) FAIL(NVFP4MOE_ERR_ALIGN, "%s: %s is not 16-byte aligned", __func__, #p); \
    } while (0)

// fp32 scalars and int32 index arrays are read element-wise: 4-byte alignment.
#define NEED_PTR4(p)                                                                   \
    do {                                                                               \
        if (!(p)) FAIL(NVFP4MOE_ERR_INVALID_ARG, "%s: %s is NULL", __func__, #p);      \
        if (reinterpret_cast<uintptr_t>(p) & 3u)                                       \
            FAIL(NVFP4MOE_ERR_ALIGN, "%s: %s is not 4-byte aligned", __func__, #p);    \
    } while (0)

#define OPT_PTR4(p)                                                                    \
    do {                                                                               \
        if ((p) && (reinterpret_cast<uintptr_t>(p) & 3u))                             \
            FAIL(NVFP4MOE_ERR_ALIGN, "%s: %s is not 4-byte aligned", __func__, #p);    \
    } while (0)

#define OPT_PTR(p)                                                                     \
    do {                                                                               \
        if ((p) && !aligned16(p))                                                      \
            FAIL(NVFP4MOE_ERR_ALIGN, "%s: %s is not 16-byte aligned", __func__, #p);   \
    } while (0)

#define NEED(cond, code, ...)                 \
    do {                                      \
        if (!(cond)) FAIL(code, __VA_ARGS__); \
    } while (0)

static nvfp4moe_status after_launch(cudaError_t e, const char *what) {
    if (e == cudaSuccess) e = cudaGetLastError();
    return cuda_status(e, what);
}

namespace nvfp4moe {

// Argument checks shared by the entry points that route and dispatch.
nvfp4moe_status check_route_permute_args(const float *logits, const uint16_t *x, int64_t T,
                                         int32_t E, int32_t k, int64_t d, int renorm,
                                         const float *x_amax_in, const int32_t *topk_idx,
                                         const float *topk_w, const int32_t *expert_off,
                                         const int32_t *pos, const int32_t *token_of,
                                         const uint8_t *xq, const uint8_t *xq_sc,
                                         const float *x_ts) {
    NEED(T >= 0 && d > 0, NVFP4MOE_ERR_INVALID_ARG, "moe_route_permute: T >= 0 and d > 0 required");
    NEED(E >= 1 && E <= 1024, NVFP4MOE_ERR_INVALID_ARG, "moe_route_permute: 1 <= E <= 1024");
    NEED(k >= 1 && k <= 32 && k <= E, NVFP4MOE_ERR_INVALID_ARG,
         "moe_route_permute: 1 <= k <= min(E, 32) required (k=%d, E=%d)", k, E);
    NEED(renorm == 0 || renorm == 1, NVFP4MOE_ERR_INVALID_ARG, "moe_route_permute: renorm 0 or 1");
    NEED(d % 64 == 0, NVFP4MOE_ERR_SHAPE, "moe_route_permute: d %% 64 == 0 required");
    NEED(T * k <= 0x7FFFFFFFLL - (int64_t)E * 128, NVFP4MOE_ERR_SHAPE,
         "moe_route_permute: T*k too large for int32 row indices");
    NEED_PTR4(expert_off);
    NEED_PTR4(token_of);
    NEED_PTR4(x_ts);
    NEED_PTR(xq);
    NEED_PTR(xq_sc);
    if (T > 0) {
        NEED_PTR4(logits);
        NEED_PTR(x);
        NEED_PTR4(topk_idx);
        NEED_PTR4(topk_w);
        NEED_PTR4(pos);
    }
    OPT_PTR4(x_amax_in);
    return NVFP4MOE_OK;
}

}  // namespace nvfp4moe

extern "C" {

int nvfp4moe_version(void) { return 100; }

const char *nvfp4moe_last_error(void) { return g_last_error; }

nvfp4moe_status nvfp4moe_device_error(int32_t *code) {
    if (!code) FAIL(NVFP4MOE_ERR_INVALID_ARG, "nvfp4moe_device_error: code is NULL");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_status(e, "nvfp4moe_device_error: synchronize");
    int32_t v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_status(e, "nvfp4moe_device_error: read");
    *code = v;
    if (v == NVFP4MOE_DEVERR_SEGMENTS)
        FAIL(NVFP4MOE_ERR_INVALID_ARG, "mxfp8_quantize_sr: segment offsets not non-decreasing in [0, rows]");
    if (v) FAIL(NVFP4MOE_ERR_TIMEOUT, "a bounded device wait ran out (wait id %d)", v);
    return NVFP4MOE_OK;
}

nvfp4moe_status nvfp4moe_selftest(int which, unsigned long long *mismatches,
                                  nvfp4moe_stream_t stream) {
    NEED(which >= 0 && which <= 3, NVFP4MOE_ERR_INVALID_ARG, "nvfp4moe_selftest: which is 0..3");
    NEED_PTR4(mismatches);
    return after_launch(launch_selftest(which, mismatches, (cudaStream_t)stream),
                        "nvfp4moe_selftest");
}

int64_t nvfp4moe_max_rows(int64_t T, int32_t k, int32_t E) {
    if (T < 0 || k < 0 || E < 0) return 0;
    return (T * k + (int64_t)E * 127 + 127) / 128 * 128;
}

nvfp4moe_status nvfp4moe_amax_bf16(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                   float *amax, nvfp4moe_stream_t stream) {
    NEED(rows >= 0 && cols >= 0, NVFP4MOE_ERR_INVALID_ARG, "amax: negative size");
    NEED(cols % 8 == 0 && ld % 8 == 0 && ld >= cols, NVFP4MOE_ERR_SHAPE,
         "amax: cols and ld must be multiples of 8, ld >= cols");
    if (rows * cols) NEED_PTR(x);
    NEED_PTR4(amax);
    return after_launch(launch_amax_bf16(x, rows, cols, ld, amax, (cudaStream_t)stream), "amax");
}

static nvfp4moe_status check_layout(int layout, int64_t rows, int64_t nsc, const char *fn) {
    NEED(layout == NVFP4MOE_LAYOUT_ROWMAJOR || layout == NVFP4MOE_LAYOUT_MMA,
         NVFP4MOE_ERR_INVALID_ARG, "%s: bad layout %d", fn, layout);
    if (layout == NVFP4MOE_LAYOUT_MMA)
        NEED(rows % 128 == 0 && nsc % 4 == 0, NVFP4MOE_ERR_SHAPE,
             "%s: MMA layout needs rows %% 128 == 0 and 4 | scales per row", fn);
    return NVFP4MOE_OK;
}

nvfp4moe_status nvfp4_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                               const float *amax_in, uint8_t *codes, uint8_t *scales,
                               float *ts_out, int layout, nvfp4moe_stream_t stream) {
    NEED(rows >= 0 && cols >= 0, NVFP4MOE_ERR_INVALID_ARG, "nvfp4_quantize: negative size");
    NEED(cols % 64 == 0 && ld % 8 == 0 && ld >= cols, NVFP4MOE_ERR_SHAPE,
         "nvfp4_quantize: cols %% 64 == 0, ld %% 8 == 0, ld >= cols required");
    nvfp4moe_status st = check_layout(layout, rows, cols / 16, "nvfp4_quantize");
    if (st) return st;
    NEED(rows * (cols / 64) < (1LL << 31), NVFP4MOE_ERR_SHAPE, "nvfp4_quantize: tensor too large");
    if (rows * cols) {
        NEED_PTR(x);
        NEED_PTR(codes);
        NEED_PTR(scales);
    }
    NEED_PTR4(ts_out);
    OPT_PTR4(amax_in);
    NEED(amax_in != ts_out, NVFP4MOE_ERR_INVALID_ARG, "nvfp4_quantize: amax_in aliases ts_out");
    return after_launch(launch_nvfp4_quantize(x, rows, cols, ld, amax_in, codes, scales, ts_out,
                                              layout, (cudaStream_t)stream),
                        "nvfp4_quantize");
}

nvfp4moe_status nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales, const float *ts,
                                 int64_t rows, int64_t cols, int layout, float *out,
                                 nvfp4moe_stream_t stream) {
    NEED(rows >= 0 && cols >= 0, NVFP4MOE_ERR_INVALID_ARG, "nvfp4_dequantize: negative size");
    NEED(cols % 16 == 0, NVFP4MOE_ERR_SHAPE, "nvfp4_dequantize: cols %% 16 == 0 required");
    nvfp4moe_status st = check_layout(layout, rows, cols / 16, "nvfp4_dequantize");
    if (st) return st;
    if (rows * cols) {
        NEED_PTR(codes);
        NEED_PTR(scales);
        NEED_PTR(out);
        NEED_PTR4(ts);
    }
    return after_launch(
        launch_nvfp4_dequantize(codes, scales, ts, rows, cols, layout, out, (cudaStream_t)stream),
        "nvfp4_dequantize");
}

int64_t nvfp4moe_mxfp8_seg_rows(int64_t rows, int32_t nseg) {
    if (rows < 0 || nseg < 1) return -1;
    return (rows + 31 * (int64_t)nseg + 31) / 32 * 32;
}

nvfp4moe_status mxfp8_quantize_sr(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                  int axis, const int32_t *seg_off, int32_t nseg, uint64_t seed,
                                  uint64_t offset, int rounding, uint8_t *codes, uint8_t *scales,
                                  int layout, nvfp4moe_stream_t stream) {
    NEED(rows >= 0 && cols >= 0, NVFP4MOE_ERR_INVALID_ARG, "mxfp8_quantize_sr: negative size");
    NEED(axis == 0 || axis == 1, NVFP4MOE_ERR_INVALID_ARG, "mxfp8_quantize_sr: axis must be 0 or 1");
    NEED(rounding == NVFP4MOE_ROUND_RNE || rounding == NVFP4MOE_ROUND_SR,
         NVFP4MOE_ERR_INVALID_ARG, "mxfp8_quantize_sr: bad rounding %d", rounding);
    NEED(ld % 8 == 0 && ld >= cols, NVFP4MOE_ERR_SHAPE, "mxfp8_quantize_sr: ld %% 8 == 0, ld >= cols");
    NEED(rows * (cols / 32 + 1) < (1LL << 31), NVFP4MOE_ERR_SHAPE, "mxfp8_quantize_sr: tensor too large");
    if (seg_off) {
        NEED(axis == 1, NVFP4MOE_ERR_INVALID_ARG, "mxfp8_quantize_sr: segments need axis 1");
        NEED(nseg >= 1 && nseg <= 1024, NVFP4MOE_ERR_INVALID_ARG,
             "mxfp8_quantize_sr: 1 <= nseg <= 1024 (got %d)", nseg);
        NEED_PTR4(seg_off);
        NEED(cols % 64 == 0, NVFP4MOE_ERR_SHAPE, "mxfp8_quantize_sr: axis 1 needs cols %% 64 == 0");
        const int64_t pitch = nvfp4moe_mxfp8_seg_rows(rows, nseg);
        NEED(pitch * (cols / 32 + 1) < (1LL << 31), NVFP4MOE_ERR_SHAPE,
             "mxfp8_quantize_sr: tensor too large");
        nvfp4moe_status st = check_layout(layout, cols, pitch / 32, "mxfp8_quantize_sr");
        if (st) return st;
        if (pitch * cols) {
            if (rows * cols) NEED_PTR(x);
            NEED_PTR(codes);
            NEED_PTR(scales);
        }
        return after_launch(launch_mxfp8_quantize_seg(x, rows, cols, ld, seg_off, nseg, pitch, seed,
                                                      offset, rounding, codes, scales, layout,
                                                      (cudaStream_t)stream),
                            "mxfp8_quantize_sr");
    }
    if (axis == 0) {
        NEED(cols % 32 == 0, NVFP4MOE_ERR_SHAPE, "mxfp8_quantize_sr: axis 0 needs cols %% 32 == 0");
        nvfp4moe_status st = check_layout(layout, rows, cols / 32, "mxfp8_quantize_sr");
        if (st) return st;
    } else {
        NEED(rows % 32 == 0 && cols % 64 == 0, NVFP4MOE_ERR_SHAPE,
             "mxfp8_quantize_sr: axis 1 needs rows %% 32 == 0 and cols %% 64 == 0");
        nvfp4moe_status st = check_layout(layout, cols, rows / 32, "mxfp8_quantize_sr");
        if (st) return st;
    }
    if (rows * cols) {
        NEED_PTR(x);
        NEED_PTR(codes);
        NEED_PTR(scales);
    }
    return after_launch(launch_mxfp8_quantize(x, rows, cols, ld, axis, seed, offset, rounding,
                                              codes, scales, layout, (cudaStream_t)stream),
                        "mxfp8_quantize_sr");
}

nvfp4moe_status mxfp8_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t n_rows,
                                 int64_t n_cols, int layout, float *out,
                                 nvfp4moe_stream_t stream) {
    NEED(n_rows >= 0 && n_cols >= 0, NVFP4MOE_ERR_INVALID_ARG, "mxfp8_dequantize: negative size");
    NEED(n_cols % 32 == 0, NVFP4MOE_ERR_SHAPE, "mxfp8_dequantize: n_cols %% 32 == 0 required");
    nvfp4moe_status st = check_layout(layout, n_rows, n_cols / 32, "mxfp8_dequantize");
    if (st) return st;
    if (n_rows * n_cols) {
        NEED_PTR(codes);
        NEED_PTR(scales);
        NEED_PTR(out);
    }
    return after_launch(launch_mxfp8_dequantize(codes, scales, n_rows, n_cols, layout, out,
                                                (cudaStream_t)stream),
                        "mxfp8_dequantize");
}

nvfp4moe_status rht32_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                               uint64_t sign_seed, int fmt, const float *amax_in,
                               uint8_t *codes, uint8_t *scales, float *ts_out, int layout,
                               nvfp4moe_stream_t stream) {
    NEED(rows >= 0 && cols >= 0, NVFP4MOE_ERR_INVALID_ARG, "rht32_quantize: negative size");
    NEED(fmt == NVFP4MOE_FMT_NVFP4 || fmt == NVFP4MOE_FMT_MXFP8, NVFP4MOE_ERR_INVALID_ARG,
         "rht32_quantize: bad fmt %d", fmt);
    NEED(layout == NVFP4MOE_LAYOUT_ROWMAJOR, NVFP4MOE_ERR_UNSUPPORTED,
         "rht32_quantize: only the ROWMAJOR scale layout is implemented");
    NEED(cols % 32 == 0 && ld % 8 == 0 && ld >= cols, NVFP4MOE_ERR_SHAPE,
         "rht32_quantize: cols %% 32 == 0, ld %% 8 == 0, ld >= cols required");
    NEED(rows * (cols / 32) < (1LL << 31), NVFP4MOE_ERR_SHAPE, "rht32_quantize: tensor too large");
    if (rows * cols) {
        NEED_PTR(x);
        NEED_PTR(codes);
        NEED_PTR(scales);
    }
    if (fmt == NVFP4MOE_FMT_NVFP4) {
        NEED_PTR4(ts_out);
        OPT_PTR4(amax_in);
        NEED(amax_in != ts_out, NVFP4MOE_ERR_INVALID_ARG, "rht32_quantize: amax_in aliases ts_out");
    }
    return after_launch(launch_rht32_quantize(x, rows, cols, ld, sign_seed, fmt,
                                              fmt == NVFP4MOE_FMT_NVFP4 ? amax_in : nullptr, codes,
                                              scales, fmt == NVFP4MOE_FMT_NVFP4 ? ts_out : nullptr,
                                              (cudaStream_t)stream),
                        "rht32_quantize");
}

nvfp4moe_status rht32_dequantize(const uint8_t *codes, const uint8_t *scales, const float *ts,
                                 int64_t rows, int64_t cols, uint64_t sign_seed, int fmt,
                                 int layout, float *out, nvfp4moe_stream_t stream) {
    NEED(rows >= 0 && cols >= 0, NVFP4MOE_ERR_INVALID_ARG, "rht32_dequantize: negative size");
    NEED(fmt == NVFP4MOE_FMT_NVFP4 || fmt == NVFP4MOE_FMT_MXFP8, NVFP4MOE_ERR_INVALID_ARG,
         "rht32_dequantize: bad fmt %d", fmt);
    NEED(layout == NVFP4MOE_LAYOUT_ROWMAJOR, NVFP4MOE_ERR_UNSUPPORTED,
         "rht32_dequantize: only the ROWMAJOR scale layout is implemented");
    NEED(cols % 32 == 0, NVFP4MOE_ERR_SHAPE, "rht32_dequantize: cols %% 32 == 0 required");
    if (rows * cols) {
        NEED_PTR(codes);
        NEED_PTR(scales);
        NEED_PTR(out);
        if (fmt == NVFP4MOE_FMT_NVFP4) NEED_PTR4(ts);
    }
    return after_launch(launch_rht32_dequantize(codes, scales, ts, rows, cols, sign_seed, fmt, out,
                                                (cudaStream_t)stream),
                        "rht32_dequantize");
}

size_t moe_route_permute_workspace_size(int64_t T, int32_t E, int32_t k) {
    if (T < 0 || E <= 0 || k <= 0) return 0;
    return route_permute_ws_bytes(T, E, k);
}

nvfp4moe_status moe_route_permute(const float *logits, const uint16_t *x, int64_t T, int32_t E,
                                  int32_t k, int64_t d, int renorm, const float *x_amax_in,
                                  int32_t *topk_idx, float *topk_w, int32_t *expert_off,
                                  int32_t *pos, int32_t *token_of, uint8_t *xq, uint8_t *xq_sc,
                                  float *x_ts, void *ws, size_t ws_bytes,
                                  nvfp4moe_stream_t stream) {
    nvfp4moe_status st = check_route_permute_args(logits, x, T, E, k, d, renorm, x_amax_in,
                                                  topk_idx, topk_w, expert_off, pos, token_of,
                                                  xq, xq_sc, x_ts);
    if (st) return st;
    NEED(ws != nullptr && ws_bytes >= route_permute_ws_bytes(T, E, k), NVFP4MOE_ERR_WORKSPACE,
         "moe_route_permute: workspace of %zu bytes needed", route_permute_ws_bytes(T, E, k));
    NEED(aligned16(ws), NVFP4MOE_ERR_ALIGN, "moe_route_permute: ws is not 16-byte aligned");
    const int64_t R = nvfp4moe_max_rows(T, k, E);
    return after_launch(launch_route_permute(logits, x, T, E, k, d, renorm, x_amax_in, topk_idx,
                                             topk_w, expert_off, pos, token_of, xq, xq_sc, x_ts,
                                             ws, R, (cudaStream_t)stream),
                        "moe_route_permute");
}

nvfp4moe_status nvfp4moe_debug_gemm(uint32_t flags, uint64_t wait_ns) {
    NEED((flags & ~1u) == 0, NVFP4MOE_ERR_INVALID_ARG, "nvfp4moe_debug_gemm: unknown flags 0x%x", flags);
    set_gemm_debug(flags, wait_ns);
    return NVFP4MOE_OK;
}

// The NVFP4 expert FFN; with ws == nullptr the requantization of h is its
// own kernel between the GEMMs, otherwise it is fused into GEMM1.
static nvfp4moe_status expert_fwd(const char *fn, const uint8_t *xq, const uint8_t *xq_sc,
                                  const float *x_ts, const int32_t *expert_off, int32_t E,
                                  int64_t d, int64_t f, const uint8_t *w1, const uint8_t *w1_sc,
                                  const float *w1_ts, const uint8_t *w2, const uint8_t *w2_sc,
                                  const float *w2_ts, uint16_t *h, uint8_t *hq, uint8_t *hq_sc,
                                  float *h_amax, float *h_ts, uint16_t *y, int64_t rows_alloc,
                                  void *ws, size_t ws_bytes, bool fused, cudaStream_t s) {
    if (!(E >= 1 && E <= 1024)) FAIL(NVFP4MOE_ERR_INVALID_ARG, "%s: 1 <= E <= 1024", fn);
    if (!(d > 0 && f > 0 && rows_alloc >= 0)) FAIL(NVFP4MOE_ERR_INVALID_ARG, "%s: sizes", fn);
    if (!(d % 256 == 0 && f % 256 == 0 && rows_alloc % 128 == 0))
        FAIL(NVFP4MOE_ERR_SHAPE, "%s: d %% 256, f %% 256 and rows_alloc %% 128 must be 0", fn);
    NEED_PTR(xq); NEED_PTR(xq_sc); NEED_PTR4(x_ts); NEED_PTR4(expert_off);
    NEED_PTR(w1); NEED_PTR(w1_sc); NEED_PTR4(w1_ts);
    NEED_PTR(w2); NEED_PTR(w2_sc); NEED_PTR4(w2_ts);
    NEED_PTR(h); NEED_PTR(hq); NEED_PTR(hq_sc); NEED_PTR4(h_amax); NEED_PTR4(h_ts); NEED_PTR(y);
    const size_t need = requant_ws_bytes(E);
    if (fused) {
        if (!ws || ws_bytes < need)
            FAIL(NVFP4MOE_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need,
                 ws ? ws_bytes : (size_t)0);
        NEED_PTR(ws);
    }
    cudaError_t e = cudaMemsetAsync(h_amax, 0, sizeof(float) * E, s);
    if (e == cudaSuccess && fused) e = cudaMemsetAsync(ws, 0, need, s);
    if (e != cudaSuccess) return cuda_status(e, fn);
    GemmArgs g1{};
    g1.kind = 0; g1.epi = EPI_SWIGLU_AMAX; g1.group_axis = NVFP4MOE_GROUP_M;
    g1.a = xq; g1.a_sc = xq_sc; g1.a_ts = x_ts; g1.a_ts_stride = 0;
    g1.b = w1; g1.b_sc = w1_sc; g1.b_ts = w1_ts;
    g1.group_off = expert_off; g1.G = E;
    g1.a_rows = rows_alloc; g1.a_cols = d; g1.N = 2 * f; g1.b_rows_per_group = 2 * f;
    g1.c = h; g1.amax = h_amax;
    if (fused) {
        g1.hq = hq; g1.hq_sc = hq_sc; g1.h_ts = h_ts; g1.rq_ws = ws;
    }
    if ((e = launch_grouped_gemm(g1, s)) != cudaSuccess) return cuda_status(e, fn);
    if (!fused && (e = launch_nvfp4_quant_grouped(h, rows_alloc, f, expert_off, E, h_amax, hq,
                                                  hq_sc, h_ts, s)) != cudaSuccess)
        return cuda_status(e, fn);
    GemmArgs g2{};
    g2.kind = 0; g2.epi = EPI_STORE_BF16; g2.group_axis = NVFP4MOE_GROUP_M;
    g2.a = hq; g2.a_sc = hq_sc; g2.a_ts = h_ts; g2.a_ts_stride = 1;
    g2.b = w2; g2.b_sc = w2_sc; g2.b_ts = w2_ts;
    g2.group_off = expert_off; g2.G = E;
    g2.a_rows = rows_alloc; g2.a_cols = f; g2.N = d; g2.b_rows_per_group = d;
    g2.c = y;
    if ((e = launch_grouped_gemm(g2, s)) != cudaSuccess) return cuda_status(e, fn);
    return after_launch(cudaSuccess, fn);
}

nvfp4moe_status moe_expert_fwd(const uint8_t *xq, const uint8_t *xq_sc, const float *x_ts,
                               const int32_t *expert_off, int32_t E, int64_t d, int64_t f,
                               const uint8_t *w1, const uint8_t *w1_sc, const float *w1_ts,
                               const uint8_t *w2, const uint8_t *w2_sc, const float *w2_ts,
                               uint16_t *h, uint8_t *hq, uint8_t *hq_sc, float *h_amax,
                               float *h_ts, uint16_t *y, int64_t rows_alloc,
                               nvfp4moe_stream_t stream) {
    return expert_fwd("moe_expert_fwd", xq, xq_sc, x_ts, expert_off, E, d, f, w1, w1_sc, w1_ts, w2,
                      w2_sc, w2_ts, h, hq, hq_sc, h_amax, h_ts, y, rows_alloc, nullptr, 0, false,
                      (cudaStream_t)stream);
}

size_t moe_expert_fwd_fused_requant_workspace_size(int32_t E) {
    return E < 0 ? 0 : requant_ws_bytes(E);
}

nvfp4moe_status moe_expert_fwd_fused_requant(
    const uint8_t *xq, const uint8_t *xq_sc, const float *x_ts, const int32_t *expert_off,
    int32_t E, int64_t d, int64_t f, const uint8_t *w1, const uint8_t *w1_sc, const float *w1_ts,
    const uint8_t *w2, const uint8_t *w2_sc, const float *w2_ts, uint16_t *h, uint8_t *hq,
    uint8_t *hq_sc, float *h_amax, float *h_ts, uint16_t *y, int64_t rows_alloc, void *ws,
    size_t ws_bytes, nvfp4moe_stream_t stream) {
    return expert_fwd("moe_expert_fwd_fused_requant", xq, xq_sc, x_ts, expert_off, E, d, f, w1,
                      w1_sc, w1_ts, w2, w2_sc, w2_ts, h, hq, hq_sc, h_amax, h_ts, y, rows_alloc, ws,
                      ws_bytes, true, (cudaStream_t)stream);
}

nvfp4moe_status moe_expert_fwd_mxfp8(const uint8_t *xq, const uint8_t *xq_sc,
                                     const int32_t *expert_off, int32_t E, int64_t d, int64_t f,
                                     const uint8_t *w1, const uint8_t *w1_sc, const uint8_t *w2,
                                     const uint8_t *w2_sc, uint16_t *h, float *h_amax,
                                     uint8_t *hq, uint8_t *hq_sc, uint16_t *y, int64_t rows_alloc,
                                     nvfp4moe_stream_t stream) {
    NEED(E >= 1 && E <= 1024, NVFP4MOE_ERR_INVALID_ARG, "moe_expert_fwd_mxfp8: 1 <= E <= 1024");
    NEED(d > 0 && f > 0 && rows_alloc >= 0, NVFP4MOE_ERR_INVALID_ARG, "moe_expert_fwd_mxfp8: sizes");
    NEED(d % 256 == 0 && f % 256 == 0 && rows_alloc % 128 == 0, NVFP4MOE_ERR_SHAPE,
         "moe_expert_fwd_mxfp8: d %% 256, f %% 256 and rows_alloc %% 128 must be 0");
    NEED_PTR(xq); NEED_PTR(xq_sc); NEED_PTR4(expert_off);
    NEED_PTR(w1); NEED_PTR(w1_sc); NEED_PTR(w2); NEED_PTR(w2_sc);
    NEED_PTR(h); NEED_PTR4(h_amax); NEED_PTR(hq); NEED_PTR(hq_sc); NEED_PTR(y);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(h_amax, 0, sizeof(float) * E, s);
    if (e != cudaSuccess) return cuda_status(e, "moe_expert_fwd_mxfp8: memset");
    GemmArgs g1{};
    g1.kind = 1; g1.epi = EPI_SWIGLU_AMAX; g1.group_axis = NVFP4MOE_GROUP_M;
    g1.a = xq; g1.a_sc = xq_sc; g1.b = w1; g1.b_sc = w1_sc;
    g1.group_off = expert_off; g1.G = E;
    g1.a_rows = rows_alloc; g1.a_cols = d; g1.N = 2 * f; g1.b_rows_per_group = 2 * f;
    g1.c = h; g1.amax = h_amax;
    if ((e = launch_grouped_gemm(g1, s)) != cudaSuccess)
        return cuda_status(e, "moe_expert_fwd_mxfp8: gemm1");
    // per-32-block scales need no expert-wide pass: one row-wise quantize of h
    if ((e = launch_mxfp8_quantize(h, rows_alloc, f, f, 0, 0, 0, NVFP4MOE_ROUND_RNE, hq, hq_sc,
                                   NVFP4MOE_LAYOUT_MMA, s)) != cudaSuccess)
        return cuda_status(e, "moe_expert_fwd_mxfp8: requantize");
    GemmArgs g2{};
    g2.kind = 1; g2.epi = EPI_STORE_BF16; g2.group_axis = NVFP4MOE_GROUP_M;
    g2.a = hq; g2.a_sc = hq_sc; g2.b = w2; g2.b_sc = w2_sc;
    g2.group_off = expert_off; g2.G = E;
    g2.a_rows = rows_alloc; g2.a_cols = f; g2.N = d; g2.b_rows_per_group = d;
    g2.c = y;
    if ((e = launch_grouped_gemm(g2, s)) != cudaSuccess)
        return cuda_status(e, "moe_expert_fwd_mxfp8: gemm2");
    return after_launch(cudaSuccess, "moe_expert_fwd_mxfp8");
}

nvfp4moe_status swiglu_bwd(const uint16_t *gu, const uint16_t *dh, int64_t rows, int64_t f,
                           uint16_t *dgu, nvfp4moe_stream_t stream) {
    NEED(rows >= 0 && f > 0, NVFP4MOE_ERR_INVALID_ARG, "swiglu_bwd: sizes");
    NEED(f % 8 == 0, NVFP4MOE_ERR_SHAPE, "swiglu_bwd: f %% 8 == 0 required");
    if (rows > 0) {
        NEED_PTR(gu); NEED_PTR(dh); NEED_PTR(dgu);
        NEED(dgu != gu && dgu != dh, NVFP4MOE_ERR_INVALID_ARG, "swiglu_bwd: dgu aliases an input");
    }
    return after_launch(launch_swiglu_bwd(gu, dh, rows, f, dgu, (cudaStream_t)stream), "swiglu_bwd");
}

nvfp4moe_status moe_expert_bwd_gemm1(const uint16_t *dgu, const uint16_t *x,
                                     const int32_t *expert_off, int32_t E, int64_t d, int64_t f,
                                     const uint8_t *w1t, const uint8_t *w1t_sc, uint64_t seed,
                                     uint64_t offset, uint8_t *gq, uint8_t *gq_sc, uint8_t *gt,
                                     uint8_t *gt_sc, uint8_t *xt, uint8_t *xt_sc, uint16_t *dx,
                                     float *dw1, int64_t rows_alloc, nvfp4moe_stream_t stream) {
    NEED(E >= 1 && E <= 1024, NVFP4MOE_ERR_INVALID_ARG, "moe_expert_bwd_gemm1: 1 <= E <= 1024");
    NEED(d > 0 && f > 0 && rows_alloc >= 0, NVFP4MOE_ERR_INVALID_ARG, "moe_expert_bwd_gemm1: sizes");
    NEED(d % 256 == 0 && f % 128 == 0 && rows_alloc % 128 == 0, NVFP4MOE_ERR_SHAPE,
         "moe_expert_bwd_gemm1: d %% 256, f %% 128 and rows_alloc %% 128 must be 0");
    NEED(rows_alloc * (2 * f / 32 + 1) < (1LL << 31) && rows_alloc * (d / 32 + 1) < (1LL << 31),
         NVFP4MOE_ERR_SHAPE, "moe_expert_bwd_gemm1: tensors too large");
    NEED_PTR4(expert_off); NEED_PTR(w1t); NEED_PTR(w1t_sc); NEED_PTR(dw1);
    if (rows_alloc > 0) {
        NEED_PTR(dgu); NEED_PTR(x); NEED_PTR(gq); NEED_PTR(gq_sc); NEED_PTR(gt); NEED_PTR(gt_sc);
        NEED_PTR(xt); NEED_PTR(xt_sc); NEED_PTR(dx);
    }
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t R = rows_alloc, f2 = 2 * f;
    cudaError_t e;
    // expert starts are multiples of 128, so no 32-row block straddles two experts
    if ((e = launch_mxfp8_quantize(dgu, R, f2, f2, 0, seed, offset, NVFP4MOE_ROUND_SR, gq, gq_sc,
                                   NVFP4MOE_LAYOUT_MMA, s)) != cudaSuccess)
        return cuda_status(e, "moe_expert_bwd_gemm1: quantize dgu rows");
    if ((e = launch_mxfp8_quantize(dgu, R, f2, f2, 1, seed, offset + 1, NVFP4MOE_ROUND_SR, gt, gt_sc,
                                   NVFP4MOE_LAYOUT_MMA, s)) != cudaSuccess)
        return cuda_status(e, "moe_expert_bwd_gemm1: quantize dgu columns");
    if ((e = launch_mxfp8_quantize(x, R, d, d, 1, 0, 0, NVFP4MOE_ROUND_RNE, xt, xt_sc,
                                   NVFP4MOE_LAYOUT_MMA, s)) != cudaSuccess)
        return cuda_status(e, "moe_expert_bwd_gemm1: quantize x columns");
    GemmArgs g1{};  // dgrad: contraction over 2f, grouped over rows
    g1.kind = 1; g1.epi = EPI_STORE_BF16; g1.group_axis = NVFP4MOE_GROUP_M;
    g1.a = gq; g1.a_sc = gq_sc; g1.b = w1t; g1.b_sc = w1t_sc;
    g1.group_off = expert_off; g1.G = E;
    g1.a_rows = R; g1.a_cols = f2; g1.M = R; g1.N = d; g1.b_rows_per_group = d; g1.c = dx;
    if ((e = launch_grouped_gemm(g1, s)) != cudaSuccess) return cuda_status(e, "moe_expert_bwd_gemm1: dgrad");
    GemmArgs g2{};  // wgrad: contraction over each expert's rows
    g2.kind = 1; g2.epi = EPI_STORE_F32; g2.group_axis = NVFP4MOE_GROUP_K;
    g2.a = gt; g2.a_sc = gt_sc; g2.b = xt; g2.b_sc = xt_sc;
    g2.group_off = expert_off; g2.G = E;
    g2.a_rows = f2; g2.a_cols = R; g2.M = f2; g2.N = d; g2.b_rows_per_group = d; g2.c = dw1;
    if ((e = launch_grouped_gemm(g2, s)) != cudaSuccess) return cuda_status(e, "moe_expert_bwd_gemm1: wgrad");
    return after_launch(cudaSuccess, "moe_expert_bwd_gemm1");
}

nvfp4moe_status moe_combine(const uint16_t *y, const int32_t *pos, const float *topk_w,
                            int64_t T, int32_t k, int64_t d, uint16_t *out,
                            nvfp4moe_stream_t stream) {
    NEED(T >= 0 && k >= 1 && d > 0, NVFP4MOE_ERR_INVALID_ARG, "moe_combine: sizes");
    NEED(d % 8 == 0, NVFP4MOE_ERR_SHAPE, "moe_combine: d %% 8 == 0 required");
    if (T > 0) {
        NEED_PTR(y); NEED_PTR4(pos); NEED_PTR4(topk_w); NEED_PTR(out);
    }
    return after_launch(launch_combine(y, pos, topk_w, T, k, d, out, (cudaStream_t)stream),
                        "moe_combine");
}

nvfp4moe_status moe_combine_rht(const uint8_t *codes, const uint8_t *scales, const float *ts,
                                int fmt, uint64_t sign_seed, const int32_t *pos,
                                const float *topk_w, int64_t T, int32_t k, int64_t d,
                                uint16_t *out, nvfp4moe_stream_t stream) {
    NEED(T >= 0 && k >= 1 && d > 0, NVFP4MOE_ERR_INVALID_ARG, "moe_combine_rht: sizes");
    NEED(fmt == NVFP4MOE_FMT_NVFP4 || fmt == NVFP4MOE_FMT_MXFP8, NVFP4MOE_ERR_INVALID_ARG,
         "moe_combine_rht: bad fmt");
    NEED(d % 32 == 0, NVFP4MOE_ERR_SHAPE, "moe_combine_rht: d %% 32 == 0 required");
    if (T > 0) {
        NEED_PTR(codes); NEED_PTR(scales); NEED_PTR4(pos); NEED_PTR4(topk_w); NEED_PTR(out);
        if (fmt == NVFP4MOE_FMT_NVFP4) NEED_PTR4(ts);
    }
    return after_launch(launch_combine_rht(codes, scales, ts, fmt, sign_seed, pos, topk_w, T, k, d,
                                           out, (cudaStream_t)stream),
                        "moe_combine_rht");
}

nvfp4moe_status nvfp4_grouped_gemm(const uint8_t *a, const uint8_t *a_sc, const float *a_ts,
                                   int32_t a_ts_stride, const uint8_t *b, const uint8_t *b_sc,
                                   const float *b_ts, const int32_t *group_off, int32_t G,
                                   int64_t R, int64_t N, int64_t K, void *c, int out_dtype,
                                   nvfp4moe_stream_t stream) {
    NEED(G >= 1 && G <= 1024, NVFP4MOE_ERR_INVALID_ARG, "nvfp4_grouped_gemm: 1 <= G <= 1024");
    NEED(R >= 0 && N > 0 && K > 0, NVFP4MOE_ERR_INVALID_ARG, "nvfp4_grouped_gemm: sizes");
    NEED(a_ts_stride == 0 || a_ts_stride == 1, NVFP4MOE_ERR_INVALID_ARG,
         "nvfp4_grouped_gemm: a_ts_stride must be 0 or 1");
    NEED(out_dtype == NVFP4MOE_OUT_BF16 || out_dtype == NVFP4MOE_OUT_F32, NVFP4MOE_ERR_INVALID_ARG,
         "nvfp4_grouped_gemm: bad out_dtype");
    NEED(K % 256 == 0 && N % 256 == 0 && R % 128 == 0, NVFP4MOE_ERR_SHAPE,
         "nvfp4_grouped_gemm: K %% 256, N %% 256, R %% 128 must be 0");
    NEED_PTR(a); NEED_PTR(a_sc); NEED_PTR4(a_ts); NEED_PTR(b); NEED_PTR(b_sc); NEED_PTR4(b_ts);
    NEED_PTR4(group_off); NEED_PTR(c);
    GemmArgs g{};
    g.kind = 0; g.epi = out_dtype == NVFP4MOE_OUT_BF16 ? EPI_STORE_BF16 : EPI_STORE_F32;
    g.group_axis = NVFP4MOE_GROUP_M;
    g.a = a; g.a_sc = a_sc; g.a_ts = a_ts; g.a_ts_stride = a_ts_stride;
    g.b = b; g.b_sc = b_sc; g.b_ts = b_ts; g.group_off = group_off; g.G = G;
    g.a_rows = R; g.a_cols = K; g.N = N; g.b_rows_per_group = N; g.c = c;
    return after_launch(launch_grouped_gemm(g, (cudaStream_t)stream), "nvfp4_grouped_gemm");
}

nvfp4moe_status mxfp8_grouped_gemm(const uint8_t *a, const uint8_t *a_sc, const uint8_t *b,
                                   const uint8_t *b_sc, const int32_t *group_off, int32_t G,
                                   int group_axis, int64_t M, int64_t N, int64_t K, void *c,
                                   int out_dtype, nvfp4moe_stream_t stream) {
    NEED(G >= 1 && G <= 1024, NVFP4MOE_ERR_INVALID_ARG, "mxfp8_grouped_gemm: 1 <= G <= 1024");
    NEED(M >= 0 && N > 0 && K >= 0, NVFP4MOE_ERR_INVALID_ARG, "mxfp8_grouped_gemm: sizes");
    NEED(group_axis == NVFP4MOE_GROUP_M || group_axis == NVFP4MOE_GROUP_K, NVFP4MOE_ERR_INVALID_ARG,
         "mxfp8_grouped_gemm: bad group_axis");
    NEED(out_dtype == NVFP4MOE_OUT_BF16 || out_dtype == NVFP4MOE_OUT_F32, NVFP4MOE_ERR_INVALID_ARG,
         "mxfp8_grouped_gemm: bad out_dtype");
    NEED(K % 128 == 0 && N % 256 == 0 && M % 128 == 0, NVFP4MOE_ERR_SHAPE,
         "mxfp8_grouped_gemm: K %% 128, N %% 256, M %% 128 must be 0");
    NEED_PTR(a); NEED_PTR(a_sc); NEED_PTR(b); NEED_PTR(b_sc); NEED_PTR4(group_off); NEED_PTR(c);
    GemmArgs g{};
    g.kind = 1; g.epi = out_dtype == NVFP4MOE_OUT_BF16 ? EPI_STORE_BF16 : EPI_STORE_F32;
    g.group_axis = group_axis;
    g.a = a; g.a_sc = a_sc; g.b = b; g.b_sc = b_sc; g.group_off = group_off; g.G = G;
    g.a_rows = M; g.a_cols = K; g.M = M; g.N = N; g.b_rows_per_group = N; g.c = c;
    return after_launch(launch_grouped_gemm(g, (cudaStream_t)stream), "mxfp8_grouped_gemm");
}

}  // extern "C"

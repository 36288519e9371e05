// Host-side launchers of the nvfp4moe kernels (all asynchronous on stream s).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nvfp4moe.h"

namespace nvfp4moe {

cudaError_t launch_amax_bf16(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                             float *amax, cudaStream_t s);
cudaError_t launch_nvfp4_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                  const float *amax_in, uint8_t *codes, uint8_t *scales,
                                  float *ts_out, int layout, cudaStream_t s);
cudaError_t launch_nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales, const float *ts,
                                    int64_t rows, int64_t cols, int layout, float *out,
                                    cudaStream_t s);
// Column-wise (axis 1) MXFP8 over segments of rows, blocks packed into an
// output of `pitch` columns; see mxfp8_quantize_sr in nvfp4moe.h.
cudaError_t launch_mxfp8_quantize_seg(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                      const int32_t *seg_off, int32_t nseg, int64_t pitch,
                                      uint64_t seed, uint64_t offset, int rounding,
                                      uint8_t *codes, uint8_t *scales, int layout, cudaStream_t s);
cudaError_t launch_mxfp8_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                  int axis, uint64_t seed, uint64_t offset, int rounding,
                                  uint8_t *codes, uint8_t *scales, int layout, cudaStream_t s);
cudaError_t launch_mxfp8_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t n_rows,
                                    int64_t n_cols, int layout, float *out, cudaStream_t s);
cudaError_t launch_rht32_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                  uint64_t sign_seed, int fmt, const float *amax_in,
                                  uint8_t *codes, uint8_t *scales, float *ts_out,
                                  cudaStream_t s);
cudaError_t launch_rht32_dequantize(const uint8_t *codes, const uint8_t *scales, const float *ts,
                                    int64_t rows, int64_t cols, uint64_t sign_seed, int fmt,
                                    float *out, cudaStream_t s);
cudaError_t launch_nvfp4_quant_grouped(const uint16_t *x, int64_t rows_alloc, int64_t cols,
                                       const int32_t *off, int32_t E, const float *amax,
                                       uint8_t *codes, uint8_t *scales, float *ts,
                                       cudaStream_t s);

cudaError_t launch_swiglu_bwd(const uint16_t *gu, const uint16_t *dh, int64_t rows, int64_t f,
                              uint16_t *dgu, cudaStream_t s);
cudaError_t launch_selftest(int which, unsigned long long *mismatches, cudaStream_t s);

// routing / permutation / combine (route.cu)
size_t route_permute_ws_bytes(int64_t T, int32_t E, int32_t k);
cudaError_t launch_route_permute(const float *logits, const uint16_t *x, int64_t T, int32_t E,
                                 int32_t k, int64_t d, int renorm, const float *x_amax_in,
                                 int32_t *topk_idx, float *topk_w, int32_t *expert_off,
                                 int32_t *pos, int32_t *token_of, uint8_t *xq, uint8_t *xq_sc,
                                 float *x_ts, void *ws, int64_t rows_alloc, cudaStream_t s);
nvfp4moe_status check_route_permute_args(const float *logits, const uint16_t *x, int64_t T,
                                         int32_t E, int32_t k, int64_t d, int renorm,
                                         const float *x_amax_in, const int32_t *topk_idx,
                                         const float *topk_w, const int32_t *expert_off,
                                         const int32_t *pos, const int32_t *token_of,
                                         const uint8_t *xq, const uint8_t *xq_sc,
                                         const float *x_ts);
cudaError_t launch_combine(const uint16_t *y, const int32_t *pos, const float *w, int64_t T,
                           int32_t k, int64_t d, uint16_t *out, cudaStream_t s);

// grouped block-scaled GEMMs (gemm.cu)
enum GemmEpi { EPI_SWIGLU_AMAX = 0, EPI_STORE_BF16 = 1, EPI_STORE_F32 = 2 };
struct GemmArgs {
    int kind;        // 0 = NVFP4 (mxf4nvf4), 1 = MXFP8 (mxf8f6f4)
    int epi;         // GemmEpi
    int group_axis;  // 0 = rows of A, 1 = contraction columns
    const uint8_t *a, *a_sc, *b, *b_sc;
    const float *a_ts, *b_ts;  // NVFP4 only
    int32_t a_ts_stride;
    const int32_t *group_off;
    int32_t G;
    int64_t a_rows;   // rows of the A matrix as stored
    int64_t a_cols;   // contraction columns of A/B as stored (elements)
    int64_t M;        // group K: rows of every output block
    int64_t N;        // output columns (SwiGLU: 2 * f acc columns, f outputs)
    int64_t b_rows_per_group;  // rows of B per group (N, or 2f for SwiGLU)
    void *c;
    float *amax;      // SwiGLU: per-group amax of h
    // SwiGLU with NVFP4: requantize h inside the same launch (hq != nullptr):
    // hq [rows x f/2], hq_sc (MMA layout), h_ts [G]; rq_ws holds the expert
    // queue, requant_ws_bytes(G) bytes, zeroed before the launch.
    uint8_t *hq = nullptr, *hq_sc = nullptr;
    float *h_ts = nullptr;
    void *rq_ws = nullptr;
};
cudaError_t launch_grouped_gemm(const GemmArgs &a, cudaStream_t s);
// Workspace of the fused requantization: per-group arrival counters, row
// cursors and queue slots (int32, each array padded to 16 bytes), then the
// two queue counters.
inline size_t requant_ws_bytes(int64_t G) { return (size_t)(3 * ((G + 3) / 4 * 4) + 4) * 4; }
// Test hook of the failure path (nvfp4moe_debug_gemm).
void set_gemm_debug(uint32_t flags, uint64_t wait_ns);

// Device address of the device error word on the current device, for kernels
// built as whole programs (they cannot name the variable itself); nullptr if
// the runtime cannot resolve it.
int32_t *device_error_word();
cudaError_t launch_combine_rht(const uint8_t *codes, const uint8_t *scales, const float *ts, int fmt,
                               uint64_t sign_seed, const int32_t *pos, const float *w, int64_t T,
                               int32_t k, int64_t d, uint16_t *out, cudaStream_t s);

}  // namespace nvfp4moe

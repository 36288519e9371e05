/*
 * nvfp4moe: NVFP4 mixture-of-experts expert layer for NVIDIA B200 (sm_100a).
 *
 * The method: write-ups of Thinking Machines Lab's "End-to-End 4-Bit
 * Training" post.
 *   - news.t0001.com, "Thinking Machines 详解 Inkling 2 Small 原生 4-bit 前向训练完整流程",
 *     list "训练数值格式分工清单": expert-layer forward passes in NVFP4 on
 *     dedicated CUDA kernels, backward gradients in MXFP8 with stochastic
 *     rounding, quantized cross-GPU traffic, non-expert modules at higher
 *     precision.
 *   - aicoder.com, "Thinking Machines Details End-to-End 4-Bit Training for
 *     Inkling 2 Small", "Key Takeaways" and "Architecture highlights": MXFP8
 *     backward with re-quantization and stochastic rounding; the
 *     expert-parallel combine is quantized after a 32-dimensional random
 *     Hadamard transform into a block-scaled format; the kernels are fully
 *     deterministic. "Background": NVFP4 costs about 4.5 bits per value.
 *   - 10100.com, "Inkling 2 Small", "PART 01": 384 experts, top-8 routing.
 * The pages print no formula. The numeric readings this library implements:
 *   NVFP4  = E2M1 codes (grid 0, .5, 1, 1.5, 2, 3, 4, 6; nearest, ties to even,
 *            saturating), one E4M3 scale per 16 elements, one fp32 decode
 *            scale per tensor: ts = amax / 2688, S_enc = 2688 / amax,
 *            s_b = E4M3_RNE((amax_b / 6) * S_enc), q = E2M1_RNE(x * S_enc / s_b),
 *            x_hat = e2m1(q) * s_b * ts (amax 0 -> S_enc = ts = 1).
 *   MXFP8  = E4M3 codes, one E8M0 scale 2^k per 32 elements, k the smallest
 *            integer in [-127, 127] with amax_b <= 448 * 2^k (nothing clips);
 *            rounding to nearest even, or stochastic with Philox4x32-10
 *            (key = seed, counter = (i / 4, offset), word i % 4, i the
 *            row-major index of the element in the source tensor): round up
 *            iff (word >> 8) * 2^-24 < (|v| - lo) / (hi - lo).
 *   RHT32  = v = fp32(1/sqrt(32)) * H32 * (s .* x) per 32-element block; H32
 *            Sylvester; s_i = -1 iff bit i of word 0 of Philox4x32-10(key =
 *            sign_seed, counter = 0); fp32 butterflies h = 1, 2, 4, 8, 16.
 *
 * Conventions (all entry points):
 *   - Every function returns an nvfp4moe_status. Arguments are validated on
 *     the host before anything is launched; a failed validation leaves every
 *     output untouched. NVFP4MOE_ERR_CUDA carries the CUDA error text in
 *     nvfp4moe_last_error() (thread-local).
 *   - All pointers named in a signature are DEVICE pointers unless the comment
 *     says "host". The caller owns all memory; the library allocates nothing.
 *     Tensor pointers (bf16 data, codes, scales, outputs, workspace) must be
 *     16-byte aligned; fp32 scalars (amax, ts) and int32 index arrays
 *     4-byte aligned (NVFP4MOE_ERR_ALIGN).
 *   - Every call is asynchronous on the given stream, performs no host
 *     synchronisation, and is deterministic (identical bits for identical
 *     inputs). The one piece of library state is a device-side error word
 *     set by a kernel whose bounded wait ran out or that found device-side
 *     arguments it could not use; nvfp4moe_device_error() reads and clears
 *     it.
 *   - bf16 tensors are passed as uint16_t bit patterns, row-major, with a row
 *     stride ld in elements (ld >= cols, ld % 8 == 0).
 *   - NVFP4 codes: rows x cols/2 bytes, element 2i in the low nibble of byte i.
 *   - Scale layouts:
 *       NVFP4MOE_LAYOUT_ROWMAJOR: scales[r * (cols / B) + b] (B = 16 or 32).
 *       NVFP4MOE_LAYOUT_MMA: the tcgen05 block-scaled MMA layout. Scales are
 *         grouped in 512-byte chunks, one per 128 rows x 4 scale columns;
 *         chunk (rt, kc) starts at byte (rt * (cols / B / 4) + kc) * 512 and
 *         the scale of row r = 128 rt + 32 r1 + r0 (r0 < 32, r1 < 4) and scale
 *         column 4 kc + c sits at byte r0 * 16 + r1 * 4 + c of its chunk.
 *         Needs rows % 128 == 0 and (cols / B) % 4 == 0.
 */
#ifndef NVFP4MOE_H
#define NVFP4MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The library is built with hidden visibility; the entry points below are
 * the only exported symbols. */
#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

typedef struct CUstream_st *nvfp4moe_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
    NVFP4MOE_OK = 0,
    NVFP4MOE_ERR_INVALID_ARG = 1, /* null pointer, negative size, k > E, bad enum, aliasing */
    NVFP4MOE_ERR_SHAPE = 2,       /* a dimension breaks the divisibility rule of the call */
    NVFP4MOE_ERR_ALIGN = 3,       /* a device pointer is not 16-byte aligned */
    NVFP4MOE_ERR_WORKSPACE = 4,   /* workspace missing or smaller than the query says */
    NVFP4MOE_ERR_CUDA = 5,        /* a CUDA call failed; see nvfp4moe_last_error() */
    NVFP4MOE_ERR_TIMEOUT = 6,     /* a bounded device wait ran out (nvfp4moe_device_error) */
    NVFP4MOE_ERR_UNSUPPORTED = 7  /* valid request this library version does not implement */
} nvfp4moe_status;

enum { NVFP4MOE_LAYOUT_ROWMAJOR = 0, NVFP4MOE_LAYOUT_MMA = 1 };
enum { NVFP4MOE_ROUND_RNE = 0, NVFP4MOE_ROUND_SR = 1 };
enum { NVFP4MOE_FMT_NVFP4 = 0, NVFP4MOE_FMT_MXFP8 = 1 };
enum { NVFP4MOE_OUT_BF16 = 0, NVFP4MOE_OUT_F32 = 1 };
enum { NVFP4MOE_GROUP_M = 0, NVFP4MOE_GROUP_K = 1 };

/* Library version, e.g. 100 for 0.1.0. */
int nvfp4moe_version(void);

/* Text of the last error on this thread ("" if none). Owned by the library. */
const char *nvfp4moe_last_error(void);

/* Synchronises the current device, then reads and clears the device error
 * word. *code (host) receives 0 if no kernel recorded an error, 1..15 for the
 * identifier of a bounded GEMM wait that ran out (returns
 * NVFP4MOE_ERR_TIMEOUT), or NVFP4MOE_DEVERR_SEGMENTS if mxfp8_quantize_sr was
 * given segment offsets that are not non-decreasing inside [0, rows]
 * (returns NVFP4MOE_ERR_INVALID_ARG). */
enum { NVFP4MOE_DEVERR_SEGMENTS = 16 };
nvfp4moe_status nvfp4moe_device_error(int32_t *code);

/* Test hook of the failure path of the grouped GEMMs (no counterpart on the
 * pages). flags = NVFP4MOE_DEBUG_WITHHOLD_LOADS makes the GEMM launches that
 * follow (in this process) issue no operand or scale load at all, so no copy
 * is ever in flight; their consumers' bounded waits then give up after
 * wait_ns nanoseconds (0: the normal 2 s), every role winds down, the launch
 * ends, and nvfp4moe_device_error() reports NVFP4MOE_ERR_TIMEOUT with the id
 * of the wait that gave up first. flags = 0 restores normal operation (and
 * the 2 s limit). Not for use while other threads launch GEMMs. */
enum { NVFP4MOE_DEBUG_WITHHOLD_LOADS = 1 };
nvfp4moe_status nvfp4moe_debug_gemm(uint32_t flags, uint64_t wait_ns);

/* Exhaustive check of the hardware conversions the kernels use against the
 * library's own encoders and decoders (which the test suite pins bit for bit
 * to the CPU reference): which = 0 checks cvt.rn.satfinite.e2m1x2.f32 and
 * which = 1 cvt.rn.satfinite.e4m3x2.f32, each over every finite fp32 input;
 * which = 2 checks the decode cvt.rn.f16x2.e2m1x2 over all 256 code pairs
 * and which = 3 cvt.rn.f16x2.e4m3x2 over all 65536 code pairs (the NaN codes
 * 0x7F / 0xFF excepted: the encoders saturate and never write them). The mismatch
 * count lands in *mismatches (device uint64, overwritten). Has no counterpart
 * on the pages; it guards the conversions on a new driver. */
nvfp4moe_status nvfp4moe_selftest(int which, unsigned long long *mismatches,
                                  nvfp4moe_stream_t stream);

/* Upper bound on the rows of a permuted, per-expert-padded activation:
 * T*k + E*127 rounded up to 128. Pure host arithmetic. */
int64_t nvfp4moe_max_rows(int64_t T, int32_t k, int32_t E);

/* ------------------------------------------------------------------------
 * max |x| over a bf16 tensor (the NVFP4 tensor amax).
 * x [rows x cols], stride ld. amax: one fp32, overwritten. */
nvfp4moe_status nvfp4moe_amax_bf16(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                   float *amax, nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------
 * NVFP4 quantization (news.t0001.com '训练数值格式分工清单': the expert forward in
 * NVFP4; aicoder.com 'Background': about 4.5 bits per value).
 * x: bf16 [rows x cols], stride ld; cols % 64 == 0.
 * amax_in: device fp32 or NULL. NULL computes max|x| first (two passes);
 *   a caller that already holds the amax passes it (one pass). Must not
 *   alias ts_out.
 * codes: [rows x cols/2]. scales: E4M3 in `layout`. ts_out: one fp32, the
 *   decode tensor scale amax / 2688. */
nvfp4moe_status nvfp4_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                               const float *amax_in, uint8_t *codes, uint8_t *scales,
                               float *ts_out, int layout, nvfp4moe_stream_t stream);

/* out[r][c] = e2m1(code) * scale * ts in fp32, out [rows x cols] fp32.
 * ts: device fp32 (one value). */
nvfp4moe_status nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales, const float *ts,
                                 int64_t rows, int64_t cols, int layout, float *out,
                                 nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------
 * MXFP8 quantization with stochastic rounding (news.t0001.com '训练数值格式分工清单':
 * MXFP8 backward with stochastic rounding; aicoder.com 'Key Takeaways':
 * re-quantization and stochastic rounding to limit gradient bias).
 * x: bf16 [rows x cols], stride ld.
 * axis 0: blocks of 32 along a row. cols % 32 == 0 (MMA layout: rows % 128,
 *   cols % 128). codes [rows x cols], scales E8M0 [rows x cols/32].
 * axis 1: blocks of 32 consecutive rows of a column, cols % 64 == 0. The
 *   output is transposed, ready to be the K-major operand of a GEMM that
 *   contracts over rows.
 *   seg_off == NULL: one segment of all rows; rows % 32 == 0 (MMA: rows %
 *     128, cols % 128); codes [cols x rows], scales [cols x rows/32].
 *   seg_off != NULL: device int32 [nseg + 1], 1 <= nseg <= 1024,
 *     non-decreasing inside [0, rows]; segment s is rows [seg_off[s],
 *     seg_off[s+1]). No block crosses a segment: each segment is cut into
 *     ceil(len / 32) blocks, the last one zero-padded, and the blocks of all
 *     segments are packed in order into an output of
 *     P = nvfp4moe_mxfp8_seg_rows(rows, nseg) columns (the most the packed
 *     blocks can need): codes [cols x P], scales [cols x P/32]; columns past
 *     the packed blocks get zero codes and zero scale codes (MMA layout: P %
 *     128 and cols % 128). The offsets are checked on the device: invalid
 *     ones give an all-zero output and NVFP4MOE_DEVERR_SEGMENTS in the device
 *     error word (nvfp4moe_device_error).
 * rounding: NVFP4MOE_ROUND_RNE or NVFP4MOE_ROUND_SR (seed, offset select the
 *   Philox stream; quantize the same tensor along two axes with two offsets).
 *   A draw follows the element's row-major index in the [rows x cols] source,
 *   with or without segments. */
nvfp4moe_status mxfp8_quantize_sr(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                  int axis, const int32_t *seg_off, int32_t nseg, uint64_t seed,
                                  uint64_t offset, int rounding, uint8_t *codes, uint8_t *scales,
                                  int layout, nvfp4moe_stream_t stream);

/* Output columns of a segmented column-wise MXFP8 quantization:
 * round_up(rows + 31 * nseg, 32); -1 for rows < 0 or nseg < 1. */
int64_t nvfp4moe_mxfp8_seg_rows(int64_t rows, int32_t nseg);

/* out = e4m3(code) * 2^(scale - 127), fp32 [n_rows x n_cols] for an MXFP8
 * tensor stored as codes [n_rows x n_cols] with ROWMAJOR or MMA scales. */
nvfp4moe_status mxfp8_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t n_rows,
                                 int64_t n_cols, int layout, float *out,
                                 nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------
 * RHT32 + block-scaled quantization of the combine payload (aicoder.com 'Key
 * Takeaways' and 'Architecture highlights': a 32-dimensional random Hadamard
 * transform before the expert-parallel combine traffic is quantized).
 * x: bf16 [rows x cols], stride ld, cols % 32 == 0. ROWMAJOR scales only.
 * fmt NVFP4: codes [rows x cols/2], scales [rows x cols/16], ts_out (decode
 *   tensor scale of the transformed values; amax_in as in nvfp4_quantize,
 *   but the amax of the TRANSFORMED values).
 * fmt MXFP8 (round to nearest even): codes [rows x cols], scales
 *   [rows x cols/32]; amax_in and ts_out unused (may be NULL). */
nvfp4moe_status rht32_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                               uint64_t sign_seed, int fmt, const float *amax_in,
                               uint8_t *codes, uint8_t *scales, float *ts_out, int layout,
                               nvfp4moe_stream_t stream);

/* Inverse: dequantize, inverse transform; out fp32 [rows x cols]. ts: device
 * fp32 for NVFP4 (ignored for MXFP8). */
nvfp4moe_status rht32_dequantize(const uint8_t *codes, const uint8_t *scales, const float *ts,
                                 int64_t rows, int64_t cols, uint64_t sign_seed, int fmt,
                                 int layout, float *out, nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Routing and dispatch with fused NVFP4 quantization (10100.com 'PART 01':
 * top-8 of 384 experts; aicoder.com 'Key Takeaways': expert-parallel
 * dispatch and combine).
 * logits fp32 [T x E]; x bf16 [T x d] (ld = d). 1 <= k <= min(E, 32),
 * E <= 1024, d % 64 == 0.
 * Top-k by logit (largest first, ties to the lower expert id). renorm = 1:
 * weights = softmax over the k chosen logits (= p_j / sum of chosen p);
 * renorm = 0: weights = softmax over all E.
 * Slots (t, j) are grouped by expert, ascending (t, j) inside an expert, each
 * expert's rows start at a multiple of 128.
 * Outputs: topk_idx int32 [T x k], topk_w fp32 [T x k], expert_off int32
 *   [E + 1] (expert_off[E] = used rows), pos int32 [T x k] (slot -> row),
 *   token_of int32 [R] (row -> token, -1 for a padding row),
 *   xq [R x d/2] and xq_sc (MMA layout, R rows) = NVFP4 of x with one tensor
 *   scale for all of x, padding rows zero; x_ts (one fp32).
 *   R = nvfp4moe_max_rows(T, k, E); rows >= expert_off[E] are not written
 *   except token_of (-1).
 * x_amax_in: device fp32 or NULL (NULL: computed here).
 * ws: device workspace of at least moe_route_permute_workspace_size() bytes. */
size_t moe_route_permute_workspace_size(int64_t T, int32_t E, int32_t k);
nvfp4moe_status moe_route_permute(const float *logits, const uint16_t *x, int64_t T, int32_t E,
                                  int32_t k, int64_t d, int renorm, const float *x_amax_in,
                                  int32_t *topk_idx, float *topk_w, int32_t *expert_off,
                                  int32_t *pos, int32_t *token_of, uint8_t *xq, uint8_t *xq_sc,
                                  float *x_ts, void *ws, size_t ws_bytes,
                                  nvfp4moe_stream_t stream);

/* The same routing and dispatch without a workspace argument. The pages have
 * no counterpart to this entry point; it exists for callers that cannot
 * allocate device memory: a process whose device memory is reserved up front
 * by another runtime's allocator (a serving engine holding almost all HBM),
 * so that a cudaMalloc would fail; code called from inside another framework
 * that must not allocate on its own; and latency-critical loops that cannot
 * afford cudaMalloc's implicit device synchronisation.
 * The scratch is a 4 MiB array inside the library (held by every GPU that
 * loads the library until the process exits); calls needing more, i.e. when
 * moe_route_permute_workspace_size(T, E, k) > 4 MiB, are rejected with
 * NVFP4MOE_ERR_WORKSPACE before anything is launched. The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress) and
 * caches it; make that first call before any stream capture. Every call on a
 * device uses the same array and the kernels overwrite all of it that they
 * read, so nothing needs clearing between calls, but two calls that overlap
 * on the GPU (different streams, no ordering between them) race on it.
 * Arguments, outputs and errors are otherwise those of moe_route_permute. */
nvfp4moe_status moe_route_permute_noalloc(const float *logits, const uint16_t *x, int64_t T,
                                          int32_t E, int32_t k, int64_t d, int renorm,
                                          const float *x_amax_in, int32_t *topk_idx,
                                          float *topk_w, int32_t *expert_off, int32_t *pos,
                                          int32_t *token_of, uint8_t *xq, uint8_t *xq_sc,
                                          float *x_ts, nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Expert FFN forward in NVFP4 (news.t0001.com '训练数值格式分工清单'; aicoder.com
 * 'Architecture highlights': NVFP4 forward in the expert layers).
 * For every expert e, rows [expert_off[e], expert_off[e+1]):
 *   [g | u] = dq(xq) . dq(W1_e)^T in fp32 on the tensor cores,
 *   h       = bf16(silu(g) * u),            silu(g) = g / (1 + exp(-g))
 *   h_amax[e] = max |h| over the expert's rows,
 *   hq      = NVFP4(h) with the per-expert tensor scale h_ts[e] = h_amax[e] / 2688,
 *   y       = bf16(dq(hq) . dq(W2_e)^T).
 * xq [R x d/2], xq_sc (MMA), x_ts (one fp32): from moe_route_permute.
 * w1 [E x 2f x d/2] codes, w1_sc MMA layout of the [E*2f x d] matrix, w1_ts
 *   fp32 [E]; rows 0..f-1 of W1_e give g, rows f..2f-1 give u.
 * w2 [E x d x f/2], w2_sc MMA layout of [E*d x f], w2_ts fp32 [E].
 *   (Quantize each expert with nvfp4_quantize, MMA layout, its own amax.)
 * Caller-provided intermediates (outputs too): h bf16 [R x f], hq [R x f/2],
 *   hq_sc MMA layout of [R x f], h_amax fp32 [E], h_ts fp32 [E].
 * y bf16 [R x d]. R = rows_alloc >= expert_off[E], R % 128 == 0.
 * d % 256 == 0, f % 256 == 0, E <= 1024.
 * Three kernel launches: GEMM1 with SwiGLU and the amax of h, the grouped
 * requantization of h, GEMM2. */
nvfp4moe_status moe_expert_fwd(const uint8_t *xq, const uint8_t *xq_sc, const float *x_ts,
                               const int32_t *expert_off, int32_t E, int64_t d, int64_t f,
                               const uint8_t *w1, const uint8_t *w1_sc, const float *w1_ts,
                               const uint8_t *w2, const uint8_t *w2_sc, const float *w2_ts,
                               uint16_t *h, uint8_t *hq, uint8_t *hq_sc, float *h_amax,
                               float *h_ts, uint16_t *y, int64_t rows_alloc,
                               nvfp4moe_stream_t stream);

/* The same expert FFN with the requantization of h fused into GEMM1 (the
 * pages' re-quantization step kept inside the first GEMM's launch: aicoder.com
 * 'Key Takeaways'): every expert is published once its last tile is stored
 * and its rows are requantized by the epilogue warps when their tiles are
 * done, while much of h is still in L2; two kernel launches. Same arguments
 * and results (bit for bit) as moe_expert_fwd, plus ws: a device workspace of
 * at least moe_expert_fwd_fused_requant_workspace_size(E) bytes (16-byte
 * aligned, a few KB), cleared by the call itself (NVFP4MOE_ERR_WORKSPACE if
 * smaller). On B200 it is slower than moe_expert_fwd, which is therefore the
 * default path. */
size_t moe_expert_fwd_fused_requant_workspace_size(int32_t E);
nvfp4moe_status moe_expert_fwd_fused_requant(
    const uint8_t *xq, const uint8_t *xq_sc, const float *x_ts, const int32_t *expert_off,
    int32_t E, int64_t d, int64_t f, const uint8_t *w1, const uint8_t *w1_sc, const float *w1_ts,
    const uint8_t *w2, const uint8_t *w2_sc, const float *w2_ts, uint16_t *h, uint8_t *hq,
    uint8_t *hq_sc, float *h_amax, float *h_ts, uint16_t *y, int64_t rows_alloc, void *ws,
    size_t ws_bytes, nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Expert FFN forward in MXFP8 (aicoder.com 'Architecture highlights': the last
 * 16.6% of layers stay in MXFP8). The same computation as moe_expert_fwd
 * with every operand in MXFP8: E4M3 codes with one E8M0 scale per 32
 * consecutive elements of a row, round-to-nearest-even, no tensor scale.
 * For every expert e, rows [expert_off[e], expert_off[e+1]):
 *   [g | u] = dq(xq) . dq(W1_e)^T in fp32 on the tensor cores,
 *   h       = bf16(silu(g) * u),  h_amax[e] = max |h| over the expert's rows,
 *   hq      = MXFP8(h) along rows (round-to-nearest-even),
 *   y       = bf16(dq(hq) . dq(W2_e)^T).
 * xq [R x d] E4M3 codes in the dispatch layout of moe_route_permute (expert
 *   blocks starting at multiples of 128 rows, padding rows zero), xq_sc the
 *   MMA layout of its [R x d/32] E8M0 scales (mxfp8_quantize, axis 0).
 * w1 [E x 2f x d] codes, w1_sc MMA layout of the [E*2f x d] matrix; rows
 *   0..f-1 of W1_e give g, rows f..2f-1 give u. w2 [E x d x f], w2_sc MMA
 *   layout of [E*d x f]. (Quantize with mxfp8_quantize, axis 0, RNE.)
 * Caller-provided intermediates (outputs too): h bf16 [R x f], h_amax fp32
 *   [E], hq [R x f] codes, hq_sc MMA layout of [R x f/32]. Rows of h and hq
 *   past expert_off[E] hold no meaning.
 * y bf16 [R x d]. R = rows_alloc >= expert_off[E], R % 128 == 0.
 * d % 256 == 0, f % 256 == 0, E <= 1024. Pointers 16-byte aligned (4 for
 * expert_off and h_amax). Errors: NVFP4MOE_ERR_INVALID_ARG, _SHAPE, _ALIGN
 * before any launch; NVFP4MOE_ERR_CUDA for a failed launch. */
nvfp4moe_status moe_expert_fwd_mxfp8(const uint8_t *xq, const uint8_t *xq_sc,
                                     const int32_t *expert_off, int32_t E, int64_t d, int64_t f,
                                     const uint8_t *w1, const uint8_t *w1_sc, const uint8_t *w2,
                                     const uint8_t *w2_sc, uint16_t *h, float *h_amax,
                                     uint8_t *hq, uint8_t *hq_sc, uint16_t *y, int64_t rows_alloc,
                                     nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------
 * SwiGLU backward (news.t0001.com '训练数值格式分工清单': the backward pass of
 * the expert layers runs in MXFP8; this is its elementwise SwiGLU step, whose
 * output is quantized with mxfp8_quantize_sr for the GEMM1 dgrad and wgrad).
 * gu bf16 [rows x 2f]: g in columns 0..f-1, u in f..2f-1 (the layout GEMM1
 * writes with out = X . W1^T, W1 = [gate; up]). dh bf16 [rows x f], the
 * gradient of h = silu(g) * u. Writes dgu bf16 [rows x 2f] = dg | du:
 *   dg = dh * u * s(g) * (1 + g * (1 - s(g))),  du = dh * g * s(g),
 *   s(g) = 1 / (1 + exp(-g)), fp32 arithmetic, bf16 round-to-nearest-even.
 * f % 8 == 0; pointers 16-byte aligned; dgu must not overlap the inputs.
 * rows = 0 is a no-op. Errors: NVFP4MOE_ERR_INVALID_ARG, _SHAPE, _ALIGN
 * before any launch; NVFP4MOE_ERR_CUDA for a failed launch. */
nvfp4moe_status swiglu_bwd(const uint16_t *gu, const uint16_t *dh, int64_t rows, int64_t f,
                           uint16_t *dgu, nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------
 * GEMM1 backward in MXFP8 (news.t0001.com '训练数值格式分工清单'; aicoder.com
 * 'Architecture highlights': MXFP8 backward with stochastic rounding of the
 * re-quantized gradients). For every expert e, rows [expert_off[e],
 * expert_off[e+1]) (starts at multiples of 128, as moe_route_permute lays
 * them out):
 *   dX_e  = dq(SR(dgu) along 2f)_e . dq(W1_e along 2f)       -> dx bf16 [R x d]
 *   dW1_e = dq(SR(dgu) along rows)_e^T . dq(RNE(x) along rows)_e -> dw1 fp32 [E x 2f x d]
 * dgu bf16 [R x 2f] (dg | du, e.g. from swiglu_bwd), x bf16 [R x d]: the
 *   experts' input rows; rows past expert_off[E] are quantized but never read.
 * w1t, w1t_sc: W1^T of every expert in MXFP8 with blocks along 2f, codes
 *   [E*d x 2f] and the MMA layout of its [E*d x 2f/32] scales
 *   (mxfp8_quantize_sr(W1_e, axis 1, RNE, MMA) per expert).
 * Stochastic draws: Philox stream (seed, offset) for the row-wise
 *   quantization of dgu, (seed, offset + 1) for the column-wise one, each
 *   element at its row-major index in [R x 2f].
 * Caller-provided intermediates (outputs too), all scales in the MMA layout:
 *   gq [R x 2f] + gq_sc (dgu along 2f), gt [2f x R] + gt_sc (dgu along rows,
 *   transposed), xt [d x R] + xt_sc (x along rows, transposed).
 * R = rows_alloc % 128 == 0, d % 256 == 0, f % 128 == 0, E <= 1024.
 * Errors: NVFP4MOE_ERR_INVALID_ARG, _SHAPE, _ALIGN before any launch;
 * NVFP4MOE_ERR_CUDA for a failed launch. */
nvfp4moe_status moe_expert_bwd_gemm1(const uint16_t *dgu, const uint16_t *x,
                                     const int32_t *expert_off, int32_t E, int64_t d, int64_t f,
                                     const uint8_t *w1t, const uint8_t *w1t_sc, uint64_t seed,
                                     uint64_t offset, uint8_t *gq, uint8_t *gq_sc, uint8_t *gt,
                                     uint8_t *gt_sc, uint8_t *xt, uint8_t *xt_sc, uint16_t *dx,
                                     float *dw1, int64_t rows_alloc, nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Weighted top-k combine (aicoder.com 'Key Takeaways': the combine step).
 * out[t] = bf16( sum_{j=0..k-1} topk_w[t,j] * y[pos[t,j]] ), fp32 accumulation
 * in slot order with fused multiply-adds; a gather, no atomics.
 * y bf16 [* x d] (row stride d); pos, topk_w [T x k]; out bf16 [T x d].
 * d % 8 == 0. */
nvfp4moe_status moe_combine(const uint16_t *y, const int32_t *pos, const float *topk_w,
                            int64_t T, int32_t k, int64_t d, uint16_t *out,
                            nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Combine straight from the RHT32-quantized payload (aicoder.com 'Key
 * Takeaways' and 'Architecture highlights': the expert-parallel combine
 * traffic travels block-scaled after a 32-point random Hadamard transform).
 * out[t] = bf16( RHT32^-1( sum_{j=0..k-1} topk_w[t,j] * v[pos[t,j]] ) ) per
 * 32-block: the dequantized payload rows v are summed in fp32 in slot order
 * with fused multiply-adds, then transformed once per token (the transform is
 * linear, so this is the combine of the inverse-transformed rows).
 * codes / scales / ts: a payload as written by rht32_quantize with the same
 * sign_seed and fmt, ROWMAJOR scales: NVFP4 codes [* x d/2], scales
 * [* x d/16], ts one device fp32; MXFP8 codes [* x d], scales [* x d/32], ts
 * unused (may be NULL). pos, topk_w [T x k]; out bf16 [T x d]. d % 32 == 0.
 * Caller owns all buffers; nothing is allocated. */
nvfp4moe_status moe_combine_rht(const uint8_t *codes, const uint8_t *scales, const float *ts,
                                int fmt, uint64_t sign_seed, const int32_t *pos,
                                const float *topk_w, int64_t T, int32_t k, int64_t d,
                                uint16_t *out, nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Grouped block-scaled GEMMs on the tcgen05 tensor cores.
 *
 * nvfp4_grouped_gemm: for every group g, rows [off[g], off[g+1]) of A
 *   (multiples of 128):  C[rows] = alpha_g * dq(A[rows]) . dq(B_g)^T with
 *   alpha_g = a_ts[g * a_ts_stride] * b_ts[g], fp32 accumulation.
 *   A [R x K/2] NVFP4 + MMA scales; B [G x N x K/2] + MMA scales of [G*N x K];
 *   C [R x N] bf16 or fp32 (out_dtype), row stride N. K % 256 == 0,
 *   N % 256 == 0, G <= 1024, R % 128 == 0.
 * mxfp8_grouped_gemm: E4M3 x E4M3 with E8M0 scales (MMA layout), fp32 accumulation.
 *   group_axis M: as above with A [R x K], B [G x N x K], C [R x N].
 *   group_axis K: group g contracts over columns [off[g], off[g+1]) of
 *     A [M x Kt] and B [N x Kt] (offsets multiples of 128) into C_g [M x N];
 *     C [G x M x N] (a group with no columns writes zeros). M % 128 == 0.
 *   K % 128 == 0 (group M), N % 256 == 0. */
nvfp4moe_status nvfp4_grouped_gemm(const uint8_t *a, const uint8_t *a_sc, const float *a_ts,
                                   int32_t a_ts_stride, const uint8_t *b, const uint8_t *b_sc,
                                   const float *b_ts, const int32_t *group_off, int32_t G,
                                   int64_t R, int64_t N, int64_t K, void *c, int out_dtype,
                                   nvfp4moe_stream_t stream);
nvfp4moe_status mxfp8_grouped_gemm(const uint8_t *a, const uint8_t *a_sc, const uint8_t *b,
                                   const uint8_t *b_sc, const int32_t *group_off, int32_t G,
                                   int group_axis, int64_t M, int64_t N, int64_t K, void *c,
                                   int out_dtype, nvfp4moe_stream_t stream);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif

#ifdef __cplusplus
}
#endif
#endif /* NVFP4MOE_H */

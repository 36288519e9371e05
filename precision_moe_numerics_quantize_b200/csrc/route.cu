// Router top-k, deterministic counting-sort dispatch with fused NVFP4
// quantization of the token rows, and the weighted top-k combine.
//
// Dispatch is a stable counting sort of the routed slots (t, j) by expert:
//   1. top-k per token (one warp per token),
//   2. per-chunk expert histograms with stable ranks inside each chunk of
//      1024 slots (one warp per chunk, warp-synchronous in slot order),
//   3. one CTA turns the histograms into per-expert row offsets (each expert
//      padded to a multiple of 128 rows) and per-chunk bases,
//   4. scatter: row = base[chunk][e] + rank; token_of[row] = t,
//   5. every token row of x is quantized to NVFP4 once and its codes and
//      scales are copied to its k rows; padding rows are zero-filled.
// No step depends on the order in which atomics land, so the result is
// identical on every run.
#include "common.cuh"
#include "quant.cuh"

namespace nvfp4moe {

static constexpr int CHUNK = 1024;

// ---------------------------------------------------------------------------
// 1. top-k: one warp per token; lane l owns experts l, l + 32, ... (PER of
// them); k rounds of a warp argmax (largest logit, ties to the lower expert
// id). Lane j keeps the j-th choice, so nothing is indexed at run time.
// ---------------------------------------------------------------------------
template <int PER>
__global__ void __launch_bounds__(256) topk_kernel(const float *__restrict__ logits, int64_t T,
                                                   int32_t E, int32_t k, int renorm,
                                                   int32_t *__restrict__ idx_out,
                                                   float *__restrict__ w_out) {
    const int lane = threadIdx.x & 31;
    const int64_t t = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float *l = logits + t * E;
    const float ninf = __int_as_float(0xff800000);
    float v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? __ldg(l + e) : ninf;
    }
    uint32_t taken = 0;  // bit i: element i of this lane already chosen
    float my_l = 0.0f, mx = 0.0f;
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
        float bv = ninf;
        int be = 0x7FFFFFFF;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = lane + 32 * i;
            const bool ok = e < E && !((taken >> i) & 1u);
            if (ok && (v[i] > bv || (v[i] == bv && e < be) || be == 0x7FFFFFFF)) {
                bv = v[i];
                be = e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
            const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, o);
            if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == j) {
            my_l = bv;
            my_e = be;
        }
        if (j == 0) mx = bv;
    }
    // weights: softmax over the chosen logits (renorm) or over all E, each
    // sum a fixed-order tree over the lanes
    float s = 0.0f;
    if (renorm) {
        s = lane < k ? expf(my_l - mx) : 0.0f;
    } else {
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = lane + 32 * i;
            if (e < E) s += expf(v[i] - mx);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    if (lane < k) {
        idx_out[t * k + lane] = my_e;
        w_out[t * k + lane] = expf(my_l - mx) / s;
    }
}

// ---------------------------------------------------------------------------
// 2. per-chunk histograms and stable in-chunk ranks (one warp per chunk).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) chunk_rank_kernel(const int32_t *__restrict__ idx,
                                                         int64_t n_slots, int32_t E,
                                                         int32_t *__restrict__ counts,
                                                         int32_t *__restrict__ rank_out) {
    extern __shared__ int32_t s_cnt[];  // [warps][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t chunk = blockIdx.x * (int64_t)(blockDim.x >> 5) + warp;
    int32_t *cnt = s_cnt + warp * E;
    for (int e = lane; e < E; e += 32) cnt[e] = 0;
    __syncwarp();
    const int64_t base = chunk * CHUNK;
    if (base < n_slots) {
        const int64_t end = (base + CHUNK < n_slots) ? base + CHUNK : n_slots;
        const uint32_t lt = (1u << lane) - 1u;
        for (int64_t s0 = base; s0 < end; s0 += 32) {
            const int64_t s = s0 + lane;
            const bool valid = s < end;
            const int e = valid ? idx[s] : -1 - lane;  // invalid lanes never match a real expert
            const uint32_t peers = __match_any_sync(0xFFFFFFFFu, e);
            const int leader = __ffs(peers) - 1;
            int b = 0;
            if (lane == leader && valid) b = cnt[e];
            b = __shfl_sync(0xFFFFFFFFu, b, leader);
            if (valid) rank_out[s] = b + __popc(peers & lt);
            __syncwarp();
            if (lane == leader && valid) cnt[e] = b + __popc(peers);
            __syncwarp();
        }
        for (int e = lane; e < E; e += 32) counts[chunk * E + e] = cnt[e];
    }
}

// ---------------------------------------------------------------------------
// 3. offsets: one CTA. Per expert: running sums over chunks (bases), total,
// padded total; exclusive scan over experts.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) offsets_kernel(int32_t *__restrict__ counts,
                                                       int64_t n_chunks, int32_t E,
                                                       int32_t *__restrict__ expert_off,
                                                       int32_t *__restrict__ expert_cnt) {
    __shared__ int32_t s_warp[32];
    const int e = threadIdx.x;
    int32_t total = 0;
    if (e < E) {
        // eight independent loads in flight per round
        int64_t c = 0;
        for (; c + 8 <= n_chunks; c += 8) {
            int32_t v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = counts[(c + u) * E + e];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                counts[(c + u) * E + e] = total;  // exclusive base within the expert
                total += v[u];
            }
        }
        for (; c < n_chunks; ++c) {
            const int32_t v = counts[c * E + e];
            counts[c * E + e] = total;
            total += v;
        }
        expert_cnt[e] = total;
    }
    int32_t pad = (e < E) ? (total + 127) / 128 * 128 : 0;
    // block-wide exclusive scan of pad (fixed order)
    const int lane = e & 31, warp = e >> 5;
    int32_t incl = pad;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int32_t n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t w = (lane < (int)(blockDim.x >> 5)) ? s_warp[lane] : 0;
        int32_t wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int32_t n = __shfl_up_sync(0xFFFFFFFFu, wi, o);
            if (lane >= o) wi += n;
        }
        s_warp[lane] = wi - w;
    }
    __syncthreads();
    const int32_t excl = s_warp[warp] + incl - pad;
    if (e < E) expert_off[e] = excl;
    if (e == E - 1) expert_off[E] = excl + pad;
}

// ---------------------------------------------------------------------------
// 4. scatter: pos and token_of.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) scatter_kernel(const int32_t *__restrict__ idx,
                                                      const int32_t *__restrict__ rank,
                                                      const int32_t *__restrict__ bases,
                                                      const int32_t *__restrict__ expert_off,
                                                      int64_t n_slots, int32_t E, int32_t k,
                                                      int32_t *__restrict__ pos,
                                                      int32_t *__restrict__ token_of) {
    for (int64_t s = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; s < n_slots;
         s += (int64_t)gridDim.x * blockDim.x) {
        const int e = idx[s];
        const int64_t chunk = s / CHUNK;
        const int32_t row = expert_off[e] + bases[chunk * E + e] + rank[s];
        pos[s] = row;
        token_of[row] = (int32_t)(s / k);
    }
}

// ---------------------------------------------------------------------------
// 5. quantize token rows once and copy to their k destination rows; zero the
// padding rows of every expert.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dispatch_quant_kernel(
    const uint16_t *__restrict__ x, int64_t T, int64_t d, int32_t k,
    const float *__restrict__ amax_p, const int32_t *__restrict__ pos,
    uint8_t *__restrict__ xq, uint8_t *__restrict__ xq_sc, float *__restrict__ x_ts,
    int write_ts) {
    __shared__ float enc_tab[128];
    const float amax = *amax_p;
    const float S_enc = nvfp4_senc(amax);
    fill_enc_table(enc_tab, S_enc);
    __syncthreads();
    if (write_ts && blockIdx.x == 0 && threadIdx.x == 0) *x_ts = nvfp4_ts(amax);
    const int64_t G = d / 64;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < T * G;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / G, g = i - t * G;
        const uint4 *pv = reinterpret_cast<const uint4 *>(x + t * d + g * 64);
        uint4 raw[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) raw[j] = __ldg(pv + j);
        uint32_t w[8], scw = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            float v[16];
            unpack_bf16x8(raw[2 * b], v);
            unpack_bf16x8(raw[2 * b + 1], v + 8);
            scw |= nvfp4_block16_tab(v, S_enc, enc_tab, w[2 * b], w[2 * b + 1]) << (8 * b);
        }
        const uint4 c0 = make_uint4(w[0], w[1], w[2], w[3]);
        const uint4 c1 = make_uint4(w[4], w[5], w[6], w[7]);
        for (int j = 0; j < k; ++j) {
            const int64_t row = pos[t * k + j];
            uint4 *co = reinterpret_cast<uint4 *>(xq + row * (d / 2) + g * 32);
            co[0] = c0;
            co[1] = c1;
            *reinterpret_cast<uint32_t *>(xq_sc + mma_sf_offset(row, g * 4, d / 16)) = scw;
        }
    }
}

// One CTA per expert: its padding rows are [off_e + cnt_e, off_{e+1}).
__global__ void __launch_bounds__(256) zero_pad_rows_kernel(
    const int32_t *__restrict__ expert_cnt, const int32_t *__restrict__ expert_off, int64_t d,
    uint8_t *__restrict__ xq, uint8_t *__restrict__ xq_sc) {
    const int e = blockIdx.x;
    const int64_t r0 = (int64_t)expert_off[e] + expert_cnt[e];
    const int64_t n = (int64_t)expert_off[e + 1] - r0;
    const int64_t G = d / 64;
    for (int64_t i = threadIdx.x; i < n * G; i += blockDim.x) {
        const int64_t r = r0 + i / G, g = i % G;
        uint4 *co = reinterpret_cast<uint4 *>(xq + r * (d / 2) + g * 32);
        co[0] = make_uint4(0, 0, 0, 0);
        co[1] = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint32_t *>(xq_sc + mma_sf_offset(r, g * 4, d / 16)) = 0u;
    }
}

// ---------------------------------------------------------------------------
// combine: one thread per (token, 8 columns); slot order, fp32 fused multiply-add.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t *__restrict__ y,
                                                      const int32_t *__restrict__ pos,
                                                      const float *__restrict__ w, int64_t T,
                                                      int32_t k, int64_t d,
                                                      uint16_t *__restrict__ out) {
    const int64_t G = d / 8;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < T * G;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / G, g = i - t * G;
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int j = 0; j < k; ++j) {
            const int64_t row = pos[t * k + j];
            const float wj = w[t * k + j];
            const uint4 q = __ldg(reinterpret_cast<const uint4 *>(y + row * d + g * 8));
            acc[0] = fmaf(wj, bf16_lo(q.x), acc[0]);
            acc[1] = fmaf(wj, bf16_hi(q.x), acc[1]);
            acc[2] = fmaf(wj, bf16_lo(q.y), acc[2]);
            acc[3] = fmaf(wj, bf16_hi(q.y), acc[3]);
            acc[4] = fmaf(wj, bf16_lo(q.z), acc[4]);
            acc[5] = fmaf(wj, bf16_hi(q.z), acc[5]);
            acc[6] = fmaf(wj, bf16_lo(q.w), acc[6]);
            acc[7] = fmaf(wj, bf16_hi(q.w), acc[7]);
        }
        uint4 o;
        o.x = f32_to_bf16_bits(acc[0]) | (f32_to_bf16_bits(acc[1]) << 16);
        o.y = f32_to_bf16_bits(acc[2]) | (f32_to_bf16_bits(acc[3]) << 16);
        o.z = f32_to_bf16_bits(acc[4]) | (f32_to_bf16_bits(acc[5]) << 16);
        o.w = f32_to_bf16_bits(acc[6]) | (f32_to_bf16_bits(acc[7]) << 16);
        *reinterpret_cast<uint4 *>(out + t * d + g * 8) = o;
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static int64_t n_chunks_of(int64_t T, int32_t k) { return (T * k + CHUNK - 1) / CHUNK; }

static size_t align256(size_t b) { return (b + 255) / 256 * 256; }

// workspace: counts/bases [n_chunks x E], ranks [T*k], expert_cnt [E], amax [1]
size_t route_permute_ws_bytes(int64_t T, int32_t E, int32_t k) {
    const int64_t nc = n_chunks_of(T, k);
    return align256(sizeof(int32_t) * nc * E) + align256(sizeof(int32_t) * T * k) +
           align256(sizeof(int32_t) * E) + align256(sizeof(float));
}

static int grid_cap(int64_t work, int per = 256) {
    int64_t g = (work + per - 1) / per;
    if (g > 148 * 16) g = 148 * 16;
    return (int)(g < 1 ? 1 : g);
}

cudaError_t launch_route_permute(const float *logits, const uint16_t *x, int64_t T, int32_t E,
                                 int32_t k, int64_t d, int renorm, const float *x_amax_in,
                                 int32_t *topk_idx, float *topk_w, int32_t *expert_off,
                                 int32_t *pos, int32_t *token_of, uint8_t *xq, uint8_t *xq_sc,
                                 float *x_ts, void *ws, int64_t rows_alloc, cudaStream_t s) {
    cudaError_t e;
    const int64_t n_slots = T * k;
    const int64_t nc = n_chunks_of(T, k);
    char *p = static_cast<char *>(ws);
    int32_t *counts = reinterpret_cast<int32_t *>(p);
    p += align256(sizeof(int32_t) * nc * E);
    int32_t *ranks = reinterpret_cast<int32_t *>(p);
    p += align256(sizeof(int32_t) * T * k);
    int32_t *expert_cnt = reinterpret_cast<int32_t *>(p);
    p += align256(sizeof(int32_t) * E);
    float *amax = reinterpret_cast<float *>(p);

    if ((e = cudaMemsetAsync(token_of, 0xFF, sizeof(int32_t) * rows_alloc, s)) != cudaSuccess)
        return e;
    if (T > 0) {
        const unsigned tgrid = (unsigned)((T + 7) / 8);
        const int per = (E + 31) / 32;
        if (per <= 4)
            topk_kernel<4><<<tgrid, 256, 0, s>>>(logits, T, E, k, renorm, topk_idx, topk_w);
        else if (per <= 8)
            topk_kernel<8><<<tgrid, 256, 0, s>>>(logits, T, E, k, renorm, topk_idx, topk_w);
        else if (per <= 12)
            topk_kernel<12><<<tgrid, 256, 0, s>>>(logits, T, E, k, renorm, topk_idx, topk_w);
        else if (per <= 16)
            topk_kernel<16><<<tgrid, 256, 0, s>>>(logits, T, E, k, renorm, topk_idx, topk_w);
        else
            topk_kernel<32><<<tgrid, 256, 0, s>>>(logits, T, E, k, renorm, topk_idx, topk_w);
        const int warps = 4;
        chunk_rank_kernel<<<(unsigned)((nc + warps - 1) / warps), 32 * warps,
                            warps * E * sizeof(int32_t), s>>>(topk_idx, n_slots, E, counts,
                                                              ranks);
    }
    offsets_kernel<<<1, 1024, 0, s>>>(counts, nc, E, expert_off, expert_cnt);
    if (T > 0)
        scatter_kernel<<<grid_cap(n_slots), 256, 0, s>>>(topk_idx, ranks, counts, expert_off,
                                                        n_slots, E, k, pos, token_of);
    const float *amax_use = x_amax_in;
    if (!x_amax_in) {
        if ((e = launch_amax_bf16(x, T, d, d, amax, s)) != cudaSuccess) return e;
        amax_use = amax;
    }
    if (T > 0)
        dispatch_quant_kernel<<<grid_cap(T * (d / 64)), 256, 0, s>>>(x, T, d, k, amax_use, pos, xq,
                                                                    xq_sc, x_ts, 1);
    else
        dispatch_quant_kernel<<<1, 32, 0, s>>>(x, 0, d, k, amax_use, pos, xq, xq_sc, x_ts, 1);
    zero_pad_rows_kernel<<<E, 256, 0, s>>>(expert_cnt, expert_off, d, xq, xq_sc);
    return cudaGetLastError();
}

cudaError_t launch_combine(const uint16_t *y, const int32_t *pos, const float *w, int64_t T,
                           int32_t k, int64_t d, uint16_t *out, cudaStream_t s) {
    if (T * d == 0) return cudaSuccess;
    combine_kernel<<<grid_cap(T * (d / 8)), 256, 0, s>>>(y, pos, w, T, k, d, out);
    return cudaGetLastError();
}

}  // namespace nvfp4moe

// ---------------------------------------------------------------------------
// Dispatch without a caller-provided workspace: the scratch lives in a
// file-scope device array of fixed size, shared by every call on a device.
// ---------------------------------------------------------------------------
#include <mutex>

namespace nvfp4moe {

static constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB

// Every GPU that loads the library keeps this array until the process exits.
static __device__ __align__(256) uint8_t g_route_scratch[kNoAllocScratchBytes];

// Device address of g_route_scratch in the current device and context. In
// host code the array's name is only a stand-in, so the address is looked up
// with cudaGetSymbolAddress on the first call in each device and driver
// context (the module, and with it the array, is loaded once per context)
// and cached.
static void *route_scratch_address(nvfp4moe_status *st) {
    static SymbolAddressCache cache;
    void *p = nullptr;
    cudaError_t e = cached_symbol_address(cache, g_route_scratch, &p);
    if (e != cudaSuccess) {
        *st = cuda_status(e, "moe_route_permute_noalloc: cudaGetSymbolAddress");
        return nullptr;
    }
    return p;
}

}  // namespace nvfp4moe

extern "C" nvfp4moe_status moe_route_permute_noalloc(
    const float *logits, const uint16_t *x, int64_t T, int32_t E, int32_t k, int64_t d,
    int renorm, const float *x_amax_in, int32_t *topk_idx, float *topk_w, int32_t *expert_off,
    int32_t *pos, int32_t *token_of, uint8_t *xq, uint8_t *xq_sc, float *x_ts,
    nvfp4moe_stream_t stream) {
    using namespace nvfp4moe;
    nvfp4moe_status st = check_route_permute_args(logits, x, T, E, k, d, renorm, x_amax_in,
                                                  topk_idx, topk_w, expert_off, pos, token_of,
                                                  xq, xq_sc, x_ts);
    if (st) return st;
    const size_t need = route_permute_ws_bytes(T, E, k);
    if (need > kNoAllocScratchBytes) {
        set_last_error(
            "moe_route_permute_noalloc: T=%lld, E=%d, k=%d needs %zu bytes of scratch, more than "
            "the built-in %zu; use moe_route_permute with a workspace",
            (long long)T, E, k, need, kNoAllocScratchBytes);
        return NVFP4MOE_ERR_WORKSPACE;
    }
    void *ws = route_scratch_address(&st);
    if (!ws) return st;
    cudaError_t e = launch_route_permute(logits, x, T, E, k, d, renorm, x_amax_in, topk_idx,
                                         topk_w, expert_off, pos, token_of, xq, xq_sc, x_ts, ws,
                                         nvfp4moe_max_rows(T, k, E), (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaGetLastError();
    return cuda_status(e, "moe_route_permute_noalloc");
}

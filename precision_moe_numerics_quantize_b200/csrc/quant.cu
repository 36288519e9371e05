// Bandwidth-bound quantizers: tensor amax, NVFP4 (16-element E4M3-scaled
// E2M1), MXFP8 (32-element E8M0-scaled E4M3, nearest or Philox stochastic
// rounding, along rows or along columns), and the 32-point random Hadamard
// transform followed by block-scaled quantization of the combine payload.
//
// Every kernel reads its input with 16-byte vector loads in a coalesced
// pattern and writes codes with 16-byte stores; scales are written either
// row-major or directly in the tcgen05 MMA layout (512-byte chunks of
// 128 rows x 4 scales) so that the GEMMs can stream them with bulk copies.
#include "common.cuh"
#include "quant.cuh"

namespace nvfp4moe {

__device__ int32_t g_device_error = 0;

// Device address of g_device_error in the current device and context.
int32_t *device_error_word() {
    static SymbolAddressCache cache;
    void *p = nullptr;
    if (cached_symbol_address(cache, &g_device_error, &p) != cudaSuccess) return nullptr;
    return static_cast<int32_t *>(p);
}

// ---------------------------------------------------------------------------
// amax of a bf16 tensor. *amax must be zero before the launch.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) amax_bf16_kernel(const uint16_t *__restrict__ x,
                                                        int64_t rows, int64_t cols, int64_t ld,
                                                        float *__restrict__ amax) {
    float m = 0.0f;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    if (ld == cols) {
        // contiguous: one flat run of 16-byte vectors, two loads in flight per step
        const uint4 *xv = reinterpret_cast<const uint4 *>(x);
        const int64_t nvec = rows * cols / 8;
        for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nvec; i += 2 * stride) {
            const uint4 v = __ldg(xv + i);
            const uint4 w = (i + stride < nvec) ? __ldg(xv + i + stride) : make_uint4(0, 0, 0, 0);
            m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))),
                               fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y)))));
            m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))),
                               fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w)))));
            m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(w.x)), fabsf(bf16_hi(w.x))),
                               fmaxf(fabsf(bf16_lo(w.y)), fabsf(bf16_hi(w.y)))));
            m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(w.z)), fabsf(bf16_hi(w.z))),
                               fmaxf(fabsf(bf16_lo(w.w)), fabsf(bf16_hi(w.w)))));
        }
    } else {
        const int64_t vpr = cols / 8;  // 16-byte vectors per row
        for (int64_t r = blockIdx.y; r < rows; r += gridDim.y)
            for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < vpr; c += stride) {
                const uint4 v = __ldg(reinterpret_cast<const uint4 *>(x + r * ld) + c);
                m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))),
                                   fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y)))));
                m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))),
                                   fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w)))));
            }
    }
    m = warp_max(m);
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
        v = warp_max(v);
        if (threadIdx.x == 0) atomic_max_nonneg(amax, v);
    }
}

// ---------------------------------------------------------------------------
// NVFP4: per-tensor S_enc from amax; one thread quantizes 64 consecutive
// elements (4 blocks of 16): 128 bytes in, 32 bytes of codes and 4 scales out.
// ---------------------------------------------------------------------------
NV_DEV void unpack8(uint4 q, float *f) { unpack_bf16x8(q, f); }

// 64 bf16 elements at p -> 32 code bytes at out_codes, 4 scale codes packed in a word.
NV_DEV uint32_t nvfp4_quant64(const uint16_t *__restrict__ p, float S_enc, uint4 &c0, uint4 &c1) {
    const uint4 *pv = reinterpret_cast<const uint4 *>(p);
    uint32_t scw = 0;
    uint32_t w[8];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        float v[16];
        unpack8(__ldg(pv + 2 * b), v);
        unpack8(__ldg(pv + 2 * b + 1), v + 8);
        uint32_t sc = nvfp4_block16(v, S_enc, w[2 * b], w[2 * b + 1]);
        scw |= sc << (8 * b);
    }
    c0 = make_uint4(w[0], w[1], w[2], w[3]);
    c1 = make_uint4(w[4], w[5], w[6], w[7]);
    return scw;
}

// Same with the per-tensor encode table; all eight 16-byte loads issued first.
NV_DEV uint32_t nvfp4_quant64_tab(const uint16_t *__restrict__ p, float S_enc, const float *enc_tab,
                                  uint4 &c0, uint4 &c1) {
    const uint4 *pv = reinterpret_cast<const uint4 *>(p);
    uint4 raw[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) raw[j] = __ldg(pv + j);
    uint32_t scw = 0;
    uint32_t w[8];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        float v[16];
        unpack8(raw[2 * b], v);
        unpack8(raw[2 * b + 1], v + 8);
        uint32_t sc = nvfp4_block16_tab(v, S_enc, enc_tab, w[2 * b], w[2 * b + 1]);
        scw |= sc << (8 * b);
    }
    c0 = make_uint4(w[0], w[1], w[2], w[3]);
    c1 = make_uint4(w[4], w[5], w[6], w[7]);
    return scw;
}

__global__ void __launch_bounds__(256) nvfp4_quant_kernel(
    const uint16_t *__restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    const float *__restrict__ amax_p, uint8_t *__restrict__ codes, uint8_t *__restrict__ scales,
    float *__restrict__ ts_out, int layout) {
    __shared__ float enc_tab[128];
    const float amax = *amax_p;
    const float S_enc = nvfp4_senc(amax);
    fill_enc_table(enc_tab, S_enc);
    __syncthreads();
    const uint32_t G = (uint32_t)(cols / 64);
    const uint32_t n = (uint32_t)(rows * G);  // < 2^31 (checked by the caller)
    if (ts_out && blockIdx.x == 0 && threadIdx.x == 0) *ts_out = nvfp4_ts(amax);
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const uint32_t r = i / G, g = i - r * G;
        uint4 c0, c1;
        const uint32_t scw = nvfp4_quant64_tab(x + (int64_t)r * ld + g * 64, S_enc, enc_tab, c0, c1);
        uint4 *co = reinterpret_cast<uint4 *>(codes + (int64_t)i * 32);
        co[0] = c0;
        co[1] = c1;
        if (layout == NVFP4MOE_LAYOUT_ROWMAJOR)
            *reinterpret_cast<uint32_t *>(scales + (int64_t)i * 4) = scw;
        else
            *reinterpret_cast<uint32_t *>(scales + mma_sf_offset(r, g * 4, G * 4)) = scw;
    }
}

// Writes ts = amax / 2688 after a two-pass quantization.
__global__ void nvfp4_finalize_ts_kernel(float *ts_inout) {
    *ts_inout = nvfp4_ts(*ts_inout);
}

__global__ void __launch_bounds__(256) nvfp4_dequant_kernel(
    const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales,
    const float *__restrict__ ts_p, int64_t rows, int64_t cols, int layout,
    float *__restrict__ out) {
    const float ts = *ts_p;
    const int64_t G = cols / 16;
    const int64_t n = rows * G;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        int64_t r = i / G, b = i - r * G;
        uint32_t sc = layout == NVFP4MOE_LAYOUT_ROWMAJOR ? scales[r * G + b]
                                                         : scales[mma_sf_offset(r, b, G)];
        float sf = e4m3_decode(sc);
        uint2 q = *reinterpret_cast<const uint2 *>(codes + r * (cols / 2) + b * 8);
        float o[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) o[j] = __fmul_rn(e2m1_decode((q.x >> (4 * j)) & 15u) * sf, ts);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            o[8 + j] = __fmul_rn(e2m1_decode((q.y >> (4 * j)) & 15u) * sf, ts);
        float4 *op = reinterpret_cast<float4 *>(out + r * cols + b * 16);
        op[0] = make_float4(o[0], o[1], o[2], o[3]);
        op[1] = make_float4(o[4], o[5], o[6], o[7]);
        op[2] = make_float4(o[8], o[9], o[10], o[11]);
        op[3] = make_float4(o[12], o[13], o[14], o[15]);
    }
}

// ---------------------------------------------------------------------------
// MXFP8 along rows: one thread per 128 consecutive elements of a row (4 blocks).
// ---------------------------------------------------------------------------
template <bool SR>
NV_DEV uint32_t mx_block32(const float (&v)[32], uint64_t seed, uint64_t offset, uint64_t idx0,
                           uint32_t (&w)[8]) {
    float amax_b = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax_b = fmaxf(amax_b, fabsf(v[i]));
    const int k = mx_scale_exp(amax_b);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        float s0 = scale_pow2(v[4 * q], k), s1 = scale_pow2(v[4 * q + 1], k);
        float s2 = scale_pow2(v[4 * q + 2], k), s3 = scale_pow2(v[4 * q + 3], k);
        if (SR) {
            // idx0 is a multiple of 4 (cols % 32 == 0): one Philox call per 4 elements
            const u32x4 r = philox_block(seed, offset, (idx0 >> 2) + q);
            s0 = e4m3_sr_value(s0, r.x);
            s1 = e4m3_sr_value(s1, r.y);
            s2 = e4m3_sr_value(s2, r.z);
            s3 = e4m3_sr_value(s3, r.w);
        }
        // on-grid values (SR) convert exactly; otherwise this is the RNE encode
        w[q] = e4m3x2_hw(s0, s1) | (e4m3x2_hw(s2, s3) << 16);
    }
    return (uint32_t)(k + 127);
}

template <bool SR>
__global__ void __launch_bounds__(256, 4) mxfp8_rows_kernel(
    const uint16_t *__restrict__ x, int64_t rows, int64_t cols, int64_t ld, uint64_t seed,
    uint64_t offset, uint8_t *__restrict__ codes, uint8_t *__restrict__ scales, int layout) {
    const uint32_t G = (uint32_t)(cols / 32);  // blocks per row
    const uint32_t n = (uint32_t)(rows * G);
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const uint32_t r = i / G, b = i - r * G;
        const uint4 *pv = reinterpret_cast<const uint4 *>(x + (int64_t)r * ld + b * 32);
        uint4 raw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) raw[j] = __ldg(pv + j);
        float v[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) unpack8(raw[j], v + 8 * j);
        uint32_t w[8];
        const uint32_t sc = mx_block32<SR>(v, seed, offset, (uint64_t)r * cols + b * 32, w);
        uint4 *co = reinterpret_cast<uint4 *>(codes + (int64_t)i * 32);
        co[0] = make_uint4(w[0], w[1], w[2], w[3]);
        co[1] = make_uint4(w[4], w[5], w[6], w[7]);
        if (layout == NVFP4MOE_LAYOUT_ROWMAJOR)
            scales[i] = (uint8_t)sc;
        else
            scales[mma_sf_offset(r, b, G)] = (uint8_t)sc;
    }
}

// ---------------------------------------------------------------------------
// MXFP8 along columns, transposed output. A warp owns a 32-row x 32-column
// patch: lane = 8 rq + cq holds rows 8 rq .. 8 rq + 7 of the patch's 32-row
// block and the four adjacent columns 4 cq .. 4 cq + 3. It reads them straight
// from global memory (each row a 64-byte run per row quarter), the block amax
// of a column joins its four row quarters with two shuffles, and the four
// elements of a row are consecutive in the source, so one Philox call per row
// gives all four their random words. No shared memory: occupancy is set by
// registers alone.
// ---------------------------------------------------------------------------
template <bool SR>
__global__ void __launch_bounds__(256, 3) mxfp8_cols_kernel(
    const uint16_t *__restrict__ x, int64_t rows, int64_t cols, int64_t ld, uint64_t seed,
    uint64_t offset, uint8_t *__restrict__ codes, uint8_t *__restrict__ scales, int layout) {
    const int lane = threadIdx.x & 31, rq = lane >> 3, cq = lane & 7;
    const int64_t G = rows / 32;          // scales per output row
    const int64_t CP = cols / 32;         // column patches
    const int64_t items = G * CP;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t it = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); it < items;
         it += warps) {
        const int64_t b = it / CP, cp = it - b * CP;
        const int64_t r0 = b * 32 + rq * 8, c = cp * 32 + cq * 4;
        uint2 q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = __ldg(reinterpret_cast<const uint2 *>(x + (r0 + i) * ld + c));
        float am0 = 0.0f, am1 = 0.0f, am2 = 0.0f, am3 = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            am0 = fmaxf(am0, fabsf(bf16_lo(q[i].x)));
            am1 = fmaxf(am1, fabsf(bf16_hi(q[i].x)));
            am2 = fmaxf(am2, fabsf(bf16_lo(q[i].y)));
            am3 = fmaxf(am3, fabsf(bf16_hi(q[i].y)));
        }
#pragma unroll
        for (int m = 8; m <= 16; m <<= 1) {
            am0 = fmaxf(am0, __shfl_xor_sync(0xFFFFFFFFu, am0, m));
            am1 = fmaxf(am1, __shfl_xor_sync(0xFFFFFFFFu, am1, m));
            am2 = fmaxf(am2, __shfl_xor_sync(0xFFFFFFFFu, am2, m));
            am3 = fmaxf(am3, __shfl_xor_sync(0xFFFFFFFFu, am3, m));
        }
        const int k0 = mx_scale_exp(am0), k1 = mx_scale_exp(am1), k2 = mx_scale_exp(am2),
                  k3 = mx_scale_exp(am3);
        // code bytes of rows r0 .. r0 + 7, per column: [column][row half]
        uint32_t w0[2] = {0u, 0u}, w1[2] = {0u, 0u}, w2[2] = {0u, 0u}, w3[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float v0 = scale_pow2(bf16_lo(q[i].x), k0), v1 = scale_pow2(bf16_hi(q[i].x), k1);
            float v2 = scale_pow2(bf16_lo(q[i].y), k2), v3 = scale_pow2(bf16_hi(q[i].y), k3);
            if (SR) {
                // elements (r0 + i, c .. c + 3): row-major index multiple of 4
                const u32x4 r4 = philox_block(seed, offset, (uint64_t)((r0 + i) * cols + c) >> 2);
                v0 = e4m3_sr_value(v0, r4.x);
                v1 = e4m3_sr_value(v1, r4.y);
                v2 = e4m3_sr_value(v2, r4.z);
                v3 = e4m3_sr_value(v3, r4.w);
            }
            const uint32_t p01 = e4m3x2_hw(v0, v1), p23 = e4m3x2_hw(v2, v3);
            const int h = i >> 2, sh = 8 * (i & 3);
            w0[h] |= (p01 & 0xFFu) << sh;
            w1[h] |= (p01 >> 8) << sh;
            w2[h] |= (p23 & 0xFFu) << sh;
            w3[h] |= (p23 >> 8) << sh;
        }
        *reinterpret_cast<uint2 *>(codes + (c + 0) * rows + r0) = make_uint2(w0[0], w0[1]);
        *reinterpret_cast<uint2 *>(codes + (c + 1) * rows + r0) = make_uint2(w1[0], w1[1]);
        *reinterpret_cast<uint2 *>(codes + (c + 2) * rows + r0) = make_uint2(w2[0], w2[1]);
        *reinterpret_cast<uint2 *>(codes + (c + 3) * rows + r0) = make_uint2(w3[0], w3[1]);
        if (rq == 0) {
            const int ks[4] = {k0, k1, k2, k3};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint8_t e8 = (uint8_t)(ks[j] + 127);
                if (layout == NVFP4MOE_LAYOUT_ROWMAJOR)
                    scales[(c + j) * G + b] = e8;
                else
                    scales[mma_sf_offset(c + j, b, G)] = e8;
            }
        }
    }
}

// Column-wise MXFP8 over segments of rows: segment s holds rows
// [seg_off[s], seg_off[s+1]) and is cut into ceil(len / 32) blocks of 32 rows,
// the last one zero-padded. The blocks of all segments are packed in order
// into an output of `pitch` columns (>= the packed total, a multiple of 32);
// output columns past the packed blocks get zero codes and zero scale codes.
// Each CTA first turns the segment lengths into block offsets in shared
// memory; each warp then quantizes one 32-row block x 32-column patch, the
// loads of rows outside the block's segment replaced by zeros. The draws
// follow every element's row-major index in the [rows x cols] source.
constexpr int MAX_SEGS = 1024;

template <bool SR>
__global__ void __launch_bounds__(256) mxfp8_cols_seg_kernel(
    const uint16_t *__restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    const int32_t *__restrict__ seg_off, int32_t nseg, int64_t pitch, uint64_t seed,
    uint64_t offset, uint8_t *__restrict__ codes, uint8_t *__restrict__ scales, int layout) {
    __shared__ int32_t blk0[MAX_SEGS + 1];  // first output block of each segment
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (warp == 0) {
        // offsets must be non-decreasing inside [0, rows]; otherwise every
        // output block is written as zeros, nothing is loaded, and the
        // device error word records it
        bool bad = lane == 0 && (seg_off[0] < 0 || seg_off[nseg] > rows);
        int32_t run = 0;
        for (int32_t base = 0; base < nseg; base += 32) {
            const int32_t sidx = base + lane;
            int32_t nb = 0;
            if (sidx < nseg) {
                const int32_t len = seg_off[sidx + 1] - seg_off[sidx];
                bad |= len < 0;
                nb = (len + 31) / 32;
            }
            int32_t incl = nb;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += t;
            }
            if (sidx < nseg) blk0[sidx] = run + incl - nb;
            run += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (__any_sync(0xFFFFFFFFu, bad)) {
            run = 0;
            if (lane == 0 && blockIdx.x == 0) atomicCAS(&g_device_error, 0, DEVERR_SEGMENTS);
        }
        if (lane == 0) blk0[nseg] = run;
    }
    __syncthreads();
    const int32_t nblk = blk0[nseg];
    const int rq = lane >> 3, cq = lane & 7;
    const int64_t G = pitch / 32;   // scales per output row
    const int64_t CP = cols / 32;   // column patches
    const int64_t items = G * CP;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t it = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp; it < items; it += warps) {
        const int64_t b = it / CP, cp = it - b * CP;
        const int64_t c = cp * 32 + cq * 4;
        int64_t r0 = 0, r_end = 0;  // source rows of this lane's 8 rows, segment end
        if (b < nblk) {
            int lo = 0, hi = nseg - 1;  // last segment whose first block <= b
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (blk0[mid] <= b) lo = mid; else hi = mid - 1;
            }
            r0 = (int64_t)seg_off[lo] + (b - blk0[lo]) * 32 + rq * 8;
            r_end = seg_off[lo + 1];
        }
        uint2 q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            q[i] = (r0 + i < r_end) ? __ldg(reinterpret_cast<const uint2 *>(x + (r0 + i) * ld + c))
                                    : make_uint2(0u, 0u);
        float am0 = 0.0f, am1 = 0.0f, am2 = 0.0f, am3 = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            am0 = fmaxf(am0, fabsf(bf16_lo(q[i].x)));
            am1 = fmaxf(am1, fabsf(bf16_hi(q[i].x)));
            am2 = fmaxf(am2, fabsf(bf16_lo(q[i].y)));
            am3 = fmaxf(am3, fabsf(bf16_hi(q[i].y)));
        }
#pragma unroll
        for (int m = 8; m <= 16; m <<= 1) {
            am0 = fmaxf(am0, __shfl_xor_sync(0xFFFFFFFFu, am0, m));
            am1 = fmaxf(am1, __shfl_xor_sync(0xFFFFFFFFu, am1, m));
            am2 = fmaxf(am2, __shfl_xor_sync(0xFFFFFFFFu, am2, m));
            am3 = fmaxf(am3, __shfl_xor_sync(0xFFFFFFFFu, am3, m));
        }
        const int k0 = mx_scale_exp(am0), k1 = mx_scale_exp(am1), k2 = mx_scale_exp(am2),
                  k3 = mx_scale_exp(am3);
        uint32_t w0[2] = {0u, 0u}, w1[2] = {0u, 0u}, w2[2] = {0u, 0u}, w3[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float v0 = scale_pow2(bf16_lo(q[i].x), k0), v1 = scale_pow2(bf16_hi(q[i].x), k1);
            float v2 = scale_pow2(bf16_lo(q[i].y), k2), v3 = scale_pow2(bf16_hi(q[i].y), k3);
            if (SR && r0 + i < r_end) {
                const u32x4 r4 = philox_block(seed, offset, (uint64_t)((r0 + i) * cols + c) >> 2);
                v0 = e4m3_sr_value(v0, r4.x);
                v1 = e4m3_sr_value(v1, r4.y);
                v2 = e4m3_sr_value(v2, r4.z);
                v3 = e4m3_sr_value(v3, r4.w);
            }
            const uint32_t p01 = e4m3x2_hw(v0, v1), p23 = e4m3x2_hw(v2, v3);
            const int h = i >> 2, sh = 8 * (i & 3);
            w0[h] |= (p01 & 0xFFu) << sh;
            w1[h] |= (p01 >> 8) << sh;
            w2[h] |= (p23 & 0xFFu) << sh;
            w3[h] |= (p23 >> 8) << sh;
        }
        const int64_t o = b * 32 + rq * 8;  // output column of this lane's first row
        *reinterpret_cast<uint2 *>(codes + (c + 0) * pitch + o) = make_uint2(w0[0], w0[1]);
        *reinterpret_cast<uint2 *>(codes + (c + 1) * pitch + o) = make_uint2(w1[0], w1[1]);
        *reinterpret_cast<uint2 *>(codes + (c + 2) * pitch + o) = make_uint2(w2[0], w2[1]);
        *reinterpret_cast<uint2 *>(codes + (c + 3) * pitch + o) = make_uint2(w3[0], w3[1]);
        if (rq == 0) {
            const int ks[4] = {k0, k1, k2, k3};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint8_t e8 = (uint8_t)(ks[j] + 127);
                if (layout == NVFP4MOE_LAYOUT_ROWMAJOR)
                    scales[(c + j) * G + b] = e8;
                else
                    scales[mma_sf_offset(c + j, b, G)] = e8;
            }
        }
    }
}

__global__ void __launch_bounds__(256) mxfp8_dequant_kernel(
    const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales, int64_t n_rows,
    int64_t n_cols, int layout, float *__restrict__ out) {
    const int64_t G = n_cols / 32;
    const int64_t n = n_rows * G;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        int64_t r = i / G, b = i - r * G;
        uint32_t sc = layout == NVFP4MOE_LAYOUT_ROWMAJOR ? scales[r * G + b]
                                                         : scales[mma_sf_offset(r, b, G)];
        int k = (int)sc - 127;
        const uint8_t *cp = codes + r * n_cols + b * 32;
        float *op = out + r * n_cols + b * 32;
        for (int j = 0; j < 32; ++j) op[j] = scale_pow2(e4m3_decode(cp[j]), -k);
    }
}

// ---------------------------------------------------------------------------
// RHT32: per 32-element block, sign flip, five butterfly stages (h = 1, 2, 4,
// 8, 16), times fp32(1/sqrt(32)); all in fp32 with one rounding per op.
// ---------------------------------------------------------------------------
NV_DEV void fwht32(float (&t)[32]) {
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            if ((j & h) == 0) {
                float a = t[j], b = t[j + h];
                t[j] = __fadd_rn(a, b);
                t[j + h] = __fsub_rn(a, b);
            }
        }
    }
}

#define RHT_C 0.17677669529663688f  // fp32 nearest to 1/sqrt(32)

NV_DEV void rht32_fwd(const uint16_t *__restrict__ p, uint32_t signs, float (&v)[32]) {
    const uint4 *pv = reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int j = 0; j < 4; ++j) unpack8(__ldg(pv + j), v + 8 * j);
#pragma unroll
    for (int i = 0; i < 32; ++i)
        if ((signs >> i) & 1u) v[i] = -v[i];
    fwht32(v);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(v[i], RHT_C);
}

NV_DEV uint32_t rht_signs_dev(uint64_t sign_seed) {
    return philox4x32_10(u32x4{0, 0, 0, 0}, (uint32_t)sign_seed, (uint32_t)(sign_seed >> 32)).x;
}

__global__ void __launch_bounds__(256) rht32_amax_kernel(const uint16_t *__restrict__ x,
                                                         int64_t rows, int64_t cols, int64_t ld,
                                                         uint64_t sign_seed,
                                                         float *__restrict__ amax) {
    const uint32_t signs = rht_signs_dev(sign_seed);
    const uint32_t G = (uint32_t)(cols / 32);
    const uint32_t n = (uint32_t)(rows * G);
    float m = 0.0f;
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const uint32_t r = i / G, b = i - r * G;
        float v[32];
        rht32_fwd(x + (int64_t)r * ld + b * 32, signs, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(v[j]));
    }
    m = warp_max(m);
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
        v = warp_max(v);
        if (threadIdx.x == 0) atomic_max_nonneg(amax, v);
    }
}

__global__ void __launch_bounds__(256) rht32_quant_kernel(
    const uint16_t *__restrict__ x, int64_t rows, int64_t cols, int64_t ld, uint64_t sign_seed,
    int fmt, const float *__restrict__ amax_p, uint8_t *__restrict__ codes,
    uint8_t *__restrict__ scales, float *__restrict__ ts_out) {
    __shared__ float enc_tab[128];
    const uint32_t signs = rht_signs_dev(sign_seed);
    const uint32_t G = (uint32_t)(cols / 32);
    const uint32_t n = (uint32_t)(rows * G);
    float S_enc = 1.0f;
    if (fmt == NVFP4MOE_FMT_NVFP4) {
        const float amax = *amax_p;
        S_enc = nvfp4_senc(amax);
        fill_enc_table(enc_tab, S_enc);
        if (ts_out && blockIdx.x == 0 && threadIdx.x == 0) *ts_out = nvfp4_ts(amax);
    }
    __syncthreads();
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const uint32_t r = i / G, b = i - r * G;
        float v[32];
        rht32_fwd(x + (int64_t)r * ld + b * 32, signs, v);
        if (fmt == NVFP4MOE_FMT_NVFP4) {
            uint32_t w0, w1, w2, w3;
            const uint32_t s0 = nvfp4_block16_tab(v, S_enc, enc_tab, w0, w1);
            const uint32_t s1 = nvfp4_block16_tab(v + 16, S_enc, enc_tab, w2, w3);
            *reinterpret_cast<uint4 *>(codes + (int64_t)i * 16) = make_uint4(w0, w1, w2, w3);
            *reinterpret_cast<uint16_t *>(scales + (int64_t)i * 2) = (uint16_t)(s0 | (s1 << 8));
        } else {
            uint32_t w[8];
            const uint32_t sc = mx_block32<false>(v, 0, 0, 0, w);
            uint4 *co = reinterpret_cast<uint4 *>(codes + (int64_t)i * 32);
            co[0] = make_uint4(w[0], w[1], w[2], w[3]);
            co[1] = make_uint4(w[4], w[5], w[6], w[7]);
            scales[i] = (uint8_t)sc;
        }
    }
}

__global__ void __launch_bounds__(256) rht32_dequant_kernel(
    const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales,
    const float *__restrict__ ts_p, int64_t rows, int64_t cols, uint64_t sign_seed, int fmt,
    float *__restrict__ out) {
    const uint32_t signs = rht_signs_dev(sign_seed);
    const int64_t G = cols / 32;
    const float ts = (fmt == NVFP4MOE_FMT_NVFP4) ? *ts_p : 1.0f;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < rows * G;
         i += (int64_t)gridDim.x * blockDim.x) {
        int64_t r = i / G, b = i - r * G;
        float t[32];
        if (fmt == NVFP4MOE_FMT_NVFP4) {
            uint4 q = *reinterpret_cast<const uint4 *>(codes + r * (cols / 2) + b * 16);
            uint32_t qs[4] = {q.x, q.y, q.z, q.w};
            float sf0 = e4m3_decode(scales[r * (cols / 16) + 2 * b]);
            float sf1 = e4m3_decode(scales[r * (cols / 16) + 2 * b + 1]);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                float sf = j < 16 ? sf0 : sf1;
                t[j] = __fmul_rn(e2m1_decode((qs[j >> 3] >> (4 * (j & 7))) & 15u) * sf, ts);
            }
        } else {
            int k = (int)scales[r * G + b] - 127;
            const uint4 *cq = reinterpret_cast<const uint4 *>(codes + r * cols + b * 32);
            uint4 q0 = cq[0], q1 = cq[1];
            uint32_t qs[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
            for (int j = 0; j < 32; ++j)
                t[j] = scale_pow2(e4m3_decode((qs[j >> 2] >> (8 * (j & 3))) & 0xFFu), -k);
        }
        fwht32(t);
        float *op = out + r * cols + b * 32;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            float u = __fmul_rn(t[j], RHT_C);
            t[j] = ((signs >> j) & 1u) ? -u : u;
        }
#pragma unroll
        for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4 *>(op + j) = make_float4(t[j], t[j + 1], t[j + 2], t[j + 3]);
    }
}

// ---------------------------------------------------------------------------
// Combine straight from the RHT32-quantized payload: per token and 32-block,
// sum_j w_j * dequant(v_j) in fp32 (slot order, fused multiply-adds), then one
// inverse transform (butterflies, times c, sign flip) -> bf16. The transform
// is linear, so this equals combining the inverse-transformed rows, with one
// transform per token instead of k.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) combine_rht_kernel(
    const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales,
    const float *__restrict__ ts_p, int fmt, uint64_t sign_seed, const int32_t *__restrict__ pos,
    const float *__restrict__ w, int64_t T, int32_t k, int64_t d, uint16_t *__restrict__ out) {
    const uint32_t signs = rht_signs_dev(sign_seed);
    const int64_t G = d / 32;
    const float ts = (fmt == NVFP4MOE_FMT_NVFP4) ? *ts_p : 1.0f;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < T * G;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / G, b = i - t * G;
        float acc[32];
#pragma unroll
        for (int m = 0; m < 32; ++m) acc[m] = 0.0f;
        for (int j = 0; j < k; ++j) {
            const int64_t r = pos[t * k + j];
            const float wj = w[t * k + j];
            if (fmt == NVFP4MOE_FMT_NVFP4) {
                const uint4 q = __ldg(reinterpret_cast<const uint4 *>(codes + r * (d / 2) + b * 16));
                const uint32_t qs[4] = {q.x, q.y, q.z, q.w};
                const uint16_t sc = __ldg(reinterpret_cast<const uint16_t *>(scales + r * (d / 16) + 2 * b));
                // w_j * (block scale * tensor scale): one coefficient per 16 values
                const float c0 = __fmul_rn(wj, __fmul_rn(e4m3_decode(sc & 0xFFu), ts));
                const float c1 = __fmul_rn(wj, __fmul_rn(e4m3_decode(sc >> 8), ts));
#pragma unroll
                for (int m = 0; m < 32; m += 2) {
                    const float2 v = e2m1x2_decode_hw((qs[m >> 3] >> (4 * (m & 7))) & 0xFFu);
                    const float cm = m < 16 ? c0 : c1;
                    acc[m] = fmaf(cm, v.x, acc[m]);
                    acc[m + 1] = fmaf(cm, v.y, acc[m + 1]);
                }
            } else {
                const float cj = scale_pow2(wj, 127 - (int)__ldg(scales + r * G + b));  // w_j * 2^(e - 127)
                const uint4 *cq = reinterpret_cast<const uint4 *>(codes + r * d + b * 32);
                const uint4 q0 = __ldg(cq), q1 = __ldg(cq + 1);
                const uint32_t qs[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
                for (int m = 0; m < 32; m += 2) {
                    const float2 v = e4m3x2_decode_hw((qs[m >> 2] >> (8 * (m & 3))) & 0xFFFFu);
                    acc[m] = fmaf(cj, v.x, acc[m]);
                    acc[m + 1] = fmaf(cj, v.y, acc[m + 1]);
                }
            }
        }
        fwht32(acc);
        uint32_t pk[16];
#pragma unroll
        for (int m = 0; m < 32; m += 2) {
            float u0 = __fmul_rn(acc[m], RHT_C), u1 = __fmul_rn(acc[m + 1], RHT_C);
            if ((signs >> m) & 1u) u0 = -u0;
            if ((signs >> (m + 1)) & 1u) u1 = -u1;
            pk[m >> 1] = f32_to_bf16_bits(u0) | (f32_to_bf16_bits(u1) << 16);
        }
        uint4 *op = reinterpret_cast<uint4 *>(out + t * d + b * 32);
#pragma unroll
        for (int v = 0; v < 4; ++v) op[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
    }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
static int grid_for(int64_t work, int per_block = 256) {
    int64_t g = (work + per_block - 1) / per_block;
    const int64_t cap = 148 * 16;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    return (int)g;
}

cudaError_t launch_amax_bf16(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                             float *amax, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), s);
    if (e != cudaSuccess) return e;
    if (rows * cols == 0) return cudaSuccess;
    if (ld == cols) {
        amax_bf16_kernel<<<grid_for(rows * cols / 16), 256, 0, s>>>(x, rows, cols, ld, amax);
    } else {
        const int64_t vpr = cols / 8;
        dim3 grid((unsigned)((vpr + 255) / 256), (unsigned)(rows < 1024 ? rows : 1024));
        amax_bf16_kernel<<<grid, 256, 0, s>>>(x, rows, cols, ld, amax);
    }
    return cudaGetLastError();
}

cudaError_t launch_nvfp4_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                  const float *amax_in, uint8_t *codes, uint8_t *scales,
                                  float *ts_out, int layout, cudaStream_t s) {
    cudaError_t e;
    if (!amax_in) {
        // ts_out holds the amax between the passes, then becomes amax / 2688
        if ((e = launch_amax_bf16(x, rows, cols, ld, ts_out, s)) != cudaSuccess) return e;
        if (rows * cols > 0)
            nvfp4_quant_kernel<<<grid_for(rows * (cols / 64)), 256, 0, s>>>(
                x, rows, cols, ld, ts_out, codes, scales, nullptr, layout);
        nvfp4_finalize_ts_kernel<<<1, 1, 0, s>>>(ts_out);
    } else {
        nvfp4_quant_kernel<<<grid_for(rows * (cols / 64)), 256, 0, s>>>(
            x, rows, cols, ld, amax_in, codes, scales, ts_out, layout);
    }
    return cudaGetLastError();
}

cudaError_t launch_nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales, const float *ts,
                                    int64_t rows, int64_t cols, int layout, float *out,
                                    cudaStream_t s) {
    if (rows * cols == 0) return cudaSuccess;
    nvfp4_dequant_kernel<<<grid_for(rows * (cols / 16)), 256, 0, s>>>(codes, scales, ts, rows,
                                                                      cols, layout, out);
    return cudaGetLastError();
}

cudaError_t launch_mxfp8_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                  int axis, uint64_t seed, uint64_t offset, int rounding,
                                  uint8_t *codes, uint8_t *scales, int layout, cudaStream_t s) {
    if (rows * cols == 0) return cudaSuccess;
    const bool sr = rounding == NVFP4MOE_ROUND_SR;
    if (axis == 0) {
        int g = grid_for(rows * (cols / 32));
        if (sr)
            mxfp8_rows_kernel<true><<<g, 256, 0, s>>>(x, rows, cols, ld, seed, offset, codes, scales,
                                                      layout);
        else
            mxfp8_rows_kernel<false><<<g, 256, 0, s>>>(x, rows, cols, ld, seed, offset, codes,
                                                       scales, layout);
    } else {
        // one warp per 32 x 32 patch, 8 warps per CTA
        const int g = grid_for((rows / 32) * (cols / 32), 8);
        if (sr)
            mxfp8_cols_kernel<true><<<g, 256, 0, s>>>(x, rows, cols, ld, seed, offset, codes, scales,
                                                      layout);
        else
            mxfp8_cols_kernel<false><<<g, 256, 0, s>>>(x, rows, cols, ld, seed, offset, codes,
                                                       scales, layout);
    }
    return cudaGetLastError();
}

cudaError_t launch_mxfp8_quantize_seg(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                      const int32_t *seg_off, int32_t nseg, int64_t pitch,
                                      uint64_t seed, uint64_t offset, int rounding,
                                      uint8_t *codes, uint8_t *scales, int layout,
                                      cudaStream_t s) {
    if (pitch * cols == 0) return cudaSuccess;
    const int g = grid_for((pitch / 32) * (cols / 32), 8);
    if (rounding == NVFP4MOE_ROUND_SR)
        mxfp8_cols_seg_kernel<true><<<g, 256, 0, s>>>(x, rows, cols, ld, seg_off, nseg, pitch, seed,
                                                      offset, codes, scales, layout);
    else
        mxfp8_cols_seg_kernel<false><<<g, 256, 0, s>>>(x, rows, cols, ld, seg_off, nseg, pitch, seed,
                                                       offset, codes, scales, layout);
    return cudaGetLastError();
}

cudaError_t launch_mxfp8_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t n_rows,
                                    int64_t n_cols, int layout, float *out, cudaStream_t s) {
    if (n_rows * n_cols == 0) return cudaSuccess;
    mxfp8_dequant_kernel<<<grid_for(n_rows * (n_cols / 32)), 256, 0, s>>>(codes, scales, n_rows,
                                                                          n_cols, layout, out);
    return cudaGetLastError();
}

cudaError_t launch_rht32_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                                  uint64_t sign_seed, int fmt, const float *amax_in,
                                  uint8_t *codes, uint8_t *scales, float *ts_out,
                                  cudaStream_t s) {
    cudaError_t e;
    const int g = grid_for(rows * (cols / 32));
    if (fmt == NVFP4MOE_FMT_NVFP4 && !amax_in) {
        if ((e = cudaMemsetAsync(ts_out, 0, sizeof(float), s)) != cudaSuccess) return e;
        if (rows * cols > 0) {
            rht32_amax_kernel<<<g, 256, 0, s>>>(x, rows, cols, ld, sign_seed, ts_out);
            rht32_quant_kernel<<<g, 256, 0, s>>>(x, rows, cols, ld, sign_seed, fmt, ts_out, codes,
                                                 scales, nullptr);
        }
        nvfp4_finalize_ts_kernel<<<1, 1, 0, s>>>(ts_out);
    } else if (rows * cols > 0) {
        rht32_quant_kernel<<<g, 256, 0, s>>>(x, rows, cols, ld, sign_seed, fmt, amax_in, codes,
                                             scales, ts_out);
    }
    return cudaGetLastError();
}

cudaError_t launch_rht32_dequantize(const uint8_t *codes, const uint8_t *scales, const float *ts,
                                    int64_t rows, int64_t cols, uint64_t sign_seed, int fmt,
                                    float *out, cudaStream_t s) {
    if (rows * cols == 0) return cudaSuccess;
    rht32_dequant_kernel<<<grid_for(rows * (cols / 32)), 256, 0, s>>>(codes, scales, ts, rows, cols,
                                                                      sign_seed, fmt, out);
    return cudaGetLastError();
}

cudaError_t launch_combine_rht(const uint8_t *codes, const uint8_t *scales, const float *ts, int fmt,
                               uint64_t sign_seed, const int32_t *pos, const float *w, int64_t T,
                               int32_t k, int64_t d, uint16_t *out, cudaStream_t s) {
    if (T * d == 0) return cudaSuccess;
    combine_rht_kernel<<<grid_for(T * (d / 32)), 256, 0, s>>>(codes, scales, ts, fmt, sign_seed, pos,
                                                              w, T, k, d, out);
    return cudaGetLastError();
}

// grouped NVFP4 quantization of the expert activations h with per-expert
// tensor scales: rows [off[e], off[e+1]) use amax[e]; ts[e] = amax[e] / 2688.
__global__ void __launch_bounds__(256) nvfp4_quant_grouped_kernel(
    const uint16_t *__restrict__ x, int64_t cols, const int32_t *__restrict__ off, int32_t E,
    const float *__restrict__ amax, uint8_t *__restrict__ codes, uint8_t *__restrict__ scales,
    float *__restrict__ ts) {
    extern __shared__ int32_t s_off[];
    for (int i = threadIdx.x; i <= E; i += blockDim.x) s_off[i] = off[i];
    __syncthreads();
    if (blockIdx.x == 0)
        for (int e = threadIdx.x; e < E; e += blockDim.x) ts[e] = nvfp4_ts(amax[e]);
    const int64_t rows = s_off[E];
    const int64_t G = cols / 64;
    // each CTA owns one contiguous range of 64-element groups, so the rows a
    // thread meets only move forward and so does their expert
    const int64_t n = rows * G;
    const int64_t chunk = (n + gridDim.x - 1) / gridDim.x;
    const int64_t i0 = (int64_t)blockIdx.x * chunk;
    const int64_t i1 = i0 + chunk < n ? i0 + chunk : n;
    int e = -1;
    float S_enc = 1.0f;
    for (int64_t i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
        const int64_t r = i / G, g = i - r * G;
        const uint4 *pv = reinterpret_cast<const uint4 *>(x + r * cols + g * 64);
        uint4 raw[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) raw[j] = __ldg(pv + j);
        int e1 = e;
        if (e1 < 0) {
            int lo = 0, hi = E;  // largest e with s_off[e] <= r
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (s_off[mid] <= r) lo = mid; else hi = mid;
            }
            e1 = lo;
        }
        while (e1 + 1 < E && s_off[e1 + 1] <= r) ++e1;
        if (e1 != e) {
            e = e1;
            S_enc = nvfp4_senc(amax[e]);
        }
        uint32_t scw = 0, w[8];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            float v[16];
            unpack8(raw[2 * b], v);
            unpack8(raw[2 * b + 1], v + 8);
            scw |= nvfp4_block16(v, S_enc, w[2 * b], w[2 * b + 1]) << (8 * b);
        }
        uint4 *co = reinterpret_cast<uint4 *>(codes + r * (cols / 2) + g * 32);
        co[0] = make_uint4(w[0], w[1], w[2], w[3]);
        co[1] = make_uint4(w[4], w[5], w[6], w[7]);
        *reinterpret_cast<uint32_t *>(scales + mma_sf_offset(r, g * 4, cols / 16)) = scw;
    }
}

cudaError_t launch_nvfp4_quant_grouped(const uint16_t *x, int64_t rows_alloc, int64_t cols,
                                       const int32_t *off, int32_t E, const float *amax,
                                       uint8_t *codes, uint8_t *scales, float *ts,
                                       cudaStream_t s) {
    int g = grid_for(rows_alloc * (cols / 64));
    nvfp4_quant_grouped_kernel<<<g, 256, (E + 1) * sizeof(int32_t), s>>>(x, cols, off, E, amax,
                                                                         codes, scales, ts);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// SwiGLU backward (the backward pass of the expert layers, news.t0001.com
// "训练数值格式分工清单"): from the saved g | u and dh,
//   dg = dh * u * s(g) * (1 + g * (1 - s(g))),  du = dh * g * s(g),
// s(g) = 1 / (1 + exp(-g)), in fp32 with IEEE division, rounded to bf16.
// One thread per 8 columns of a row: three 16-byte loads, two 16-byte stores.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) swiglu_bwd_kernel(const uint16_t *__restrict__ gu,
                                                         const uint16_t *__restrict__ dh,
                                                         int64_t rows, int64_t f,
                                                         uint16_t *__restrict__ dgu) {
    const int64_t G = f / 8;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < rows * G;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / G, c = (i - r * G) * 8;
        const uint16_t *row = gu + r * 2 * f;
        const uint4 qg = __ldg(reinterpret_cast<const uint4 *>(row + c));
        const uint4 qu = __ldg(reinterpret_cast<const uint4 *>(row + f + c));
        const uint4 qd = __ldg(reinterpret_cast<const uint4 *>(dh + r * f + c));
        float g[8], u[8], d[8];
        unpack_bf16x8(qg, g);
        unpack_bf16x8(qu, u);
        unpack_bf16x8(qd, d);
        float dg[8], du[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float sg = 1.0f / (1.0f + expf(-g[j]));
            const float ds = sg * (1.0f + g[j] * (1.0f - sg));  // d silu / d g
            dg[j] = d[j] * u[j] * ds;
            du[j] = d[j] * (g[j] * sg);
        }
        uint16_t *orow = dgu + r * 2 * f;
        *reinterpret_cast<uint4 *>(orow + c) =
            make_uint4(bf16x2_rn(dg[0], dg[1]), bf16x2_rn(dg[2], dg[3]), bf16x2_rn(dg[4], dg[5]),
                       bf16x2_rn(dg[6], dg[7]));
        *reinterpret_cast<uint4 *>(orow + f + c) =
            make_uint4(bf16x2_rn(du[0], du[1]), bf16x2_rn(du[2], du[3]), bf16x2_rn(du[4], du[5]),
                       bf16x2_rn(du[6], du[7]));
    }
}

cudaError_t launch_swiglu_bwd(const uint16_t *gu, const uint16_t *dh, int64_t rows, int64_t f,
                              uint16_t *dgu, cudaStream_t s) {
    if (rows * f == 0) return cudaSuccess;
    swiglu_bwd_kernel<<<grid_for(rows * (f / 8)), 256, 0, s>>>(gu, dh, rows, f, dgu);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Self-test of the hardware conversions the quantizers use: every finite fp32
// input, hardware result against the library's software encoders.
// which 0: cvt.rn.satfinite.e2m1x2.f32; which 1: cvt.rn.satfinite.e4m3x2.f32.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) selftest_cvt_kernel(int which,
                                                           unsigned long long *mismatches) {
    unsigned long long bad = 0;
    // which 2 / 3: the decodes cvt.rn.f16x2.e2m1x2 / .e4m3x2 over every packed
    // pair against the software decoders, bit for bit
    if (which >= 2) {
        const uint32_t n = which == 2 ? 256u : 65536u;
        for (uint32_t c = blockIdx.x * blockDim.x + threadIdx.x; c < n; c += gridDim.x * blockDim.x) {
            float2 hw;
            float lo, hi;
            if (which == 2) {
                hw = e2m1x2_decode_hw(c);
                lo = e2m1_decode(c & 15u);
                hi = e2m1_decode(c >> 4);
            } else {
                hw = e4m3x2_decode_hw(c);
                lo = e4m3_decode(c & 0xFFu);
                hi = e4m3_decode(c >> 8);
            }
            // E4M3 codes 0x7F / 0xFF are NaN; the library's encoders saturate
            // and never write them, and its decoder is defined on the others
            const bool skip_lo = which == 3 && (c & 0x7Fu) == 0x7Fu;
            const bool skip_hi = which == 3 && ((c >> 8) & 0x7Fu) == 0x7Fu;
            const bool ok_lo = skip_lo || __float_as_uint(lo) == __float_as_uint(hw.x);
            const bool ok_hi = skip_hi || __float_as_uint(hi) == __float_as_uint(hw.y);
            bad += (ok_lo ? 0 : 1) + (ok_hi ? 0 : 1);
        }
    }
    const uint64_t groups = which >= 2 ? 0 : 1ull << 29;  // 8 consecutive bit patterns per group
    for (uint64_t g = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; g < groups;
         g += (uint64_t)gridDim.x * blockDim.x) {
        const uint32_t base = (uint32_t)(g << 3);
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(base + j);
        if (which == 0) {
            const uint32_t hw = e2m1x8_hw(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (isfinite(v[j]) && ((hw >> (4 * j)) & 15u) != e2m1_encode(v[j])) ++bad;
        } else {
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const uint32_t hw = e4m3x2_hw(v[2 * p], v[2 * p + 1]);
                if (isfinite(v[2 * p]) && (hw & 0xFFu) != e4m3_encode(v[2 * p])) ++bad;
                if (isfinite(v[2 * p + 1]) && (hw >> 8) != e4m3_encode(v[2 * p + 1])) ++bad;
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xFFFFFFFFu, bad, o);
    if ((threadIdx.x & 31) == 0 && bad) atomicAdd(mismatches, bad);
}

cudaError_t launch_selftest(int which, unsigned long long *mismatches, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(mismatches, 0, sizeof(unsigned long long), s);
    if (e != cudaSuccess) return e;
    selftest_cvt_kernel<<<148 * 8, 256, 0, s>>>(which, mismatches);
    return cudaGetLastError();
}

}  // namespace nvfp4moe

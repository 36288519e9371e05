// Device-side building blocks shared by the nvfp4moe kernels: status
// plumbing, bf16 loads, the E2M1 / E4M3 / E8M0 encoders, Philox4x32-10, and
// thin inline-PTX wrappers for mbarriers, TMA and tcgen05 (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <mutex>

#include "../../include/nvfp4moe.h"

#define NV_DEV __device__ __forceinline__

namespace nvfp4moe {

// ---------------------------------------------------------------------------
// host-side error plumbing (defined in abi.cu)
// ---------------------------------------------------------------------------
void set_last_error(const char *fmt, ...);
nvfp4moe_status cuda_status(cudaError_t e, const char *what);

// Device addresses of a __device__ variable, one per (device, driver context)
// the library has run in: looked up with cudaGetSymbolAddress on the first
// call in that device and context, then reused.
struct SymbolAddressCache {
    static constexpr int kEntries = 64;
    struct Entry {
        int dev;
        void *ctx;
        void *addr;
    };
    std::mutex mu;
    Entry entry[kEntries];
    int n = 0, next = 0;
};
cudaError_t cached_symbol_address(SymbolAddressCache &cache, const void *symbol, void **out);

// Device error word: a kernel whose bounded wait ran out stores the id of the
// wait here (first writer wins) and returns early.
#ifndef NVFP4MOE_WHOLE_PROGRAM
extern __device__ int32_t g_device_error;
#endif

enum WaitId : int32_t {
    WAIT_NONE = 0,
    WAIT_GEMM_FULL = 1,
    WAIT_GEMM_EMPTY = 2,
    WAIT_GEMM_ACC_FULL = 3,
    WAIT_GEMM_ACC_EMPTY = 4,
    WAIT_GEMM_DRAIN = 5,
    WAIT_GEMM_SF_SLOT = 6,
    WAIT_GEMM_SF_FULL = 7,
    WAIT_GEMM_SF_FREE = 8,
    // not a wait: a kernel found device-side arguments it could not use
    DEVERR_SEGMENTS = NVFP4MOE_DEVERR_SEGMENTS,  // mxfp8 columns: bad segment offsets
    DEVERR_REQUANT = 17,  // fused requantization: a queue entry outside its expert
};

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------
NV_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
NV_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// fp32 -> bf16 bits, nearest with ties to even (finite inputs; NaN -> quiet NaN).
NV_DEV uint32_t f32_to_bf16_bits(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0u;
    u += 0x7FFFu + ((u >> 16) & 1u);
    return u >> 16;
}

// Hardware decodes of packed low-precision pairs to two fp32 values: the low
// nibble / byte lands in .x. Exact (every E2M1 and E4M3 value is an fp16).
NV_DEV float2 e2m1x2_decode_hw(uint32_t byte) {
    uint32_t h;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u16 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(h)
        : "h"((uint16_t)byte));
    return __half22float2(*reinterpret_cast<const __half2 *>(&h));
}
NV_DEV float2 e4m3x2_decode_hw(uint32_t two_bytes) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)two_bytes));
    return __half22float2(*reinterpret_cast<const __half2 *>(&h));
}

// Two floats to a bf16 pair, round to nearest even (lo in bits 0..15).
NV_DEV uint32_t bf16x2_rn(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

NV_DEV float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Non-negative floats order like their bit patterns: max via unsigned atomics.
NV_DEV void atomic_max_nonneg(float *addr, float v) {
    atomicMax(reinterpret_cast<unsigned int *>(addr), __float_as_uint(v));
}

// ---------------------------------------------------------------------------
// E2M1: magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}. Nearest value, ties to the
// even code, saturating; the sign bit is the input's sign. The decision
// points are the midpoints between neighbouring magnitudes; a midpoint goes
// to the neighbour with the even code.
// ---------------------------------------------------------------------------
NV_DEV uint32_t e2m1_encode(float v) {
    float a = fabsf(v);
    uint32_t m = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) +
                 (a >= 3.5f) + (a > 5.0f);
    return m | ((__float_as_uint(v) >> 28) & 8u);
}

NV_DEV float e2m1_decode(uint32_t nib) {
    // magnitude m: 0..3 -> m/2, 4 -> 2, 5 -> 3, 6 -> 4, 7 -> 6
    uint32_t m = nib & 7u;
    float mag = (m < 4u) ? 0.5f * (float)m : (m == 7u ? 6.0f : (float)(m - 2u));
    return (nib & 8u) ? -mag : mag;
}

// ---------------------------------------------------------------------------
// E4M3 (bias 7, max 448, no infinities). Encoding of a non-negative finite
// value: nearest, ties to even, saturating at 448.
//   a >= 448         -> 0x7E
//   a <  2^-6        -> subnormal: mantissa = round(a * 2^9) (0..8; 8 is 2^-6)
//   otherwise        -> exponent e = floor(log2 a) from the fp32 exponent
//                       field, 3-bit mantissa rounded from the 23-bit one.
// ---------------------------------------------------------------------------
NV_DEV uint32_t e4m3_encode_pos(float a) {
    if (a >= 448.0f) return 0x7Eu;
    if (a < 0.015625f) return (uint32_t)__float2int_rn(a * 512.0f);
    uint32_t u = __float_as_uint(a);
    int e = (int)((u >> 23) & 0xFF) - 127;  // -6 .. 8
    uint32_t man = u & 0x7FFFFFu;
    uint32_t m3 = man >> 20, rem = man & 0xFFFFFu;
    uint32_t code = ((uint32_t)(e + 7) << 3) | m3;
    if (rem > 0x80000u || (rem == 0x80000u && (m3 & 1u))) code += 1u;
    return code;
}

NV_DEV uint32_t e4m3_encode(float v) {
    return e4m3_encode_pos(fabsf(v)) | ((__float_as_uint(v) >> 24) & 0x80u);
}

NV_DEV float e4m3_decode_pos(uint32_t c) {  // c in 0..126
    uint32_t e = (c >> 3) & 15u, m = c & 7u;
    if (e == 0) return (float)m * 0.001953125f;  // m * 2^-9
    return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

NV_DEV float e4m3_decode(uint32_t c) {
    float v = e4m3_decode_pos(c & 0x7Fu);
    return (c & 0x80u) ? -v : v;
}

// ---------------------------------------------------------------------------
// Hardware conversions (sm_100a cvt.rn.satfinite). They round to nearest with
// ties to even and saturate, as the encoders above do; nvfp4moe_selftest
// compares them with those encoders over every finite fp32 input.
// ---------------------------------------------------------------------------
// Eight floats -> eight E2M1 codes in one word, v[0] in the lowest nibble.
NV_DEV uint32_t e2m1x8_hw(float v0, float v1, float v2, float v3, float v4, float v5, float v6,
                          float v7) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
    return r;
}

// Two floats -> two E4M3 codes, lo in the low byte.
NV_DEV uint32_t e4m3x2_hw(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// 2^e as an fp32 for e in [-126, 127].
NV_DEV float exp2i(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// ---------------------------------------------------------------------------
// MXFP8 block exponent: smallest k in [-127, 127] with amax <= 448 * 2^k.
// amax = m * 2^E (m in [1, 2)); 448 = 1.75 * 2^8: k = E - 8 if m <= 1.75,
// else E - 7. Zero and subnormal amax clamp to -127.
// ---------------------------------------------------------------------------
NV_DEV int mx_scale_exp(float amax) {
    uint32_t u = __float_as_uint(amax);
    int ef = (int)((u >> 23) & 0xFF);
    if (ef == 0) return -127;
    int E = ef - 127;
    uint32_t man = u & 0x7FFFFFu;
    int k = (man <= 0x600000u) ? E - 8 : E - 7;  // 0x600000 = 0.75 * 2^23
    return k < -127 ? -127 : (k > 127 ? 127 : k);
}

// v * 2^-k exactly (k in [-127, 127]).
NV_DEV float scale_pow2(float v, int k) {
    int nk = -k;
    if (nk > 127) return (v * exp2i(127)) * exp2i(nk - 127);
    if (nk < -126) return (v * exp2i(-126)) * exp2i(nk + 126);
    return v * exp2i(nk);
}

// v rounded stochastically onto the E4M3 grid (sign kept), as an fp32 value,
// driven by the 32-bit word r: with lo <= |v| <= hi the neighbouring E4M3
// values, round up iff (r >> 8) * 2^-24 < (|v| - lo) / (hi - lo). |v| <= 448.
// E4M3 normal range (|v| >= 2^-6): E4M3 keeps 3 of the 23 fp32 mantissa bits,
// the fraction is the 20 dropped bits / 2^20, and the test is the integer
// comparison (r >> 8) < dropped << 4; a carry out of the kept mantissa moves to
// the next binade, which is the correct neighbour. Below 2^-6 the spacing is
// 2^-9 and the fraction is taken in exact fp32 arithmetic.
NV_DEV float e4m3_sr_value(float v, uint32_t r) {
    const uint32_t u = __float_as_uint(v);
    const uint32_t a = u & 0x7FFFFFFFu;
    const uint32_t r24 = r >> 8;
    if (a >= 0x3C800000u) {
        const uint32_t low = a & 0xFFFFFu;
        uint32_t kept = a & ~0xFFFFFu;
        if (r24 < (low << 4)) kept += 0x100000u;
        return __uint_as_float(kept | (u & 0x80000000u));
    }
    const float m = __uint_as_float(a) * 512.0f;  // exact
    const float lo = floorf(m);
    const float frac = m - lo;                    // exact
    const float rr = (float)r24 * 5.9604644775390625e-08f;
    const float mag = (rr < frac) ? lo + 1.0f : lo;
    return copysignf(mag * 0.001953125f, v);      // exact
}

// E4M3 code of v with stochastic rounding (see e4m3_sr_value).
NV_DEV uint32_t e4m3_encode_sr(float v, uint32_t r) { return e4m3_encode(e4m3_sr_value(v, r)); }

// ---------------------------------------------------------------------------
// NVFP4 block of 16: per-tensor S_enc, block scale s = E4M3((amax_b / 6) * S_enc),
// codes E2M1(x * S_enc / s). Returns the scale code; 8 code bytes in w0, w1.
// ---------------------------------------------------------------------------
NV_DEV float nvfp4_senc(float amax) {
    return (amax > 0.0f && amax <= 3.402823466e38f) ? __fdiv_rn(2688.0f, amax) : 1.0f;
}
NV_DEV float nvfp4_ts(float amax) {
    return (amax > 0.0f && amax <= 3.402823466e38f) ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}

NV_DEV uint32_t nvfp4_block16(const float *v, float S_enc, uint32_t &w0, uint32_t &w1) {
    float amax_b = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax_b = fmaxf(amax_b, fabsf(v[i]));
    const float t = __fmul_rn(__fdiv_rn(amax_b, 6.0f), S_enc);
    const uint32_t sc = e4m3_encode_pos(t);
    const float sf = e4m3_decode_pos(sc);
    const float enc = (sf == 0.0f) ? 0.0f : __fdiv_rn(S_enc, sf);
    w0 = e2m1x8_hw(__fmul_rn(v[0], enc), __fmul_rn(v[1], enc), __fmul_rn(v[2], enc),
                   __fmul_rn(v[3], enc), __fmul_rn(v[4], enc), __fmul_rn(v[5], enc),
                   __fmul_rn(v[6], enc), __fmul_rn(v[7], enc));
    w1 = e2m1x8_hw(__fmul_rn(v[8], enc), __fmul_rn(v[9], enc), __fmul_rn(v[10], enc),
                   __fmul_rn(v[11], enc), __fmul_rn(v[12], enc), __fmul_rn(v[13], enc),
                   __fmul_rn(v[14], enc), __fmul_rn(v[15], enc));
    return sc;
}

// Same block quantization with the per-tensor table enc_tab[c] = S_enc / e4m3(c)
// (enc_tab[0] = 0), built once per CTA with the same correctly rounded division,
// and the scale code from the hardware conversion: identical results.
NV_DEV uint32_t nvfp4_block16_tab(const float *v, float S_enc, const float *enc_tab, uint32_t &w0,
                                  uint32_t &w1) {
    float amax_b = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax_b = fmaxf(amax_b, fabsf(v[i]));
    const float t = __fmul_rn(__fdiv_rn(amax_b, 6.0f), S_enc);
    const uint32_t sc = e4m3x2_hw(t, 0.0f) & 0xFFu;
    const float enc = enc_tab[sc];
    w0 = e2m1x8_hw(__fmul_rn(v[0], enc), __fmul_rn(v[1], enc), __fmul_rn(v[2], enc),
                   __fmul_rn(v[3], enc), __fmul_rn(v[4], enc), __fmul_rn(v[5], enc),
                   __fmul_rn(v[6], enc), __fmul_rn(v[7], enc));
    w1 = e2m1x8_hw(__fmul_rn(v[8], enc), __fmul_rn(v[9], enc), __fmul_rn(v[10], enc),
                   __fmul_rn(v[11], enc), __fmul_rn(v[12], enc), __fmul_rn(v[13], enc),
                   __fmul_rn(v[14], enc), __fmul_rn(v[15], enc));
    return sc;
}

// enc_tab for one tensor scale, filled by the threads of a CTA (then sync).
NV_DEV void fill_enc_table(float *enc_tab, float S_enc) {
    for (int c = threadIdx.x; c < 128; c += blockDim.x)
        enc_tab[c] = (c == 0 || c == 127) ? 0.0f : __fdiv_rn(S_enc, e4m3_decode_pos((uint32_t)c));
}

NV_DEV void unpack_bf16x8(uint4 q, float *f) {
    f[0] = bf16_lo(q.x); f[1] = bf16_hi(q.x); f[2] = bf16_lo(q.y); f[3] = bf16_hi(q.y);
    f[4] = bf16_lo(q.z); f[5] = bf16_hi(q.z); f[6] = bf16_lo(q.w); f[7] = bf16_hi(q.w);
}

// Byte offset of scale (row r, scale column c) in the MMA layout of a matrix
// whose rows carry nsc scales (nsc % 4 == 0).
NV_DEV size_t mma_sf_offset(int64_t r, int64_t c, int64_t nsc) {
    int64_t chunk = (r >> 7) * (nsc >> 2) + (c >> 2);
    return (size_t)chunk * 512 + (size_t)((r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3));
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon et al., SC'11): 10 rounds of the multiply-xor bijection
// with the published multipliers and Weyl key increments.
// ---------------------------------------------------------------------------
struct u32x4 { uint32_t x, y, z, w; };

NV_DEV u32x4 philox4x32_10(u32x4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int i = 0; i < 10; ++i) {
        // one 32x32 -> 64-bit multiply gives both halves of each product
        const uint64_t p0 = (uint64_t)0xD2511F53u * c.x;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c.z;
        c = u32x4{(uint32_t)(p1 >> 32) ^ c.y ^ k0, (uint32_t)p1, (uint32_t)(p0 >> 32) ^ c.w ^ k1,
                  (uint32_t)p0};
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c;
}

// The four words for elements 4*blk .. 4*blk+3 of the (seed, offset) stream.
NV_DEV u32x4 philox_block(uint64_t seed, uint64_t offset, uint64_t blk) {
    return philox4x32_10(u32x4{(uint32_t)blk, (uint32_t)(blk >> 32), (uint32_t)offset,
                               (uint32_t)(offset >> 32)},
                         (uint32_t)seed, (uint32_t)(seed >> 32));
}

// ---------------------------------------------------------------------------
// PTX wrappers: shared-memory addresses, mbarriers, TMA, tcgen05.
// ---------------------------------------------------------------------------
NV_DEV uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

NV_DEV void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

NV_DEV void fence_mbarrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

NV_DEV void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

NV_DEV void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

NV_DEV bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

NV_DEV uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase with the given parity to complete, giving up after about
// two seconds: on timeout the wait id goes to the device error word `err` and
// the caller returns false so the kernel can wind down instead of hanging.
NV_DEV bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, int32_t *err, int32_t wait_id) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > 2000000000ull) {
            atomicCAS(err, 0, wait_id);
            return false;
        }
    }
}

// TMA tiled 2D load into shared memory, completion counted on an mbarrier.
NV_DEV void tma_load_2d(void *dst, const CUtensorMap *map, int32_t x, int32_t y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Plain bulk copy global -> shared (16-byte aligned, size % 16 == 0).
NV_DEV void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Per-thread asynchronous copies global -> shared (cp.async), with their
// completion counted on an mbarrier: the arrival is made when all of this
// thread's earlier cp.async copies have landed, and does not increment the
// barrier's pending count (it was initialised with one count per thread).
NV_DEV void cp_async_16(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
NV_DEV void cp_async_4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
NV_DEV void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

NV_DEV void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// --- clusters ----------------------------------------------------------------
NV_DEV uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address in the shared::cluster window of the same variable in CTA `rank`.
NV_DEV uint32_t cluster_addr(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
// Arrive on an mbarrier of any CTA of the cluster without release semantics:
// for hand-offs of TMEM whose reads or writes this thread has already waited
// for (tcgen05.wait::ld / ::st, then tcgen05.fence::before_thread_sync). A
// cluster-scope release would also wait for every generic store of the thread
// to become visible, which costs about a thousand cycles while the SM streams
// epilogue stores.
NV_DEV void mbar_arrive_cluster_relaxed(uint32_t cbar) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cbar)
                 : "memory");
}
// All threads of every CTA of the cluster.
NV_DEV void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA tiled loads issued by either CTA of a pair into its own shared memory,
// the completed bytes counted on an mbarrier given by its shared::cluster
// address (the pair's first CTA holds it).
NV_DEV void tma_load_2d_pair(void *dst, const CUtensorMap *map, int32_t x, int32_t y,
                             uint32_t cbar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(cbar)
        : "memory");
}
NV_DEV void tma_load_5d_pair(void *dst, const CUtensorMap *map, int32_t c0, int32_t c1, int32_t c2,
                             int32_t c3, int32_t c4, uint32_t cbar) {
    asm volatile(
        "cp.async.bulk.tensor.5d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
        "r"(cbar)
        : "memory");
}

// Per-warpgroup register budget (all four warps of the warpgroup execute it).
template <uint32_t N> NV_DEV void regs_shrink() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N> NV_DEV void regs_grow() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// --- tcgen05 (CTA pairs: every tcgen05 op of a kernel uses one cta_group) ----
NV_DEV void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
NV_DEV void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
NV_DEV void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
NV_DEV void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
NV_DEV void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive on an mbarrier (shared::cluster address, either CTA of the pair) once
// every tcgen05 op issued so far by this thread has completed.
NV_DEV void tc_commit_pair(uint32_t cbar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     cbar)
                 : "memory");
}
// The same, arriving on the mbarrier at this shared::cta offset in every CTA
// of `cta_mask` (one tensor-core commit, no memory load involved).
NV_DEV void tc_commit_pair_mc(uint32_t cbar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
        "[%0], %1;" ::"r"(cbar),
        "h"(cta_mask)
        : "memory");
}
NV_DEV void tc_mma_nvf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                             uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], "
        "[%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}
NV_DEV void tc_mma_mxf8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                             uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], "
        "p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns -> 32 registers per thread.
NV_DEV void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
NV_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// 32 lanes x 16 consecutive 32-bit columns <- 16 registers per thread.
NV_DEV void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}
// 32 lanes x 32 columns <- 32 registers per thread.
NV_DEV void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
NV_DEV void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
                     taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                 "r"(r[7])
                 : "memory");
}
NV_DEV void tmem_st_32x32b_x4(uint32_t taddr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(r0),
                 "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
}
NV_DEV void tmem_st_32x32b_x1(uint32_t taddr, uint32_t r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(r) : "memory");
}
NV_DEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor (tcgen05 format): start address, leading and
// stride byte offsets in 16-byte units, descriptor version 1 (bit 46), swizzle
// mode in bits 61..63 (0 none, 2 = 128-byte swizzle).
NV_DEV uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                          uint32_t swizzle) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)(swizzle & 7u) << 61;
    return d;
}

}  // namespace nvfp4moe

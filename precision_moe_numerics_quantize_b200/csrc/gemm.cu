// Grouped block-scaled GEMM on the sm_100a tensor cores (tcgen05).
//
// One persistent CTA per SM walks a list of 128 x 256 output tiles. Tiles are
// enumerated group by group (an expert is a group), N-tile major and M-tile
// minor, so neighbouring CTAs share the weight tile through L2. The tile list
// is derived on the device from the group offsets: no host synchronisation.
//
// Roles (448 threads, 14 warps):
//   warp 0       TMA producer: per 128-byte K stage, the A tile (128 rows),
//                the B tile (two 128-row halves) with 128-byte swizzle, and
//                the block scales (stored in the MMA chunk layout) with plain
//                bulk copies. STAGES-deep mbarrier ring.
//   warps 2..5   scale warps, one per TMEM lane quarter: they move each stage's
//                scales from shared memory into a TMEM ring with tcgen05.st,
//                in the replicated layout the block-scaled MMA reads (lane r of
//                every quarter holds the scales of rows r, r+32, r+64, ...).
//                Doing this with thread stores rather than tcgen05.cp keeps the
//                tensor pipe for MMAs only: a tcgen05.cp occupies the in-order
//                tensor pipe about as long as an MMA.
//   warp 1       MMA issuer (one thread): four block-scaled MMAs per stage
//                (kind::mxf4nvf4 block16 for NVFP4, kind::mxf8f6f4 with E8M0
//                scales for MXFP8) into the TMEM accumulator; tcgen05.commit
//                frees the stage and finally signals the accumulator.
//   warps 6..13  epilogue: tcgen05.ld of the fp32 accumulator (warp w reads
//                lanes 32*(w%4)..+31, two warps per quarter split the columns),
//                released back to the MMA warp as soon as it is in registers;
//                then SwiGLU with a fused per-group amax, or a bf16 / fp32 store.
// TMEM: columns [0, 256) accumulator, [256, 512) scale ring, 64 columns per
// stage: B scales of MMA kb at +8kb .. +8kb+7 (every lane quarter holds all 256
// B rows); A scales of MMA kb at the 4-column group +32+4kb (lane quarter q,
// which computes rows 32q..32q+31, reads column +32+4kb+q, so each quarter
// writes only that one column). Scale addresses given to the MMA and the
// column of every multi-column tcgen05.st stay 4-column aligned.
//
// Every wait is bounded (about 2 s); a wait that runs out records its id in
// the device error word, raises a CTA-wide abort flag and the kernel winds
// down, releasing TMEM.
#include "common.cuh"
#include "quant.cuh"

#include <mutex>

namespace nvfp4moe {

namespace {

constexpr int BM = 128, BN = 256, KBYTES = 128, STAGES = 4;
constexpr int A_STAGE = BM * KBYTES;   // 16 KB
constexpr int B_STAGE = BN * KBYTES;   // 32 KB
constexpr int SFA_STAGE = 2048, SFB_STAGE = 4096;
constexpr int NUM_THREADS = 448;
constexpr int MAX_GROUPS = 1024;
constexpr uint32_t TMEM_COLS = 512, TMEM_SF = 256, SF_SLOT_COLS = 64;

constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
constexpr int OFF_SFA = OFF_B + STAGES * B_STAGE;
constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_STAGE;
// barriers: full[S] (operands), sf_loaded[S] (scales in smem), sf_full[S]
// (scales in TMEM), empty[S], acc_full, acc_empty
constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_STAGE;
constexpr int OFF_MISC = OFF_BAR + 8 * (4 * STAGES + 2);  // tmem base, abort flag
constexpr int OFF_PREFIX = OFF_MISC + 16;
constexpr int SMEM_BYTES = OFF_PREFIX + 4 * (MAX_GROUPS + 1);
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;  // slack for 1024-byte alignment

struct Params {
    int kind, epi, group_axis;
    const uint8_t *a_sc, *b_sc;
    const float *a_ts, *b_ts;
    int32_t a_ts_stride;
    const int32_t *group_off;
    int32_t G;
    int64_t M;             // group K: rows of each output block
    int64_t N;             // accumulator columns per group (SwiGLU: 2f)
    int64_t f_out;         // SwiGLU: f
    int64_t ldc;           // output row stride (elements)
    int64_t b_rows_per_group;
    int64_t a_nkc, b_nkc;  // 512-byte scale chunks per 128-row block
    int32_t kt_total;      // K stages (group M)
    void *c;
    float *amax;
};

struct Tile {
    int g;
    int64_t a_row;          // TMA row of A
    int64_t b_row0, b_row1; // TMA rows of the two B halves
    int64_t k0;             // first contraction element (group K)
    int kt;                 // number of K stages
    int64_t out_row, out_col;
    int nt, mt;
};

__device__ __forceinline__ int upper_group(const int32_t *prefix, int G, int64_t t) {
    int lo = 0, hi = G;  // largest g with prefix[g] <= t
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (prefix[mid] <= t) lo = mid; else hi = mid;
    }
    return lo;
}

__device__ __forceinline__ Tile tile_info(const Params &p, const int32_t *prefix, int64_t t) {
    Tile T;
    const int g = upper_group(prefix, p.G, t);
    const int64_t local = t - prefix[g];
    T.g = g;
    if (p.group_axis == NVFP4MOE_GROUP_M) {
        const int64_t r0 = p.group_off[g];
        const int64_t mtiles = ((int64_t)p.group_off[g + 1] - r0) / BM;
        const int64_t nt = local / mtiles, mt = local - nt * mtiles;
        T.nt = (int)nt;
        T.mt = (int)mt;
        T.a_row = r0 + mt * BM;
        if (p.epi == EPI_SWIGLU_AMAX) {
            T.b_row0 = (int64_t)g * p.b_rows_per_group + nt * 128;
            T.b_row1 = T.b_row0 + p.f_out;
            T.out_col = nt * 128;
        } else {
            T.b_row0 = (int64_t)g * p.b_rows_per_group + nt * BN;
            T.b_row1 = T.b_row0 + 128;
            T.out_col = nt * BN;
        }
        T.k0 = 0;
        T.kt = p.kt_total;
        T.out_row = T.a_row;
    } else {
        const int64_t mtiles = p.M / BM;
        const int64_t nt = local / mtiles, mt = local - nt * mtiles;
        T.nt = (int)nt;
        T.mt = (int)mt;
        T.a_row = mt * BM;
        T.b_row0 = nt * BN;
        T.b_row1 = T.b_row0 + 128;
        T.k0 = p.group_off[g];
        T.kt = (int)(((int64_t)p.group_off[g + 1] - T.k0) / 128);
        T.out_row = (int64_t)g * p.M + T.a_row;
        T.out_col = nt * BN;
    }
    return T;
}

// Bounded wait that also gives up when another role raised the abort flag.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity,
                                              volatile int32_t *abort_flag, int32_t id) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > 2000000000ull) {
            atomicCAS(&g_device_error, 0, id);
            *abort_flag = 1;
            return false;
        }
    }
}

__device__ __forceinline__ uint32_t idesc_nvf4() {
    // a/b format E2M1 (1), N >> 3 at bit 17, scale format UE4M3 (0) at bit 23,
    // M >> 4 at bit 24; K-major A and B; dense.
    return (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}
__device__ __forceinline__ uint32_t idesc_mxf8(uint32_t sf_id) {
    // a/b format E4M3 (0), scale format UE8M0 (1) at bit 23, scale-factor ids
    // (byte of the 32-bit TMEM scale word) at bits 29..30 (A) and 4..5 (B).
    return ((uint32_t)(BN >> 3) << 17) | (1u << 23) | ((uint32_t)(BM >> 4) << 24) |
           (sf_id << 29) | (sf_id << 4);
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *empty = full + STAGES;
    uint64_t *sf_full = empty + STAGES;
    uint64_t *sf_loaded = sf_full + STAGES;
    uint64_t *acc_full = sf_loaded + STAGES;
    uint64_t *acc_empty = acc_full + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int32_t *abort_flag = reinterpret_cast<int32_t *>(smem + OFF_MISC + 4);
    int32_t *prefix = reinterpret_cast<int32_t *>(smem + OFF_PREFIX);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- tile prefix over the groups (all threads) ----
    const int G = p.G;
    for (int g = threadIdx.x; g < G; g += NUM_THREADS) {
        int64_t tiles;
        if (p.group_axis == NVFP4MOE_GROUP_M) {
            int64_t mt = ((int64_t)p.group_off[g + 1] - p.group_off[g]) / BM;
            int64_t nt = (p.epi == EPI_SWIGLU_AMAX) ? p.f_out / 128 : p.N / BN;
            tiles = mt * nt;
        } else {
            tiles = (p.M / BM) * (p.N / BN);
        }
        prefix[g + 1] = (int32_t)tiles;
    }
    if (threadIdx.x == 0) {
        prefix[0] = 0;
        *abort_flag = 0;
    }
    __syncthreads();
    if (warp == 0) {
        // inclusive scan of prefix[1..G] in chunks of `per` entries per lane
        const int per = (G + 31) / 32;
        int32_t s = 0;
        for (int i = 0; i < per; ++i) {
            int idx = lane * per + i + 1;
            if (idx <= G) s += prefix[idx];
        }
        int32_t incl = s;
        for (int o = 1; o < 32; o <<= 1) {
            int32_t n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += n;
        }
        int32_t run = incl - s;
        for (int i = 0; i < per; ++i) {
            int idx = lane * per + i + 1;
            if (idx <= G) {
                run += prefix[idx];
                prefix[idx] = run;
            }
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, TMEM_COLS);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_full[s], 4);
            mbar_init(&sf_loaded[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 8);
        fence_mbarrier_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int64_t total = prefix[G];
    const bool nvf4 = p.kind == 0;
    const uint32_t sfa_bytes = nvf4 ? 2048u : 512u;  // per 128-row block per stage
    const uint32_t op_tx = A_STAGE + B_STAGE;

    if (warp == 0) {
        // ======================= TMA producer =======================
        if (lane == 0) {
            prefetch_tmap(&tmA);
            prefetch_tmap(&tmB);
            int s = 0;
            uint32_t phase = 0;
            for (int64_t t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
                const Tile T = tile_info(p, prefix, t);
                for (int kt = 0; kt < T.kt; ++kt) {
                    if (!wait_or_abort(&empty[s], phase ^ 1u, abort_flag, WAIT_GEMM_EMPTY)) break;
                    // scales first, on their own barrier: they are small, land
                    // early, and the scale warps move them into TMEM while the
                    // operand tiles are still in flight
                    // (NVFP4 stage = 4 chunks (256 K) per 128 rows; MXFP8 = 1 chunk (128 K))
                    const int64_t kc = nvf4 ? (int64_t)kt * 4 : (T.k0 / 128 + kt);
                    const uint8_t *srcA = p.a_sc + ((T.a_row / 128) * p.a_nkc + kc) * 512;
                    const uint8_t *srcB0 = p.b_sc + ((T.b_row0 / 128) * p.b_nkc + kc) * 512;
                    const uint8_t *srcB1 = p.b_sc + ((T.b_row1 / 128) * p.b_nkc + kc) * 512;
                    uint8_t *ssfa = smem + OFF_SFA + s * SFA_STAGE;
                    uint8_t *ssfb = smem + OFF_SFB + s * SFB_STAGE;
                    mbar_arrive_expect_tx(&sf_loaded[s], 3 * sfa_bytes);
                    bulk_load(ssfa, srcA, sfa_bytes, &sf_loaded[s]);
                    bulk_load(ssfb, srcB0, sfa_bytes, &sf_loaded[s]);
                    bulk_load(ssfb + sfa_bytes, srcB1, sfa_bytes, &sf_loaded[s]);
                    mbar_arrive_expect_tx(&full[s], op_tx);
                    const int32_t kx = (int32_t)(T.k0 + (int64_t)kt * 128);  // byte column
                    uint8_t *sa = smem + OFF_A + s * A_STAGE;
                    uint8_t *sb = smem + OFF_B + s * B_STAGE;
                    tma_load_2d(sa, &tmA, kx, (int32_t)T.a_row, &full[s]);
                    tma_load_2d(sb, &tmB, kx, (int32_t)T.b_row0, &full[s]);
                    tma_load_2d(sb + B_STAGE / 2, &tmB, kx, (int32_t)T.b_row1, &full[s]);
                    if (++s == STAGES) { s = 0; phase ^= 1u; }
                }
            }
        }
    } else if (warp >= 2 && warp <= 5) {
        // ======================= scale warps =======================
        // In a 512-byte scale chunk the word (4 scales) of row r0 + 32 r1 sits
        // at byte r0 * 16 + r1 * 4, so lane r0 reads 16 contiguous bytes per
        // chunk: the B words of tile rows r0 + 32 j, and from the A chunk the
        // word of row r0 + 32 q, the only A row this lane quarter computes.
        const int q = warp & 3;
        const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
        int s = 0;
        uint32_t phase = 0;
        for (int64_t t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
            const Tile T = tile_info(p, prefix, t);
            for (int kt = 0; kt < T.kt; ++kt) {
                if (!wait_or_abort(&sf_loaded[s], phase, abort_flag, WAIT_GEMM_FULL)) break;
                const uint8_t *ssfa = smem + OFF_SFA + s * SFA_STAGE;
                const uint8_t *ssfb = smem + OFF_SFB + s * SFB_STAGE;
                const uint32_t slot = lane_addr + TMEM_SF + s * SF_SLOT_COLS;
                if (nvf4) {
                    uint32_t b[32], a[4];
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        const uint4 b0 = *reinterpret_cast<const uint4 *>(ssfb + kb * 512 + lane * 16);
                        const uint4 b1 = *reinterpret_cast<const uint4 *>(ssfb + 2048 + kb * 512 + lane * 16);
                        b[8 * kb + 0] = b0.x; b[8 * kb + 1] = b0.y; b[8 * kb + 2] = b0.z; b[8 * kb + 3] = b0.w;
                        b[8 * kb + 4] = b1.x; b[8 * kb + 5] = b1.y; b[8 * kb + 6] = b1.z; b[8 * kb + 7] = b1.w;
                        a[kb] = *reinterpret_cast<const uint32_t *>(ssfa + kb * 512 + lane * 16 + q * 4);
                    }
                    tmem_st_32x32b_x32(slot, b);
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) tmem_st_32x32b_x1(slot + 32 + 4 * kb + q, a[kb]);
                } else {
                    // one chunk per stage: the four scale bytes of a word serve
                    // the four MMAs (byte kb selected by the MMA's scale id)
                    const uint4 b0 = *reinterpret_cast<const uint4 *>(ssfb + lane * 16);
                    const uint4 b1 = *reinterpret_cast<const uint4 *>(ssfb + 512 + lane * 16);
                    const uint32_t b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                    tmem_st_32x32b_x8(slot, b);
                    tmem_st_32x32b_x1(slot + 32 + q,
                                      *reinterpret_cast<const uint32_t *>(ssfa + lane * 16 + q * 4));
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_full[s]);
                if (++s == STAGES) { s = 0; phase ^= 1u; }
            }
        }
    } else if (warp == 1) {
        // ======================= MMA issuer =======================
        if (lane == 0) {
            int s = 0;
            uint32_t phase = 0, acc_phase = 0;
            const uint32_t d_tmem = tmem_base;
            for (int64_t t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
                const Tile T = tile_info(p, prefix, t);
                if (T.kt == 0) continue;
                if (!wait_or_abort(acc_empty, acc_phase ^ 1u, abort_flag, WAIT_GEMM_ACC_EMPTY)) break;
                tc_fence_after();
                bool ok = true;
                for (int kt = 0; kt < T.kt; ++kt) {
                    if (!wait_or_abort(&full[s], phase, abort_flag, WAIT_GEMM_FULL) ||
                        !wait_or_abort(&sf_full[s], phase, abort_flag, WAIT_GEMM_FULL)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + OFF_A + s * A_STAGE);
                    const uint32_t sb = smem_u32(smem + OFF_B + s * B_STAGE);
                    const uint32_t sf = tmem_base + TMEM_SF + s * SF_SLOT_COLS;
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        const uint64_t ad = smem_desc(sa + 32 * kb, 16, 1024, 2);
                        const uint64_t bd = smem_desc(sb + 32 * kb, 16, 1024, 2);
                        if (nvf4) {
                            tc_mma_nvf4(d_tmem, ad, bd, idesc_nvf4(), sf + 32 + 4 * kb, sf + 8 * kb,
                                        (kt | kb) != 0);
                        } else {
                            const uint32_t sub = (uint32_t)kb << 30;  // byte kb of the scale word
                            tc_mma_mxf8(d_tmem, ad, bd, idesc_mxf8((uint32_t)kb), (sf + 32) | sub,
                                        sf | sub, (kt | kb) != 0);
                        }
                    }
                    tc_commit(&empty[s]);
                    if (++s == STAGES) { s = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit(acc_full);
                acc_phase ^= 1u;
            }
        }
    } else {
        // ======================= epilogue =======================
        const int q = warp & 3;          // TMEM lane quarter this warp may access
        const int half = (warp - 6) >> 2;
        const int row_in_tile = q * 32 + lane;
        const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
        uint32_t acc_phase = 0;
        for (int64_t t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
            const Tile T = tile_info(p, prefix, t);
            const int64_t row = T.out_row + row_in_tile;
            float alpha = 1.0f;
            if (nvf4) alpha = __fmul_rn(p.a_ts[(int64_t)T.g * p.a_ts_stride], p.b_ts[T.g]);
            const bool have_acc = T.kt > 0;
            if (have_acc) {
                if (!wait_or_abort(acc_full, acc_phase, abort_flag, WAIT_GEMM_ACC_FULL)) break;
                tc_fence_after();
            }
            if (p.epi == EPI_SWIGLU_AMAX) {
                // two rounds of (32 gate + 32 up) columns; the accumulator goes
                // back to the MMA warp once the second round is in registers
                uint16_t *h = static_cast<uint16_t *>(p.c);
                float amax = 0.0f;
                uint32_t pk[2][16];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int hc = half * 64 + c * 32;
                    uint32_t g[32], u[32];
                    tmem_ld_32x32b_x32(lane_addr + hc, g);
                    tmem_ld_32x32b_x32(lane_addr + 128 + hc, u);
                    tmem_wait_ld();
                    if (c == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(acc_empty);
                    }
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        float hv[2];
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const float gq = __fmul_rn(__uint_as_float(g[i + j]), alpha);
                            const float uq = __fmul_rn(__uint_as_float(u[i + j]), alpha);
                            const float den = fminf(1.0f + __expf(-gq), 1e30f);
                            hv[j] = __fmul_rn(__fdividef(gq, den), uq);
                        }
                        const uint32_t b0 = f32_to_bf16_bits(hv[0]), b1 = f32_to_bf16_bits(hv[1]);
                        amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(b0 << 16)),
                                                 fabsf(__uint_as_float(b1 << 16))));
                        pk[c][i >> 1] = b0 | (b1 << 16);
                    }
                }
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint4 *dst = reinterpret_cast<uint4 *>(h + row * p.ldc + T.out_col + half * 64 + c * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        dst[v] = make_uint4(pk[c][4 * v], pk[c][4 * v + 1], pk[c][4 * v + 2], pk[c][4 * v + 3]);
                }
                amax = warp_max(amax);
                if (lane == 0) atomic_max_nonneg(p.amax + T.g, amax);
            } else if (p.epi == EPI_STORE_BF16) {
                // two rounds of 64 columns, converted to bf16 as they arrive
                uint32_t pk[4][16];
#pragma unroll
                for (int rd = 0; rd < 2; ++rd) {
                    uint32_t r0[32], r1[32];
                    if (have_acc) {
                        tmem_ld_32x32b_x32(lane_addr + half * 128 + rd * 64, r0);
                        tmem_ld_32x32b_x32(lane_addr + half * 128 + rd * 64 + 32, r1);
                        tmem_wait_ld();
                        if (rd == 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(acc_empty);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) r0[i] = r1[i] = 0u;
                    }
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        pk[2 * rd][i >> 1] =
                            f32_to_bf16_bits(__fmul_rn(__uint_as_float(r0[i]), alpha)) |
                            (f32_to_bf16_bits(__fmul_rn(__uint_as_float(r0[i + 1]), alpha)) << 16);
                        pk[2 * rd + 1][i >> 1] =
                            f32_to_bf16_bits(__fmul_rn(__uint_as_float(r1[i]), alpha)) |
                            (f32_to_bf16_bits(__fmul_rn(__uint_as_float(r1[i + 1]), alpha)) << 16);
                    }
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.c) + row * p.ldc +
                                                           T.out_col + half * 128 + c * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        dst[v] = make_uint4(pk[c][4 * v], pk[c][4 * v + 1], pk[c][4 * v + 2], pk[c][4 * v + 3]);
                }
            } else {
                // fp32 out: two rounds of 64 columns stored as they arrive
#pragma unroll
                for (int rd = 0; rd < 2; ++rd) {
                    uint32_t r0[32], r1[32];
                    if (have_acc) {
                        tmem_ld_32x32b_x32(lane_addr + half * 128 + rd * 64, r0);
                        tmem_ld_32x32b_x32(lane_addr + half * 128 + rd * 64 + 32, r1);
                        tmem_wait_ld();
                        if (rd == 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(acc_empty);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) r0[i] = r1[i] = 0u;
                    }
                    float *cp = static_cast<float *>(p.c) + row * p.ldc + T.out_col + half * 128 + rd * 64;
                    float4 *d0 = reinterpret_cast<float4 *>(cp);
                    float4 *d1 = reinterpret_cast<float4 *>(cp + 32);
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        d0[v] = make_float4(__fmul_rn(__uint_as_float(r0[4 * v]), alpha),
                                            __fmul_rn(__uint_as_float(r0[4 * v + 1]), alpha),
                                            __fmul_rn(__uint_as_float(r0[4 * v + 2]), alpha),
                                            __fmul_rn(__uint_as_float(r0[4 * v + 3]), alpha));
                        d1[v] = make_float4(__fmul_rn(__uint_as_float(r1[4 * v]), alpha),
                                            __fmul_rn(__uint_as_float(r1[4 * v + 1]), alpha),
                                            __fmul_rn(__uint_as_float(r1[4 * v + 2]), alpha),
                                            __fmul_rn(__uint_as_float(r1[4 * v + 3]), alpha));
                    }
                }
            }
            if (have_acc) acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// --- host side: tensor maps through the driver entry point -------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// A [rows x cols_bytes] uint8 matrix, 128-byte x 128-row boxes, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols_bytes) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols_bytes};
    cuuint32_t box[2] = {128, 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int sm_count() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

}  // namespace

cudaError_t launch_grouped_gemm(const GemmArgs &a, cudaStream_t s) {
    const bool nvf4 = a.kind == 0;
    Params p{};
    p.kind = a.kind;
    p.epi = a.epi;
    p.group_axis = a.group_axis;
    p.a_sc = a.a_sc;
    p.b_sc = a.b_sc;
    p.a_ts = a.a_ts;
    p.b_ts = a.b_ts;
    p.a_ts_stride = a.a_ts_stride;
    p.group_off = a.group_off;
    p.G = a.G;
    p.M = a.M;
    p.N = a.N;
    p.f_out = (a.epi == EPI_SWIGLU_AMAX) ? a.N / 2 : a.N;
    p.ldc = p.f_out;
    p.b_rows_per_group = a.b_rows_per_group;
    p.c = a.c;
    p.amax = a.amax;
    // contraction bytes per row and scale chunks per 128-row block
    const int64_t kbytes = nvf4 ? a.a_cols / 2 : a.a_cols;
    p.a_nkc = nvf4 ? a.a_cols / 64 : a.a_cols / 128;
    p.b_nkc = p.a_nkc;
    p.kt_total = (int32_t)(kbytes / 128);
    const int64_t b_rows =
        (a.group_axis == NVFP4MOE_GROUP_M) ? (int64_t)a.G * a.b_rows_per_group : a.N;
    CUtensorMap ma, mb;
    if (!make_map(&ma, a.a, a.a_rows, kbytes) || !make_map(&mb, a.b, b_rows, kbytes))
        return cudaErrorInvalidValue;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    grouped_gemm_kernel<<<sm_count(), NUM_THREADS, SMEM_ALLOC, s>>>(ma, mb, p);
    return cudaGetLastError();
}

}  // namespace nvfp4moe

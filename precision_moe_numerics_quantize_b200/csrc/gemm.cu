// Grouped block-scaled GEMM on the sm_100a tensor cores, one CTA pair per
// tile (tcgen05.mma.cta_group::2).
//
// Every product in this file has the form
//     out[x, w] = alpha_g * sum_k X[x, k] * W[w, k]
// with X the token-side operand (activations or gradients: rows grouped by
// expert, or one row set whose contraction columns are split by group) and W
// the weights of group g. The MMA's M side is W: a cluster of two CTAs on two
// SMs computes a tile of 256 W rows x n X rows. Each CTA stages 128 W rows and
// n/2 X rows per k-block; the MMA reads the operands from both CTAs' shared
// memory, and each CTA's TMEM receives the fp32 accumulator of its 128 W rows
// over all n X rows. A group's (128-padded) X rows are cut into the fewest
// tiles of at most 192 rows, of equal size rounded up to 64: a 384-row expert
// becomes 2 x 192, not 256 + 128. A pair MMA of N = 192 runs at the full
// tensor rate, one of N = 128 is limited by how fast one thread can issue it.
//
// A pipeline stage is 256 bytes of K (two 128-byte k-blocks, eight MMAs): the
// MMA-issuing thread pays one barrier wait, one fence and one commit per stage,
// and issues the eight MMAs from straight-line code (a loop over k-blocks with
// a per-MMA branch on the format ran them about half again as slowly).
// Every barrier operation costs a few hundred cycles while the tensor cores
// and TMA keep shared memory busy, so each role does as few per stage as the
// protocol allows.
//
// Roles (640 threads, 20 warps, in both CTAs of the pair):
//   warp 0       TMA producer: first the X block scales of the stage (plain
//                bulk copies of the one or two 128-row chunk rows) into this
//                CTA, counted on its own `sf_loaded`; then this CTA's W and X
//                halves (128-byte swizzle), counted on the first CTA's `full`:
//                one box per operand covers both k-blocks of the stage, so a
//                stage is two tensor loads per CTA, not four.
//   warps 4..7   scale warps, one per TMEM lane quarter, one set for every
//                stage (the barriers assume one set). Each lane reads the stage's X
//                scale words from shared memory and the W scale words of its
//                own TMEM lane, loaded from L2 one stage ahead, and writes them
//                with tcgen05.st into the stage's scale slot in this CTA's
//                TMEM, in the layout the block-scaled MMA reads (the X scales
//                of all n rows in every lane quarter; the W scale word of lane
//                32q + l in column q of a 4-column group). One scale slot per
//                shared-memory stage: the producer only loads a stage once the
//                MMAs of the stage that last used its slot are done, so the
//                one wait for the stage's X scales also frees the slot. The
//                scale warps do not wait for the operands: each arrives once
//                per stage on the first CTA's `full`, the barrier the TMA
//                operand bytes complete on, so the MMA thread has a single
//                wait per stage and the scale writes run while the operands
//                are in flight. Thread stores keep the in-order tensor pipe
//                for MMAs only.
//   warp 1       first CTA only: the MMA issuer (one thread), eight
//                block-scaled MMAs per stage (kind::mxf4nvf4 block16 for
//                NVFP4, kind::mxf8f6f4 with E8M0 scales for MXFP8) after one
//                wait on `full`; one commit multicast to both CTAs' `empty`
//                barriers per stage and, after a tile's last stage, to both
//                `acc_full` barriers.
//   warps 8..19  epilogue: three warps per lane quarter, at most two
//                32-column blocks each, read with tcgen05.ld in one round
//                trip; the accumulator goes back to the MMA warp (arrival on
//                the first CTA's acc_empty) as soon as they are in registers,
//                before any arithmetic, and SwiGLU or the bf16 / fp32
//                conversion and the stores follow. Lane =
//                output column, register = output row, so every store
//                instruction of a warp writes one contiguous run of an output
//                row.
// SwiGLU (first GEMM of the expert FFN): W = [gate; up]. The W box of a CTA
// holds, per lane quarter, 16 gate rows followed by the 16 up rows of the same
// h columns (one 5-D TMA box), so lanes l and l ^ 16 of a warp hold g and u of
// one h column and trade half their values with one shuffle each.
// TMEM: columns [0, 192) accumulator, then one scale slot of 96 columns per
// shared-memory stage, 48 per k-block j: X scales of MMA kb at +48j+8kb (8
// columns = 256 rows), W scales of MMA kb at +48j+32+4kb (column q is read by
// lane quarter q). Every multi-column tcgen05.st and every scale address given
// to the MMA is 4-column aligned.
//
// Arrivals between the CTAs of a pair are relaxed: what they hand over is
// TMEM, ordered by tcgen05.wait and the tcgen05 fences; a cluster-scope
// release would also wait for the epilogue's global stores.
//
// Every wait is bounded (about 2 s): a wait that runs out records its id in
// the device error word and raises this CTA's abort flag; the CTA winds down
// and the other CTA of the pair then runs out on its own waits. Both CTAs meet
// at a final cluster barrier before TMEM is released.
// Built as a whole program (not relocatable device code) so that ptxas
// applies the setmaxnreg register split; the device error word is reached
// through a pointer in the kernel parameters.
#define NVFP4MOE_WHOLE_PROGRAM 1
#include "common.cuh"
#include "quant.cuh"

#include <atomic>
#include <mutex>

namespace nvfp4moe {

namespace {

constexpr int STAGES = 3;                // shared-memory stages of 2 k-blocks
constexpr int MAX_N = 192;               // X rows per tile
constexpr int W_KBLK = 128 * 128;        // one k-block (128 bytes of K) of 128 W rows
constexpr int X_KBLK = (MAX_N / 2) * 128;  // one k-block of up to 96 X rows
constexpr int W_STAGE = 2 * W_KBLK;
constexpr int X_STAGE = 2 * X_KBLK;
// X block scales of a stage: two 128-row chunk rows x 8 chunks of 512 bytes
// (NVFP4: 4 chunks per k-block; MXFP8: 1)
constexpr int SFX_CHUNKS = 8, SFX_STAGE = 2 * SFX_CHUNKS * 512;
// scale warps come in SCALE_SETS sets of four taking turns by stage; the
// epilogue's warps follow them.
// Warpgroups: 0 = producer, MMA issuer and two idle warps; 1 = scale warps
// (SCALE_SETS sets of four); then the epilogue, three warps per TMEM lane
// quarter, each owning at most two 32-column blocks of a tile of up to
// MAX_N = 192 columns. The kernel launches with 96 registers a thread
// (640 x 96 = 61440); setmaxnreg moves some from warpgroup 0 to the
// epilogue within that budget.
constexpr int SCALE_SETS = 1;
// the MMA thread waits on full[i % STAGES]: one scale-warp set
static_assert(SCALE_SETS == 1, "the scale warps arrive on the MMA thread's `full` barrier");
constexpr int SCALE_WARP0 = 4, EPI_WARP0 = SCALE_WARP0 + 4 * SCALE_SETS;
constexpr int EPI_PER_QUARTER = 3, EPI_WARPS = 4 * EPI_PER_QUARTER;
constexpr int NUM_THREADS = 32 * (EPI_WARP0 + EPI_WARPS);
// Measured on the full-size expert FFN (same box): 56 / 96 / 104 took
// 3.44 ms, no split 3.45 ms, 64 / 88 / 104 3.50 ms, 48 / 88 / 112 3.71 ms
// (the MMA and producer loops spill at 48).
constexpr uint32_t REGS_LAUNCH = 96, REGS_CONTROL = 56, REGS_EPILOGUE = 104;
static_assert(NUM_THREADS == 640, "register split below assumes 20 warps");
static_assert(128 * REGS_CONTROL + 128 * REGS_LAUNCH + 32 * EPI_WARPS * REGS_EPILOGUE <= NUM_THREADS * REGS_LAUNCH,
              "setmaxnreg split exceeds the registers the block launches with");
constexpr int MAX_GROUPS = 1024;
constexpr uint32_t TMEM_COLS = 512, TMEM_SF = MAX_N, SF_KB_COLS = 48, SF_SLOT_COLS = 96;

constexpr int OFF_W = 0;
constexpr int OFF_X = OFF_W + STAGES * W_STAGE;
constexpr int OFF_SFX = OFF_X + STAGES * X_STAGE;
// barriers: full[SETS S], empty[S], sf_loaded[SETS S], acc_full, acc_empty.
// `sf_loaded` is waited on by the scale-warp set that handles the stage: stage i uses barrier stage_bar(i) = (i % SETS) S +
// (i / SETS) % S, so every barrier is waited on by one set, in order, and a
// parity wait can never alias a phase two uses ahead.
constexpr int OFF_BAR = OFF_SFX + STAGES * SFX_STAGE;
constexpr int NUM_BARS = (2 * SCALE_SETS + 1) * STAGES + 2;
constexpr int OFF_MISC = (OFF_BAR + 8 * NUM_BARS + 15) & ~15;  // tmem base, abort flag
constexpr int OFF_GTAB = OFF_MISC + 16;  // per-group tile table (int4), one sentinel
static_assert(OFF_BAR % 8 == 0 && OFF_GTAB % 16 == 0, "barriers and the int4 tile table stay aligned");
constexpr int SMEM_BYTES = OFF_GTAB + 16 * (MAX_GROUPS + 1);
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;  // slack for 1024-byte alignment
static_assert(SMEM_ALLOC <= 232448, "shared memory per CTA");
static_assert(X_KBLK % 1024 == 0, "k-block areas stay 1024-byte aligned");
static_assert(TMEM_SF + STAGES * SF_SLOT_COLS <= TMEM_COLS, "TMEM columns");

// the first CTA's `full` completes when the operand bytes of both CTAs have
// landed and the scale warps of both CTAs (4 each) have written the stage's
// block scales into TMEM: the producer's arrival plus eight.
constexpr uint32_t FULL_COUNT = 1 + 8;
constexpr uint32_t ACC_EMPTY_COUNT = 2 * EPI_WARPS;  // every epilogue warp of both CTAs

__host__ __device__ constexpr uint32_t stage_bar(uint32_t i) {
    return (i % SCALE_SETS) * STAGES + (i / SCALE_SETS) % STAGES;
}
__host__ __device__ constexpr uint32_t stage_par(uint32_t i) { return ((i / SCALE_SETS) / STAGES) & 1u; }

// Test hook flags (nvfp4moe_debug_gemm): normal operation uses none.
constexpr uint32_t GEMM_DEBUG_WITHHOLD_LOADS = 1;  // producers issue nothing

struct Params {
    int kind, epi, group_axis;
    const uint8_t *w_sc, *x_sc;
    const float *w_ts, *x_ts;
    int32_t x_ts_stride;
    const int32_t *group_off;
    int32_t G;
    int64_t x_rows;        // group K: X rows, the output rows of every group
    int64_t w_rows_group;  // W rows per group (SwiGLU: 2f); 0 when W is shared
    int64_t f_out;         // SwiGLU: f
    int64_t ldc;           // output row stride (elements)
    int64_t w_nkc, x_nkc;  // 512-byte scale chunks per 128-row block
    int32_t kt_total;      // 128-byte k-blocks of K (group M)
    int32_t wtiles;        // 256-row W tiles per group (SwiGLU: f / 128)
    void *c;
    float *amax;
    int32_t *err;  // device error word
    uint64_t wait_ns;  // limit of every bounded wait
    uint32_t debug;    // GEMM_DEBUG_* (test hook; 0 in normal operation)
    // fused requantization of h (SwiGLU, NVFP4): hq == nullptr switches it off
    uint8_t *hq, *hq_sc;
    float *h_ts;
    int32_t *rq_tiles;   // per group: epilogue-warp arrivals so far
    int32_t *rq_cursor;  // per group: rows handed out so far
    int32_t *rq_queue;   // published groups in order, g + 1 (0: slot not written yet)
    int32_t *rq_ctr;     // [0] queue slots reserved, [1] head of the queue
};

struct Tile {
    int g;
    int n;            // X rows of the tile: a multiple of 64, at most MAX_N
    int mt;           // W tile within the group
    int kt;           // 128-byte k-blocks of K
    int64_t x_row;    // first X row (a multiple of 64)
    int64_t out_row;  // output row of X row x_row
    int64_t k0;       // first contraction element (group K)
};

// the tiles of `rows` X rows: count, and rows per tile (a multiple of 64)
__device__ __forceinline__ int32_t x_tiles(int32_t rows) { return (rows + MAX_N - 1) / MAX_N; }
__device__ __forceinline__ int32_t x_tile_rows(int32_t rows, int32_t ntiles) {
    return ntiles ? ((rows + ntiles - 1) / ntiles + 63) / 64 * 64 : 0;
}

// Per-group tile table in shared memory, one int4 per group:
//   x = tiles of the group, y = first X row (group M) or first contraction
//   element (group K), z = X tiles | rows per X tile << 16,
//   w = X rows (group M) or 128-byte k-blocks (group K).
// Every role walks its tiles t = pair, pair + npairs, ... with a cursor
// (group g, tile within the group) that only moves forward, one table read
// per group it crosses.
struct Cursor {
    int g;
    int32_t local;
    int4 e;
};
__device__ __forceinline__ void cursor_settle(const int4 *gtab, int G, Cursor &c) {
    while (c.g < G && c.local >= c.e.x) {
        c.local -= c.e.x;
        c.e = gtab[++c.g];
    }
}
__device__ __forceinline__ Cursor cursor_first(const int4 *gtab, int G, int32_t pair) {
    Cursor c;
    c.g = 0;
    c.local = pair;
    c.e = gtab[0];
    cursor_settle(gtab, G, c);
    return c;
}
__device__ __forceinline__ void cursor_next(const int4 *gtab, int G, int32_t npairs, Cursor &c) {
    c.local += npairs;
    cursor_settle(gtab, G, c);
}

__device__ __forceinline__ Tile cursor_tile(const Params &p, const Cursor &c) {
    Tile T;
    const int32_t ntiles = c.e.z & 0xFFFF, nb = c.e.z >> 16;
    const bool gm = p.group_axis == NVFP4MOE_GROUP_M;
    const int32_t rows = gm ? c.e.w : (int32_t)p.x_rows;
    const int32_t mt = c.local / ntiles, nt = c.local - mt * ntiles;
    T.g = c.g;
    T.mt = mt;
    T.n = min(nb, rows - nt * nb);
    if (gm) {
        T.x_row = (int64_t)c.e.y + (int64_t)nt * nb;
        T.out_row = T.x_row;
        T.k0 = 0;
        T.kt = p.kt_total;
    } else {
        T.x_row = (int64_t)nt * nb;
        T.out_row = (int64_t)c.g * p.x_rows + T.x_row;
        T.k0 = c.e.y;
        T.kt = c.e.w;
    }
    return T;
}

// Bounded wait (limit_ns) that also gives up when another role of this CTA
// raised the abort flag.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int32_t *abort_flag,
                                              int32_t *err, int32_t id, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            atomicCAS(err, 0, id);
            *abort_flag = 1;
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_3d_pair(void *dst, const CUtensorMap *map, int32_t c0, int32_t c1,
                                                 int32_t c2, uint32_t cbar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(cbar)
        : "memory");
}

// Instruction descriptors, M = 256 (two CTAs), N = n, K-major A and B, dense.
__device__ __forceinline__ uint32_t idesc_nvf4(int n) {
    // a/b format E2M1 (1) at bits 7 and 10, N >> 3 at bit 17, scale format
    // UE4M3 (0) at bit 23, M >> 4 at bit 24
    return (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | (16u << 24);
}
__device__ __forceinline__ uint32_t idesc_mxf8(int n, uint32_t sf_id) {
    // a/b format E4M3 (0), scale format UE8M0 (1) at bit 23, scale-factor ids
    // (byte of the 32-bit TMEM scale word) at bits 29..30 (A) and 4..5 (B)
    return ((uint32_t)(n >> 3) << 17) | (1u << 23) | (16u << 24) | (sf_id << 29) | (sf_id << 4);
}

// ---------------------------------------------------------------------------
// Fused requantization of h (the first GEMM of the expert FFN, NVFP4; the
// entry point moe_expert_fwd_fused_requant).
// An expert's NVFP4 tensor scale is amax(h) over all of its rows, known only
// once the last of its tiles is stored. Every epilogue warp counts its tiles
// per expert: one atomic per warp and tile, preceded by a fence that
// publishes its h stores and its amax update, and deferred until the warp
// has released the next accumulator, so that the stores have long drained.
// The warp that makes the expert's last arrival publishes it: the decode
// scale h_ts, then the expert's id in the next slot of a queue of experts.
// When all epilogue warps of a CTA are done with their tiles they meet at a
// CTA-local barrier and take rows from the queue until its head slot is not
// written yet or everything is taken: rows are handed out by a fetch-and-add
// on the head expert's row cursor (it never fails, so takers do not
// serialize); the head moves on, with one compare-and-swap, only when its
// expert has no rows left. Nothing ever waits on another CTA: every row still
// gets requantized, because the warp that writes a queue slot is inside its
// epilogue and drains the queue after it.
// Measured on B200, this is slower than the standalone requantization after
// GEMM1 (moe_expert_fwd): taking rows while tiles are still in flight, from
// the epilogue or from otherwise idle warps, lengthens the GEMM's TMA
// latency-bound pipeline by more than the separate pass costs.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int32_t ld_volatile_i32(const int32_t *p) {
    return *reinterpret_cast<const volatile int32_t *>(p);
}

// Called by a whole warp after it stored its part of a tile of group g.
__device__ __forceinline__ void requant_arrive(const Params &p, const int4 *gtab, int g, int lane) {
    __threadfence();  // this lane's h stores (and lane 0's amax update) before the count
    __syncwarp();
    int last = 0;
    if (lane == 0) last = atomicAdd(p.rq_tiles + g, 1) == gtab[g].x * (2 * EPI_WARPS) - 1;
    last = __shfl_sync(0xFFFFFFFFu, last, 0);
    if (!last) return;
    if (lane == 0) {
        __threadfence();  // every other warp's h and amax of g, seen through the count
        p.h_ts[g] = nvfp4_ts(*reinterpret_cast<const volatile float *>(p.amax + g));
        __threadfence();  // h_ts before the queue slot
        const int32_t slot = atomicAdd(p.rq_ctr, 1);
        *reinterpret_cast<volatile int32_t *>(p.rq_queue + slot) = g + 1;
    }
    __syncwarp();
}

// Takes up to max_rows rows of the expert at the head of the queue and
// requantizes them (codes and MMA-layout scale words, as the standalone
// grouped requantization writes them). Returns false, the same in every
// lane, when the head slot is not written yet or the queue is used up. A slot
// holding an impossible group is recorded (DEVERR_REQUANT) and passed over.
__device__ __forceinline__ bool requant_take(const Params &p, const int4 *gtab, int G, int lane,
                                             int max_rows, int &cg) {
    int g = -1;
    int32_t r = 0;
    if (lane == 0) {
        // the expert this warp took rows of last time: one fetch-and-add
        if (cg >= 0) {
            const int32_t got = atomicAdd(p.rq_cursor + cg, max_rows);
            if (got < gtab[cg].w) {
                g = cg;
                r = got;
            }
        }
        // else the head of the queue. Finite: every pass either hands out
        // rows, stops, or finds the head moved past an exhausted expert (by
        // this warp's CAS or another's)
        while (g < 0) {
            const int32_t s = ld_volatile_i32(p.rq_ctr + 1);
            if (s >= G) break;
            const int32_t e1 = ld_volatile_i32(p.rq_queue + s);
            if (e1 == 0) break;
            if (e1 < 1 || e1 > G) {
                atomicCAS(p.err, 0, DEVERR_REQUANT);
                atomicCAS(p.rq_ctr + 1, s, s + 1);
                continue;
            }
            const int32_t got = atomicAdd(p.rq_cursor + (e1 - 1), max_rows);
            if (got < gtab[e1 - 1].w) {
                g = e1 - 1;
                r = got;
                break;
            }
            atomicCAS(p.rq_ctr + 1, s, s + 1);
        }
        cg = g;
    }
    g = __shfl_sync(0xFFFFFFFFu, g, 0);
    if (g < 0) return false;
    r = __shfl_sync(0xFFFFFFFFu, r, 0);
    const int32_t row0 = gtab[g].y + r;
    const int n = min(max_rows, gtab[g].w - r);
    __threadfence();  // the slot was written after the group's amax was final
    const float S_enc = nvfp4_senc(*reinterpret_cast<const volatile float *>(p.amax + g));
    const int64_t f = p.f_out;
    const int32_t G64 = (int32_t)(f / 64);
    const uint16_t *h = static_cast<const uint16_t *>(p.c);
    for (int32_t it = lane; it < n * G64; it += 32) {
        const int64_t rr = row0 + it / G64;
        const int32_t gr = it % G64;
        const uint4 *pv = reinterpret_cast<const uint4 *>(h + rr * f + (int64_t)gr * 64);
        uint4 raw[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) raw[j] = __ldcg(pv + j);
        uint32_t scw = 0, w[8];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            float v[16];
            unpack_bf16x8(raw[2 * b], v);
            unpack_bf16x8(raw[2 * b + 1], v + 8);
            scw |= nvfp4_block16(v, S_enc, w[2 * b], w[2 * b + 1]) << (8 * b);
        }
        uint4 *co = reinterpret_cast<uint4 *>(p.hq + rr * (f / 2) + (int64_t)gr * 32);
        co[0] = make_uint4(w[0], w[1], w[2], w[3]);
        co[1] = make_uint4(w[4], w[5], w[6], w[7]);
        *reinterpret_cast<uint32_t *>(p.hq_sc + mma_sf_offset(rr, (int64_t)gr * 4, f / 16)) = scw;
    }
    __syncwarp();
    return true;
}

// Epilogue warps only: CTA-local barrier (named barrier 1) of the 12
// epilogue warps, all of which reach it after their tile loop (the warp is
// reconverged first; the barrier itself is the non-aligned form).
__device__ __forceinline__ void epilogue_barrier() {
    __syncwarp();
    asm volatile("barrier.sync 1, %0;" ::"n"(32 * EPI_WARPS) : "memory");
}

__device__ __forceinline__ float swiglu_value(float g, float u, float alpha) {
    const float gq = __fmul_rn(g, alpha);
    const float uq = __fmul_rn(u, alpha);
    const float den = fminf(1.0f + __expf(-gq), 1e30f);
    return __fmul_rn(__fdividef(gq, den), uq);
}

// REQUANT: the first GEMM of moe_expert_fwd_fused_requant, whose epilogue
// warps also requantize h. It is its own instantiation: compiled into every
// launch, the unused requantization code alone made the fp32-output GEMM
// nearly twice as slow (3.98 ms against 7.6 ms for the full-size MXFP8 wgrad).
template <bool REQUANT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmW,
                             const __grid_constant__ CUtensorMap tmX32,
                             const __grid_constant__ CUtensorMap tmX64,
                             const __grid_constant__ CUtensorMap tmX96, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *empty = full + SCALE_SETS * STAGES;
    uint64_t *sf_loaded = empty + STAGES;
    uint64_t *acc_full = sf_loaded + SCALE_SETS * STAGES;
    uint64_t *acc_empty = acc_full + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int32_t *abort_flag = reinterpret_cast<int32_t *>(smem + OFF_MISC + 4);
    int4 *gtab = reinterpret_cast<int4 *>(smem + OFF_GTAB);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    // ---- per-group tile table (both CTAs compute the same one) ----
    const int G = p.G;
    const int32_t npairs32 = (int32_t)npairs;
    for (int g = threadIdx.x; g <= G; g += NUM_THREADS) {
        int4 e = make_int4(0, 0, 0, 0);
        if (g < G) {
            const int32_t o0 = p.group_off[g], o1 = p.group_off[g + 1];
            const bool gm = p.group_axis == NVFP4MOE_GROUP_M;
            const int32_t rows = gm ? ((o1 - o0) / 128) * 128 : (int32_t)p.x_rows;
            const int32_t nx = x_tiles(rows);
            e.x = p.wtiles * nx;
            e.y = o0;
            e.z = nx | (x_tile_rows(rows, nx) << 16);
            e.w = gm ? rows : (o1 - o0) / 128;
        }
        gtab[g] = e;
    }
    if (threadIdx.x == 0) *abort_flag = 0;
    constexpr bool requant = REQUANT;
    // groups without rows are never published: their decode scale is 1
    if (requant && blockIdx.x == 0)
        for (int g = threadIdx.x; g < G; g += NUM_THREADS)
            if (gtab[g].x == 0) p.h_ts[g] = 1.0f;
    __syncthreads();
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, TMEM_COLS);
        tmem_relinquish_pair();
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < SCALE_SETS * STAGES; ++s) {
            mbar_init(&full[s], FULL_COUNT);
            mbar_init(&sf_loaded[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, ACC_EMPTY_COUNT);
        fence_mbarrier_init();
    }
    // both CTAs' barriers exist before any arrival from the other CTA
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const bool nvf4 = p.kind == 0;
    const bool swiglu = p.epi == EPI_SWIGLU_AMAX;

    if (warp == 0) {
        regs_shrink<REGS_CONTROL>();
        // ======================= TMA producer =======================
        if (lane == 0) {
            prefetch_tmap(&tmW);
            prefetch_tmap(&tmX32);
            prefetch_tmap(&tmX64);
            prefetch_tmap(&tmX96);
            const uint32_t cfull = cluster_addr(full, 0);
            const uint32_t sfc = nvf4 ? 4 : 1;  // scale chunks per k-block
            const int32_t gu_groups = (int32_t)(2 * p.f_out / 16);  // 16-row groups of W1 per expert
            int s = 0;
            uint32_t phase = 0, i = 0;
            // test hook: withhold every load (nothing is ever in flight), so
            // that the consumers' bounded waits run out
            bool ok = (p.debug & GEMM_DEBUG_WITHHOLD_LOADS) == 0;
            for (Cursor c = cursor_first(gtab, G, (int32_t)pair); c.g < G && ok && !*abort_flag;
                 cursor_next(gtab, G, npairs32, c)) {
                const Tile T = cursor_tile(p, c);
                const int64_t w_row = (int64_t)T.g * p.w_rows_group + (int64_t)T.mt * 256 + 128 * rank;
                const uint32_t kblk_tx = 2u * W_KBLK + (uint32_t)T.n * 128u;  // both CTAs
                const int hn = T.n / 2;  // this CTA's X rows: 32, 64 or 96
                const int32_t xr = (int32_t)(T.x_row + (int64_t)rank * hn);
                // X scale chunk rows of the tile: a, and a + 1 if the tile
                // reaches into it
                const int64_t xa = T.x_row / 128;
                const int xcr = (int)((T.x_row + T.n - 1) / 128 - xa) + 1;
                for (int kb0 = 0; kb0 < T.kt; kb0 += 2) {
                    const int nkb = T.kt - kb0 >= 2 ? 2 : 1;
                    if (!wait_or_abort(&empty[s], phase ^ 1u, abort_flag, p.err, WAIT_GEMM_EMPTY, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    // the X block scales first, on this CTA's own sf_loaded:
                    // the scale warps start on them while the operands are
                    // still in flight
                    const uint32_t sf_bytes = (uint32_t)xcr * nkb * sfc * 512u;
                    const uint32_t sb = stage_bar(i);
                    mbar_arrive_expect_tx(&sf_loaded[sb], sf_bytes);
                    const int64_t kc0 = nvf4 ? (int64_t)kb0 * 4 : (T.k0 / 128 + kb0);
                    uint8_t *ssf = smem + OFF_SFX + s * SFX_STAGE;
                    for (int cr = 0; cr < xcr; ++cr)
                        bulk_load(ssf + cr * (SFX_CHUNKS * 512), p.x_sc + ((xa + cr) * p.x_nkc + kc0) * 512,
                                  nkb * sfc * 512u, &sf_loaded[sb]);
                    // both k-blocks always: a lone last k-block brings its
                    // neighbour (or the zero fill past the tensor) along
                    if (rank == 0) mbar_arrive_expect_tx(&full[sb], 2u * kblk_tx);
                    const uint32_t cbar = cfull + 8u * sb;
                    {
                        // one box per operand brings both k-blocks of the stage
                        const int32_t kc = (int32_t)(T.k0 / 128 + kb0);  // k-block coordinate
                        uint8_t *sw = smem + OFF_W + s * W_STAGE;
                        uint8_t *sx = smem + OFF_X + s * X_STAGE;
                        if (swiglu)
                            tma_load_5d_pair(sw, &tmW, 0, 0, 0, T.g * gu_groups + 8 * T.mt + 4 * (int32_t)rank, kc, cbar);
                        else
                            tma_load_3d_pair(sw, &tmW, 0, (int32_t)w_row, kc, cbar);
                        const CUtensorMap *mx = hn == 96 ? &tmX96 : (hn == 64 ? &tmX64 : &tmX32);
                        tma_load_3d_pair(sx, mx, 0, xr, kc, cbar);
                    }
                    ++i;
                    if (++s == STAGES) { s = 0; phase ^= 1u; }
                }
            }
        }
    } else if (warp >= SCALE_WARP0 && warp < EPI_WARP0) {
        // ======================= scale warps (launch registers) =======================
        // In a 512-byte scale chunk the word (4 scales) of row r0 + 32 r1 sits
        // at byte r0 * 16 + r1 * 4, so lane r0 reads 16 contiguous bytes per X
        // chunk (the words of X rows r0 + 32 j) and one word of each W chunk:
        // that of the W row TMEM lane 32 q + r0 of this CTA holds.
        const int q = warp & 3;
        const uint32_t set = (uint32_t)(warp - SCALE_WARP0) >> 2;  // stages i with i % SCALE_SETS == set
        const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
        // this lane's W row inside its 128-row scale block; SwiGLU: lanes
        // 0..15 hold gate rows, lanes 16..31 the up rows of the same h columns
        const int w_rib = swiglu ? 64 * (int)rank + 16 * q + (lane & 15) : 32 * q + lane;
        const int64_t w_up = (swiglu && lane >= 16) ? p.f_out : 0;
        const uint32_t w_word = (uint32_t)((w_rib & 31) * 16 + (w_rib >> 5) * 4);
        const uint32_t c_full = cluster_addr(full, 0);
        const int chunks = nvf4 ? 4 : 1;  // scale chunks per k-block

        // a pipeline stage: tile at cursor c (T), k-blocks kb0 and kb0 + 1
        struct Stage {
            Cursor c;
            Tile T;
            int kb0;
        };
        // next stage after `st`, skipping tiles without K
        auto next_stage = [&](Stage &st) -> bool {
            st.kb0 += 2;
            if (st.kb0 < st.T.kt) return true;
            for (cursor_next(gtab, G, npairs32, st.c); st.c.g < G; cursor_next(gtab, G, npairs32, st.c)) {
                st.T = cursor_tile(p, st.c);
                if (st.T.kt > 0) {
                    st.kb0 = 0;
                    return true;
                }
            }
            return false;
        };
        // W scale words of the stage's k-blocks: [k-block j][MMA kb]
        auto fetch_w = [&](const Stage &st, uint32_t (&w)[2][4]) {
            const Tile &T = st.T;
            const int64_t wrow = swiglu ? (int64_t)T.g * p.w_rows_group + (int64_t)T.mt * 128 + w_up
                                        : (int64_t)T.g * p.w_rows_group + (int64_t)T.mt * 256 + 128 * rank;
            const int nkb = T.kt - st.kb0 >= 2 ? 2 : 1;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int64_t kc = nvf4 ? (int64_t)(st.kb0 + j) * 4 : (T.k0 / 128 + st.kb0 + j);
                const uint8_t *ws = p.w_sc + ((wrow / 128) * p.w_nkc + kc) * 512 + w_word;
#pragma unroll
                for (int kb = 0; kb < 4; ++kb)
                    w[j][kb] = (j < nkb && kb < chunks) ? __ldg(reinterpret_cast<const uint32_t *>(ws + kb * 512))
                                                       : 0u;
            }
        };
        // write stage i (slot s = i % STAGES) into TMEM and hand it over
        auto put = [&](const Stage &st, uint32_t i, const uint32_t (&w)[2][4]) -> bool {
            const Tile &T = st.T;
            const uint32_t s = i % STAGES, sb = stage_bar(i), par = stage_par(i);
            // the stage's X scales landed; the producer only loaded them
            // after the MMAs that last read slot s were done, so the slot is
            // free. The operands may still be in flight.
            if (!wait_or_abort(&sf_loaded[sb], par, abort_flag, p.err, WAIT_GEMM_SF_SLOT, p.wait_ns)) return false;
            tc_fence_after();
            const int nkb = T.kt - st.kb0 >= 2 ? 2 : 1;
            // tile rows start at 128 a + 64 h: column j holds word (2h + j) % 4
            // of chunk row (2h + j) / 4
            const bool h = (T.x_row & 64) != 0;
            const bool need_b = (h ? 2 : 0) + T.n / 32 > 4;
            const uint8_t *ssf = smem + OFF_SFX + s * SFX_STAGE + lane * 16;
            for (int j = 0; j < nkb; ++j) {
                const uint32_t slot = lane_addr + TMEM_SF + s * SF_SLOT_COLS + j * SF_KB_COLS;
                if (nvf4) {
                    uint32_t b[32];
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        const int c = j * 4 + kb;
                        const uint4 A = *reinterpret_cast<const uint4 *>(ssf + c * 512);
                        const uint4 B = need_b ? *reinterpret_cast<const uint4 *>(ssf + (SFX_CHUNKS + c) * 512)
                                               : make_uint4(0u, 0u, 0u, 0u);
                        b[8 * kb + 0] = h ? A.z : A.x; b[8 * kb + 1] = h ? A.w : A.y;
                        b[8 * kb + 2] = h ? B.x : A.z; b[8 * kb + 3] = h ? B.y : A.w;
                        b[8 * kb + 4] = h ? B.z : B.x; b[8 * kb + 5] = h ? B.w : B.y;
                        b[8 * kb + 6] = B.z;           b[8 * kb + 7] = B.w;
                    }
                    tmem_st_32x32b_x32(slot, b);
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) tmem_st_32x32b_x1(slot + 32 + 4 * kb + q, w[j][kb]);
                } else {
                    // one chunk per k-block: the four scale bytes of a word
                    // serve its four MMAs (byte kb selected by the scale id)
                    const uint4 A = *reinterpret_cast<const uint4 *>(ssf + j * 512);
                    const uint4 B = need_b ? *reinterpret_cast<const uint4 *>(ssf + (SFX_CHUNKS + j) * 512)
                                           : make_uint4(0u, 0u, 0u, 0u);
                    const uint32_t b[8] = {h ? A.z : A.x, h ? A.w : A.y, h ? B.x : A.z, h ? B.y : A.w,
                                           h ? B.z : B.x, h ? B.w : B.y, B.z, B.w};
                    tmem_st_32x32b_x8(slot, b);
                    tmem_st_32x32b_x1(slot + 32 + q, w[j][0]);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) mbar_arrive(&full[sb]);
                else mbar_arrive_cluster_relaxed(c_full + 8u * sb);
            }
            return true;
        };
        // this set's stages: i = set, set + SCALE_SETS, ...; the W words of
        // the next one are loaded before the current one is written
        auto skip = [&](Stage &st) -> bool {
            bool ok = true;
            for (int k = 0; k < SCALE_SETS && ok; ++k) ok = next_stage(st);
            return ok;
        };
        Stage cur;
        cur.c.g = 0;
        cur.c.local = (int32_t)pair - npairs32;
        cur.c.e = gtab[0];
        cur.T.kt = 0;
        cur.kb0 = 0;
        bool more = next_stage(cur);
        uint32_t i = 0;
        for (uint32_t k = 0; k < set && more; ++k) {
            more = next_stage(cur);
            ++i;
        }
        uint32_t wa[2][4], wb[2][4];
        if (more) fetch_w(cur, wa);
        // two stages per iteration so the word buffers swap roles without
        // register copies
        while (more && !*abort_flag) {
            Stage nxt = cur;
            bool more2 = skip(nxt);
            if (more2) fetch_w(nxt, wb);
            if (!put(cur, i, wa)) break;
            if (!more2 || *abort_flag) break;
            cur = nxt;
            i += SCALE_SETS;
            nxt = cur;
            more = skip(nxt);
            if (more) fetch_w(nxt, wa);
            if (!put(cur, i, wb)) break;
            cur = nxt;
            i += SCALE_SETS;
        }
    } else if (warp == 1) {
        regs_shrink<REGS_CONTROL>();
        // ======================= MMA issuer (first CTA) =======================
        if (rank == 0 && lane == 0) {
            const uint32_t c_empty = cluster_addr(empty, 0), c_acc = cluster_addr(acc_full, 0);
            const uint64_t wdesc0 = smem_desc(smem_u32(smem + OFF_W), 16, 1024, 2);
            const uint64_t xdesc0 = smem_desc(smem_u32(smem + OFF_X), 16, 1024, 2);
            int s = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (Cursor c = cursor_first(gtab, G, (int32_t)pair); c.g < G && ok && !*abort_flag;
                 cursor_next(gtab, G, npairs32, c)) {
                const Tile T = cursor_tile(p, c);
                if (T.kt == 0) continue;
                if (!wait_or_abort(acc_empty, acc_phase ^ 1u, abort_flag, p.err, WAIT_GEMM_ACC_EMPTY, p.wait_ns)) break;
                tc_fence_after();
                const uint32_t idesc4 = idesc_nvf4(T.n);
                for (int kb0 = 0; kb0 < T.kt; kb0 += 2) {
                    const int nkb = T.kt - kb0 >= 2 ? 2 : 1;
                    // one wait: both CTAs' operands landed and both CTAs'
                    // scale warps wrote the stage's scales into TMEM
                    if (!wait_or_abort(&full[s], phase, abort_flag, p.err, WAIT_GEMM_FULL, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // descriptors advance in 16-byte units: 32 bytes of K per MMA
                    const uint64_t wd = wdesc0 + (uint64_t)((s * W_STAGE) >> 4);
                    const uint64_t xd = xdesc0 + (uint64_t)((s * X_STAGE) >> 4);
                    const uint32_t sf = tmem_base + TMEM_SF + s * SF_SLOT_COLS;
                    const uint32_t acc0 = kb0 != 0;
                    if (nvf4) {
                        tc_mma_nvf4_pair(tmem_base, wd, xd, idesc4, sf + 32, sf, acc0);
                        tc_mma_nvf4_pair(tmem_base, wd + 2, xd + 2, idesc4, sf + 36, sf + 8, 1u);
                        tc_mma_nvf4_pair(tmem_base, wd + 4, xd + 4, idesc4, sf + 40, sf + 16, 1u);
                        tc_mma_nvf4_pair(tmem_base, wd + 6, xd + 6, idesc4, sf + 44, sf + 24, 1u);
                        if (nkb == 2) {
                            const uint64_t w1 = wd + (uint64_t)(W_KBLK >> 4), x1 = xd + (uint64_t)(T.n * 4);
                            const uint32_t s1 = sf + SF_KB_COLS;
                            tc_mma_nvf4_pair(tmem_base, w1, x1, idesc4, s1 + 32, s1, 1u);
                            tc_mma_nvf4_pair(tmem_base, w1 + 2, x1 + 2, idesc4, s1 + 36, s1 + 8, 1u);
                            tc_mma_nvf4_pair(tmem_base, w1 + 4, x1 + 4, idesc4, s1 + 40, s1 + 16, 1u);
                            tc_mma_nvf4_pair(tmem_base, w1 + 6, x1 + 6, idesc4, s1 + 44, s1 + 24, 1u);
                        }
                    } else {
                        for (int j = 0; j < nkb; ++j) {
                            const uint32_t sfj = sf + j * SF_KB_COLS;
#pragma unroll
                            for (int kb = 0; kb < 4; ++kb) {
                                const uint64_t woff = (uint64_t)((j * W_KBLK + 32 * kb) >> 4);
                                const uint64_t xoff = (uint64_t)((j * (T.n / 2) * 128 + 32 * kb) >> 4);
                                const uint32_t acc = (kb0 | j | kb) != 0;
                                const uint32_t sub = (uint32_t)kb << 30;  // byte kb of the scale word
                                tc_mma_mxf8_pair(tmem_base, wd + woff, xd + xoff, idesc_mxf8(T.n, (uint32_t)kb),
                                                 (sfj + 32) | sub, sfj | sub, acc);
                            }
                        }
                    }
                    tc_commit_pair_mc(c_empty + 8u * s, 0x3);
                    if (++s == STAGES) { s = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit_pair_mc(c_acc, 0x3);
                acc_phase ^= 1u;
            }
        }
    } else if (warp >= EPI_WARP0) {
        regs_grow<REGS_EPILOGUE>();
        // ======================= epilogue =======================
        const int q = warp & 3;                   // TMEM lane quarter this warp may access
        const int sub = (warp - EPI_WARP0) >> 2;  // which pair of 32-column blocks
        const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
        const uint32_t c_acc_empty = cluster_addr(acc_empty, 0);
        const bool up_lane = lane >= 16;
        const bool f32_out = p.epi == EPI_STORE_F32;
        uint32_t acc_phase = 0;
        // fused requantization state: the group whose tile this warp stored
        // last and has not counted yet (its count, with the fence before it,
        // waits until the next tile so the stores have long drained), and the
        // expert this warp takes rows of (lane 0)
        int pend_g = -1, take_g = -1;
        for (Cursor c = cursor_first(gtab, G, (int32_t)pair); c.g < G && !*abort_flag;
             cursor_next(gtab, G, npairs32, c)) {
            const Tile T = cursor_tile(p, c);
            float alpha = 1.0f;
            if (nvf4) alpha = __fmul_rn(p.x_ts[(int64_t)T.g * p.x_ts_stride], p.w_ts[T.g]);
            const bool have_acc = T.kt > 0;
            // this warp's accumulator columns (X rows): blocks 2 sub and
            // 2 sub + 1 of the tile's n / 32
            const int b0 = 2 * sub;
            const int nb = max(0, min(2, T.n / 32 - b0));
            const int64_t row0 = T.out_row + 32 * b0;  // output row of the first column
            if (have_acc) {
                if (!wait_or_abort(acc_full, acc_phase, abort_flag, p.err, WAIT_GEMM_ACC_FULL, p.wait_ns)) break;
                tc_fence_after();
            }
            uint32_t va[32], vb[32];
            if (have_acc && nb > 0) {
                tmem_ld_32x32b_x32(lane_addr + 32 * b0, va);
                if (nb > 1) tmem_ld_32x32b_x32(lane_addr + 32 * b0 + 32, vb);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int k = 0; k < 32; ++k) va[k] = vb[k] = 0u;
            }
            if (have_acc) {
                // the accumulator goes back before any arithmetic
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster_relaxed(c_acc_empty);
                acc_phase ^= 1u;
            }
            if (requant && pend_g >= 0) {
                requant_arrive(p, gtab, pend_g, lane);
                pend_g = -1;
            }
            float amax = 0.0f;
            // finish and store block b (0 or 1 of this warp) from its 32
            // accumulator columns v
            auto finish = [&](int b, const uint32_t (&v)[32]) {
                const int64_t r = row0 + 32 * b;  // output row of column 0 of the block
                if (swiglu) {
                    // lane l < 16: gate of an h column, lane l + 16: up of the
                    // same column; the gate lane finishes X rows 0..15 of the
                    // block, the up lane rows 16..31
                    const int64_t hc = (int64_t)T.mt * 128 + 64 * rank + 16 * q + (lane & 15);
                    uint16_t *dst = static_cast<uint16_t *>(p.c) + (r + (up_lane ? 16 : 0)) * p.ldc + hc;
#pragma unroll
                    for (int j = 0; j < 16; j += 2) {
                        float hv[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const uint32_t send = up_lane ? v[j + e] : v[16 + j + e];
                            const uint32_t x = __shfl_xor_sync(0xFFFFFFFFu, send, 16);
                            const float g = __uint_as_float(up_lane ? x : v[j + e]);
                            const float u = __uint_as_float(up_lane ? v[16 + j + e] : x);
                            hv[e] = swiglu_value(g, u, alpha);
                        }
                        const uint32_t w = bf16x2_rn(hv[0], hv[1]);
                        amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w << 16)),
                                                 fabsf(__uint_as_float(w & 0xFFFF0000u))));
                        *dst = (uint16_t)w;
                        dst += p.ldc;
                        *dst = (uint16_t)(w >> 16);
                        dst += p.ldc;
                    }
                } else {
                    const int64_t col = (int64_t)T.mt * 256 + 128 * rank + 32 * q + lane;
                    if (!f32_out) {
                        uint16_t *dst = static_cast<uint16_t *>(p.c) + r * p.ldc + col;
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            const uint32_t w = bf16x2_rn(__fmul_rn(__uint_as_float(v[j]), alpha),
                                                         __fmul_rn(__uint_as_float(v[j + 1]), alpha));
                            *dst = (uint16_t)w;
                            dst += p.ldc;
                            *dst = (uint16_t)(w >> 16);
                            dst += p.ldc;
                        }
                    } else {
                        float *dst = static_cast<float *>(p.c) + r * p.ldc + col;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            *dst = __fmul_rn(__uint_as_float(v[j]), alpha);
                            dst += p.ldc;
                        }
                    }
                }
            };
            if (nb > 0) finish(0, va);
            if (nb > 1) finish(1, vb);
            if (swiglu) {
                amax = warp_max(amax);
                if (lane == 0 && nb > 0) atomic_max_nonneg(p.amax + T.g, amax);
                if (requant) pend_g = T.g;
            }
        }
        if (requant) {
            if (pend_g >= 0) requant_arrive(p, gtab, pend_g, lane);
            // every epilogue warp of this CTA is past its tiles: take rows
            // until the head of the queue is not written yet or all is taken
            epilogue_barrier();
            while (requant_take(p, gtab, G, lane, 4, take_g)) {
            }
        }
    } else {
        regs_shrink<REGS_CONTROL>();  // warps 2 and 3: idle
    }

    // No CTA leaves (or frees TMEM) while the other may still arrive on its
    // barriers or the MMA may still write its TMEM.
    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
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

// A [rows x cols_bytes] uint8 matrix seen as 3-D (128 bytes, rows, 128-byte
// k-block): one box of (128, box_rows, 2) brings two k-blocks, each a
// contiguous [box_rows x 128] block with 128-byte swizzle.
bool make_map_3d_kb(CUtensorMap *m, const void *base, int64_t rows, int64_t cols_bytes,
                    uint32_t box_rows) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)rows, (cuuint64_t)(cols_bytes / 128)};
    cuuint64_t strides[2] = {(cuuint64_t)cols_bytes, 128};
    cuuint32_t box[3] = {128, box_rows, 2};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The [E x 2f x cols_bytes] gate/up weights seen as 5-D (128 bytes, 16 rows,
// gate|up, 16-row group counted across experts, 128-byte k-block): one box of
// (128, 16, 2, 4, 2) brings, for two k-blocks, 4 x (16 gate rows, the 16
// matching up rows) = 128 rows in the order the SwiGLU epilogue pairs them.
bool make_map_swiglu_kb(CUtensorMap *m, const void *base, int64_t E, int64_t f, int64_t cols_bytes) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    const cuuint64_t rb = (cuuint64_t)cols_bytes;
    cuuint64_t dims[5] = {128, 16, 2, (cuuint64_t)(E * 2 * f / 16), rb / 128};
    cuuint64_t strides[4] = {rb, (cuuint64_t)f * rb, 16 * rb, 128};
    cuuint32_t box[5] = {128, 16, 2, 4, 2};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Per-device launch set-up, done once per device (a process may drive
// several GPUs): the shared-memory attribute, the register check, and the
// grid, two CTAs for every cluster the device keeps resident at once (the
// tile loop is persistent, so a cluster left waiting for a free pair of SMs
// would double the tail).
cudaError_t launch_setup(int &grid) {
    constexpr int kMaxDevices = 64;
    static int grids[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (grids[dev] == 0) {
        for (const void *k : {reinterpret_cast<const void *>(grouped_gemm_pair_kernel<false>),
                              reinterpret_cast<const void *>(grouped_gemm_pair_kernel<true>)}) {
            e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
            if (e != cudaSuccess) return e;
            // setmaxnreg only redistributes the registers the block launched
            // with: a build that gave the kernel fewer than REGS_LAUNCH would
            // leave the epilogue's increase waiting forever
            cudaFuncAttributes fa;
            e = cudaFuncGetAttributes(&fa, k);
            if (e != cudaSuccess) return e;
            if (fa.numRegs < (int)REGS_LAUNCH) return cudaErrorInvalidConfiguration;
        }
        int sms = 0;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 1) sms = 148;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(sms & ~1));
        cfg.blockDim = dim3(NUM_THREADS);
        cfg.dynamicSmemBytes = SMEM_ALLOC;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, grouped_gemm_pair_kernel<false>, &cfg) != cudaSuccess ||
            clusters <= 0) {
            cudaGetLastError();
            clusters = sms / 2;
        }
        grids[dev] = 2 * (clusters < sms / 2 ? clusters : sms / 2);
    }
    grid = grids[dev];
    return cudaSuccess;
}

}  // namespace

// Test hook state, set by nvfp4moe_debug_gemm (abi.cu).
std::atomic<uint32_t> g_gemm_debug{0};
std::atomic<uint64_t> g_gemm_debug_wait_ns{2000000000ull};

void set_gemm_debug(uint32_t flags, uint64_t wait_ns) {
    g_gemm_debug_wait_ns.store(wait_ns ? wait_ns : 2000000000ull);
    g_gemm_debug.store(flags);
}

cudaError_t launch_grouped_gemm(const GemmArgs &a, cudaStream_t s) {
    const bool nvf4 = a.kind == 0;
    const bool swiglu = a.epi == EPI_SWIGLU_AMAX;
    if (swiglu && (a.group_axis != NVFP4MOE_GROUP_M || (a.N / 2) % 128 != 0 || !a.amax))
        return cudaErrorInvalidValue;
    if (a.N % 256 != 0) return cudaErrorInvalidValue;
    // the per-group tile table packs the X-tile count of a group into 16 bits
    if (a.a_rows >= (int64_t)MAX_N * 65535) return cudaErrorInvalidValue;
    Params p{};
    p.kind = a.kind;
    p.epi = a.epi;
    p.group_axis = a.group_axis;
    // X = the token-side operand (argument "a"), W = the weights (argument "b")
    p.x_sc = a.a_sc;
    p.w_sc = a.b_sc;
    p.x_ts = a.a_ts;
    p.w_ts = a.b_ts;
    p.x_ts_stride = a.a_ts_stride;
    p.group_off = a.group_off;
    p.G = a.G;
    p.x_rows = a.M;
    p.f_out = swiglu ? a.N / 2 : a.N;
    p.ldc = p.f_out;
    p.w_rows_group = (a.group_axis == NVFP4MOE_GROUP_M) ? a.b_rows_per_group : 0;
    p.wtiles = (int32_t)(swiglu ? p.f_out / 128 : a.N / 256);
    p.c = a.c;
    p.amax = a.amax;
    if (a.hq) {
        if (!swiglu || !nvf4 || !a.hq_sc || !a.h_ts || !a.rq_ws) return cudaErrorInvalidValue;
        p.hq = a.hq;
        p.hq_sc = a.hq_sc;
        p.h_ts = a.h_ts;
        int32_t *w = static_cast<int32_t *>(a.rq_ws);
        const int64_t per = (a.G + 3) / 4 * 4;  // int32 arrays padded to 16 bytes
        p.rq_tiles = w;
        p.rq_cursor = w + per;
        p.rq_queue = w + 2 * per;
        p.rq_ctr = w + 3 * per;
    }
    p.err = device_error_word();
    p.debug = g_gemm_debug.load();
    p.wait_ns = p.debug ? g_gemm_debug_wait_ns.load() : 2000000000ull;
    if (!p.err) return cudaErrorInvalidSymbol;
    // contraction bytes per row and scale chunks per 128-row block
    const int64_t kbytes = nvf4 ? a.a_cols / 2 : a.a_cols;
    p.x_nkc = nvf4 ? a.a_cols / 64 : a.a_cols / 128;
    p.w_nkc = p.x_nkc;
    p.kt_total = (int32_t)(kbytes / 128);
    const int64_t w_rows =
        (a.group_axis == NVFP4MOE_GROUP_M) ? (int64_t)a.G * a.b_rows_per_group : a.N;
    CUtensorMap mw, mx32, mx64, mx96;
    const bool okw = swiglu ? make_map_swiglu_kb(&mw, a.b, a.G, p.f_out, kbytes)
                            : make_map_3d_kb(&mw, a.b, w_rows, kbytes, 128);
    if (!okw || !make_map_3d_kb(&mx32, a.a, a.a_rows, kbytes, 32) ||
        !make_map_3d_kb(&mx64, a.a, a.a_rows, kbytes, 64) || !make_map_3d_kb(&mx96, a.a, a.a_rows, kbytes, 96))
        return cudaErrorInvalidValue;
    int grid = 0;
    cudaError_t e = launch_setup(grid);
    if (e != cudaSuccess) return e;
    if (p.hq)
        grouped_gemm_pair_kernel<true><<<grid, NUM_THREADS, SMEM_ALLOC, s>>>(mw, mx32, mx64, mx96, p);
    else
        grouped_gemm_pair_kernel<false><<<grid, NUM_THREADS, SMEM_ALLOC, s>>>(mw, mx32, mx64, mx96, p);
    return cudaGetLastError();
}

}  // namespace nvfp4moe

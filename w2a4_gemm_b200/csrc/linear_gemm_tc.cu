// linear_gemm_tc.cu -- qift_linear at prefill batch sizes: a fused W2A4 GEMM on the sm_100a
// tensor cores (tcgen05, int8 x int8 -> int32 in tensor memory).
//
// "Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
// Inference", Abstract: 2-bit weights with fixed levels ({+-1,+-3} or {+-1,+-4} times the
// per-channel scale) applied to 4-bit activations.
//
//   y[t][n] = ((float)acc[t][n] * s_w[n]) * s_a[t],  acc = sum_k q[t][k] * L(code[n][k]).
//
// Every mbarrier wait is bounded: a wait that runs out of time sets a shared abort flag and
// the device error word, every role drains what it started, tensor memory is freed and the CTA
// exits.
#include <cudaTypedefs.h>

#include <algorithm>

#include "internal.h"
#include "tc.cuh"

namespace qift {

__device__ int g_qift_error = 0;  // QIFT_ERR_TIMEOUT-style bits, read by qift_device_error()
#ifdef QIFT_CHECK
__device__ int g_qift_check_line = 0;  // bounds-checked build: source line of the first failed check
#endif

// =====================================================================================
// CTA-pair GEMM, persistent.  A cluster of two CTAs on two SMs computes 256-weight-row x
// 256-token tiles with pair MMAs (tcgen05.mma.cta_group::2, M = 256, N = 256): each CTA decodes
// its own 128 weight rows into its own tensor memory and stages only its half of the activation
// tile (128 tokens); the two tensor cores exchange the B halves on chip, which halves the
// activation bytes each SM fetches per multiply-add.  Each cluster walks a list of tiles; the
// TMA ring and the decoders run straight on from one tile into the next, and dedicated epilogue
// warps drain the accumulator into shared memory, release it to the next tile's MMAs and write
// the tile out while those run, so per-tile start-up and write-out are hidden.
//   warp 0          TMA producer of this CTA (4-stage ring: 128 tokens x 256 B + 128 x 64 B codes)
//   warp 1          TMEM owner of this CTA; in rank 0 also the MMA issuer for the pair
//   warps 2..9      decoders: group g (4 warps) fills ring stages g and g + 2
//   warps 10..25    epilogue: four warps per TMEM lane quarter, a quarter of the columns each
// One ring of STAGES slots covers both the shared-memory stages and the tensor-memory A stages,
// so a single commit per K block (`consumed`, arriving in both CTAs) frees both.  Rank 0's
// decoders also wait for the pair's activation halves (both CTAs' loads complete on rank 0's
// `full`), so the decoders' `afull` (eight arrivals: four warps per CTA) is the only barrier the
// MMA issuer waits on inside a tile; the single MMA-issuing thread otherwise paces the tensor
// core with its own instruction latency.
// =====================================================================================
namespace gemm_pair {

constexpr int BMW = 128;                          // weight rows per CTA (pair MMA M = 256)
constexpr int BNT = 256;                          // tokens per pair tile (MMA N)
constexpr int BNH = BNT / 2;                      // tokens of B staged by each CTA
constexpr int BK = 256;                           // K bytes per block: two 128-byte swizzled columns
constexpr int STAGES = 4;                         // shared-memory slots = tensor-memory A stages
constexpr int kGroups = 2;
constexpr int kDecWarps = 4 * kGroups;
constexpr int kEpiWarps = 16;
constexpr int kEpiBase = 2 + kDecWarps;           // first epilogue warp
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = 32 * (kEpiBase + kEpiWarps);
constexpr int ACT_HALF = BNH * 128;               // one 128-byte column of the activation block: 16 KB
constexpr int ACT_BYTES = BNH * BK;               // 32 KB
constexpr int COD_BYTES = BMW * (BK / 16) * 4;    // 8 KB (64-byte rows, 64-byte swizzle)
constexpr int STG_BYTES = 64 * 1024;              // epilogue staging: [columns of a pass][128 rows]
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = STAGES * (ACT_BYTES + COD_BYTES) + STG_BYTES + 1024 + BAR_BYTES + BNT * 4;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;
constexpr uint32_t A_COL = 256;                   // A stage s at A_COL + 64 * s (BK / 4 columns)
static_assert(A_COL + (BK / 4) * STAGES <= TMEM_COLS, "tensor memory");
static_assert((4 * STAGES + 4) * 8 + 8 <= BAR_BYTES, "barrier area");
static_assert(SMEM_BYTES <= 232448, "shared memory");
static_assert(STAGES % kGroups == 0, "decoder group g fills ring stages g, g + kGroups, ...");
static_assert(BK == 256, "the MMA loop issues eight K = 32 steps per block");
static_assert(kEpiThreads >= BNT, "one epilogue thread per token scale");

constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 2 GHz before a wait gives up

// Test hooks (qift_debug.h), per host thread: a shorter wait limit, and a one-shot stall that
// makes the MMA thread wait on a barrier nothing arrives on, so the timeout path runs without
// any fault.
static thread_local long long g_wait_limit = kWaitCycles;
static thread_local bool g_stall_next = false;

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, int* abort, long long limit) {
    if (tc::mbar_wait_bounded(bar, parity, abort, limit)) return true;
    if (!*reinterpret_cast<volatile int*>(abort)) {
        atomicOr(&g_qift_error, 1);
        *reinterpret_cast<volatile int*>(abort) = 1;
    }
    return false;
}

template <typename OutT>
__device__ __forceinline__ void store_one(OutT* p, float v);
template <>
__device__ __forceinline__ void store_one<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_one<__half>(__half* p, float v) { *p = __float2half_rn(v); }


struct Smem {
    uint8_t* act;
    uint8_t* cod;
    uint8_t* stg;
    uint64_t* full;      // [STAGES] rank 0: both CTAs' activation halves landed
    uint64_t* cfull;     // [STAGES] this CTA's codes landed
    uint64_t* afull;     // [STAGES] rank 0: decoded weights of both CTAs in tensor memory
    uint64_t* consumed;  // [STAGES] pair MMAs done with the slot and the A stage (both CTAs)
    uint64_t* accfull;   // the tile's MMAs are complete (both CTAs)
    uint64_t* accfree;   // rank 0: both CTAs' epilogues have read the accumulator
    uint64_t* done;      // every MMA issued has completed (both CTAs)
    uint64_t* never;
    uint32_t* tmem_base;
    int* abort;
    float* sa;           // [BNT] activation scales of the tile being written out
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    Smem s;
    s.act = base;
    s.cod = s.act + STAGES * ACT_BYTES;
    s.stg = s.cod + STAGES * COD_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(s.stg + STG_BYTES);
    s.full = bars;
    s.cfull = s.full + STAGES;
    s.afull = s.cfull + STAGES;
    s.consumed = s.afull + STAGES;
    s.accfull = s.consumed + STAGES;
    s.accfree = s.accfull + 1;
    s.done = s.accfree + 1;
    s.never = s.done + 1;
    s.tmem_base = reinterpret_cast<uint32_t*>(s.never + 1);
    s.abort = reinterpret_cast<int*>(s.tmem_base + 1);
    s.sa = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + BAR_BYTES);
    return s;
}

// One non-blocking probe, then the bounded wait (which records a timeout).
__device__ __forceinline__ bool wait_fast(uint64_t* bar, uint32_t parity, int* abort, long long limit) {
    return tc::mbar_try_wait(bar, parity) || wait_or_abort(bar, parity, abort, limit);
}

// int32 -> fp32 without the conversion pipe: exact for |v| < 2^22 (|acc| <= 4 * 7 * n_in <= 2^20
// here), since 1.5 * 2^23 + v is then an fp32 integer and the subtraction is exact.
__device__ __forceinline__ float i2f_exact(int v) {
    return __fsub_rn(__int_as_float(0x4B400000 + v), 12582912.0f);
}

// The accumulator word as acc: W4 accumulates 16 x acc (an exact multiple of 16).
template <bool W4>
__device__ __forceinline__ int unscale(uint32_t a) {
    return W4 ? ((int)a >> 4) : (int)a;
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, %0;" ::"r"(kEpiThreads) : "memory"); }

struct Tile {
    int n0;  // this CTA's first weight row
    int t0;  // the pair tile's first token
};

__device__ __forceinline__ Tile tile_of(int i, int pairs_x, uint32_t rank) {
    const int tile = (int)(blockIdx.x >> 1) + i * (int)(gridDim.x >> 1);
    Tile t;
    t.n0 = (tile % pairs_x) * (2 * BMW) + (int)rank * BMW;
    t.t0 = (tile / pairs_x) * BNT;
    return t;
}

// W4: 4-bit weights (QIFT_SET_INT4, eight two's-complement nibbles per word, byte j = inputs j
// (low) and j + 4 (high)).  A ring stage then covers 128 inputs -- the same 64 code bytes per
// row, one 128-byte activation column, four MMAs -- and the decoders turn a word into two int8x4
// registers with a shift and two masks: 16 x the levels of inputs 0..3 and 4..7.  The
// accumulator holds 16 x acc exactly (|16 acc| <= 16 * 49 * 32768 < 2^31); the epilogue shifts it
// back before the scales.
template <typename OutT, bool W4>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    w2a4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_c,
                          const float* __restrict__ s_a, const float* __restrict__ s_w, uint32_t lut, int T, int N,
                          int K, OutT* __restrict__ y, long long wait_limit, int stall) {
    extern __shared__ uint8_t smem_raw[];
    const Smem sm = carve(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = tc::cluster_ctarank();
    const int pairs_x = (N + 2 * BMW - 1) / (2 * BMW);
    const int tiles = pairs_x * ((T + BNT - 1) / BNT);
    const int cl = (int)(blockIdx.x >> 1), clusters = (int)(gridDim.x >> 1);
    const int my_tiles = cl < tiles ? (tiles - 1 - cl) / clusters + 1 : 0;
    constexpr int BKI = W4 ? 128 : BK;    // inputs per ring stage
    const int num_kb = (K + BKI - 1) / BKI;
    const int total = my_tiles * num_kb;  // K blocks this cluster streams through the ring

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(&sm.full[s], 1);
            tc::mbar_init(&sm.cfull[s], 1);
            tc::mbar_init(&sm.afull[s], 8);  // four decoder warps in each CTA
            tc::mbar_init(&sm.consumed[s], 1);
        }
        tc::mbar_init(sm.accfull, 1);
        tc::mbar_init(sm.accfree, 2 * kEpiWarps);
        tc::mbar_init(sm.done, 1);
        tc::mbar_init(sm.never, 1);
        *sm.abort = 0;
        tc::fence_mbar_init();
        tc::prefetch_tensormap(&tmap_x);
        tc::prefetch_tensormap(&tmap_c);
    }
    if (warp == 1) {
        tc::tmem_alloc_pair(sm.tmem_base, TMEM_COLS);
        tc::tmem_relinquish_pair();
    }
    tc::tc_fence_before();
    tc::cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrive or copy
    tc::tc_fence_after();
    // Programmatic dependent launch: the next kernel on the stream may be scheduled now; it
    // waits for this grid's completion before it reads what this grid writes.
    griddep_launch_dependents();
    const uint32_t tmem = *sm.tmem_base;
    volatile int* abort_v = reinterpret_cast<volatile int*>(sm.abort);

    if (warp == 0) {
        if (lane == 0) {  // ------------------------------------------------ TMA producer
            const uint32_t full0 = tc::cluster_addr(sm.full, 0);
            // The codes of the first ring stages (weights: nothing a previous kernel on the stream
            // writes) are requested before the wait for that kernel; the activations after it.
            const int pre = total < STAGES ? total : STAGES;
            for (int gp = 0; gp < pre; ++gp) {
                const int ip = gp / num_kb, kbp = gp - ip * num_kb;
                const Tile tp = tile_of(ip, pairs_x, rank);
                const bool cod = tp.n0 < N;
                tc::mbar_arrive_expect_tx(&sm.cfull[gp], cod ? COD_BYTES : 0);
                if (cod && QIFT_CK(kbp * 16 * (W4 ? 8 : 16) < K && tp.n0 >= 0 && tp.n0 < N))
                    tc::tma_load_2d(sm.cod + gp * COD_BYTES, &tmap_c, &sm.cfull[gp], kbp * 16, tp.n0);
            }
            griddep_wait();
            int g = 0;
            bool ok = true;
            for (int i = 0; ok && i < my_tiles; ++i) {
                const Tile tl = tile_of(i, pairs_x, rank);
                const int tb = tl.t0 + (int)rank * BNH;  // this CTA's B half
                // A box lying wholly outside the matrix is not fetched: its rows/tokens are never
                // stored.  Rank 0 expects the activation bytes of both CTAs; the second 128-byte
                // column of the last block is neither fetched nor multiplied when wholly past K.
                const bool has_act = tb < T, has_cod = tl.n0 < N;
                const uint32_t act_ctas = tl.t0 + BNH < T ? 2u : 1u;
                for (int kb = 0; kb < num_kb; ++kb, ++g) {
                    const uint32_t s = g & (STAGES - 1), ph = (g / STAGES) & 1;
                    if (g >= STAGES && !wait_fast(&sm.consumed[s], ph ^ 1, sm.abort, wait_limit)) {
                        ok = false;
                        break;
                    }
                    const bool second = !W4 && kb * BK + 128 < K;
                    if (rank == 0) tc::mbar_arrive_expect_tx(&sm.full[s], act_ctas * (second ? 2u : 1u) * ACT_HALF);
                    if (g >= pre) tc::mbar_arrive_expect_tx(&sm.cfull[s], has_cod ? COD_BYTES : 0);
                    // tensor-map coordinates: x a 16-byte multiple inside the row, y inside the matrix
                    if (has_act && QIFT_CK((kb * BKI) % 16 == 0 && kb * BKI < K && tb >= 0 && tb < T)) {
                        tc::tma_load_2d_pair(sm.act + s * ACT_BYTES, &tmap_x, full0 + 8 * s, kb * BKI, tb);
                        if (second)
                            tc::tma_load_2d_pair(sm.act + s * ACT_BYTES + ACT_HALF, &tmap_x, full0 + 8 * s,
                                                 kb * BK + 128, tb);
                    }
                    if (g >= pre && has_cod && QIFT_CK(kb * 16 * (W4 ? 8 : 16) < K && tl.n0 >= 0 && tl.n0 < N))
                        tc::tma_load_2d(sm.cod + s * COD_BYTES, &tmap_c, &sm.cfull[s], kb * 16, tl.n0);
                }
            }
            if (*abort_v) {
                // Drain: the copies this thread started land before the CTA exits.  Rank 0 sees
                // both halves of the activations on its own barriers; each CTA sees its codes.
                int zero = 0;
                for (int q = g > STAGES ? g - STAGES : 0; q < g; ++q) {
                    const uint32_t s = q & (STAGES - 1), ph = (q / STAGES) & 1;
                    if (rank == 0) tc::mbar_wait_bounded(&sm.full[s], ph, &zero, wait_limit);
                    tc::mbar_wait_bounded(&sm.cfull[s], ph, &zero, wait_limit);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {  // -------------------------------------- pair MMA issuer
            constexpr uint32_t idesc = tc::idesc_i8(2 * BMW, BNT);
            const uint64_t desc0 = tc::smem_desc_sw128(tc::smem_u32(sm.act));
            if (stall) wait_or_abort(sm.never, 0, sm.abort, wait_limit);  // test hook
            // The wait for block g + 1 sits between the MMAs of block g, so it overlaps the MMAs
            // already queued; a tile's first MMA also waits until the epilogue has drained the
            // previous tile's accumulator.
            bool ok = !*abort_v && (total == 0 || wait_fast(&sm.afull[0], 0, sm.abort, wait_limit));
            int g = 0;
            for (int i = 0; ok && i < my_tiles; ++i) {
                if (i > 0 && !wait_fast(sm.accfree, (i - 1) & 1, sm.abort, wait_limit)) break;
                for (int kb = 0; kb < num_kb; ++kb, ++g) {
                    const uint32_t s = g & (STAGES - 1);
                    tc::tc_fence_after();
                    const uint64_t d = desc0 + (uint64_t)((s * ACT_BYTES) >> 4);
                    const uint64_t d2 = d + (uint64_t)(ACT_HALF >> 4);
                    const uint32_t a = tmem + A_COL + (BK / 4) * s;
                    // the A stage's columns and the accumulator's lie inside the allocation
                    if (!QIFT_CK(A_COL + (BK / 4) * (s + 1) <= TMEM_COLS && ACC_COL + BNT <= A_COL)) {
                        ok = false;
                        break;
                    }
                    tc::mma_i8_ts_pair(tmem + ACC_COL, a, d, idesc, kb != 0 ? 1u : 0u);
#pragma unroll
                    for (int k = 1; k < 4; ++k) tc::mma_i8_ts_pair(tmem + ACC_COL, a + 8 * k, d + 2 * k, idesc, 1u);
                    if (g + 1 < total)
                        ok = wait_fast(&sm.afull[(g + 1) & (STAGES - 1)], ((g + 1) / STAGES) & 1, sm.abort, wait_limit);
                    if (!W4 && kb * BK + 128 < K) {
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            tc::mma_i8_ts_pair(tmem + ACC_COL, a + 32 + 8 * k, d2 + 2 * k, idesc, 1u);
                    }
                    tc::mma_commit_pair(&sm.consumed[s], 0x3);
                    if (!ok) break;
                }
                if (!ok) break;
                tc::mma_commit_pair(sm.accfull, 0x3);
            }
            if (*abort_v) {  // the peer must not store its tiles either
                tc::st_cluster_u32(sm.abort, 1, 1u);
                asm volatile("fence.acq_rel.cluster;" ::: "memory");
            }
            tc::mma_commit_pair(sm.done, 0x3);  // also after an abort, so both CTAs see the MMAs drained
        }
    } else if (warp < kEpiBase) {
        const int grp = (warp - 2) >> 2;  // fills ring stages grp, grp + kGroups, ...
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int swz = (r >> 1) & 3;  // 64-byte TMA swizzle: chunk c of row r sits at c ^ swz
        for (int g = grp; g < total; g += kGroups) {  // ---------------------- decoders
            const uint32_t s = g & (STAGES - 1), ph = (g / STAGES) & 1;
            bool ok = wait_fast(&sm.cfull[s], ph, sm.abort, wait_limit) &&
                      (g < STAGES || wait_fast(&sm.consumed[s], ph ^ 1, sm.abort, wait_limit)) &&
                      (rank != 0 || wait_fast(&sm.full[s], ph, sm.abort, wait_limit));
            if (!__all_sync(0xffffffffu, ok)) break;
            const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + A_COL + (BK / 4) * s;
            if (!QIFT_CK(quarter == (warp & 3) && A_COL + (BK / 4) * (s + 1) <= TMEM_COLS)) break;
            const uint8_t* crow = sm.cod + s * COD_BYTES + r * 64;
            tc::tc_fence_after();
            if constexpr (W4) {  // 128 inputs (sixteen code words) in one tensor-memory store
                uint32_t v[32];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const uint4 w = *reinterpret_cast<const uint4*>(crow + 16 * (h ^ swz));
                    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        v[8 * h + 2 * c] = (words[c] << 4) & 0xF0F0F0F0u;
                        v[8 * h + 2 * c + 1] = words[c] & 0xF0F0F0F0u;
                    }
                }
                tc::tmem_st_32x32b_x32(taddr, v);
            } else {
#pragma unroll
                for (int h = 0; h < 2; ++h) {  // 128 K bytes (eight code words) per tensor-memory store
                    const uint4 w0 = *reinterpret_cast<const uint4*>(crow + 16 * ((2 * h) ^ swz));
                    const uint4 w1 = *reinterpret_cast<const uint4*>(crow + 16 * ((2 * h + 1) ^ swz));
                    const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                    uint32_t v[32];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint32_t d[4];
                        decode_word_natural(words[c], lut, d);
                        v[4 * c] = d[0];
                        v[4 * c + 1] = d[1];
                        v[4 * c + 2] = d[2];
                        v[4 * c + 3] = d[3];
                    }
                    tc::tmem_st_32x32b_x32(taddr + 32 * h, v);
                }
            }
            tc::tmem_st_wait();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive_cluster_relaxed(&sm.afull[s], 0);
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        // Warp (quarter, column group): 32 weight rows, a quarter of each pass's columns.  Per tile:
        // drain the accumulator (scaled, converted) into the staging buffer -- fp16 as packed
        // token pairs [token/2][row][2], fp32 as [token][row] in two passes of 128 columns --
        // release the accumulator after the last pass's reads, then write 16-byte pieces along n.
        // The drain stalls the next tile's MMAs, so it keeps off the conversion pipe (exact
        // integer-to-float by magic number, one packed two-value fp16 conversion).  Every
        // epilogue warp runs every named barrier of every tile, also after an abort (`alive`
        // only skips the work).
        constexpr int CPP = STG_BYTES / (BMW * (int)sizeof(OutT));  // columns per pass: 256 / 128
        constexpr int PASSES = BNT / CPP;
        constexpr int EPP = 16 / sizeof(OutT);                      // elements per 16-byte piece
        constexpr int PPR = BMW / EPP;                              // pieces per token row
        constexpr int CPW = CPP / 4;                                // columns per warp per pass
        const int et = threadIdx.x - 32 * kEpiBase;                 // 0 .. kEpiThreads - 1
        const int quarter = warp & 3, cgrp = (warp - kEpiBase) >> 2;
        const int r = quarter * 32 + lane;
        OutT* stg = reinterpret_cast<OutT*>(sm.stg);
        const bool vec_ok = ((int64_t)N * sizeof(OutT)) % 16 == 0;
        bool alive = true;
        griddep_wait();  // the activation scales, and y, may belong to the previous kernel
        for (int i = 0; i < my_tiles; ++i) {
            const Tile tl = tile_of(i, pairs_x, rank);
            if (et < BNT) sm.sa[et] = tl.t0 + et < T ? s_a[tl.t0 + et] : 0.0f;
            const float sw = tl.n0 + r < N ? s_w[tl.n0 + r] : 0.0f;
            epi_bar();  // token scales in place
            bool ok = alive && wait_fast(sm.accfull, i & 1, sm.abort, wait_limit) && !*abort_v;
            alive = __all_sync(0xffffffffu, ok);
            for (int p = 0; p < PASSES; ++p) {
                if (alive) {
                    tc::tc_fence_after();
#pragma unroll 1
                    for (int cc = 0; cc < CPW / 32; ++cc) {
                        const int cl0 = cgrp * CPW + cc * 32;  // column within the pass
                        const int c0 = p * CPP + cl0;         // column within the tile
                        uint32_t acc[32];
                        if (!QIFT_CK(c0 + 32 <= BNT && quarter == (warp & 3))) continue;
                        tc::tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + ACC_COL + c0, acc);
                        tc::tmem_ld_wait();
                        if constexpr (sizeof(OutT) == 2) {
                            uint32_t* stg32 = reinterpret_cast<uint32_t*>(sm.stg);
#pragma unroll
                            for (int j = 0; j < 32; j += 2) {
                                const float v0 = __fmul_rn(__fmul_rn(i2f_exact(unscale<W4>(acc[j])), sw), sm.sa[c0 + j]);
                                const float v1 =
                                    __fmul_rn(__fmul_rn(i2f_exact(unscale<W4>(acc[j + 1])), sw), sm.sa[c0 + j + 1]);
                                const __half2 h = __floats2half2_rn(v0, v1);  // .x = token c0 + j
                                stg32[((cl0 + j) / 2) * BMW + r] = *reinterpret_cast<const uint32_t*>(&h);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                const float v = __fmul_rn(__fmul_rn(i2f_exact(unscale<W4>(acc[j])), sw), sm.sa[c0 + j]);
                                store_one<OutT>(stg + (cl0 + j) * BMW + r, v);
                            }
                        }
                    }
                    if (p == PASSES - 1) {  // every column of the accumulator has been read
                        tc::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive_cluster_relaxed(sm.accfree, 0);
                    }
                }
                epi_bar();  // staging complete
                if (alive) {
                    if constexpr (sizeof(OutT) == 2) {
                        // Piece (token pair jp, 8 rows): 32 staged bytes hold both tokens' halves,
                        // split with byte permutes into one 16-byte row piece per token.
                        const uint32_t* stg32 = reinterpret_cast<const uint32_t*>(sm.stg);
#pragma unroll 2
                        for (int q = et; q < (CPP / 2) * PPR; q += kEpiThreads) {
                            const int jp = q / PPR, sub = q % PPR;
                            const int t = tl.t0 + p * CPP + 2 * jp, nn = tl.n0 + sub * EPP;
                            if (t < T) {
                                const uint4 u0 = *reinterpret_cast<const uint4*>(stg32 + jp * BMW + sub * 8);
                                const uint4 u1 = *reinterpret_cast<const uint4*>(stg32 + jp * BMW + sub * 8 + 4);
                                const uint32_t u[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                                uint32_t lo[4], hi[4];
#pragma unroll
                                for (int k = 0; k < 4; ++k) {
                                    lo[k] = __byte_perm(u[2 * k], u[2 * k + 1], 0x5410);
                                    hi[k] = __byte_perm(u[2 * k], u[2 * k + 1], 0x7632);
                                }
                                for (int tt = 0; tt < 2 && t + tt < T; ++tt) {
                                    const uint32_t* w = tt ? hi : lo;
                                    OutT* dst = y + (int64_t)(t + tt) * N + nn;
                                    const int64_t off = (int64_t)(t + tt) * N + nn;
                                    if (vec_ok && nn + EPP <= N) {
                                        if (QIFT_CK_RANGE(off, EPP, (int64_t)T * N))
                                            *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
                                    } else {
                                        const __half* hv = reinterpret_cast<const __half*>(w);
                                        for (int e = 0; e < EPP; ++e)
                                            if (nn + e < N && QIFT_CK_RANGE(off + e, 1, (int64_t)T * N)) dst[e] = hv[e];
                                    }
                                }
                            }
                        }
                    } else {
#pragma unroll 2
                        for (int q = et; q < CPP * PPR; q += kEpiThreads) {
                            const int j = q / PPR, sub = q % PPR;
                            const int t = tl.t0 + p * CPP + j, nn = tl.n0 + sub * EPP;
                            if (t < T) {
                                OutT* dst = y + (int64_t)t * N + nn;
                                const OutT* src = stg + j * BMW + sub * EPP;
                                const int64_t off = (int64_t)t * N + nn;
                                if (vec_ok && nn + EPP <= N) {
                                    if (QIFT_CK_RANGE(off, EPP, (int64_t)T * N))
                                        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
                                } else {
                                    for (int e = 0; e < EPP; ++e)
                                        if (nn + e < N && QIFT_CK_RANGE(off + e, 1, (int64_t)T * N)) dst[e] = src[e];
                                }
                            }
                        }
                    }
                }
                epi_bar();  // staging free again
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        // The pair MMAs read this CTA's shared and tensor memory: wait for the last of them.
        int zero = 0;
        tc::mbar_wait_bounded(sm.done, 0, &zero, wait_limit);
        __syncwarp();
    }
    // Neither CTA leaves (or frees its tensor memory) while the other may still read its
    // memory or arrive on its barriers.
    tc::cluster_sync();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

// Largest number of co-resident pair clusters of this kernel (cached per device and type).
template <typename OutT, bool W4>
static int max_clusters() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (!cached[dev]) {
        cudaLaunchConfig_t cfg = {};
        int sms = 148;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cfg.gridDim = dim3((unsigned)(sms & ~1));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = SMEM_BYTES;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, w2a4_gemm_pair_kernel<OutT, W4>, &cfg) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = sms / 2;
        }
        cached[dev] = n;
    }
    return cached[dev];
}

template <typename OutT, bool W4>
static cudaError_t launch_t(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, uint32_t lut,
                            int64_t T, int64_t N, int64_t K, OutT* y, cudaStream_t s) {
    constexpr int CPW = W4 ? 8 : 16;  // codes per 32-bit word
    auto encode = tensor_map_encoder();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap mx, mc;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)T};
        const cuuint64_t strides[1] = {(cuuint64_t)K};
        const cuuint32_t box[2] = {128, BNH};
        const cuuint32_t es[2] = {1, 1};
        if (encode(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(q), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)(K / CPW), (cuuint64_t)N};
        const cuuint64_t strides[1] = {(cuuint64_t)(K / CPW) * 4};
        const cuuint32_t box[2] = {16, BMW};  // 64 code bytes per row and stage
        const cuuint32_t es[2] = {1, 1};
        if (encode(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(codes), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const cudaError_t e = ensure_smem(w2a4_gemm_pair_kernel<OutT, W4>, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int64_t tiles = ((N + 2 * BMW - 1) / (2 * BMW)) * ((T + BNT - 1) / BNT);
    if (tiles > 0x3fffffff) return cudaErrorInvalidValue;
    const int clusters = (int)std::min<int64_t>(tiles, std::max(1, max_clusters<OutT, W4>()));
    const int stall = g_stall_next ? 1 : 0;
    g_stall_next = false;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * clusters));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, w2a4_gemm_pair_kernel<OutT, W4>, mx, mc, s_a, s_w, lut, (int)T, (int)N, (int)K, y,
                              g_wait_limit, stall);
}

}  // namespace gemm_pair

cudaError_t launch_linear_gemm_pair(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, int set,
                                    int64_t T, int64_t N, int64_t K, void* y, bool f16, cudaStream_t s) {
    if (T == 0 || N == 0) return cudaSuccess;
    const uint32_t lut = level_lut(set);
    if (set == kSetInt4) {
        if (f16) return gemm_pair::launch_t<__half, true>(q, s_a, codes, s_w, lut, T, N, K, static_cast<__half*>(y), s);
        return gemm_pair::launch_t<float, true>(q, s_a, codes, s_w, lut, T, N, K, static_cast<float*>(y), s);
    }
    if (f16) return gemm_pair::launch_t<__half, false>(q, s_a, codes, s_w, lut, T, N, K, static_cast<__half*>(y), s);
    return gemm_pair::launch_t<float, false>(q, s_a, codes, s_w, lut, T, N, K, static_cast<float*>(y), s);
}

bool linear_gemm_supported(int64_t T, int64_t N, int64_t K) {
    // TMA needs 16-byte row strides for the code matrix (K % 64), and the kernel indexes tokens
    // and rows in 32-bit integers.
    return K % 64 == 0 && T <= (int64_t)0x7fffff00 && N <= (int64_t)0x7fffff00;
}

void debug_set_gemm_wait_limit(long long cycles) {
    gemm_pair::g_wait_limit = cycles > 0 ? cycles : gemm_pair::kWaitCycles;
}
void debug_stall_next_gemm() { gemm_pair::g_stall_next = true; }

cudaError_t read_and_clear_check_line(int* line) {
    *line = 0;
#ifdef QIFT_CHECK
    cudaError_t e = cudaMemcpyFromSymbol(line, g_qift_check_line, sizeof(int));
    if (e != cudaSuccess || *line == 0) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_qift_check_line, &zero, sizeof(int));
#else
    return cudaSuccess;
#endif
}

cudaError_t read_and_clear_device_error(int* word) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_qift_error, sizeof(int));
    if (e != cudaSuccess) return e;
    if (v != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_qift_error, &zero, sizeof(int));
    }
    *word = v;
    return e;
}

}  // namespace qift

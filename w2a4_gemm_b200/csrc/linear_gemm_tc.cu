// linear_gemm_tc.cu -- qift_linear at prefill batch sizes: a fused W2A4 GEMM on the sm_100a
// tensor cores (tcgen05, int8 x int8 -> int32 in tensor memory).
//
// "Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
// Inference", Abstract: 2-bit weights with fixed levels ({+-1,+-3} or {+-1,+-4} times the
// per-channel scale) applied to 4-bit activations.
//
//   y[t][n] = ((float)acc[t][n] * s_w[n]) * s_a[t],  acc = sum_k q[t][k] * L(code[n][k]).
//
// One CTA computes a 128-token x 256-output tile, walking K in 128-byte blocks.  Two rings of
// shared memory: STAGES slots for what TMA brings (the int8 activation tile and the packed
// code tile), deep enough to cover the L2/HBM round trip, and BSTAGES slots for the decoded
// int8 weight tile, which only has to run ahead of the tensor core by one block:
//   warp 0      TMA producer: the int8 activation tile (128 x 128 B, 128-byte swizzle) and the
//               packed code tile (256 rows x 8 words) land on one mbarrier per stage;
//   warps 2..9  decoders (one weight row per thread): expand 2-bit codes to int8 weights in
//               registers (byte permutes against the level table) and write them in the tensor
//               core's 128-byte swizzled K-major layout; then, after the last block, the
//               epilogue: tcgen05.ld of the int32 accumulators, the fp32 scale product, stores;
//   warp 1      allocates 256 TMEM columns and one elected thread issues tcgen05.mma
//               (kind::i8, M=128, N=256, K=32 per instruction, 4 per block), committing each
//               stage back to the producer.
// Every mbarrier wait is bounded: a wait that runs out of time sets a shared abort flag and
// the device error word, every role drains what it started, TMEM is freed and the CTA exits.
#include <cudaTypedefs.h>

#include <algorithm>

#include "internal.h"
#include "tc.cuh"

namespace qift {

__device__ int g_qift_error = 0;  // QIFT_ERR_TIMEOUT-style bits, read by qift_device_error()

namespace gemm {

constexpr int BM = 128;          // tokens per tile (MMA M, TMEM lanes)
constexpr int BN = 256;          // output features per tile (MMA N, TMEM columns)
constexpr int BK = 128;          // K bytes per stage (one 128-byte swizzle row)
constexpr int STAGES = 5;        // TMA ring (activations + codes)
constexpr int BSTAGES = 3;       // decoded-weight ring
constexpr int kDecWarps = 8;     // one weight row of the tile per decoder thread
constexpr int kThreads = 64 + 32 * kDecWarps;
constexpr int A_BYTES = BM * BK;             // 16 KB
constexpr int B_BYTES = BN * BK;             // 32 KB
constexpr int C_BYTES = BN * (BK / 16) * 4;  // 8 KB of packed codes
constexpr int SMEM_BYTES = STAGES * (A_BYTES + C_BYTES) + BSTAGES * B_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t TMEM_COLS = 256;
constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 2 GHz before a wait gives up

// Test hooks (qift_debug.h): a shorter wait limit, and a one-shot stall that makes the MMA
// thread wait on a barrier nothing arrives on, so the timeout path runs without any fault.
static long long g_wait_limit = kWaitCycles;
static bool g_stall_next = false;

struct Smem {
    uint8_t* a;
    uint8_t* b;
    uint8_t* c;
    uint64_t* full;     // [STAGES]  TMA landed
    uint64_t* empty;    // [STAGES]  MMA done with the slot
    uint64_t* decoded;  // [BSTAGES] decoded weights written
    uint64_t* bempty;   // [BSTAGES] MMA done with the decoded weights
    uint64_t* accum;
    uint64_t* never;
    uint32_t* tmem_base;
    int* abort;
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    Smem s;
    s.a = base;
    s.b = s.a + STAGES * A_BYTES;
    s.c = s.b + BSTAGES * B_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(s.c + STAGES * C_BYTES);
    s.full = bars;
    s.empty = bars + STAGES;
    s.decoded = bars + 2 * STAGES;
    s.bempty = bars + 2 * STAGES + BSTAGES;
    s.accum = bars + 2 * STAGES + 2 * BSTAGES;
    s.never = s.accum + 1;
    s.tmem_base = reinterpret_cast<uint32_t*>(s.never + 1);
    s.abort = reinterpret_cast<int*>(s.tmem_base + 1);
    return s;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, int* abort, long long limit) {
    if (tc::mbar_wait_bounded(bar, parity, abort, limit)) return true;
    if (!*reinterpret_cast<volatile int*>(abort)) {
        atomicOr(&g_qift_error, 1);
        *reinterpret_cast<volatile int*>(abort) = 1;
    }
    return false;
}

template <typename OutT>
__device__ __forceinline__ void store_row16(OutT* y, int64_t row, int64_t n0, int64_t N, const float* v);

template <>
__device__ __forceinline__ void store_row16<__half>(__half* y, int64_t row, int64_t n0, int64_t N, const float* v) {
    __half* p = y + row * N + n0;
    if ((N & 7) == 0 && n0 + 16 <= N) {
        uint4 t0, t1;
        __half2* h0 = reinterpret_cast<__half2*>(&t0);
        __half2* h1 = reinterpret_cast<__half2*>(&t1);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            h0[j] = __floats2half2_rn(v[2 * j], v[2 * j + 1]);
            h1[j] = __floats2half2_rn(v[8 + 2 * j], v[8 + 2 * j + 1]);
        }
        reinterpret_cast<uint4*>(p)[0] = t0;
        reinterpret_cast<uint4*>(p)[1] = t1;
    } else {
        for (int j = 0; j < 16; ++j)
            if (n0 + j < N) p[j] = __float2half_rn(v[j]);
    }
}

template <>
__device__ __forceinline__ void store_row16<float>(float* y, int64_t row, int64_t n0, int64_t N, const float* v) {
    float* p = y + row * N + n0;
    if ((N & 3) == 0 && n0 + 16 <= N) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            reinterpret_cast<float4*>(p)[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    } else {
        for (int j = 0; j < 16; ++j)
            if (n0 + j < N) p[j] = v[j];
    }
}

template <typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
    w2a4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_c,
                     const float* __restrict__ s_a, const float* __restrict__ s_w, uint32_t lut, int T, int N,
                     int K, OutT* __restrict__ y, long long wait_limit, int stall) {
    extern __shared__ uint8_t smem_raw[];
    const Smem sm = carve(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BN;
    const int m0 = blockIdx.y * BM;
    const int num_kb = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(&sm.full[s], 1);
            tc::mbar_init(&sm.empty[s], 1);
        }
        for (int s = 0; s < BSTAGES; ++s) {
            tc::mbar_init(&sm.decoded[s], kDecWarps);  // one arrive per decoder warp
            tc::mbar_init(&sm.bempty[s], 1);
        }
        tc::mbar_init(sm.accum, 1);
        tc::mbar_init(sm.never, 1);
        *sm.abort = 0;
        tc::fence_mbar_init();
        tc::prefetch_tensormap(&tmap_a);
        tc::prefetch_tensormap(&tmap_c);
    }
    if (warp == 1) {
        tc::tmem_alloc(sm.tmem_base, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_d = *sm.tmem_base;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int kb = 0; kb < num_kb; ++kb) {
                const int s = kb % STAGES;
                const uint32_t round = kb / STAGES;
                if (!wait_or_abort(&sm.empty[s], (round & 1) ^ 1, sm.abort, wait_limit)) break;
                tc::mbar_arrive_expect_tx(&sm.full[s], A_BYTES + C_BYTES);
                tc::tma_load_2d(sm.a + s * A_BYTES, &tmap_a, &sm.full[s], kb * BK, m0);
                tc::tma_load_2d(sm.c + s * C_BYTES, &tmap_c, &sm.full[s], kb * (BK / 16), n0);
                ++issued;
            }
            if (*reinterpret_cast<volatile int*>(sm.abort)) {
                // Drain: let every copy this thread started land before the CTA exits.
                int zero = 0;
                for (int kb = issued > STAGES ? issued - STAGES : 0; kb < issued; ++kb)
                    tc::mbar_wait_bounded(&sm.full[kb % STAGES], (kb / STAGES) & 1, &zero, wait_limit);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_i8(BM, BN);
            if (stall) wait_or_abort(sm.never, 0, sm.abort, wait_limit);  // test hook: always times out
            for (int kb = 0; kb < num_kb && !*reinterpret_cast<volatile int*>(sm.abort); ++kb) {
                const int s = kb % STAGES, sb = kb % BSTAGES;
                if (!wait_or_abort(&sm.full[s], (kb / STAGES) & 1, sm.abort, wait_limit)) break;
                if (!wait_or_abort(&sm.decoded[sb], (kb / BSTAGES) & 1, sm.abort, wait_limit)) break;
                tc::tc_fence_after();
                const uint32_t a_addr = tc::smem_u32(sm.a + s * A_BYTES);
                const uint32_t b_addr = tc::smem_u32(sm.b + sb * B_BYTES);
#pragma unroll
                for (int k = 0; k < BK / 32; ++k) {
                    tc::mma_i8_ss(tmem_d, tc::smem_desc_sw128(a_addr + 32 * k), tc::smem_desc_sw128(b_addr + 32 * k),
                                  idesc, (kb > 0 || k > 0) ? 1u : 0u);
                }
                tc::mma_commit(&sm.empty[s]);
                tc::mma_commit(&sm.bempty[sb]);
            }
            tc::mma_commit(sm.accum);  // also issued after an abort, so TMEM is idle before it is freed
        }
    } else {
        // ---------------------------------------------------------------- decoders
        const int r = threadIdx.x - 64;  // 0..255: this thread's row of the weight tile
        // Rows r and r+4 of a quarter-warp would hit the same banks reading 32-byte code rows;
        // every other group of four rows reads its second 16 bytes first.
        const int first = (r >> 2) & 1;
        for (int kb = 0; kb < num_kb; ++kb) {
            const int s = kb % STAGES, sb = kb % BSTAGES;
            bool ok = wait_or_abort(&sm.full[s], (kb / STAGES) & 1, sm.abort, wait_limit) &&
                      wait_or_abort(&sm.bempty[sb], ((kb / BSTAGES) & 1) ^ 1, sm.abort, wait_limit);
            if (!__all_sync(0xffffffffu, ok)) break;  // the whole warp leaves together (it syncs below)
            const uint8_t* crow = sm.c + s * C_BYTES + r * 32;
            const uint4 wa = *reinterpret_cast<const uint4*>(crow + 16 * first);
            const uint4 wb = *reinterpret_cast<const uint4*>(crow + 16 * (first ^ 1));
            const uint4 w0 = first ? wb : wa, w1 = first ? wa : wb;
            const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            uint8_t* brow = sm.b + sb * B_BYTES + r * BK;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t v[4];
                decode_word_natural(words[c], lut, v);
                *reinterpret_cast<uint4*>(brow + ((c ^ (r & 7)) << 4)) = make_uint4(v[0], v[1], v[2], v[3]);
            }
            tc::fence_proxy_async_smem();  // this lane's generic writes -> async proxy
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.decoded[sb]);
        }
        // ---------------------------------------------------------------- epilogue
        bool ok = wait_or_abort(sm.accum, 0, sm.abort, wait_limit) && !*reinterpret_cast<volatile int*>(sm.abort);
        ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld is warp-collective: decide per warp
        if (ok) {
            tc::tc_fence_after();
            const int quarter = warp & 3;             // TMEM lanes 32*quarter .. +31
            const int half = (warp - 2) >> 2;         // warps 2..5: columns 0..127, 6..9: 128..255
            const int row = m0 + quarter * 32 + lane;  // token
            const float sa = row < T ? s_a[row] : 0.0f;
#pragma unroll 1
            for (int cc = half * (BN / 32); cc < (half + 1) * (BN / 32); ++cc) {
                uint32_t acc[16];
                tc::tmem_ld_32x32b_x16(tmem_d + ((uint32_t)(quarter * 32) << 16) + cc * 16, acc);
                tc::tmem_ld_wait();
                const int nb = n0 + cc * 16;
                if (row < T && nb < N) {
                    float v[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float sw = (nb + j < N) ? s_w[nb + j] : 0.0f;
                        v[j] = __fmul_rn(__fmul_rn((float)(int)acc[j], sw), sa);
                    }
                    store_row16<OutT>(y, row, nb, N, v);
                }
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        // Every MMA this CTA issued has been committed to sm.accum; make sure they are done.
        __syncwarp();
        int zero = 0;
        tc::mbar_wait_bounded(sm.accum, 0, &zero, wait_limit);
        __syncwarp();
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_d, TMEM_COLS);
    }
}

// ---------------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() { return tensor_map_encoder(); }

template <typename OutT>
static cudaError_t launch_t(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, uint32_t lut,
                            int64_t T, int64_t N, int64_t K, OutT* y, cudaStream_t s) {
    auto encode = get_encode();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap ma, mc;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)T};
        const cuuint64_t strides[1] = {(cuuint64_t)K};
        const cuuint32_t box[2] = {BK, BM};
        const cuuint32_t es[2] = {1, 1};
        if (encode(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(q), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)(K / 16), (cuuint64_t)N};
        const cuuint64_t strides[1] = {(cuuint64_t)(K / 16) * 4};
        const cuuint32_t box[2] = {BK / 16, BN};
        const cuuint32_t es[2] = {1, 1};
        if (encode(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(codes), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const cudaError_t e = ensure_smem(w2a4_gemm_kernel<OutT>, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((N + BN - 1) / BN), (unsigned)((T + BM - 1) / BM));
    const int stall = g_stall_next ? 1 : 0;
    g_stall_next = false;
    w2a4_gemm_kernel<OutT><<<grid, kThreads, SMEM_BYTES, s>>>(ma, mc, s_a, s_w, lut, (int)T, (int)N, (int)K, y,
                                                              g_wait_limit, stall);
    return cudaGetLastError();
}

}  // namespace gemm

// =====================================================================================
// Variant with the decoded weights as the tensor core's A operand in TENSOR MEMORY.
//
// D[w][t] = sum_k W[w][k] * X[t][k]: the MMA's M = 128 weight rows (TMEM lanes), N = 256
// tokens (TMEM columns).  Decoder threads own one weight row each; they expand its 128 codes of
// a K block to int8 in 32 registers and write them with one tcgen05.st into that row's TMEM
// lane -- the weights never touch shared memory, and per multiply-accumulate the decode work is
// half that of the shared-memory variant (128 weight rows feed 256 tokens).  Shared memory only
// carries what TMA brings: the activation tile (256 tokens x 128 B, 128-byte swizzle, the MMA's
// B operand) and the packed codes (128 rows x 32 B).
//   warp 0      TMA producer over a 6-stage ring
//   warp 1      TMEM allocation (512 columns: accumulator 0..255, five A stages of 32 from
//               256) and the single MMA-issuing thread (4 x K=32 per block)
//   warps 2..17 four decoder groups of four warps (K blocks round-robin, so each group has four
//               MMA periods for its decode); afterwards, the epilogue (tcgen05.ld of D, scales,
//               y[t][w] stores coalesced along w).
// =====================================================================================
namespace gemm_ts {

constexpr int BMW = 128;                          // weight rows per tile (MMA M)
constexpr int BNT = 256;                          // tokens per tile (MMA N)
constexpr int BK = 128;                           // K bytes per block
constexpr int STAGES = 6;                         // TMA ring
constexpr int ASTAGES = 5;                        // decoded-weight stages in TMEM
constexpr int kGroups = 4;                        // decoder groups, K blocks round-robin
constexpr int kDecWarps = 4 * kGroups;
constexpr int kThreads = 64 + 32 * kDecWarps;
constexpr int ACT_BYTES = BNT * BK;               // 32 KB
constexpr int COD_BYTES = BMW * (BK / 16) * 4;    // 4 KB
constexpr int SMEM_BYTES = STAGES * (ACT_BYTES + COD_BYTES) + 1024 + 256 + BNT * 4 /*token scales*/;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;
constexpr uint32_t A_COL = 256;                   // A stage sa at A_COL + 32 * sa

struct Smem {
    uint8_t* act;
    uint8_t* cod;
    uint64_t* full;    // [STAGES]  TMA landed
    uint64_t* empty;   // [STAGES]  MMA done with the slot
    uint64_t* afull;   // [ASTAGES] decoded weights stored in TMEM
    uint64_t* aempty;  // [ASTAGES] MMA done with the TMEM stage
    uint64_t* accum;
    uint64_t* never;
    uint32_t* tmem_base;
    int* abort;
    float* sa;         // [BNT] activation scales of this tile's tokens
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    Smem s;
    s.act = base;
    s.cod = s.act + STAGES * ACT_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(s.cod + STAGES * COD_BYTES);
    s.full = bars;
    s.empty = bars + STAGES;
    s.afull = bars + 2 * STAGES;
    s.aempty = bars + 2 * STAGES + ASTAGES;
    s.accum = bars + 2 * STAGES + 2 * ASTAGES;
    s.never = s.accum + 1;
    s.tmem_base = reinterpret_cast<uint32_t*>(s.never + 1);
    s.abort = reinterpret_cast<int*>(s.tmem_base + 1);
    s.sa = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 256);
    return s;
}

template <typename OutT>
__device__ __forceinline__ void store_one(OutT* p, float v);
template <>
__device__ __forceinline__ void store_one<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_one<__half>(__half* p, float v) { *p = __float2half_rn(v); }

template <typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
    w2a4_gemm_ts_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_c,
                        const float* __restrict__ s_a, const float* __restrict__ s_w, uint32_t lut, int T, int N,
                        int K, OutT* __restrict__ y, long long wait_limit, int stall) {
    extern __shared__ uint8_t smem_raw[];
    const Smem sm = carve(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BMW;   // first weight row
    const int t0 = blockIdx.y * BNT;   // first token
    const int num_kb = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(&sm.full[s], 1);
            tc::mbar_init(&sm.empty[s], 1);
        }
        for (int s = 0; s < ASTAGES; ++s) {
            tc::mbar_init(&sm.afull[s], 4);  // the four warps of one decoder group
            tc::mbar_init(&sm.aempty[s], 1);
        }
        tc::mbar_init(sm.accum, 1);
        tc::mbar_init(sm.never, 1);
        *sm.abort = 0;
        tc::fence_mbar_init();
        tc::prefetch_tensormap(&tmap_x);
        tc::prefetch_tensormap(&tmap_c);
    }
    if (warp == 1) {
        tc::tmem_alloc(sm.tmem_base, TMEM_COLS);
        tc::tmem_relinquish();
    }
    if (threadIdx.x >= 64 && threadIdx.x < 64 + BNT) {
        const int t = t0 + threadIdx.x - 64;
        sm.sa[threadIdx.x - 64] = t < T ? s_a[t] : 0.0f;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *sm.tmem_base;

    if (warp == 0) {
        if (lane == 0) {  // ------------------------------------------------ TMA producer
            int issued = 0;
            for (int kb = 0; kb < num_kb; ++kb) {
                const int s = kb % STAGES;
                if (!gemm::wait_or_abort(&sm.empty[s], ((kb / STAGES) & 1) ^ 1, sm.abort, wait_limit)) break;
                tc::mbar_arrive_expect_tx(&sm.full[s], ACT_BYTES + COD_BYTES);
                tc::tma_load_2d(sm.act + s * ACT_BYTES, &tmap_x, &sm.full[s], kb * BK, t0);
                tc::tma_load_2d(sm.cod + s * COD_BYTES, &tmap_c, &sm.full[s], kb * (BK / 16), n0);
                ++issued;
            }
            if (*reinterpret_cast<volatile int*>(sm.abort)) {
                int zero = 0;  // drain: every copy this thread started lands before the CTA exits
                for (int kb = issued > STAGES ? issued - STAGES : 0; kb < issued; ++kb)
                    tc::mbar_wait_bounded(&sm.full[kb % STAGES], (kb / STAGES) & 1, &zero, wait_limit);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {  // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = tc::idesc_i8(BMW, BNT);
            if (stall) gemm::wait_or_abort(sm.never, 0, sm.abort, wait_limit);  // test hook
            for (int kb = 0; kb < num_kb && !*reinterpret_cast<volatile int*>(sm.abort); ++kb) {
                const int s = kb % STAGES, sa = kb % ASTAGES;
                if (!gemm::wait_or_abort(&sm.full[s], (kb / STAGES) & 1, sm.abort, wait_limit)) break;
                if (!gemm::wait_or_abort(&sm.afull[sa], (kb / ASTAGES) & 1, sm.abort, wait_limit)) break;
                tc::tc_fence_after();
                const uint32_t x_addr = tc::smem_u32(sm.act + s * ACT_BYTES);
#pragma unroll
                for (int k = 0; k < BK / 32; ++k)
                    tc::mma_i8_ts(tmem + ACC_COL, tmem + A_COL + 32 * sa + 8 * k, tc::smem_desc_sw128(x_addr + 32 * k),
                                  idesc, (kb > 0 || k > 0) ? 1u : 0u);
                tc::mma_commit(&sm.empty[s]);
                tc::mma_commit(&sm.aempty[sa]);
            }
            tc::mma_commit(sm.accum);  // also after an abort, so TMEM is idle before it is freed
        }
    } else {
        const int grp = (warp - 2) >> 2;      // decoder group: K blocks grp, grp + kGroups, ...
        const int quarter = warp & 3;         // TMEM lanes 32*quarter .. +31
        const int r = quarter * 32 + lane;    // weight row of the tile
        const int first = (r >> 2) & 1;       // staggered 16-byte halves: no bank conflicts
        for (int kb = grp; kb < num_kb; kb += kGroups) {  // ---------------- decoders
            const int s = kb % STAGES, sa = kb % ASTAGES;
            bool ok = gemm::wait_or_abort(&sm.full[s], (kb / STAGES) & 1, sm.abort, wait_limit) &&
                      gemm::wait_or_abort(&sm.aempty[sa], ((kb / ASTAGES) & 1) ^ 1, sm.abort, wait_limit);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc::tc_fence_after();
            const uint8_t* crow = sm.cod + s * COD_BYTES + r * 32;
            const uint4 wa = *reinterpret_cast<const uint4*>(crow + 16 * first);
            const uint4 wb = *reinterpret_cast<const uint4*>(crow + 16 * (first ^ 1));
            const uint4 w0 = first ? wb : wa, w1 = first ? wa : wb;
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
            tc::tmem_st_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + A_COL + 32 * sa, v);
            tc::tmem_st_wait();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.afull[sa]);
        }
        // ---------------------------------------------------------------- epilogue
        bool ok = gemm::wait_or_abort(sm.accum, 0, sm.abort, wait_limit) &&
                  !*reinterpret_cast<volatile int*>(sm.abort);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc::tc_fence_after();
            const int n = n0 + r;
            const float sw = n < N ? s_w[n] : 0.0f;
#pragma unroll 1
            for (int cc = 0; cc < BNT / (16 * kGroups); ++cc) {
                const int c0 = grp * (BNT / kGroups) + cc * 16;  // token column within the tile
                uint32_t acc[16];
                tc::tmem_ld_32x32b_x16(tmem + ((uint32_t)(quarter * 32) << 16) + ACC_COL + c0, acc);
                tc::tmem_ld_wait();
                if (n < N) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int t = t0 + c0 + j;
                        if (t < T) {
                            const float v = __fmul_rn(__fmul_rn((float)(int)acc[j], sw), sm.sa[c0 + j]);
                            store_one<OutT>(y + (int64_t)t * N + n, v);
                        }
                    }
                }
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        int zero = 0;
        tc::mbar_wait_bounded(sm.accum, 0, &zero, wait_limit);
        __syncwarp();
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <typename OutT>
static cudaError_t launch_t(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, uint32_t lut,
                            int64_t T, int64_t N, int64_t K, OutT* y, cudaStream_t s) {
    auto encode = gemm::get_encode();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap mx, mc;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)T};
        const cuuint64_t strides[1] = {(cuuint64_t)K};
        const cuuint32_t box[2] = {BK, BNT};
        const cuuint32_t es[2] = {1, 1};
        if (encode(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(q), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)(K / 16), (cuuint64_t)N};
        const cuuint64_t strides[1] = {(cuuint64_t)(K / 16) * 4};
        const cuuint32_t box[2] = {BK / 16, BMW};
        const cuuint32_t es[2] = {1, 1};
        if (encode(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(codes), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const cudaError_t e = ensure_smem(w2a4_gemm_ts_kernel<OutT>, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((N + BMW - 1) / BMW), (unsigned)((T + BNT - 1) / BNT));
    const int stall = gemm::g_stall_next ? 1 : 0;
    gemm::g_stall_next = false;
    w2a4_gemm_ts_kernel<OutT><<<grid, kThreads, SMEM_BYTES, s>>>(mx, mc, s_a, s_w, lut, (int)T, (int)N, (int)K, y,
                                                                 gemm::g_wait_limit, stall);
    return cudaGetLastError();
}

}  // namespace gemm_ts

// =====================================================================================
// Persistent variant of the tensor-memory-A GEMM: one CTA per SM walks a list of
// 128-weight-row x 128-token tiles.  Two accumulators in TMEM (columns 0..127 and 128..255)
// let four dedicated epilogue warps drain tile i while the MMAs of tile i+1 run, and the TMA
// ring and the decoders run straight on into the next tile, so no pipeline fill or epilogue
// is exposed between tiles.
//   warp 0        TMA producer (8-stage ring: 128 tokens x 128 B activations + 128 x 32 B codes)
//   warp 1        TMEM owner and MMA issuer (M = 128 weight rows, N = 128 tokens)
//   warps 2..17   decoders, four groups taking K blocks round-robin across tiles
//   warps 18..21  epilogue: tcgen05.ld, scales, y stores; frees an accumulator per tile
// =====================================================================================
namespace gemm_tsp {

constexpr int BMW = 128;
constexpr int BNT = 128;
constexpr int BK = 128;
constexpr int STAGES = 8;
constexpr int ASTAGES = 5;
constexpr int kGroups = 4;
constexpr int kDecWarps = 4 * kGroups;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * (kDecWarps + kEpiWarps);
constexpr int ACT_BYTES = BNT * BK;               // 16 KB
constexpr int COD_BYTES = BMW * (BK / 16) * 4;    // 4 KB
constexpr int SMEM_BYTES = STAGES * (ACT_BYTES + COD_BYTES) + 1024 + 512 + 2 * BNT * 4;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t A_COL = 2 * BNT;               // accumulators at 0 and BNT

struct Smem {
    uint8_t* act;
    uint8_t* cod;
    uint64_t* full;
    uint64_t* empty;
    uint64_t* afull;
    uint64_t* aempty;
    uint64_t* accfull;   // [2]
    uint64_t* accempty;  // [2]
    uint64_t* done;
    uint64_t* never;
    uint32_t* tmem_base;
    int* abort;
    float* sa;           // [2][BNT] token scales of the tile held in each accumulator
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    Smem s;
    s.act = base;
    s.cod = s.act + STAGES * ACT_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(s.cod + STAGES * COD_BYTES);
    s.full = bars;
    s.empty = s.full + STAGES;
    s.afull = s.empty + STAGES;
    s.aempty = s.afull + ASTAGES;
    s.accfull = s.aempty + ASTAGES;
    s.accempty = s.accfull + 2;
    s.done = s.accempty + 2;
    s.never = s.done + 1;
    s.tmem_base = reinterpret_cast<uint32_t*>(s.never + 1);
    s.abort = reinterpret_cast<int*>(s.tmem_base + 1);
    s.sa = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 512);
    return s;
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, %0;" ::"r"(kEpiWarps * 32) : "memory"); }

template <typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
    w2a4_gemm_tsp_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_c,
                         const float* __restrict__ s_a, const float* __restrict__ s_w, uint32_t lut, int T, int N,
                         int K, OutT* __restrict__ y, long long wait_limit, int stall) {
    extern __shared__ uint8_t smem_raw[];
    const Smem sm = carve(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_kb = (K + BK - 1) / BK;
    const int n_tiles_w = (N + BMW - 1) / BMW;
    const int n_tiles = n_tiles_w * ((T + BNT - 1) / BNT);
    const int my_tiles = blockIdx.x < n_tiles ? (n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(&sm.full[s], 1);
            tc::mbar_init(&sm.empty[s], 1);
        }
        for (int s = 0; s < ASTAGES; ++s) {
            tc::mbar_init(&sm.afull[s], 4);
            tc::mbar_init(&sm.aempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&sm.accfull[b], 1);
            tc::mbar_init(&sm.accempty[b], kEpiWarps);
        }
        tc::mbar_init(sm.done, 1);
        tc::mbar_init(sm.never, 1);
        *sm.abort = 0;
        tc::fence_mbar_init();
        tc::prefetch_tensormap(&tmap_x);
        tc::prefetch_tensormap(&tmap_c);
    }
    if (warp == 1) {
        tc::tmem_alloc(sm.tmem_base, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *sm.tmem_base;
    volatile int* abort_v = reinterpret_cast<volatile int*>(sm.abort);

    if (warp == 0) {
        if (lane == 0) {  // ------------------------------------------------ TMA producer
            int g = 0, issued = 0;
            for (int i = 0; i < my_tiles && !*abort_v; ++i) {
                const int tile = blockIdx.x + i * gridDim.x;
                const int n0 = (tile % n_tiles_w) * BMW, t0 = (tile / n_tiles_w) * BNT;
                for (int kb = 0; kb < num_kb; ++kb, ++g) {
                    const int s = g % STAGES;
                    if (!gemm::wait_or_abort(&sm.empty[s], ((g / STAGES) & 1) ^ 1, sm.abort, wait_limit)) break;
                    tc::mbar_arrive_expect_tx(&sm.full[s], ACT_BYTES + COD_BYTES);
                    tc::tma_load_2d(sm.act + s * ACT_BYTES, &tmap_x, &sm.full[s], kb * BK, t0);
                    tc::tma_load_2d(sm.cod + s * COD_BYTES, &tmap_c, &sm.full[s], kb * (BK / 16), n0);
                    ++issued;
                }
            }
            if (*abort_v) {
                int zero = 0;  // drain every copy this thread started
                for (int q = issued > STAGES ? issued - STAGES : 0; q < issued; ++q)
                    tc::mbar_wait_bounded(&sm.full[q % STAGES], (q / STAGES) & 1, &zero, wait_limit);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {  // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = tc::idesc_i8(BMW, BNT);
            if (stall) gemm::wait_or_abort(sm.never, 0, sm.abort, wait_limit);  // test hook
            int g = 0;
            for (int i = 0; i < my_tiles && !*abort_v; ++i) {
                const int ab = i & 1;
                if (!gemm::wait_or_abort(&sm.accempty[ab], ((i >> 1) & 1) ^ 1, sm.abort, wait_limit)) break;
                tc::tc_fence_after();
                const uint32_t acc = tmem + ab * BNT;
                bool ok = true;
                for (int kb = 0; kb < num_kb; ++kb, ++g) {
                    const int s = g % STAGES, sa = g % ASTAGES;
                    if (!gemm::wait_or_abort(&sm.full[s], (g / STAGES) & 1, sm.abort, wait_limit) ||
                        !gemm::wait_or_abort(&sm.afull[sa], (g / ASTAGES) & 1, sm.abort, wait_limit)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t x_addr = tc::smem_u32(sm.act + s * ACT_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k)
                        tc::mma_i8_ts(acc, tmem + A_COL + 32 * sa + 8 * k, tc::smem_desc_sw128(x_addr + 32 * k), idesc,
                                      (kb > 0 || k > 0) ? 1u : 0u);
                    tc::mma_commit(&sm.empty[s]);
                    tc::mma_commit(&sm.aempty[sa]);
                }
                if (!ok) break;
                tc::mma_commit(&sm.accfull[ab]);
            }
            tc::mma_commit(sm.done);  // every MMA issued, also after an abort
        }
    } else if (warp < 2 + kDecWarps) {
        const int grp = (warp - 2) >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int first = (r >> 2) & 1;
        const int total = my_tiles * num_kb;
        for (int g = grp; g < total; g += kGroups) {  // ------------------------- decoders
            const int s = g % STAGES, sa = g % ASTAGES;
            bool ok = gemm::wait_or_abort(&sm.full[s], (g / STAGES) & 1, sm.abort, wait_limit) &&
                      gemm::wait_or_abort(&sm.aempty[sa], ((g / ASTAGES) & 1) ^ 1, sm.abort, wait_limit);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc::tc_fence_after();
            const uint8_t* crow = sm.cod + s * COD_BYTES + r * 32;
            const uint4 wa = *reinterpret_cast<const uint4*>(crow + 16 * first);
            const uint4 wb = *reinterpret_cast<const uint4*>(crow + 16 * (first ^ 1));
            const uint4 w0 = first ? wb : wa, w1 = first ? wa : wb;
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
            tc::tmem_st_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + A_COL + 32 * sa, v);
            tc::tmem_st_wait();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.afull[sa]);
        }
    } else {
        const int quarter = warp & 3;  // ------------------------------------------ epilogue
        const int r = quarter * 32 + lane;
        const int et = threadIdx.x - 32 * (2 + kDecWarps);  // 0..127
        // Every epilogue warp runs every iteration (and both named barriers of it) even after an
        // abort, so the barrier counts always match; `alive` only skips the work.
        bool alive = true;
        for (int i = 0; i < my_tiles; ++i) {
            const int ab = i & 1;
            const int tile = blockIdx.x + i * gridDim.x;
            const int n0 = (tile % n_tiles_w) * BMW, t0 = (tile / n_tiles_w) * BNT;
            {
                const int t = t0 + et;
                sm.sa[ab * BNT + et] = t < T ? s_a[t] : 0.0f;
            }
            epi_bar();
            bool ok = alive && gemm::wait_or_abort(&sm.accfull[ab], (i >> 1) & 1, sm.abort, wait_limit) && !*abort_v;
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                tc::tc_fence_after();
                const int n = n0 + r;
                const float sw = n < N ? s_w[n] : 0.0f;
#pragma unroll 1
                for (int cc = 0; cc < BNT / 16; ++cc) {
                    uint32_t acc[16];
                    tc::tmem_ld_32x32b_x16(tmem + ((uint32_t)(quarter * 32) << 16) + ab * BNT + cc * 16, acc);
                    tc::tmem_ld_wait();
                    if (cc == BNT / 16 - 1) {  // every column of this accumulator is in registers
                        tc::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive(&sm.accempty[ab]);
                    }
                    if (n < N) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int t = t0 + cc * 16 + j;
                            if (t < T) {
                                const float v =
                                    __fmul_rn(__fmul_rn((float)(int)acc[j], sw), sm.sa[ab * BNT + cc * 16 + j]);
                                gemm_ts::store_one<OutT>(y + (int64_t)t * N + n, v);
                            }
                        }
                    }
                }
            } else {
                alive = false;
            }
            epi_bar();  // sa[ab] is rewritten two tiles later, after every warp has used it
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        int zero = 0;
        tc::mbar_wait_bounded(sm.done, 0, &zero, wait_limit);
        __syncwarp();
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, TMEM_COLS);
    }
}

static int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int v = 0;
        cached[dev] = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0 ? v : 148;
    }
    return cached[dev];
}

template <typename OutT>
static cudaError_t launch_t(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, uint32_t lut,
                            int64_t T, int64_t N, int64_t K, OutT* y, cudaStream_t s) {
    auto encode = gemm::get_encode();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap mx, mc;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)T};
        const cuuint64_t strides[1] = {(cuuint64_t)K};
        const cuuint32_t box[2] = {BK, BNT};
        const cuuint32_t es[2] = {1, 1};
        if (encode(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(q), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)(K / 16), (cuuint64_t)N};
        const cuuint64_t strides[1] = {(cuuint64_t)(K / 16) * 4};
        const cuuint32_t box[2] = {BK / 16, BMW};
        const cuuint32_t es[2] = {1, 1};
        if (encode(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(codes), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const cudaError_t e = ensure_smem(w2a4_gemm_tsp_kernel<OutT>, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int64_t tiles = ((N + BMW - 1) / BMW) * ((T + BNT - 1) / BNT);
    if (tiles > 0x7fffffff) return cudaErrorInvalidValue;
    const int grid = (int)std::min<int64_t>(tiles, num_sms());
    const int stall = gemm::g_stall_next ? 1 : 0;
    gemm::g_stall_next = false;
    w2a4_gemm_tsp_kernel<OutT><<<grid, kThreads, SMEM_BYTES, s>>>(mx, mc, s_a, s_w, lut, (int)T, (int)N, (int)K, y,
                                                                  gemm::g_wait_limit, stall);
    return cudaGetLastError();
}

}  // namespace gemm_tsp

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
    return tc::mbar_try_wait(bar, parity) || gemm::wait_or_abort(bar, parity, abort, limit);
}

// int32 -> fp32 without the conversion pipe: exact for |v| < 2^22 (|acc| <= 4 * 7 * n_in <= 2^20
// here), since 1.5 * 2^23 + v is then an fp32 integer and the subtraction is exact.
__device__ __forceinline__ float i2f_exact(int v) {
    return __fsub_rn(__int_as_float(0x4B400000 + v), 12582912.0f);
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

template <typename OutT>
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
    const int num_kb = (K + BK - 1) / BK;
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
    const uint32_t tmem = *sm.tmem_base;
    volatile int* abort_v = reinterpret_cast<volatile int*>(sm.abort);

    if (warp == 0) {
        if (lane == 0) {  // ------------------------------------------------ TMA producer
            const uint32_t full0 = tc::cluster_addr(sm.full, 0);
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
                    const bool second = kb * BK + 128 < K;
                    if (rank == 0) tc::mbar_arrive_expect_tx(&sm.full[s], act_ctas * (second ? 2u : 1u) * ACT_HALF);
                    tc::mbar_arrive_expect_tx(&sm.cfull[s], has_cod ? COD_BYTES : 0);
                    if (has_act) {
                        tc::tma_load_2d_pair(sm.act + s * ACT_BYTES, &tmap_x, full0 + 8 * s, kb * BK, tb);
                        if (second)
                            tc::tma_load_2d_pair(sm.act + s * ACT_BYTES + ACT_HALF, &tmap_x, full0 + 8 * s,
                                                 kb * BK + 128, tb);
                    }
                    if (has_cod)
                        tc::tma_load_2d(sm.cod + s * COD_BYTES, &tmap_c, &sm.cfull[s], kb * (BK / 16), tl.n0);
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
            if (stall) gemm::wait_or_abort(sm.never, 0, sm.abort, wait_limit);  // test hook
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
                    tc::mma_i8_ts_pair(tmem + ACC_COL, a, d, idesc, kb != 0 ? 1u : 0u);
#pragma unroll
                    for (int k = 1; k < 4; ++k) tc::mma_i8_ts_pair(tmem + ACC_COL, a + 8 * k, d + 2 * k, idesc, 1u);
                    if (g + 1 < total)
                        ok = wait_fast(&sm.afull[(g + 1) & (STAGES - 1)], ((g + 1) / STAGES) & 1, sm.abort, wait_limit);
                    if (kb * BK + 128 < K) {
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
            const uint8_t* crow = sm.cod + s * COD_BYTES + r * 64;
            tc::tc_fence_after();
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
                        tc::tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + ACC_COL + c0, acc);
                        tc::tmem_ld_wait();
                        if constexpr (sizeof(OutT) == 2) {
                            uint32_t* stg32 = reinterpret_cast<uint32_t*>(sm.stg);
#pragma unroll
                            for (int j = 0; j < 32; j += 2) {
                                const float v0 = __fmul_rn(__fmul_rn(i2f_exact((int)acc[j]), sw), sm.sa[c0 + j]);
                                const float v1 = __fmul_rn(__fmul_rn(i2f_exact((int)acc[j + 1]), sw), sm.sa[c0 + j + 1]);
                                const __half2 h = __floats2half2_rn(v0, v1);  // .x = token c0 + j
                                stg32[((cl0 + j) / 2) * BMW + r] = *reinterpret_cast<const uint32_t*>(&h);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                const float v = __fmul_rn(__fmul_rn(i2f_exact((int)acc[j]), sw), sm.sa[c0 + j]);
                                gemm_ts::store_one<OutT>(stg + (cl0 + j) * BMW + r, v);
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
                                    if (vec_ok && nn + EPP <= N) {
                                        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
                                    } else {
                                        const __half* hv = reinterpret_cast<const __half*>(w);
                                        for (int e = 0; e < EPP; ++e)
                                            if (nn + e < N) dst[e] = hv[e];
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
                                if (vec_ok && nn + EPP <= N) {
                                    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
                                } else {
                                    for (int e = 0; e < EPP; ++e)
                                        if (nn + e < N) dst[e] = src[e];
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
template <typename OutT>
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
        if (cudaOccupancyMaxActiveClusters(&n, w2a4_gemm_pair_kernel<OutT>, &cfg) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = sms / 2;
        }
        cached[dev] = n;
    }
    return cached[dev];
}

template <typename OutT>
static cudaError_t launch_t(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, uint32_t lut,
                            int64_t T, int64_t N, int64_t K, OutT* y, cudaStream_t s) {
    auto encode = gemm::get_encode();
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
        const cuuint64_t dims[2] = {(cuuint64_t)(K / 16), (cuuint64_t)N};
        const cuuint64_t strides[1] = {(cuuint64_t)(K / 16) * 4};
        const cuuint32_t box[2] = {BK / 16, BMW};
        const cuuint32_t es[2] = {1, 1};
        if (encode(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(codes), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const cudaError_t e = ensure_smem(w2a4_gemm_pair_kernel<OutT>, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int64_t tiles = ((N + 2 * BMW - 1) / (2 * BMW)) * ((T + BNT - 1) / BNT);
    if (tiles > 0x3fffffff) return cudaErrorInvalidValue;
    const int clusters = (int)std::min<int64_t>(tiles, std::max(1, max_clusters<OutT>()));
    const int stall = gemm::g_stall_next ? 1 : 0;
    gemm::g_stall_next = false;
    w2a4_gemm_pair_kernel<OutT><<<2 * clusters, kThreads, SMEM_BYTES, s>>>(mx, mc, s_a, s_w, lut, (int)T, (int)N,
                                                                            (int)K, y, gemm::g_wait_limit, stall);
    return cudaGetLastError();
}

}  // namespace gemm_pair

cudaError_t launch_linear_gemm_pair(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, int set,
                                    int64_t T, int64_t N, int64_t K, void* y, bool f16, cudaStream_t s) {
    if (T == 0 || N == 0) return cudaSuccess;
    const uint32_t lut = level_lut(set);
    if (f16) return gemm_pair::launch_t<__half>(q, s_a, codes, s_w, lut, T, N, K, static_cast<__half*>(y), s);
    return gemm_pair::launch_t<float>(q, s_a, codes, s_w, lut, T, N, K, static_cast<float*>(y), s);
}

cudaError_t launch_linear_gemm_tsp(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, int set,
                                   int64_t T, int64_t N, int64_t K, void* y, bool f16, cudaStream_t s) {
    if (T == 0 || N == 0) return cudaSuccess;
    const uint32_t lut = level_lut(set);
    if (f16) return gemm_tsp::launch_t<__half>(q, s_a, codes, s_w, lut, T, N, K, static_cast<__half*>(y), s);
    return gemm_tsp::launch_t<float>(q, s_a, codes, s_w, lut, T, N, K, static_cast<float*>(y), s);
}

cudaError_t launch_linear_gemm_ts(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, int set,
                                  int64_t T, int64_t N, int64_t K, void* y, bool f16, cudaStream_t s) {
    if (T == 0 || N == 0) return cudaSuccess;
    const uint32_t lut = level_lut(set);
    if (f16) return gemm_ts::launch_t<__half>(q, s_a, codes, s_w, lut, T, N, K, static_cast<__half*>(y), s);
    return gemm_ts::launch_t<float>(q, s_a, codes, s_w, lut, T, N, K, static_cast<float*>(y), s);
}

bool linear_gemm_supported(int64_t T, int64_t N, int64_t K) {
    // TMA needs 16-byte row strides for the code matrix (K % 64) and the grid fits.
    return K % 64 == 0 && T <= (int64_t)65535 * gemm::BM && N <= (int64_t)0x7fffffff;
}

cudaError_t launch_linear_gemm(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, int set,
                               int64_t T, int64_t N, int64_t K, void* y, bool f16, cudaStream_t s) {
    if (T == 0 || N == 0) return cudaSuccess;
    const uint32_t lut = level_lut(set);
    if (f16) return gemm::launch_t<__half>(q, s_a, codes, s_w, lut, T, N, K, static_cast<__half*>(y), s);
    return gemm::launch_t<float>(q, s_a, codes, s_w, lut, T, N, K, static_cast<float*>(y), s);
}

void debug_set_gemm_wait_limit(long long cycles) { gemm::g_wait_limit = cycles > 0 ? cycles : gemm::kWaitCycles; }
void debug_stall_next_gemm() { gemm::g_stall_next = true; }

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

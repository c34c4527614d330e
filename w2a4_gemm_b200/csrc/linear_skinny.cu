// linear_skinny.cu -- qift_linear for small batches (2..16 tokens): a tensor-core skinny GEMM
// that streams the packed codes from HBM straight into mma fragments.
//
// "Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
// Inference", Abstract: fixed 2-bit levels (Qift {+-1,+-3}, power-of-two {+-1,+-4}) applied to
// 4-bit activations.  acc[t][n] = sum_k q[t][k] L(code[n][k]) in int32, then the fp32 scales.
//
// Work split.  A thread-block cluster of C CTAs shares one block of 128 output rows; CTA r of
// the cluster owns the K slice [r*KS, (r+1)*KS).  Each 16-row group of the block is owned by
// one warp, or by two warps taking alternate 256-input chunks when the grid leaves an SM per
// CTA (more warps in flight per SM).  The CTA stages its slice of every token's int8
// activations once in shared memory, permuted per 16-byte group to the decode order, so the
// weights never touch shared memory: a lane loads 16 bytes (4 words = 64 codes) of each of its
// two rows, decodes a word into four int8x4 registers with two masks, two shifts and four byte
// permutes against the level table, and those registers ARE the A fragments of
// mma.m16n8k32 (s8 x s8 -> s32).  Each warp pushes its
// partial int32 sums into the shared memory of the cluster CTA that finishes those rows
// (distributed shared memory); after one cluster barrier every CTA adds the partials it
// received (exact, order-free) and finishes 128/C rows with the fp32 epilogue.  No global
// scratch.
//
// Fragment bookkeeping (g = lane/4, q = lane%4).  For chunk c (16 words of a row) and sub-step
// j = 0..3, thread q handles word w = 16c + 4q + j of rows g and g+8; decode_word gives
// d[0] = codes {0,2,4,6}, d[1] = {8,..,14}, d[2] = {1,3,5,7}, d[3] = {9,..,15} of w.  The MMA's
// k-slots 4q..4q+3 / 16+4q..16+4q+3 are (d[0], d[1]) in the first MMA and (d[2], d[3]) in the
// second; the B fragment of token g comes from the same activation group w, permuted the same
// way.  Every thread pairs A and B on identical k positions, so the dot products are exact.
//
// 4-bit weights (W4 = true; the Abstract's mixed W2/W4 layers).  A word holds 8 inputs as
// two's-complement nibbles, byte i = inputs i (low) and i+4 (high), so (word << 4) & 0xF0F0F0F0
// and word & 0xF0F0F0F0 are int8x4 registers holding 16 x the levels of inputs 0..3 and 4..7:
// A fragments with no table and no permute.  Thread q's 16-byte load (4 words) covers two
// activation groups of 16 inputs, j = 0, 1 (chunk c = 16 words = 128 inputs, group 8c + 2q + j);
// the two words of group j give the k-slots (inputs 0..3, 4..7) of the first MMA and (8..11,
// 12..15) of the second, against the activations in natural order.  The int32 sum is 16 x acc,
// exactly (|16 acc| < 2^31 for n_in <= 32768); the epilogue shifts it right by 4.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace qift {
namespace skinny {

namespace cg = cooperative_groups;

constexpr int ROW_WARPS = 8;                    // warps along the rows: 16 rows each
constexpr int RB = ROW_WARPS * 16;              // output rows per cluster
constexpr int CHUNK_WORDS = 16;  // 256 K values per chunk
constexpr int PF = 4;            // chunks of codes in flight per lane

__device__ __forceinline__ void mma_s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared-memory slot of activation group G (16 bytes) within a token row: the low two bits
// of G are XOR-ed with bits 2..3 so the four lanes of a quad and the next token row land on
// distinct 16-byte bank groups.
__device__ __forceinline__ int act_slot(int G) { return G ^ ((G >> 2) & 3); }

template <typename OutT>
__device__ __forceinline__ void store_y(OutT* p, float v);
template <>
__device__ __forceinline__ void store_y<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_y<__half>(__half* p, float v) { *p = __float2half_rn(v); }

// NT token tiles of 8 (T <= 8*NT).  KS: K slice per CTA in bytes (multiple of 256).  KSPLIT
// warps share each 16-row group, taking alternate K chunks: 2 when the grid has at most one CTA
// per SM (16 warps hide more latency), 1 otherwise (two CTAs of 8 warps fit on an SM).
template <int NT, int KSPLIT, bool W4, typename OutT>
__global__ void __launch_bounds__(32 * ROW_WARPS * KSPLIT) skinny_kernel(const int8_t* __restrict__ q,
                                                            const float* __restrict__ s_a,
                                                            const uint32_t* __restrict__ codes,
                                                            const float* __restrict__ s_w, uint32_t lut, int T,
                                                            int N, int K, int KS, OutT* __restrict__ y) {
    constexpr int TP = NT * 8;  // padded tokens
    constexpr int THREADS = 32 * ROW_WARPS * KSPLIT;
    extern __shared__ __align__(16) uint8_t smem[];
    const int S = KS + 64;                            // token row stride (== 64 mod 128)
    uint8_t* acts = smem;                             // TP x S bytes
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    // The CTA finishes RB/C rows of the block; C is a power of two, so RB/C is too.
    const int lg_rows = 7 - (__ffs(C) - 1);  // log2(RB / C), RB = 128
    const int rows_per = 1 << lg_rows;
    const int RPS = rows_per + 4;            // row stride of the partial sums (conflict-free writes)
    // part[s][token][row]: the int32 partial sums this CTA's rows receive, one slot s per source
    // CTA of the cluster and K parity of its warps.
    int* part = reinterpret_cast<int*>(smem + TP * S);
    float* sa_s = reinterpret_cast<float*>(part + KSPLIT * C * TP * RPS);  // [TP] activation scales
    float* sw_s = sa_s + TP;                                                // [RB] weight scales of the block
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, qd = lane & 3;
    const int row_block = blockIdx.x / C;
    constexpr int CPW = W4 ? 8 : 16;                   // codes per word
    constexpr int CHUNK_K = CHUNK_WORDS * CPW;         // inputs per chunk: 256, or 128 for W4
    const int KW = K / CPW;
    const int kw0 = rank * (KS / CPW);                 // first word of this CTA's slice
    const int nchunks = KS / CHUNK_K;
    const int rw = warp % ROW_WARPS, ks = warp / ROW_WARPS;  // row warp, K parity
    const int my_n = (nchunks - ks + KSPLIT - 1) / KSPLIT;   // this warp's chunks: ks, ks+2, ...
    const int64_t r_lo = (int64_t)row_block * RB + rw * 16 + g;
    const int64_t r_hi = r_lo + 8;

    auto load_chunk = [&](int c, uint4& lo, uint4& hi) {
        const int wi = kw0 + c * CHUNK_WORDS + 4 * qd;
        lo = make_uint4(0u, 0u, 0u, 0u);
        hi = make_uint4(0u, 0u, 0u, 0u);
        if (wi + 4 <= KW) {
            if (r_lo < N && QIFT_CK_RANGE(r_lo * KW + wi, 4, N * KW)) lo = ldg_stream_v4(codes + r_lo * KW + wi);
            if (r_hi < N && QIFT_CK_RANGE(r_hi * KW + wi, 4, N * KW)) hi = ldg_stream_v4(codes + r_hi * KW + wi);
        }
    };

    // Announce that this CTA has started; the matching wait below, before the first write into a
    // peer's shared memory, guarantees every peer exists by then.
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

    // Weights do not depend on the previous kernel: start streaming them before waiting.  A
    // ring of PF chunks per lane keeps PF KB of codes per warp in flight.
    uint4 buf[PF][2];
#pragma unroll
    for (int u = 0; u < PF; ++u) load_chunk(ks + KSPLIT * u, buf[u][0], buf[u][1]);
    griddep_launch_dependents();
    griddep_wait();

    // Stage this CTA's K slice of every token, permuted to the decode order (eight loads in
    // flight per thread before any is used), and the scales the epilogue needs.  Element i is
    // group G = i % groups of token t = i / groups; a thread steps its (t, G) by THREADS with one
    // division up front.
    const int groups = KS / 16;
    const int dt = THREADS / groups, dg = THREADS - dt * groups;
    int t_i = (int)threadIdx.x / groups, g_i = (int)threadIdx.x - t_i * groups;
    const uint8_t* q_slice = reinterpret_cast<const uint8_t*>(q) + (int64_t)rank * KS;
    const int64_t rest = ((int64_t)K - (int64_t)rank * KS) / 16;  // groups of the slice inside the row
    const int g_lim = rest < groups ? (int)rest : groups;
    for (int i0 = 0; i0 < TP * groups; i0 += 8 * THREADS) {
        uint4 a[8];
        int tt[8], gg[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            tt[u] = t_i;
            gg[u] = g_i;
            a[u] = make_uint4(0u, 0u, 0u, 0u);
            if (t_i < T && g_i < g_lim &&
                QIFT_CK_RANGE((int64_t)t_i * K + (int64_t)rank * KS + 16 * g_i, 16, (int64_t)T * K))
                a[u] = __ldg(reinterpret_cast<const uint4*>(q_slice + (int64_t)t_i * K + 16 * g_i));
            t_i += dt;
            g_i += dg;
            if (g_i >= groups) {
                g_i -= groups;
                ++t_i;
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (tt[u] < TP) {
                uint4 v = a[u];
                if constexpr (!W4) {
                    uint32_t p[4];
                    permute_acts(a[u], p);
                    v = make_uint4(p[0], p[1], p[2], p[3]);
                }
                *reinterpret_cast<uint4*>(acts + tt[u] * S + act_slot(gg[u]) * 16) = v;
            }
        }
    }
    if (threadIdx.x < TP) sa_s[threadIdx.x] = (int)threadIdx.x < T ? s_a[threadIdx.x] : 0.0f;
    if (threadIdx.x >= 32 && threadIdx.x < 32 + RB) {
        const int64_t n = (int64_t)row_block * RB + threadIdx.x - 32;
        sw_s[threadIdx.x - 32] = n < N ? s_w[n] : 0.0f;
    }
    __syncthreads();

    // The two MMAs of each word pair go to separate accumulators (no dependence between them);
    // the sets are added after the loop.
    int acc[NT][4], acc2[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = acc2[nt][i] = 0;

    for (int i0 = 0; i0 < my_n; i0 += PF) {
#pragma unroll
        for (int u = 0; u < PF; ++u) {
            const int i = i0 + u, c = ks + KSPLIT * i;
            if (i < my_n) {
                const uint32_t wl[4] = {buf[u][0].x, buf[u][0].y, buf[u][0].z, buf[u][0].w};
                const uint32_t wh[4] = {buf[u][1].x, buf[u][1].y, buf[u][1].z, buf[u][1].w};
                if (i + PF < my_n) load_chunk(c + KSPLIT * PF, buf[u][0], buf[u][1]);
                if constexpr (W4) {
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        constexpr uint32_t M = 0xF0F0F0F0u;
                        const uint32_t a1[4] = {(wl[2 * j] << 4) & M, (wh[2 * j] << 4) & M, wl[2 * j] & M, wh[2 * j] & M};
                        const uint32_t a2[4] = {(wl[2 * j + 1] << 4) & M, (wh[2 * j + 1] << 4) & M, wl[2 * j + 1] & M,
                                                wh[2 * j + 1] & M};
                        const int slot = act_slot(c * (CHUNK_WORDS / 2) + 2 * qd + j);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint4 p = *reinterpret_cast<const uint4*>(acts + (nt * 8 + g) * S + slot * 16);
                            mma_s8(acc[nt], a1, p.x, p.y);
                            mma_s8(acc2[nt], a2, p.z, p.w);
                        }
                    }
                    continue;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t dl[4], dh[4];
                    decode_word(wl[j], lut, dl);
                    decode_word(wh[j], lut, dh);
                    const uint32_t a1[4] = {dl[0], dh[0], dl[1], dh[1]};
                    const uint32_t a2[4] = {dl[2], dh[2], dl[3], dh[3]};
                    const int slot = act_slot(c * CHUNK_WORDS + 4 * qd + j);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint4 p = *reinterpret_cast<const uint4*>(acts + (nt * 8 + g) * S + slot * 16);
                        mma_s8(acc[nt], a1, p.x, p.y);
                        mma_s8(acc2[nt], a2, p.z, p.w);
                    }
                }
            }
        }
    }

#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] += acc2[nt][i];
    // Each warp pushes its partial sums into the shared memory of the CTA that finishes its rows
    // (distributed shared memory), into the slot of its source CTA and K parity, so one cluster
    // barrier (release/acquire) suffices and no CTA reads another's memory after it.
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    {
        const int rl = rw * 16 + g;                     // rl and rl + 8 have the same owner
        const int owner = rl >> lg_rows, r0 = rl & (rows_per - 1);
        int* dst = cluster.map_shared_rank(part, owner) + (rank * KSPLIT + ks) * TP * RPS;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int t0 = nt * 8 + 2 * qd;
            if (QIFT_CK(owner < C && (t0 + 1) * RPS + r0 + 8 < TP * RPS)) {
                dst[t0 * RPS + r0] = acc[nt][0];
                dst[(t0 + 1) * RPS + r0] = acc[nt][1];
                dst[t0 * RPS + r0 + 8] = acc[nt][2];
                dst[(t0 + 1) * RPS + r0 + 8] = acc[nt][3];
            }
        }
    }
    cluster.sync();

    // CTA `rank` finishes rows [rank*RB/C, (rank+1)*RB/C) of the block: add the received
    // partials; consecutive threads take consecutive rows of one token, so the stores run along n.
#pragma unroll 4
    for (int i = threadIdx.x; i < rows_per * TP; i += THREADS) {
        const int t = i >> lg_rows, r0 = i & (rows_per - 1), rl = rank * rows_per + r0;
        int sum = 0;
        for (int sl = 0; sl < KSPLIT * C; ++sl) sum += part[(sl * TP + t) * RPS + r0];
        if constexpr (W4) sum >>= 4;  // exact: every product was 16 x level x q
        const int64_t n = (int64_t)row_block * RB + rl;
        if (t < T && n < N && QIFT_CK_RANGE((int64_t)t * N + n, 1, (int64_t)T * N)) {
            const float v = __fmul_rn(__fmul_rn((float)sum, sw_s[rl]), sa_s[t]);
            store_y<OutT>(y + (int64_t)t * N + n, v);
        }
    }
}

static int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int v = 0;
        cached[dev] = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0 ? v : 148;
    }
    return cached[dev];
}

template <int NT, int KSPLIT, bool W4, typename OutT>
static cudaError_t launch_k(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, uint32_t lut,
                            int64_t T, int64_t N, int64_t K, int C, int KS, OutT* y, cudaStream_t s) {
    const size_t smem = (size_t)NT * 8 * (KS + 64) + (size_t)KSPLIT * C * NT * 8 * (RB / C + 4) * sizeof(int) +
                        (size_t)(NT * 8 + RB) * 4;
    cudaError_t e = ensure_smem(skinny_kernel<NT, KSPLIT, W4, OutT>, smem);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (N + RB - 1) / RB;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(blocks * C));
    cfg.blockDim = dim3(32 * ROW_WARPS * KSPLIT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, skinny_kernel<NT, KSPLIT, W4, OutT>, q, s_a, codes, s_w, lut, (int)T, (int)N,
                              (int)K, KS, y);
}

template <int NT, bool W4, typename OutT>
static cudaError_t launch_t(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, uint32_t lut,
                            int64_t T, int64_t N, int64_t K, OutT* y, cudaStream_t s) {
    // Cluster size C, a power of two <= 8 (so it divides RB): the smallest whose grid of
    // blocks x C CTAs covers at least 80% of the SMs -- K is split, and partial sums reduced
    // across the cluster, only as far as needed to fill the GPU -- and whose K slice of the
    // activations fits shared memory.  Two warps share each 16-row group (16 warps per CTA)
    // when the grid leaves an SM per CTA and the CTA has at least four K chunks; otherwise two
    // 8-warp CTAs share an SM.  (A sweep of C and the warp split over the LLaMA shapes at 4-16
    // tokens on B200 picked these within a few percent of the best for every shape.)
    const int64_t blocks = (N + RB - 1) / RB;
    const int sms = sm_count();
    constexpr int CHUNK_K = CHUNK_WORDS * (W4 ? 8 : 16);
    auto slice = [&](int c) { return (int)(((K + c - 1) / c + 255) / 256 * 256); };
    int C = 1;
    while (C < 8 && (blocks * C * 5 < (int64_t)sms * 4 || (size_t)NT * 8 * (slice(C) + 64) > 160 * 1024)) C *= 2;
    const int KS = slice(C);
    const int64_t ctas = blocks * C;
    if (ctas <= sms && KS / CHUNK_K >= 4)
        return launch_k<NT, 2, W4, OutT>(q, s_a, codes, s_w, lut, T, N, K, C, KS, y, s);
    return launch_k<NT, 1, W4, OutT>(q, s_a, codes, s_w, lut, T, N, K, C, KS, y, s);
}

}  // namespace skinny

bool linear_skinny_supported(int64_t T, int64_t N, int64_t K) {
    return T >= 1 && T <= 16 && K % 64 == 0 && K <= 32768 && N <= (int64_t)0x7fffffff / 8;
}

cudaError_t launch_linear_skinny(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, int set,
                                 int64_t T, int64_t N, int64_t K, void* y, bool f16, cudaStream_t s) {
    if (T == 0 || N == 0) return cudaSuccess;
    const uint32_t lut = level_lut(set);
    if (set == kSetInt4) {
        if (T <= 8) {
            if (f16) return skinny::launch_t<1, true, __half>(q, s_a, codes, s_w, lut, T, N, K, static_cast<__half*>(y), s);
            return skinny::launch_t<1, true, float>(q, s_a, codes, s_w, lut, T, N, K, static_cast<float*>(y), s);
        }
        if (f16) return skinny::launch_t<2, true, __half>(q, s_a, codes, s_w, lut, T, N, K, static_cast<__half*>(y), s);
        return skinny::launch_t<2, true, float>(q, s_a, codes, s_w, lut, T, N, K, static_cast<float*>(y), s);
    }
    if (T <= 8) {
        if (f16) return skinny::launch_t<1, false, __half>(q, s_a, codes, s_w, lut, T, N, K, static_cast<__half*>(y), s);
        return skinny::launch_t<1, false, float>(q, s_a, codes, s_w, lut, T, N, K, static_cast<float*>(y), s);
    }
    if (f16) return skinny::launch_t<2, false, __half>(q, s_a, codes, s_w, lut, T, N, K, static_cast<__half*>(y), s);
    return skinny::launch_t<2, false, float>(q, s_a, codes, s_w, lut, T, N, K, static_cast<float*>(y), s);
}

}  // namespace qift

// linear_one_token.cu -- one activation token: qift_linear (from q and s_a) and
// qift_decode_linear (rotation + INT4 + linear from x, in one launch).
//
// "Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
// Inference", Abstract: rotated W2A4 inference with the fixed 2-bit weight levels.
//
//   acc[n] = sum_k q[k] * L(code[n][k])  (int32),   y[n] = ((float)acc[n] * s_w[n]) * s_a.
//
// One token means one multiply-add per packed weight: the time is what it takes to get the
// codes on chip plus the chain of latencies after the wait for whatever produced the
// activations.  Everything that does not depend on the activations goes before that wait:
//   - one CTA per SM (two for very tall matrices) takes a contiguous run of rows; one thread
//     issues bulk copies (cp.async.bulk) of all of them into shared memory, completing on one
//     mbarrier, before griddepcontrol.wait -- so they overlap the previous kernel on the stream;
//   - a CTA holds at most half an SM's registers (and, up to ~14K x 4K matrices, half its
//     shared memory), so the next launch on the stream becomes resident beside it and starts
//     its own copies while this one computes;
//   - after the wait the token is staged once per CTA in shared memory -- read from q, or
//     rotated and quantized from x by warps 0-7 with the device code of qift_quantize_acts
//     (same bits) -- and each thread keeps one 64-activation group in registers while it walks
//     the CTA's rows.
// Qift levels are affine in the code, L(c) = 2c - 3 (codes 0..3 = -3, -1, +1, +3), so
// sum q L(c) = 2 sum q c - 3 sum q.  Masking a code word with 0x03030303 << 2m leaves code
// 4j+m in byte j, scaled by 4^m: one unsigned x signed dp4a per mask against the matching four
// activations, no decode at all.  The PoT levels {-4,-1,+1,+4} are not affine in c; their codes
// are decoded by byte permutes against the level table and meet the activations in signed dp4a.
// Either way the int32 sum is exact, so every path gives the same bits.
// 4-bit weights (SET = kSetInt4, the mixed W2/W4 layers): eight nibbles per word, byte j = inputs
// j and j + 4; (w << 4) & 0xF0F0F0F0 and w & 0xF0F0F0F0 are 16 x the levels of inputs 0..3 and
// 4..7 as signed bytes, met by the activations in natural order; the row sum is 16 x acc and is
// shifted back (exact) in the epilogue.  A 16-byte code group then covers 32 inputs, not 64.
#include <math.h>

#include <algorithm>

#include "act_quant.cuh"
#include "internal.h"
#include "tc.cuh"

namespace qift {
namespace one {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr uint32_t kPiece = 4096;               // bytes per bulk copy
constexpr int64_t kMaxCodeBytes = 100 * 1024;   // packed codes one CTA stages
constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 2 GHz before the wait gives up

__device__ int g_error = 0;  // bit 0: a CTA's wait for its codes ran out (QIFT_ERR_TIMEOUT)

// Test hooks (qift_debug.h), per host thread.
static thread_local long long g_wait_limit = kWaitCycles;
static thread_local bool g_stall_next = false;

template <typename OutT>
__device__ __forceinline__ void store_out(OutT* p, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_out<__half>(__half* p, float v) { *p = __float2half_rn(v); }

__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     tc::smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
                 : "memory");
}

// Sixteen activations (natural order) -> the four words the set's code application meets.
// Qift: word m = activations 4j+m, j = 0..3 (a 4x4 byte transpose).  PoT: decode_word order.
template <int SET>
__device__ __forceinline__ uint4 arrange(uint4 a) {
    if constexpr (SET == kSetInt4) {
        return a;  // natural order
    } else if constexpr (SET == kSetQift) {
        const uint32_t t0 = prmt(a.x, a.y, 0x5140u), t1 = prmt(a.z, a.w, 0x5140u);
        const uint32_t t2 = prmt(a.x, a.y, 0x7362u), t3 = prmt(a.z, a.w, 0x7362u);
        return make_uint4(prmt(t0, t1, 0x5410u), prmt(t0, t1, 0x7632u), prmt(t2, t3, 0x5410u),
                          prmt(t2, t3, 0x7632u));
    } else {
        uint32_t p[4];
        permute_acts(a, p);
        return make_uint4(p[0], p[1], p[2], p[3]);
    }
}

__device__ __forceinline__ int sum16(uint4 a, int s) {
    s = dp4a(a.x, 0x01010101u, s);
    s = dp4a(a.y, 0x01010101u, s);
    s = dp4a(a.z, 0x01010101u, s);
    return dp4a(a.w, 0x01010101u, s);
}

// One 16-byte code group (64 weights) against its four arranged activation words a[0..3].
// Qift: returns sum q c (the affine terms are applied per row); PoT: returns sum q L(c).
template <int SET>
__device__ __forceinline__ int dot_group(uint4 wv, const uint4 (&a)[4]) {
    const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
    if constexpr (SET == kSetInt4) {  // 32 inputs: a[0], a[1] hold their activations in order
        constexpr uint32_t M = 0xF0F0F0F0u;
        int s = 0;
        s = dp4a((wd[0] << 4) & M, a[0].x, s);
        s = dp4a(wd[0] & M, a[0].y, s);
        s = dp4a((wd[1] << 4) & M, a[0].z, s);
        s = dp4a(wd[1] & M, a[0].w, s);
        s = dp4a((wd[2] << 4) & M, a[1].x, s);
        s = dp4a(wd[2] & M, a[1].y, s);
        s = dp4a((wd[3] << 4) & M, a[1].z, s);
        return dp4a(wd[3] & M, a[1].w, s);
    } else if constexpr (SET == kSetQift) {
        int s0 = 0, s1 = 0, s2 = 0, s3 = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            s0 = dp4a_us(wd[u] & 0x03030303u, a[u].x, s0);
            s1 = dp4a_us(wd[u] & 0x0C0C0C0Cu, a[u].y, s1);
            s2 = dp4a_us(wd[u] & 0x30303030u, a[u].z, s2);
            s3 = dp4a_us(wd[u] & 0xC0C0C0C0u, a[u].w, s3);
        }
        return s0 + (s1 >> 2) + (s2 >> 4) + (s3 >> 6);  // each s_m is an exact multiple of 4^m
    } else {
        int s = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            uint32_t d[4];
            decode_word(wd[u], level_lut(SET), d);
            s = dp4a(d[0], a[u].x, s);
            s = dp4a(d[1], a[u].y, s);
            s = dp4a(d[2], a[u].z, s);
            s = dp4a(d[3], a[u].w, s);
        }
        return s;
    }
}

// Shared memory after the static part: codes [R][K/64] x 16 B ([R][K/32] for 4-bit weights),
// arranged activations (K bytes), row sums and row scales [R rounded to 4] each, and for ROT the
// rotated fp16 token + the rotation's transpose buffer.
__host__ __device__ inline size_t code_bytes(int64_t R, int64_t K, bool w4) {
    return (size_t)R * (size_t)(w4 ? K / 2 : K / 4);
}
__host__ __device__ inline size_t rowacc_offset(int64_t R, int64_t K, bool w4) { return code_bytes(R, K, w4) + (size_t)K; }
__host__ __device__ inline size_t sw_offset(int64_t R, int64_t K, bool w4) {
    return rowacc_offset(R, K, w4) + (size_t)((R + 3) & ~3) * 4;
}
__host__ __device__ inline size_t xs_offset(int64_t R, int64_t K, bool w4) {
    return sw_offset(R, K, w4) + (size_t)((R + 3) & ~3) * 4;
}

template <bool ROT, int LOGB, int SET, typename OutT>
__global__ void __launch_bounds__(kThreads, 2)
    one_token_kernel(const __half* __restrict__ x, float c, const int8_t* __restrict__ q,
                     const float* __restrict__ s_a, const uint32_t* __restrict__ codes,
                     const float* __restrict__ s_w, int64_t N, int64_t K, int G, OutT* __restrict__ y,
                     int8_t* __restrict__ q_out, float* __restrict__ sa_out, long long wait_limit,
                     int stall) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bar, never_bar;  // never_bar: nothing arrives (test hook)
    __shared__ int qsum, never;
    __shared__ float sa_s;
    __shared__ float red[kActThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr bool W4 = SET == kSetInt4;
    const int64_t KW = K / 16;                    // 16-byte activation groups
    const int64_t CW = K / (W4 ? 8 : 16);         // code words per row
    const int CPR = (int)(K / (W4 ? 32 : 64));    // 16-byte code groups per row
    constexpr int AG = W4 ? 2 : 4;                // activation groups per code group
    const int64_t R = (N + G - 1) / G;
    const int64_t r0 = (int64_t)blockIdx.x * N / G, r1 = (int64_t)(blockIdx.x + 1) * N / G;
    const int nrows = (int)(r1 - r0);
    const uint4* cs = reinterpret_cast<const uint4*>(smem);
    uint4* as = reinterpret_cast<uint4*>(smem + code_bytes(R, K, W4));
    int* row_acc = reinterpret_cast<int*>(smem + rowacc_offset(R, K, W4));
    float* sw_s = reinterpret_cast<float*>(smem + sw_offset(R, K, W4));

    // 1. Before the wait: the barrier, this CTA's codes in flight, its weight scales, the
    //    activations' lines into L2.
    if (tid == 0) {
        tc::mbar_init(&bar, 1);
        tc::mbar_init(&never_bar, 1);
        tc::fence_mbar_init();
        qsum = 0;
        never = 0;
    }
    for (int i = tid; i < nrows; i += kThreads) {
        row_acc[i] = 0;
        sw_s[i] = QIFT_CK_RANGE(r0 + i, 1, N) ? __ldg(s_w + r0 + i) : 0.0f;
    }
    __syncthreads();
    const uint32_t bytes = (uint32_t)code_bytes(nrows, K, W4);
    if (tid == 0 && bytes && QIFT_CK_RANGE(r0 * CW * 4, bytes, N * CW * 4) && QIFT_CK(bytes % 16 == 0) &&
        QIFT_CK(code_bytes(R, K, W4) >= bytes)) {
        tc::mbar_arrive_expect_tx(&bar, bytes);
        const uint8_t* src = reinterpret_cast<const uint8_t*>(codes + r0 * CW);
        for (uint32_t off = 0; off < bytes; off += kPiece)
            bulk_g2s(smem + off, src + off, bytes - off < kPiece ? bytes - off : kPiece, &bar);
    }
    if constexpr (ROT) {
        prefetch_l2_grid(x, K * 2);
    } else {
        prefetch_l2_grid(q, K);
        if (blockIdx.x == gridDim.x - 1 && tid == 0) asm volatile("prefetch.global.L2 [%0];" ::"l"(s_a));
    }
    griddep_launch_dependents();
    griddep_wait();

    // 2. The token, arranged for the set, in shared memory (and sum q for Qift).
    int qs = 0;
    if constexpr (ROT) {
        if (tid < kActThreads) {
            __half* xs = reinterpret_cast<__half*>(smem + xs_offset(R, K, W4));
            float* tbuf = reinterpret_cast<float*>(smem + xs_offset(R, K, W4) + (size_t)K * 2);
            const float m = rotate_token_f16<LOGB, GroupSync<kActThreads>>(x, K, c, xs, tbuf, red);
            const float inv = m == 0.0f ? 0.0f : __fdiv_rn(7.0f, m);
            for (int g = tid; g < (int)KW; g += kActThreads) {
                const uint4 v = m == 0.0f ? make_uint4(0u, 0u, 0u, 0u) : quant16(xs + 16 * g, inv);
                if (blockIdx.x == 0 && q_out && QIFT_CK_RANGE(16 * (int64_t)g, 16, K))
                    *reinterpret_cast<uint4*>(q_out + 16 * g) = v;
                as[(g % AG) * CPR + g / AG] = arrange<SET>(v);
                if constexpr (SET == kSetQift) qs = sum16(v, qs);
            }
            if (tid == 0) {
                sa_s = m == 0.0f ? 0.0f : __fdiv_rn(m, 7.0f);
                if (blockIdx.x == 0 && sa_out) *sa_out = sa_s;
            }
        }
    } else {
        for (int g = tid; g < (int)KW; g += kThreads) {
            const uint4 v = QIFT_CK_RANGE(16 * (int64_t)g, 16, K) ? __ldg(reinterpret_cast<const uint4*>(q) + g)
                                                                   : make_uint4(0u, 0u, 0u, 0u);
            as[(g % AG) * CPR + g / AG] = arrange<SET>(v);
            if constexpr (SET == kSetQift) qs = sum16(v, qs);
        }
        if (tid == 0) sa_s = __ldg(s_a);
    }
    if constexpr (SET == kSetQift) {
        qs = __reduce_add_sync(0xffffffffu, qs);
        if (lane == 0 && qs != 0) atomicAdd(&qsum, qs);
    }
    __syncthreads();

    // 3. Codes on chip (bounded wait), then the dot products.  Thread (rg, c) owns 16-byte
    //    group c of every row rg, rg + RG, ...: its 64 arranged activations stay in registers
    //    and each row costs one 16-byte code load.  Rows are padded to whole warps (CPRp
    //    groups), so a warp never spans two rows: one warp reduction and one shared atomic per
    //    row and warp.
    bool ok = true;
    if (bytes) ok = tc::mbar_wait_bounded(stall ? &never_bar : &bar, 0, &never, wait_limit);
    ok = __syncthreads_and(ok) != 0;  // one verdict for the whole CTA
    const int CPRp = (CPR + 31) & ~31;
    const int RG = kThreads / CPRp;  // >= 2 for K <= 16384
    const int rg = tid / CPRp, ch = tid - rg * CPRp;
    if (ok && rg < RG) {
        uint4 a[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) a[u] = u < AG && ch < CPR ? as[u * CPR + ch] : make_uint4(0u, 0u, 0u, 0u);
        for (int row0 = rg; row0 < nrows; row0 += 4 * RG) {  // four independent rows per pass
            int v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int row = row0 + j * RG;
                v[j] = row < nrows && ch < CPR ? dot_group<SET>(cs[row * CPR + ch], a) : 0;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int row = row0 + j * RG;  // warp-uniform
                const int t = __reduce_add_sync(0xffffffffu, v[j]);
                if (lane == 0 && row < nrows) atomicAdd(&row_acc[row], t);
            }
        }
    }
    __syncthreads();
    if (!ok) {
        // Report, and let the copies already issued land before the CTA's shared memory is
        // released (a second bounded wait; the output is left unwritten).
        if (tid == 0) {
            atomicOr(&g_error, 1);
            tc::mbar_wait_bounded(&bar, 0, &never, wait_limit);
        }
        __syncthreads();
        return;
    }

    // 4. Epilogue: y = ((float)acc * s_w) * s_a.
    for (int t = tid; t < nrows; t += kThreads) {
        const int acc = SET == kSetQift ? 2 * row_acc[t] - 3 * qsum : (W4 ? row_acc[t] >> 4 : row_acc[t]);
        if (QIFT_CK_RANGE(r0 + t, 1, N)) store_out<OutT>(y + r0 + t, __fmul_rn(__fmul_rn((float)acc, sw_s[t]), sa_s));
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

// Grid: one CTA per SM (two when the codes of one CTA would pass kMaxCodeBytes), never more
// CTAs than rows.  Returns 0 when the matrix is too tall for this kernel.
static int plan_grid(int64_t N, int64_t K, size_t extra_smem, size_t* smem, bool w4) {
    if (N <= 0 || K <= 0 || K % 64 != 0 || K > 16384) return 0;
    const int sm = sm_count();
    for (int mult = 1; mult <= 2; ++mult) {
        const int64_t G = std::min<int64_t>(N, (int64_t)sm * mult);
        const int64_t R = (N + G - 1) / G;
        if ((int64_t)code_bytes(R, K, w4) > kMaxCodeBytes) continue;
        const size_t bytes = xs_offset(R, K, w4) + extra_smem;
        if (bytes > 200 * 1024) continue;
        *smem = bytes;
        return (int)G;
    }
    return 0;
}

template <bool ROT, int LOGB, int SET, typename OutT>
static cudaError_t launch(const __half* x, float c, const int8_t* q, const float* s_a, const uint32_t* codes,
                          const float* s_w, int64_t N, int64_t K, OutT* y, int8_t* q_out, float* sa_out,
                          cudaStream_t s) {
    size_t smem = 0;
    const size_t extra = ROT ? (size_t)K * 2 + act_tbuf_bytes<LOGB>() : 0;
    const int G = plan_grid(N, K, extra, &smem, SET == kSetInt4);
    if (!G) return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem(one_token_kernel<ROT, LOGB, SET, OutT>, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)G);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    const int stall = g_stall_next ? 1 : 0;  // wait on a barrier nothing arrives on: it runs out
    g_stall_next = false;
    return cudaLaunchKernelEx(&cfg, one_token_kernel<ROT, LOGB, SET, OutT>, x, c, q, s_a, codes, s_w, N, K, G, y,
                              q_out, sa_out, g_wait_limit, stall);
}

template <int LOGB, typename OutT>
static cudaError_t decode_by_set(const __half* x, float c, const uint32_t* codes, const float* s_w, int set,
                                 int64_t N, int64_t K, OutT* y, int8_t* q_out, float* sa_out, cudaStream_t s) {
    if (set == kSetQift)
        return launch<true, LOGB, kSetQift, OutT>(x, c, nullptr, nullptr, codes, s_w, N, K, y, q_out, sa_out, s);
    if (set == kSetInt4)
        return launch<true, LOGB, kSetInt4, OutT>(x, c, nullptr, nullptr, codes, s_w, N, K, y, q_out, sa_out, s);
    return launch<true, LOGB, kSetPot, OutT>(x, c, nullptr, nullptr, codes, s_w, N, K, y, q_out, sa_out, s);
}

template <typename OutT>
static cudaError_t decode_by_block(const __half* x, int block, const uint32_t* codes, const float* s_w, int set,
                                   int64_t N, int64_t K, OutT* y, int8_t* q_out, float* sa_out, cudaStream_t s) {
    const float c = block ? (float)(1.0 / sqrt((double)block)) : 1.0f;
    switch (block ? ilog2(block) : 0) {
        case 0: return decode_by_set<0, OutT>(x, c, codes, s_w, set, N, K, y, q_out, sa_out, s);
        case 1: return decode_by_set<1, OutT>(x, c, codes, s_w, set, N, K, y, q_out, sa_out, s);
        case 2: return decode_by_set<2, OutT>(x, c, codes, s_w, set, N, K, y, q_out, sa_out, s);
        case 3: return decode_by_set<3, OutT>(x, c, codes, s_w, set, N, K, y, q_out, sa_out, s);
        case 4: return decode_by_set<4, OutT>(x, c, codes, s_w, set, N, K, y, q_out, sa_out, s);
        case 5: return decode_by_set<5, OutT>(x, c, codes, s_w, set, N, K, y, q_out, sa_out, s);
        case 6: return decode_by_set<6, OutT>(x, c, codes, s_w, set, N, K, y, q_out, sa_out, s);
        case 7: return decode_by_set<7, OutT>(x, c, codes, s_w, set, N, K, y, q_out, sa_out, s);
        case 8: return decode_by_set<8, OutT>(x, c, codes, s_w, set, N, K, y, q_out, sa_out, s);
        case 9: return decode_by_set<9, OutT>(x, c, codes, s_w, set, N, K, y, q_out, sa_out, s);
        case 10: return decode_by_set<10, OutT>(x, c, codes, s_w, set, N, K, y, q_out, sa_out, s);
        case 11: return decode_by_set<11, OutT>(x, c, codes, s_w, set, N, K, y, q_out, sa_out, s);
        case 12: return decode_by_set<12, OutT>(x, c, codes, s_w, set, N, K, y, q_out, sa_out, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace one

bool linear_one_token_supported(int64_t n_out, int64_t n_in) {
    size_t smem = 0;
    return one::plan_grid(n_out, n_in, 0, &smem, false) != 0;
}

// The warp-per-row GEMV (8 rows per 128-thread CTA, ~110 registers: four CTAs per SM) decodes
// all its codes into registers before the wait when n_in <= 4096 and its grid fits one wave;
// after the wait it then only multiplies, and at 4096 x 4096 it takes 2.55 us against 3.0 us
// here.  Past one wave, or with longer rows that it streams after the wait, this kernel wins:
// 3.4 against 4.4 us at 6144 x 4096, 8.8 against 13.8 us at 28672 x 4096 (CUDA-graph chains of
// launches on cycled weights, B200 at 1965 MHz).
bool linear_one_token_preferred(int64_t n_out, int64_t n_in) {
    return (n_in > 4096 || n_out > 4 * 8 * (int64_t)one::sm_count()) && linear_one_token_supported(n_out, n_in);
}

static size_t rotation_tbuf_bytes(int block) {
    switch (block ? ilog2(block) : 0) {
        case 0: return act_tbuf_bytes<0>();
        case 1: return act_tbuf_bytes<1>();
        case 2: return act_tbuf_bytes<2>();
        case 3: return act_tbuf_bytes<3>();
        case 4: return act_tbuf_bytes<4>();
        case 5: return act_tbuf_bytes<5>();
        case 6: return act_tbuf_bytes<6>();
        case 7: return act_tbuf_bytes<7>();
        case 8: return act_tbuf_bytes<8>();
        case 9: return act_tbuf_bytes<9>();
        case 10: return act_tbuf_bytes<10>();
        case 11: return act_tbuf_bytes<11>();
        default: return act_tbuf_bytes<12>();
    }
}

bool decode_one_token_supported(int64_t n_out, int64_t n_in, int block, int set) {
    size_t smem = 0;
    return one::plan_grid(n_out, n_in, (size_t)n_in * 2 + rotation_tbuf_bytes(block), &smem, set == kSetInt4) != 0;
}

cudaError_t launch_linear_one_token(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w,
                                    int set, int64_t N, int64_t K, void* y, bool f16, cudaStream_t s) {
    if (set == kSetQift) {
        if (f16)
            return one::launch<false, 0, kSetQift, __half>(nullptr, 1.0f, q, s_a, codes, s_w, N, K,
                                                           static_cast<__half*>(y), nullptr, nullptr, s);
        return one::launch<false, 0, kSetQift, float>(nullptr, 1.0f, q, s_a, codes, s_w, N, K,
                                                      static_cast<float*>(y), nullptr, nullptr, s);
    }
    if (f16)
        return one::launch<false, 0, kSetPot, __half>(nullptr, 1.0f, q, s_a, codes, s_w, N, K,
                                                      static_cast<__half*>(y), nullptr, nullptr, s);
    return one::launch<false, 0, kSetPot, float>(nullptr, 1.0f, q, s_a, codes, s_w, N, K, static_cast<float*>(y),
                                                 nullptr, nullptr, s);
}

cudaError_t launch_decode_one_token(const void* x, int64_t K, int block, const uint32_t* codes, const float* s_w,
                                    int set, int64_t N, void* y, bool f16, int8_t* q_out, float* sa_out,
                                    cudaStream_t s) {
    const __half* xh = static_cast<const __half*>(x);
    if (f16)
        return one::decode_by_block<__half>(xh, block, codes, s_w, set, N, K, static_cast<__half*>(y), q_out, sa_out, s);
    return one::decode_by_block<float>(xh, block, codes, s_w, set, N, K, static_cast<float*>(y), q_out, sa_out, s);
}

void debug_set_one_token_wait_limit(long long cycles) {
    one::g_wait_limit = cycles > 0 ? cycles : one::kWaitCycles;
}
void debug_stall_next_one_token() { one::g_stall_next = true; }

cudaError_t read_and_clear_one_token_error(int* word) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, one::g_error, sizeof(int));
    if (e != cudaSuccess) return e;
    if (v != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(one::g_error, &zero, sizeof(int));
    }
    *word = v;
    return e;
}

}  // namespace qift

// linear_w4.cu -- qift_linear for 4-bit weights (levels {-7..7} * s per output channel, stored
// as two's-complement nibbles, eight per word) at decode batch sizes (1..16 tokens): a CUDA-core
// W4A4 GEMV.
//
// "Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
// Inference", Abstract: the evaluation mixes 2-bit and 4-bit layers ("L-layer mixed W2/W4"),
// both applied to the rotated 4-bit activations.
//
//   acc[t][n] = sum_k q[t][k] level[n][k]                                 (exact, int32)
//   y[t][n]   = ((float)acc * s_w[n]) * s_a[t].
//
// The codes are applied without a decode.  Byte j of a word holds input j in its low nibble and
// input j + 4 in its high nibble, so the word masked with 0xF0F0F0F0 holds, as signed bytes,
// 16 x the levels of inputs 4..7 and the word shifted left by 4 and masked 16 x those of inputs
// 0..3: each meets one 32-bit word of INT4 activations in a signed dp4a.  The total is 16 x acc
// exactly (|16 acc| <= 16 * 8 * 7 * 32768 < 2^31), and an arithmetic shift by 4 recovers acc.
//
// One token (w4_gemv1_kernel): each warp owns R rows, and all of a chunk's codes are loaded and
// split before the wait for the previous kernel on the stream (programmatic dependent launch).
// Several tokens (w4_gemv_kernel, reached when the GEMV path is pinned): each warp owns R rows
// and TC tokens; lane l streams 16-byte groups (32 codes) g = l, l+32, ... of its rows, and the
// codes of the first group are requested before the wait.
#include "common.cuh"
#include "internal.h"

namespace qift {
namespace w4 {

// Warps per CTA: 8 (256 CTAs at 4096 x 4096 for one token) measured 2.27 us per launch against
// 2.32 us for 4.
constexpr int kWarps = 8;

template <typename OutT>
__device__ __forceinline__ void store_out(OutT* p, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_out<__half>(__half* p, float v) { *p = __float2half_rn(v); }

template <int R, int TC, typename OutT>
__global__ void __launch_bounds__(kWarps * 32) w4_gemv_kernel(const int8_t* __restrict__ q,
                                                              const float* __restrict__ s_a,
                                                              const uint32_t* __restrict__ codes,
                                                              const float* __restrict__ s_w, int64_t T, int64_t N,
                                                              int64_t K, OutT* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int64_t row0 = ((int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5)) * R;
    const int64_t t0 = (int64_t)blockIdx.y * TC;
    const int64_t KW = K / 8, KG = K / 32;  // words and 16-byte groups per row
    int acc[R][TC];
#pragma unroll
    for (int t = 0; t < TC; ++t)
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r][t] = 0;
    uint4 cw[R];
    auto load_codes = [&](int64_t g) {
#pragma unroll
        for (int r = 0; r < R; ++r)
            cw[r] = (row0 + r < N && g < KG && QIFT_CK_RANGE((row0 + r) * KW + 4 * g, 4, N * KW))
                        ? ldg_stream_v4(codes + (row0 + r) * KW + 4 * g)
                        : make_uint4(0u, 0u, 0u, 0u);
    };
    load_codes(lane);
    griddep_launch_dependents();
    griddep_wait();
    for (int64_t g = lane; g < KG; g += 32) {
        if (g != lane) load_codes(g);
        // 16 x levels as signed bytes: lo[r][w] for inputs 8w..8w+3, hi[r][w] for 8w+4..8w+7
        uint32_t lo[R][4], hi[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const uint32_t wd[4] = {cw[r].x, cw[r].y, cw[r].z, cw[r].w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                lo[r][w] = (wd[w] << 4) & 0xF0F0F0F0u;
                hi[r][w] = wd[w] & 0xF0F0F0F0u;
            }
        }
#pragma unroll
        for (int t = 0; t < TC; ++t) {
            uint4 a0 = make_uint4(0u, 0u, 0u, 0u), a1 = a0;
            if (t0 + t < T && QIFT_CK_RANGE((t0 + t) * K + 32 * g, 32, T * K)) {
                const uint4* src = reinterpret_cast<const uint4*>(q + (t0 + t) * K + 32 * g);
                a0 = __ldg(src);
                a1 = __ldg(src + 1);
            }
            const uint32_t av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
            for (int w = 0; w < 4; ++w)
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    acc[r][t] = dp4a(lo[r][w], av[2 * w], acc[r][t]);
                    acc[r][t] = dp4a(hi[r][w], av[2 * w + 1], acc[r][t]);
                }
        }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int t = 0; t < TC; ++t) {
            const int sum = __reduce_add_sync(0xffffffffu, acc[r][t]) >> 4;  // exact: a multiple of 16
            const int64_t n = row0 + r, tt = t0 + t;
            if (lane == ((r * TC + t) & 31) && n < N && tt < T && QIFT_CK_RANGE(tt * N + n, 1, T * N))
                store_out<OutT>(y + tt * N + n, __fmul_rn(__fmul_rn((float)sum, __ldg(s_w + n)), __ldg(s_a + tt)));
        }
    }
}

// One token.  Lane l holds the 16-byte code groups g = c + l + 32 j (j < J) of each of its R
// rows for the chunk that starts at group c; group g is inputs 32 g .. 32 g + 31.  Every code
// of a chunk is loaded and split into its two signed-byte registers before the kernel waits
// for its predecessor, so after the wait only the token (staged once per CTA in shared memory),
// the dp4a products, the warp reduction and the epilogue remain.  The token's 16-byte halves
// h = 0, 1 of group g sit at slot 2 c + 32 (2 j + h) + l: a warp's read of one (j, h) covers 512
// contiguous bytes, and a thread staging group g writes both halves (conflict-free stores).
// ONE: the row is a single chunk (n_in <= 1024 J), so no loop over chunks is compiled.
template <int R, int J, bool ONE, typename OutT>
__global__ void __launch_bounds__(kWarps * 32) w4_gemv1_kernel(const int8_t* __restrict__ q,
                                                               const float* __restrict__ s_a,
                                                               const uint32_t* __restrict__ codes,
                                                               const float* __restrict__ s_w, int64_t N, int64_t K,
                                                               OutT* __restrict__ y) {
    extern __shared__ __align__(16) uint4 acts_s[];  // 2 K/32 token halves (chunk-padded)
    constexpr int CG = 32 * J;                       // groups per chunk
    constexpr uint32_t M = 0xF0F0F0F0u;
    const int lane = threadIdx.x & 31;
    const int64_t row0 = ((int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5)) * R;
    const int64_t KW = K / 8, KG = K / 32;

    // lo: 16 x the levels of inputs 8w..8w+3 of word w of the group, hi: of 8w+4..8w+7.
    uint32_t lo[R][J][4], hi[R][J][4];
    auto load_split = [&](int64_t c) {
        uint4 cw[R][J];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int64_t g = c + lane + 32 * j;
                cw[r][j] = (row0 + r < N && g < KG && QIFT_CK_RANGE((row0 + r) * KW + 4 * g, 4, N * KW))
                               ? ldg_stream_v4(codes + (row0 + r) * KW + 4 * g)
                               : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const uint32_t wd[4] = {cw[r][j].x, cw[r][j].y, cw[r][j].z, cw[r][j].w};
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    lo[r][j][w] = (wd[w] << 4) & M;
                    hi[r][j][w] = wd[w] & M;
                }
            }
    };
    load_split(0);
    griddep_launch_dependents();
    griddep_wait();

    float sw[R];
#pragma unroll
    for (int r = 0; r < R; ++r) sw[r] = row0 + r < N ? __ldg(s_w + row0 + r) : 0.0f;
    const float sa = __ldg(s_a);
    for (int i = threadIdx.x; i < (int)KG; i += kWarps * 32) {
        const uint4* src = reinterpret_cast<const uint4*>(q) + 2 * (int64_t)i;
        const bool ok = QIFT_CK_RANGE(32 * (int64_t)i, 32, K);
        const uint4 a0 = ok ? __ldg(src) : make_uint4(0u, 0u, 0u, 0u);
        const uint4 a1 = ok ? __ldg(src + 1) : make_uint4(0u, 0u, 0u, 0u);
        const int in = i % CG;  // group within its chunk: lane in % 32, slice in / 32
        const int slot = 2 * (i - in) + 64 * (in >> 5) + (in & 31);
        acts_s[slot] = a0;
        acts_s[slot + 32] = a1;
    }
    // A partial last chunk leaves slots no group maps to; they are read only for groups past
    // the row, which the reads below replace by zeros.
    __syncthreads();

    int acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0;
    for (int64_t c = 0; c < (ONE ? 1 : KG); c += CG) {
        if (!ONE && c > 0) load_split(c);
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const bool in_row = c + lane + 32 * j < KG;
            const uint4 a0 = in_row ? acts_s[2 * c + 64 * j + lane] : make_uint4(0u, 0u, 0u, 0u);
            const uint4 a1 = in_row ? acts_s[2 * c + 64 * j + 32 + lane] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                int v = acc[r];
                v = dp4a(lo[r][j][0], a0.x, v);
                v = dp4a(hi[r][j][0], a0.y, v);
                v = dp4a(lo[r][j][1], a0.z, v);
                v = dp4a(hi[r][j][1], a0.w, v);
                v = dp4a(lo[r][j][2], a1.x, v);
                v = dp4a(hi[r][j][2], a1.y, v);
                v = dp4a(lo[r][j][3], a1.z, v);
                v = dp4a(hi[r][j][3], a1.w, v);
                acc[r] = v;
            }
        }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int sum = __reduce_add_sync(0xffffffffu, acc[r]) >> 4;  // exact: a multiple of 16
        if (lane == r && row0 + r < N && QIFT_CK_RANGE(row0 + r, 1, N))
            store_out<OutT>(y + row0 + r, __fmul_rn(__fmul_rn((float)sum, sw[r]), sa));
    }
}

template <int R, int J, bool ONE, typename OutT>
static cudaError_t launch1_t(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, int64_t N,
                             int64_t K, OutT* y, cudaStream_t s) {
    const int64_t gx = (N + R * kWarps - 1) / (R * kWarps);
    if (gx > 0x7fffffff) return cudaErrorInvalidValue;
    const int64_t KG = K / 32, chunk = 32 * J;
    const size_t smem = (size_t)((KG + chunk - 1) / chunk * chunk) * 32;  // whole chunks of 32-byte groups
    cudaError_t e = ensure_smem(w4_gemv1_kernel<R, J, ONE, OutT>, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)gx);
    cfg.blockDim = dim3(kWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, w4_gemv1_kernel<R, J, ONE, OutT>, q, s_a, codes, s_w, N, K, y);
}

template <int R, int TC, typename OutT>
static cudaError_t launch(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, int64_t T,
                          int64_t N, int64_t K, OutT* y, cudaStream_t s) {
    const int64_t gx = (N + R * kWarps - 1) / (R * kWarps);
    const int64_t gy = (T + TC - 1) / TC;
    if (gx > 0x7fffffff || gy > 65535) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)gx, (unsigned)gy);
    cfg.blockDim = dim3(kWarps * 32);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, w4_gemv_kernel<R, TC, OutT>, q, s_a, codes, s_w, T, N, K, y);
}

template <typename OutT>
static cudaError_t dispatch(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, int64_t T,
                            int64_t N, int64_t K, OutT* y, cudaStream_t s) {
    if (T == 1 && K <= 4096) return launch1_t<2, 4, true, OutT>(q, s_a, codes, s_w, N, K, y, s);
    if (T == 1) return launch1_t<2, 4, false, OutT>(q, s_a, codes, s_w, N, K, y, s);
    if (T <= 4) return launch<2, 4, OutT>(q, s_a, codes, s_w, T, N, K, y, s);
    return launch<4, 8, OutT>(q, s_a, codes, s_w, T, N, K, y, s);
}

}  // namespace w4

// Any batch: one token on this kernel, 2..16 on the skinny tensor-core kernel, more on the
// tcgen05 pair GEMM; all need n_in % 64 == 0.
bool linear_w4_supported(int64_t tokens, int64_t n_in) { return tokens >= 1 && n_in % 64 == 0; }

cudaError_t launch_linear_w4(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, int64_t T,
                             int64_t N, int64_t K, void* y, bool f16, cudaStream_t s) {
    if (T == 0 || N == 0) return cudaSuccess;
    if (f16) return w4::dispatch<__half>(q, s_a, codes, s_w, T, N, K, static_cast<__half*>(y), s);
    return w4::dispatch<float>(q, s_a, codes, s_w, T, N, K, static_cast<float*>(y), s);
}

}  // namespace qift

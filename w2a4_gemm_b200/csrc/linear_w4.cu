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
// Each warp owns R rows and TC tokens; lane l streams 16-byte groups (32 codes) g = l, l+32, ...
// of its rows.  The codes of the first group are requested before the wait for the previous
// kernel on the stream (programmatic dependent launch).
#include "common.cuh"
#include "internal.h"

namespace qift {
namespace w4 {

constexpr int kWarps = 4;

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
    if (T == 1) return launch<2, 1, OutT>(q, s_a, codes, s_w, T, N, K, y, s);
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

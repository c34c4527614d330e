// decode_fused.cu -- qift_decode_linear: the whole online path of a decode step in one launch.
//
// "Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
// Inference", Abstract: rotated W2A4 inference -- the activation is Hadamard-rotated and
// quantized to 4 bits, then meets the fixed 2-bit weight levels.
//
// For 1..4 tokens the activation work is tiny next to streaming the packed weights, so every
// CTA does it itself instead of waiting for a separate kernel:
//   1. load this CTA's code rows and decode them to int8 registers -- before waiting for the
//      previous kernel on the stream (programmatic dependent launch), so the weight stream and
//      the decode overlap its tail;
//   2. rotate + quantize the tokens into shared memory (the same device code, and therefore
//      the same bits, as qift_quantize_acts), stored permuted to the decode order;
//   3. decode the codes to int8 (byte permutes against the level table) and dp4a them with the
//      shared activations; warp reduction; fp32 epilogue.
// The grid has one CTA per SM (or more for very tall matrices) and spreads the rows evenly,
// so each SM streams the same share of the weights.  CTA 0 can also write q and s_a out.
// 4-bit weights (W4, the Abstract's mixed W2/W4 layers): a word holds eight inputs as
// two's-complement nibbles (byte j = inputs j and j + 4), so (w << 4) & 0xF0F0F0F0 and
// w & 0xF0F0F0F0 are the int8x4 operands 16 x level of inputs 0..3 and 4..7; they meet the
// activations in natural order, and the sum is shifted back by 4 (exact) before the epilogue.
#include <math.h>

#include <algorithm>

#include "act_quant.cuh"
#include "internal.h"

namespace qift {
namespace fused {

constexpr int WARPS = kActThreads / 32;  // 8
constexpr int RMAX = 2;                  // rows per warp

template <typename OutT>
__device__ __forceinline__ void store_out(OutT* p, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_out<__half>(__half* p, float v) { *p = __float2half_rn(v); }

// TC: tokens handled (T <= TC); J: 128-word slices per K chunk.
template <int LOGB, int TC, int J, bool W4, typename OutT>
__global__ void __launch_bounds__(kActThreads) decode_kernel(const __half* __restrict__ x, int T, int64_t K, float c,
                                                             const uint32_t* __restrict__ codes,
                                                             const float* __restrict__ s_w, uint32_t lut, int64_t N,
                                                             int rows_per_cta, OutT* __restrict__ y,
                                                             int8_t* __restrict__ q_out, float* __restrict__ sa_out) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ float red[WARPS];
    __shared__ float sa_s[TC];
    const size_t xs_bytes = ((size_t)K * 2 + 15) / 16 * 16;
    __half* xs = reinterpret_cast<__half*>(smem);
    float* tbuf = reinterpret_cast<float*>(smem + xs_bytes);
    uint8_t* qs = smem + xs_bytes + act_tbuf_bytes<LOGB>();  // TC x K int8, permuted per 16-group

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t KW = K / (W4 ? 8 : 16);  // code words per row
    const int64_t cta_r0 = (int64_t)blockIdx.x * rows_per_cta;
    const int64_t cta_r1 = min(N, cta_r0 + rows_per_cta);
    const int rpw = (rows_per_cta + WARPS - 1) / WARPS;
    const int64_t row0 = cta_r0 + (int64_t)warp * rpw;
    const int nr = (int)max((int64_t)0, min((int64_t)rpw, cta_r1 - row0));

    // Codes of the first K chunk are loaded and decoded to int8 registers before waiting for
    // the previous kernel: only the activation work and the dp4a products remain after it.
    uint32_t dec[RMAX][J][4][4];
    auto load_decode = [&](int64_t base) {
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int64_t wi = base + 4 * lane + 128 * j;
                const uint4 v = (r < nr && wi + 4 <= KW && QIFT_CK_RANGE((row0 + r) * KW + wi, 4, N * KW))
                                    ? ldg_stream_v4(codes + (row0 + r) * KW + wi)
                                    : make_uint4(0u, 0u, 0u, 0u);
                if constexpr (W4) {
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        dec[r][j][u][0] = (w[u] << 4) & 0xF0F0F0F0u;
                        dec[r][j][u][1] = w[u] & 0xF0F0F0F0u;
                    }
                } else {
                    decode_word(v.x, lut, dec[r][j][0]);
                    decode_word(v.y, lut, dec[r][j][1]);
                    decode_word(v.z, lut, dec[r][j][2]);
                    decode_word(v.w, lut, dec[r][j][3]);
                }
            }
        }
    };
    // 1. weights first (and x's lines into L2), then wait for the producer of x.
    load_decode(0);
    prefetch_l2_grid(x, (int64_t)T * K * 2);
    griddep_launch_dependents();
    griddep_wait();
    float sw[RMAX];
#pragma unroll
    for (int r = 0; r < RMAX; ++r) sw[r] = r < nr && QIFT_CK_RANGE(row0 + r, 1, N) ? __ldg(s_w + row0 + r) : 0.0f;

    // 2. rotation + INT4 of every token, identical arithmetic to qift_quantize_acts.
    for (int t = 0; t < TC; ++t) {
        uint8_t* qt = qs + (int64_t)t * K;
        if (t < T) {
            const float m = rotate_token_f16<LOGB>(x + (int64_t)t * K, K, c, xs, tbuf, red);
            const float inv = m == 0.0f ? 0.0f : __fdiv_rn(7.0f, m);
            for (int64_t i = (int64_t)tid * 16; i < K; i += kActThreads * 16) {
                const uint4 v = m == 0.0f ? make_uint4(0u, 0u, 0u, 0u) : quant16(xs + i, inv);
                if (blockIdx.x == 0 && q_out && QIFT_CK_RANGE((int64_t)t * K + i, 16, (int64_t)T * K))
                    *reinterpret_cast<uint4*>(q_out + (int64_t)t * K + i) = v;
                if constexpr (W4) {
                    *reinterpret_cast<uint4*>(qt + i) = v;  // natural order
                } else {
                    uint32_t p[4];
                    permute_acts(v, p);
                    *reinterpret_cast<uint4*>(qt + i) = make_uint4(p[0], p[1], p[2], p[3]);
                }
            }
            if (tid == 0) {
                sa_s[t] = m == 0.0f ? 0.0f : __fdiv_rn(m, 7.0f);
                if (blockIdx.x == 0 && sa_out) sa_out[t] = sa_s[t];
            }
            __syncthreads();  // xs is reused by the next token
        } else {
            for (int64_t i = (int64_t)tid * 16; i < K; i += kActThreads * 16)
                *reinterpret_cast<uint4*>(qt + i) = make_uint4(0u, 0u, 0u, 0u);
            if (tid == 0) sa_s[t] = 0.0f;
        }
    }
    __syncthreads();

    // 3. decode + dp4a against the shared activations.
    int acc[RMAX][TC];
#pragma unroll
    for (int r = 0; r < RMAX; ++r)
#pragma unroll
        for (int t = 0; t < TC; ++t) acc[r][t] = 0;
    for (int64_t base = 0; base < KW && W4; base += 128 * J) {
        if (base > 0) load_decode(base);
        uint2 pa[TC][J][4];  // the eight activations of each word, natural order
#pragma unroll
        for (int t = 0; t < TC; ++t)
#pragma unroll
            for (int j = 0; j < J; ++j)
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int64_t wi = base + 4 * lane + 128 * j + u;
                    pa[t][j][u] = wi < KW ? *reinterpret_cast<const uint2*>(qs + (int64_t)t * K + wi * 8)
                                          : make_uint2(0u, 0u);
                }
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
            if (r >= nr) break;
#pragma unroll
            for (int j = 0; j < J; ++j)
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int t = 0; t < TC; ++t)
                        acc[r][t] = dp4a(dec[r][j][u][1], pa[t][j][u].y, dp4a(dec[r][j][u][0], pa[t][j][u].x, acc[r][t]));
        }
    }
    for (int64_t base = 0; base < KW && !W4; base += 128 * J) {
        if (base > 0) load_decode(base);
        uint4 pa[TC][J][4];
#pragma unroll
        for (int t = 0; t < TC; ++t)
#pragma unroll
            for (int j = 0; j < J; ++j)
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int64_t wi = base + 4 * lane + 128 * j + u;
                    pa[t][j][u] = wi < KW ? *reinterpret_cast<const uint4*>(qs + (int64_t)t * K + wi * 16)
                                          : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
            if (r >= nr) break;
#pragma unroll
            for (int j = 0; j < J; ++j) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
#pragma unroll
                    for (int t = 0; t < TC; ++t) {
                        int a = acc[r][t];
                        a = dp4a(dec[r][j][u][0], pa[t][j][u].x, a);
                        a = dp4a(dec[r][j][u][1], pa[t][j][u].y, a);
                        a = dp4a(dec[r][j][u][2], pa[t][j][u].z, a);
                        a = dp4a(dec[r][j][u][3], pa[t][j][u].w, a);
                        acc[r][t] = a;
                    }
                }
            }
        }
    }

    // 4. warp reduction and the fp32 epilogue.
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        if (r >= nr) break;
#pragma unroll
        for (int t = 0; t < TC; ++t) {
            int sum = __reduce_add_sync(0xffffffffu, acc[r][t]);
            if constexpr (W4) sum >>= 4;  // exact: every product was 16 x level x q
            if (lane == ((r * TC + t) & 31) && t < T && QIFT_CK_RANGE((int64_t)t * N + row0 + r, 1, (int64_t)T * N)) {
                const float v = __fmul_rn(__fmul_rn((float)sum, sw[r]), sa_s[t]);
                store_out<OutT>(y + (int64_t)t * N + row0 + r, v);
            }
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

template <int LOGB, int TC, int J, bool W4, typename OutT>
static cudaError_t launch_t(const __half* x, int64_t T, int64_t K, float c, const uint32_t* codes, const float* s_w,
                            uint32_t lut, int64_t N, OutT* y, int8_t* q_out, float* sa_out, cudaStream_t s) {
    const int64_t min_ctas = (N + WARPS * RMAX - 1) / (WARPS * RMAX);
    const int64_t ctas = std::max<int64_t>(std::min<int64_t>(sm_count(), (N + WARPS - 1) / WARPS), min_ctas);
    const int64_t rows_per_cta = (N + ctas - 1) / ctas;
    const int64_t grid = (N + rows_per_cta - 1) / rows_per_cta;
    const size_t smem = ((size_t)K * 2 + 15) / 16 * 16 + act_tbuf_bytes<LOGB>() + (size_t)TC * K;
    cudaError_t e = ensure_smem(decode_kernel<LOGB, TC, J, W4, OutT>, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kActThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode_kernel<LOGB, TC, J, W4, OutT>, x, (int)T, K, c, codes, s_w, lut, N,
                              (int)rows_per_cta, y, q_out, sa_out);
}

template <int LOGB, typename OutT>
static cudaError_t by_tokens(const __half* x, int64_t T, int64_t K, float c, const uint32_t* codes, const float* s_w,
                             uint32_t lut, int64_t N, OutT* y, int8_t* q_out, float* sa_out, cudaStream_t s) {
    if (lut == 0) {  // 4-bit weights
        if (T == 1) return launch_t<LOGB, 1, 2, true, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
        return launch_t<LOGB, 4, 1, true, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
    }
    if (T == 1) return launch_t<LOGB, 1, 2, false, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
    return launch_t<LOGB, 4, 1, false, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
}

template <typename OutT>
static cudaError_t by_block(const __half* x, int64_t T, int64_t K, int block, const uint32_t* codes, const float* s_w,
                            uint32_t lut, int64_t N, OutT* y, int8_t* q_out, float* sa_out, cudaStream_t s) {
    const float c = block ? (float)(1.0 / sqrt((double)block)) : 1.0f;
    switch (block ? ilog2(block) : 0) {
        case 0: return by_tokens<0, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
        case 1: return by_tokens<1, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
        case 2: return by_tokens<2, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
        case 3: return by_tokens<3, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
        case 4: return by_tokens<4, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
        case 5: return by_tokens<5, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
        case 6: return by_tokens<6, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
        case 7: return by_tokens<7, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
        case 8: return by_tokens<8, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
        case 9: return by_tokens<9, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
        case 10: return by_tokens<10, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
        case 11: return by_tokens<11, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
        case 12: return by_tokens<12, OutT>(x, T, K, c, codes, s_w, lut, N, y, q_out, sa_out, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace fused

cudaError_t launch_decode_linear(const void* x, int64_t T, int64_t K, int block, const uint32_t* codes,
                                 const float* s_w, int set, int64_t N, void* y, bool f16, int8_t* q_out,
                                 float* sa_out, cudaStream_t s) {
    const __half* xh = static_cast<const __half*>(x);
    const uint32_t lut = set == kSetInt4 ? 0u : level_lut(set);  // 0 selects the 4-bit form
    if (f16) return fused::by_block<__half>(xh, T, K, block, codes, s_w, lut, N, static_cast<__half*>(y), q_out, sa_out, s);
    return fused::by_block<float>(xh, T, K, block, codes, s_w, lut, N, static_cast<float*>(y), q_out, sa_out, s);
}

}  // namespace qift

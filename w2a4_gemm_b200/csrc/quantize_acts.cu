// quantize_acts.cu -- qift_quantize_acts: fused activation rotation + symmetric per-token INT4.
//
// "Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
// Inference", Abstract: rotated W2A4 inference (4-bit activations).  One CTA owns one token:
//   1. block Walsh-Hadamard of every length-b segment (fp32), one rounding to fp16;
//   2. m = max |x'| over the token (CTA reduction);
//   3. q = clamp(rint(x' * (7/m)), -7, 7), s_a = m / 7 (IEEE division, round half even).
// The rotated fp16 token stays in shared memory between the passes, so HBM sees one fp16
// read and one int8 write per element.
#include <math.h>

#include "fwht.cuh"
#include "internal.h"

namespace qift {

constexpr int kActThreads = 256;

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < (kActThreads / 32) ? red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[0] = v;
    }
    __syncthreads();
    return red[0];
}

// LOGB == 0: the input is already rotated (no stages, no multiply).
template <int LOGB>
__global__ void __launch_bounds__(kActThreads) quant_acts_kernel(const __half* __restrict__ x, int64_t K,
                                                                 int8_t* __restrict__ q, float* __restrict__ scales,
                                                                 float c) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ float red[kActThreads / 32];
    __half* xs = reinterpret_cast<__half*>(smem_raw);  // K rotated fp16 values
    const int tid = threadIdx.x, lane = tid & 31;
    const int64_t token = blockIdx.x;
    const __half* xt = x + token * K;
    float amax = 0.0f;
    // Launched as a programmatic dependent: wait for the previous kernel on the stream before
    // touching memory, then let the next one (the linear) start its weight stream early.
    griddep_wait();
    griddep_launch_dependents();

    if constexpr (LOGB == 0) {
        for (int64_t i = (int64_t)tid * 8; i < K; i += kActThreads * 8) {
            const uint4 t = *reinterpret_cast<const uint4*>(xt + i);
            *reinterpret_cast<uint4*>(xs + i) = t;
            const __half2* h = reinterpret_cast<const __half2*>(&t);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __half22float2(h[j]);
                amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
        }
    } else {
        using S = FwhtShape<LOGB>;
        constexpr int SPC = kActThreads / S::TPS;
        float* tbuf = reinterpret_cast<float*>(smem_raw + ((K * 2 + 15) / 16) * 16);
        const int seg_local = tid >> S::LOGT;
        const int ts = tid & (S::TPS - 1);
        const int64_t nseg = K / S::B;
        for (int64_t p = 0; p < nseg; p += SPC) {
            const int64_t seg = p + seg_local;
            const bool active = seg < nseg;
            float v[S::E];
            if (active) {
                load_contig<S::E>(xt + seg * S::B + ts * S::E, v);
            } else {
#pragma unroll
                for (int i = 0; i < S::E; ++i) v[i] = 0.0f;
            }
            float out[S::W][S::R];
            fwht_segment<LOGB>(v, ts, lane, c, tbuf + (S::W > 1 ? seg_local * S::B : 0), out);
            if (active) {
#pragma unroll
                for (int j = 0; j < S::W; ++j) {
                    float hv[S::R];
#pragma unroll
                    for (int r = 0; r < S::R; ++r) {
                        hv[r] = __half2float(__float2half_rn(out[j][r]));
                        amax = fmaxf(amax, fabsf(hv[r]));
                    }
                    store_contig<S::R>(xs + seg * S::B + ts * S::R + j * S::COL, hv);
                }
            }
            if constexpr (S::W > 1) __syncthreads();  // tbuf is reused by the next pass
        }
    }
    __syncthreads();
    const float m = block_max(amax, red);

    int8_t* qt = q + token * K;
    if (m == 0.0f) {
        for (int64_t i = (int64_t)tid * 16; i < K; i += kActThreads * 16)
            *reinterpret_cast<uint4*>(qt + i) = make_uint4(0u, 0u, 0u, 0u);
        if (tid == 0) scales[token] = 0.0f;
        return;
    }
    const float inv = __fdiv_rn(7.0f, m);
    for (int64_t i = (int64_t)tid * 16; i < K; i += kActThreads * 16) {
        const uint4 a = *reinterpret_cast<const uint4*>(xs + i);
        const uint4 b = *reinterpret_cast<const uint4*>(xs + i + 8);
        const __half2* ha = reinterpret_cast<const __half2*>(&a);
        const __half2* hb = reinterpret_cast<const __half2*>(&b);
        uint32_t packed[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const __half2* h = w < 2 ? ha + 2 * w : hb + 2 * (w - 2);
            const float2 f0 = __half22float2(h[0]);
            const float2 f1 = __half22float2(h[1]);
            const float f[4] = {f0.x, f0.y, f1.x, f1.y};
            uint32_t word = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                int v = __float2int_rn(__fmul_rn(f[e], inv));
                v = v > 7 ? 7 : (v < -7 ? -7 : v);
                word |= (uint32_t)(v & 0xff) << (8 * e);
            }
            packed[w] = word;
        }
        *reinterpret_cast<uint4*>(qt + i) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
    if (tid == 0) scales[token] = __fdiv_rn(m, 7.0f);
}

template <int LOGB>
static cudaError_t launch_qa(const __half* x, int64_t tokens, int64_t K, int8_t* q, float* scales, float c,
                             cudaStream_t s) {
    size_t smem = (size_t)((K * 2 + 15) / 16) * 16;
    if constexpr (LOGB > 0) {
        using S = FwhtShape<LOGB>;
        if (S::W > 1) smem += (size_t)(kActThreads / S::TPS) * S::B * sizeof(float);
    }
    {
        const cudaError_t e = ensure_smem(quant_acts_kernel<LOGB>, smem);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)tokens);
    cfg.blockDim = dim3(kActThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, quant_acts_kernel<LOGB>, x, K, q, scales, c);
}

cudaError_t launch_quantize_acts(const void* x, int64_t tokens, int64_t n_in, int block, int8_t* q, float* scales,
                                 cudaStream_t s) {
    if (tokens == 0) return cudaSuccess;
    const __half* xh = static_cast<const __half*>(x);
    const float c = block ? (float)(1.0 / sqrt((double)block)) : 1.0f;
    switch (block ? ilog2(block) : 0) {
        case 0: return launch_qa<0>(xh, tokens, n_in, q, scales, c, s);
        case 1: return launch_qa<1>(xh, tokens, n_in, q, scales, c, s);
        case 2: return launch_qa<2>(xh, tokens, n_in, q, scales, c, s);
        case 3: return launch_qa<3>(xh, tokens, n_in, q, scales, c, s);
        case 4: return launch_qa<4>(xh, tokens, n_in, q, scales, c, s);
        case 5: return launch_qa<5>(xh, tokens, n_in, q, scales, c, s);
        case 6: return launch_qa<6>(xh, tokens, n_in, q, scales, c, s);
        case 7: return launch_qa<7>(xh, tokens, n_in, q, scales, c, s);
        case 8: return launch_qa<8>(xh, tokens, n_in, q, scales, c, s);
        case 9: return launch_qa<9>(xh, tokens, n_in, q, scales, c, s);
        case 10: return launch_qa<10>(xh, tokens, n_in, q, scales, c, s);
        case 11: return launch_qa<11>(xh, tokens, n_in, q, scales, c, s);
        case 12: return launch_qa<12>(xh, tokens, n_in, q, scales, c, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace qift

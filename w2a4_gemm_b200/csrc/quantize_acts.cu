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

#include "act_quant.cuh"
#include "internal.h"

namespace qift {

// LOGB == 0: the input is already rotated (no stages, no multiply).  PACK: the codes are
// stored two per byte (KV4), q then points at [tokens][K/2] bytes.
template <int LOGB, bool PACK>
__global__ void __launch_bounds__(kActThreads) quant_acts_kernel(const __half* __restrict__ x, int64_t K,
                                                                 int8_t* __restrict__ q, float* __restrict__ scales,
                                                                 float c) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ float red[kActThreads / 32];
    __half* xs = reinterpret_cast<__half*>(smem_raw);  // K rotated fp16 values
    float* tbuf = reinterpret_cast<float*>(smem_raw + ((K * 2 + 15) / 16) * 16);
    const int tid = threadIdx.x;
    const int64_t token = blockIdx.x;
    // Launched as a programmatic dependent: the token's lines are requested into L2 while the
    // previous kernel on the stream finishes; the values are read only after waiting for it.
    // Only then is the next kernel (the linear) released to start its weight stream: the linear
    // reads the weights before its own wait, so the kernel before this one (which may have
    // written them) must have completed by the time the linear starts.
    prefetch_l2_cta(x + token * K, K * 2);
    griddep_wait();
    griddep_launch_dependents();

    const float m = rotate_token_f16<LOGB>(x + token * K, K, c, xs, tbuf, red);
    int8_t* qt = q + token * (PACK ? K / 2 : K);
    if (m == 0.0f) {
        for (int64_t i = (int64_t)tid * 16; i < K; i += kActThreads * 16) {
            if (!QIFT_CK_RANGE(i, 16, K)) continue;
            if constexpr (PACK) *reinterpret_cast<uint2*>(qt + i / 2) = make_uint2(0u, 0u);
            else *reinterpret_cast<uint4*>(qt + i) = make_uint4(0u, 0u, 0u, 0u);
        }
        if (tid == 0) scales[token] = 0.0f;
        return;
    }
    const float inv = __fdiv_rn(7.0f, m);
    for (int64_t i = (int64_t)tid * 16; i < K; i += kActThreads * 16) {
        if (!QIFT_CK_RANGE(i, 16, K)) continue;
        if constexpr (PACK) *reinterpret_cast<uint2*>(qt + i / 2) = pack_int4_16(quant16(xs + i, inv));
        else *reinterpret_cast<uint4*>(qt + i) = quant16(xs + i, inv);
    }
    if (tid == 0) scales[token] = __fdiv_rn(m, 7.0f);
}

// KV4 dequantization of one token per CTA: unpack the nibbles, (float)q * s in binary32 (the
// conversion by the exact magic-number add), then the inverse rotation -- the rotation itself,
// H/sqrt(b) being symmetric and orthogonal -- with qift_rotate's stages, and one rounding to
// fp16.  LOGB == 0: no rotation.
template <int LOGB>
__global__ void __launch_bounds__(kActThreads) dequant_kv_kernel(const uint8_t* __restrict__ packed,
                                                                 const float* __restrict__ scales, int64_t K,
                                                                 float c, __half* __restrict__ out) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ float red[kActThreads / 32];
    float* xf = reinterpret_cast<float*>(smem_raw);                    // K floats
    __half* xs = reinterpret_cast<__half*>(smem_raw + (size_t)K * 4);  // K rotated fp16 values
    float* tbuf = reinterpret_cast<float*>(smem_raw + (size_t)K * 6);
    const int tid = threadIdx.x;
    const int64_t token = blockIdx.x;
    griddep_wait();  // the codes may come from the previous kernel on the stream
    griddep_launch_dependents();
    const float s = __ldg(scales + token);
    const uint8_t* pt = packed + token * (K / 2);
    __half* ot = out + token * K;
    for (int64_t i = (int64_t)tid * 16; i < K; i += kActThreads * 16) {
        if (!QIFT_CK_RANGE(i, 16, K)) continue;
        const uint2 p = *reinterpret_cast<const uint2*>(pt + i / 2);
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const uint32_t w = j < 8 ? p.x : p.y;
            const int sh = 4 * (j & 7);
            const int qv = (int)(w << (28 - sh)) >> 28;  // sign-extended nibble j
            v[j] = __fmul_rn(__fsub_rn(__int_as_float(0x4B400000 + qv), 12582912.0f), s);
        }
        if constexpr (LOGB == 0) {
            uint32_t h[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const __half2 t = __floats2half2_rn(v[2 * j], v[2 * j + 1]);
                h[j] = *reinterpret_cast<const uint32_t*>(&t);
            }
            *reinterpret_cast<uint4*>(ot + i) = make_uint4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<uint4*>(ot + i + 8) = make_uint4(h[4], h[5], h[6], h[7]);
        } else {
#pragma unroll
            for (int j = 0; j < 16; j += 4)
                *reinterpret_cast<float4*>(xf + i + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        }
    }
    if constexpr (LOGB > 0) {
        __syncthreads();
        rotate_token_f16<LOGB, CtaSync, float>(xf, K, c, xs, tbuf, red);
        for (int64_t i = (int64_t)tid * 8; i < K; i += kActThreads * 8)
            if (QIFT_CK_RANGE(i, 8, K)) *reinterpret_cast<uint4*>(ot + i) = *reinterpret_cast<const uint4*>(xs + i);
    }
}

template <int LOGB, bool PACK = false>
static cudaError_t launch_qa(const __half* x, int64_t tokens, int64_t K, int8_t* q, float* scales, float c,
                             cudaStream_t s) {
    const size_t smem = (size_t)((K * 2 + 15) / 16) * 16 + act_tbuf_bytes<LOGB>();
    {
        const cudaError_t e = ensure_smem(quant_acts_kernel<LOGB, PACK>, smem);
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
    return cudaLaunchKernelEx(&cfg, quant_acts_kernel<LOGB, PACK>, x, K, q, scales, c);
}

template <int LOGB>
static cudaError_t launch_dq(const uint8_t* packed, const float* scales, int64_t tokens, int64_t K, float c,
                             __half* out, cudaStream_t s) {
    const size_t smem = LOGB ? (size_t)K * 6 + act_tbuf_bytes<LOGB>() : 0;
    {
        const cudaError_t e = ensure_smem(dequant_kv_kernel<LOGB>, smem);
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
    return cudaLaunchKernelEx(&cfg, dequant_kv_kernel<LOGB>, packed, scales, K, c, out);
}

template <bool PACK>
static cudaError_t quantize_by_block(const __half* xh, int64_t tokens, int64_t n_in, int block, int8_t* q,
                                     float* scales, cudaStream_t s) {
    const float c = block ? (float)(1.0 / sqrt((double)block)) : 1.0f;
    switch (block ? ilog2(block) : 0) {
        case 0: return launch_qa<0, PACK>(xh, tokens, n_in, q, scales, c, s);
        case 1: return launch_qa<1, PACK>(xh, tokens, n_in, q, scales, c, s);
        case 2: return launch_qa<2, PACK>(xh, tokens, n_in, q, scales, c, s);
        case 3: return launch_qa<3, PACK>(xh, tokens, n_in, q, scales, c, s);
        case 4: return launch_qa<4, PACK>(xh, tokens, n_in, q, scales, c, s);
        case 5: return launch_qa<5, PACK>(xh, tokens, n_in, q, scales, c, s);
        case 6: return launch_qa<6, PACK>(xh, tokens, n_in, q, scales, c, s);
        case 7: return launch_qa<7, PACK>(xh, tokens, n_in, q, scales, c, s);
        case 8: return launch_qa<8, PACK>(xh, tokens, n_in, q, scales, c, s);
        case 9: return launch_qa<9, PACK>(xh, tokens, n_in, q, scales, c, s);
        case 10: return launch_qa<10, PACK>(xh, tokens, n_in, q, scales, c, s);
        case 11: return launch_qa<11, PACK>(xh, tokens, n_in, q, scales, c, s);
        case 12: return launch_qa<12, PACK>(xh, tokens, n_in, q, scales, c, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_quantize_kv(const void* x, int64_t tokens, int64_t n, int block, uint8_t* packed, float* scales,
                               cudaStream_t s) {
    if (tokens == 0) return cudaSuccess;
    return quantize_by_block<true>(static_cast<const __half*>(x), tokens, n, block,
                                   reinterpret_cast<int8_t*>(packed), scales, s);
}

cudaError_t launch_dequantize_kv(const uint8_t* packed, const float* scales, int64_t tokens, int64_t n, int block,
                                 void* out, cudaStream_t s) {
    if (tokens == 0) return cudaSuccess;
    __half* o = static_cast<__half*>(out);
    const float c = block ? (float)(1.0 / sqrt((double)block)) : 1.0f;
    switch (block ? ilog2(block) : 0) {
        case 0: return launch_dq<0>(packed, scales, tokens, n, c, o, s);
        case 1: return launch_dq<1>(packed, scales, tokens, n, c, o, s);
        case 2: return launch_dq<2>(packed, scales, tokens, n, c, o, s);
        case 3: return launch_dq<3>(packed, scales, tokens, n, c, o, s);
        case 4: return launch_dq<4>(packed, scales, tokens, n, c, o, s);
        case 5: return launch_dq<5>(packed, scales, tokens, n, c, o, s);
        case 6: return launch_dq<6>(packed, scales, tokens, n, c, o, s);
        case 7: return launch_dq<7>(packed, scales, tokens, n, c, o, s);
        case 8: return launch_dq<8>(packed, scales, tokens, n, c, o, s);
        case 9: return launch_dq<9>(packed, scales, tokens, n, c, o, s);
        case 10: return launch_dq<10>(packed, scales, tokens, n, c, o, s);
        case 11: return launch_dq<11>(packed, scales, tokens, n, c, o, s);
        case 12: return launch_dq<12>(packed, scales, tokens, n, c, o, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_quantize_acts(const void* x, int64_t tokens, int64_t n_in, int block, int8_t* q, float* scales,
                                 cudaStream_t s) {
    if (tokens == 0) return cudaSuccess;
    return quantize_by_block<false>(static_cast<const __half*>(x), tokens, n_in, block, q, scales, s);
}

}  // namespace qift

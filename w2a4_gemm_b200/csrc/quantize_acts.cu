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

// LOGB == 0: the input is already rotated (no stages, no multiply).
template <int LOGB>
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
    // Then the next kernel (the linear) may start its weight stream early.
    prefetch_l2_cta(x + token * K, K * 2);
    griddep_wait();
    griddep_launch_dependents();

    const float m = rotate_token_f16<LOGB>(x + token * K, K, c, xs, tbuf, red);
    int8_t* qt = q + token * K;
    if (m == 0.0f) {
        for (int64_t i = (int64_t)tid * 16; i < K; i += kActThreads * 16)
            *reinterpret_cast<uint4*>(qt + i) = make_uint4(0u, 0u, 0u, 0u);
        if (tid == 0) scales[token] = 0.0f;
        return;
    }
    const float inv = __fdiv_rn(7.0f, m);
    for (int64_t i = (int64_t)tid * 16; i < K; i += kActThreads * 16)
        *reinterpret_cast<uint4*>(qt + i) = quant16(xs + i, inv);
    if (tid == 0) scales[token] = __fdiv_rn(m, 7.0f);
}

template <int LOGB>
static cudaError_t launch_qa(const __half* x, int64_t tokens, int64_t K, int8_t* q, float* scales, float c,
                             cudaStream_t s) {
    const size_t smem = (size_t)((K * 2 + 15) / 16) * 16 + act_tbuf_bytes<LOGB>();
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

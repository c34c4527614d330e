// rotate.cu -- qift_rotate: block-diagonal normalised Walsh-Hadamard rotation, fp32 or fp16.
//
// "Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
// Inference", Abstract ("Hadamard-rotated quantization pipeline"): W' = W H_b^T offline (fp32),
// x' = H_b x online (fp16).  HBM-bound: each element is read once and written once.
#include <math.h>

#include "fwht.cuh"
#include "internal.h"

namespace qift {

constexpr int kRotThreads = 256;

template <int LOGB, typename T>
__global__ void __launch_bounds__(kRotThreads) rotate_kernel(const T* x, T* y,
                                                             int64_t n_segments, float c) {
    using S = FwhtShape<LOGB>;
    constexpr int SPC = kRotThreads / S::TPS;  // segments per CTA
    extern __shared__ float tbuf_all[];        // SPC * B floats, only when W > 1
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int seg_local = tid >> S::LOGT;
    const int ts = tid & (S::TPS - 1);
    const int64_t seg = (int64_t)blockIdx.x * SPC + seg_local;
    const bool active = seg < n_segments;

    float v[S::E];
    if (active && QIFT_CK_RANGE(seg * S::B + ts * S::E, S::E, n_segments * S::B)) {
        load_contig<S::E>(x + seg * S::B + ts * S::E, v);
    } else {
#pragma unroll
        for (int i = 0; i < S::E; ++i) v[i] = 0.0f;
    }
    float out[S::W][S::R];
    fwht_segment<LOGB>(v, ts, lane, c, tbuf_all + (S::W > 1 ? seg_local * S::B : 0), out);
    if (active) {
        T* base = y + seg * S::B + ts * S::R;
#pragma unroll
        for (int j = 0; j < S::W; ++j)
            if (QIFT_CK_RANGE(seg * S::B + ts * S::R + j * S::COL, S::R, n_segments * S::B))
                store_contig<S::R>(base + j * S::COL, out[j]);
    }
}

template <int LOGB, typename T>
static cudaError_t launch_rotate_t(const T* x, T* y, int64_t n_segments, float c, cudaStream_t s) {
    using S = FwhtShape<LOGB>;
    constexpr int SPC = kRotThreads / S::TPS;
    const size_t smem = S::W > 1 ? (size_t)SPC * S::B * sizeof(float) : 0;
    const int64_t blocks = (n_segments + SPC - 1) / SPC;
    if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
    if (blocks == 0) return cudaSuccess;
    {
        const cudaError_t e = ensure_smem(rotate_kernel<LOGB, T>, smem);
        if (e != cudaSuccess) return e;
    }
    rotate_kernel<LOGB, T><<<(unsigned)blocks, kRotThreads, smem, s>>>(x, y, n_segments, c);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t dispatch_rotate(const T* x, T* y, int64_t n_segments, int logb, float c, cudaStream_t s) {
    switch (logb) {
        case 1: return launch_rotate_t<1, T>(x, y, n_segments, c, s);
        case 2: return launch_rotate_t<2, T>(x, y, n_segments, c, s);
        case 3: return launch_rotate_t<3, T>(x, y, n_segments, c, s);
        case 4: return launch_rotate_t<4, T>(x, y, n_segments, c, s);
        case 5: return launch_rotate_t<5, T>(x, y, n_segments, c, s);
        case 6: return launch_rotate_t<6, T>(x, y, n_segments, c, s);
        case 7: return launch_rotate_t<7, T>(x, y, n_segments, c, s);
        case 8: return launch_rotate_t<8, T>(x, y, n_segments, c, s);
        case 9: return launch_rotate_t<9, T>(x, y, n_segments, c, s);
        case 10: return launch_rotate_t<10, T>(x, y, n_segments, c, s);
        case 11: return launch_rotate_t<11, T>(x, y, n_segments, c, s);
        case 12: return launch_rotate_t<12, T>(x, y, n_segments, c, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_rotate(const void* x, void* y, bool f16, int64_t rows, int64_t n, int block, cudaStream_t s) {
    const int logb = ilog2(block);
    const int64_t n_segments = rows * (n / block);
    // Normalisation constant: binary64 1/sqrt(b) rounded once to binary32.
    const float c = (float)(1.0 / sqrt((double)block));
    if (f16)
        return dispatch_rotate<__half>(static_cast<const __half*>(x), static_cast<__half*>(y), n_segments, logb, c, s);
    return dispatch_rotate<float>(static_cast<const float*>(x), static_cast<float*>(y), n_segments, logb, c, s);
}

}  // namespace qift

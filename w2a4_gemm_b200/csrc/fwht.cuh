// fwht.cuh -- register/shuffle/shared-memory block Walsh-Hadamard transform for sm_100a.
//
// "Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
// Inference", Abstract: weights and activations are Hadamard-rotated.  Every length-B
// segment is multiplied by the normalised Sylvester matrix H_B / sqrt(B).
//
// The fp32 butterfly stages run in the fixed order h = 1, 2, ..., B/2 with (u, v) -> (u+v, u-v)
// and one multiply by the normalisation constant at the end, so every output is the same
// sequence of IEEE operations wherever a stage runs:
//   index bits [0, LOGE)            live in a thread's registers       -> register butterflies
//   next LANE_BITS bits (<= 5)      live in the lanes of one warp      -> __shfl_xor butterflies
//   top WARP_BITS bits (B > 512)    live in different warps            -> one shared-memory
//                                   transpose brings them into registers for the last stages.
// A segment is owned by TPS = B / E consecutive threads (E = min(B, 16) elements each).
#pragma once

#include "common.cuh"

namespace qift {

template <int LOGB>
struct FwhtShape {
    static constexpr int B = 1 << LOGB;
    static constexpr int LOGE = LOGB < 4 ? LOGB : 4;
    static constexpr int E = 1 << LOGE;           // elements per thread
    static constexpr int LOGT = LOGB - LOGE;      // log2 threads per segment
    static constexpr int TPS = 1 << LOGT;
    static constexpr int LANE_BITS = LOGT < 5 ? LOGT : 5;
    static constexpr int WARP_BITS = LOGT - LANE_BITS;
    static constexpr int W = 1 << WARP_BITS;      // warps per segment
    static constexpr int R = E / W;               // groups per thread after the transpose
    static constexpr int COL = B / W;             // stride of the warp index bits
    static_assert(LOGB >= 1 && LOGB <= 12, "block must be 2..4096");
};

template <int E>
__device__ __forceinline__ void reg_stages(float (&v)[E]) {
#pragma unroll
    for (int h = 1; h < E; h <<= 1) {
#pragma unroll
        for (int i = 0; i < E; ++i) {
            if (i & h) continue;
            const float a = v[i], b = v[i + h];
            v[i] = __fadd_rn(a, b);
            v[i + h] = __fsub_rn(a, b);
        }
    }
}

// Butterflies across lanes: the lane without bit m holds u, the lane with it holds v; the
// lower lane keeps u + v, the upper one u - v.  Both are fma(sgn, own, partner) with sgn = +1
// or -1: sgn * own is exact, so the one rounding gives the same bits as the add or subtract.
template <int E, int LANE_BITS>
__device__ __forceinline__ void lane_stages(float (&v)[E], int lane) {
#pragma unroll
    for (int j = 0; j < LANE_BITS; ++j) {
        const int m = 1 << j;
        const float sgn = (lane & m) ? -1.0f : 1.0f;
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const float p = __shfl_xor_sync(0xffffffffu, v[i], m);
            v[i] = __fmaf_rn(sgn, v[i], p);
        }
    }
}

// ---- vector loads / stores of E contiguous elements -----------------------------------
template <int E>
__device__ __forceinline__ void load_contig(const float* __restrict__ p, float (&v)[E]) {
    if constexpr (E >= 4) {
#pragma unroll
        for (int i = 0; i < E; i += 4) {
            const float4 t = *reinterpret_cast<const float4*>(p + i);
            v[i] = t.x; v[i + 1] = t.y; v[i + 2] = t.z; v[i + 3] = t.w;
        }
    } else {
        const float2 t = *reinterpret_cast<const float2*>(p);
        v[0] = t.x; v[1] = t.y;
    }
}

template <int E>
__device__ __forceinline__ void load_contig(const __half* __restrict__ p, float (&v)[E]) {
    if constexpr (E >= 8) {
#pragma unroll
        for (int i = 0; i < E; i += 8) {
            const uint4 t = *reinterpret_cast<const uint4*>(p + i);
            const __half2* h = reinterpret_cast<const __half2*>(&t);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __half22float2(h[j]);
                v[i + 2 * j] = f.x; v[i + 2 * j + 1] = f.y;
            }
        }
    } else if constexpr (E == 4) {
        const uint2 t = *reinterpret_cast<const uint2*>(p);
        const __half2* h = reinterpret_cast<const __half2*>(&t);
        const float2 a = __half22float2(h[0]), b = __half22float2(h[1]);
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    } else {
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(p));
        v[0] = a.x; v[1] = a.y;
    }
}

template <int N>
__device__ __forceinline__ void store_contig(float* __restrict__ p, const float* v) {
    if constexpr (N >= 4) {
#pragma unroll
        for (int i = 0; i < N; i += 4)
            *reinterpret_cast<float4*>(p + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    } else if constexpr (N == 2) {
        *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
    } else {
        p[0] = v[0];
    }
}

// Rounds each value to binary16 (nearest even).
template <int N>
__device__ __forceinline__ void store_contig(__half* __restrict__ p, const float* v) {
    if constexpr (N >= 8) {
#pragma unroll
        for (int i = 0; i < N; i += 8) {
            uint4 t;
            __half2* h = reinterpret_cast<__half2*>(&t);
#pragma unroll
            for (int j = 0; j < 4; ++j) h[j] = __floats2half2_rn(v[i + 2 * j], v[i + 2 * j + 1]);
            *reinterpret_cast<uint4*>(p + i) = t;
        }
    } else if constexpr (N == 4) {
        uint2 t;
        __half2* h = reinterpret_cast<__half2*>(&t);
        h[0] = __floats2half2_rn(v[0], v[1]);
        h[1] = __floats2half2_rn(v[2], v[3]);
        *reinterpret_cast<uint2*>(p) = t;
    } else if constexpr (N == 2) {
        *reinterpret_cast<__half2*>(p) = __floats2half2_rn(v[0], v[1]);
    } else {
        p[0] = __float2half_rn(v[0]);
    }
}

// Transform one segment owned by TPS consecutive threads.  On entry v holds the thread's E
// contiguous inputs (elements ts*E .. ts*E+E-1).  On exit out[j][r] is the normalised output
// element ts*R + r + j*COL, i.e. W runs of R contiguous elements (one run of E when W == 1).
// `tbuf` is this segment's B-float shared buffer (only used when W > 1); every thread that
// Bar synchronises must call this function the same number of times, and the caller must
// synchronise them again before reusing tbuf.
template <int LOGB, typename Bar = CtaSync>
__device__ __forceinline__ void fwht_segment(float (&v)[FwhtShape<LOGB>::E], int ts, int lane, float c,
                                             float* tbuf,
                                             float (&out)[FwhtShape<LOGB>::W][FwhtShape<LOGB>::R]) {
    using S = FwhtShape<LOGB>;
    reg_stages<S::E>(v);
    lane_stages<S::E, S::LANE_BITS>(v, lane);
    if constexpr (S::W == 1) {
#pragma unroll
        for (int i = 0; i < S::E; ++i) out[0][i] = __fmul_rn(v[i], c);
    } else {
#pragma unroll
        for (int i = 0; i < S::E; i += 4)
            *reinterpret_cast<float4*>(tbuf + ts * S::E + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        Bar::sync();
#pragma unroll
        for (int r = 0; r < S::R; ++r) {
            float u[S::W];
#pragma unroll
            for (int j = 0; j < S::W; ++j) u[j] = tbuf[ts * S::R + r + j * S::COL];
            reg_stages<S::W>(u);
#pragma unroll
            for (int j = 0; j < S::W; ++j) out[j][r] = __fmul_rn(u[j], c);
        }
    }
}

}  // namespace qift

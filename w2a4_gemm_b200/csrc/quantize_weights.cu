// quantize_weights.cu -- qift_quantize_weights: per-output-channel MSE scale search, nearest-
// level encoding and 2-bit packing for the Qift {+-1,+-3}, power-of-two {+-1,+-4} and
// standard {-2,-1,0,+1} level sets.
//
// "Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
// Inference", Abstract: a fixed two-bit code-to-level mapping with the standard per-channel
// scale (no zero point, no group grid).
//
// One CTA owns a few output rows, staged in shared memory; the thread of (row, candidate g)
// evaluates scale s_g by walking the row in index order and accumulating the fp32 squared
// error into fp64 -- the fixed order makes the argmin reproducible bit for bit.  This pass is
// ALU-bound (G candidates x K elements per row), not HBM-bound; the fp32 -> fp64 widening, one
// per evaluation, runs on the conversion unit, which sets the pace.
//
// Level thresholds are compared in fp32 against products rounded DOWN: for a float x and a
// real threshold tau = c*s, x > tau exactly when x > RD(c*s), because no float lies strictly
// between RD(c*s) and RU(c*s).  That decides every weight exactly as an exact comparison would.
#include <math.h>

#include <algorithm>

#include "fwht.cuh"
#include "internal.h"

namespace qift {

template <int SET>
struct Encoder {
    float s, thr1, thr2, l_in, l_out;
    float thr[7];  // W4: midpoints (j + 0.5) s rounded down, j = 0..6
    int z;         // asymmetric: the zero point
    __device__ __forceinline__ explicit Encoder(float s_, int z_ = 0) : s(s_), z(z_) {
        if constexpr (SET == kSetAsym) {
            // (c - z) * s: nothing to precompute; the code comes from one IEEE division
        } else if constexpr (SET == kSetInt4) {        // levels {-7..7} s; midpoints (j + 0.5) s
#pragma unroll
            for (int j = 0; j < 7; ++j) thr[j] = __fmul_rd((float)j + 0.5f, s);
        } else if constexpr (SET == kSetQift) {  // levels +-0.5 s, +-1.5 s; midpoint s
            thr1 = s;
            l_in = __fmul_rn(0.5f, s);
            l_out = __fmul_rn(1.5f, s);
        } else if constexpr (SET == kSetPot) {  // levels +-s, +-4 s; midpoint 2.5 s
            thr1 = __fmul_rd(2.5f, s);
            l_in = s;
            l_out = __fmul_rn(4.0f, s);
        } else {                                // levels -2s, -s, 0, s; midpoints -1.5s, -0.5s, 0.5s
            thr1 = __fmul_rd(1.5f, s);
            thr2 = __fmul_rd(0.5f, s);
        }
    }
    // W4: the level's magnitude -- the number of midpoints strictly below |w| (ties stay low).
    __device__ __forceinline__ int w4_mag(float a) const {
        int j = 0;
#pragma unroll
        for (int i = 0; i < 7; ++i) j += a > thr[i] ? 1 : 0;
        return j;
    }
    // Code: 0..3 in increasing level order, or (W4) the level's two's-complement nibble.  Ties go
    // to the smaller magnitude; w >= 0 is positive.
    __device__ __forceinline__ uint32_t code(float w) const {
        if constexpr (SET == kSetAsym) {  // clamp(rint(w / s) + z, 0, 3); c = z when s = 0
            if (!(s > 0.0f)) return (uint32_t)z;
            const int c = (int)rintf(__fdiv_rn(w, s)) + z;
            return (uint32_t)(c < 0 ? 0 : (c > 3 ? 3 : c));
        } else if constexpr (SET == kSetInt4) {
            const int j = w4_mag(fabsf(w));
            return (uint32_t)(w >= 0.0f ? j : -j) & 0xFu;
        } else if constexpr (SET == kSetStd) {
            const float nw = -w;
            if (nw > thr1) return 0u;   // w < -1.5 s
            if (nw > thr2) return 1u;   // w < -0.5 s
            if (w > thr2) return 3u;    // w > +0.5 s
            return 2u;
        } else {
            const bool outer = fabsf(w) > thr1;
            return w >= 0.0f ? (outer ? 3u : 2u) : (outer ? 0u : 1u);
        }
    }
    // Squared reconstruction error of w, in fp32, for its code.
    __device__ __forceinline__ float sq_err(float w) const {
        float e;
        if constexpr (SET == kSetAsym) {
            e = __fsub_rn(w, __fmul_rn((float)((int)code(w) - z), s));
        } else if constexpr (SET == kSetInt4) {
            const float a = fabsf(w);
            // (float)j by the exact magic-number add (j <= 7), off the conversion unit
            const float jf = __fsub_rn(__int_as_float(0x4B400000 + w4_mag(a)), 12582912.0f);
            e = __fsub_rn(a, __fmul_rn(jf, s));
        } else if constexpr (SET == kSetStd) {
            const float l = __fmul_rn((float)((int)code(w) - 2), s);
            e = __fsub_rn(w, l);
        } else {
            const float a = fabsf(w);
            e = __fsub_rn(a, a > thr1 ? l_out : l_in);
        }
        return __fmul_rn(e, e);
    }
};

constexpr int kQwMaxRows = 4;   // rows per CTA
constexpr int kQwMaxG = 256;     // candidates per row (API limit)

// Block Walsh-Hadamard of every length-2^logb segment of the staged rows, in place (the fused
// offline rotation): stages h = 1, 2, ..., b/2 of (lo + hi, lo - hi) in fp32, then one
// multiply by c -- the operations and the order of qift_rotate, so the rows come out the same
// bits as W H_b^T.
//
// b <= 512: a segment lives in the registers of b/16 lanes of one warp (fwht_segment: register
// and shuffle stages, no barrier).  Every lane of a warp runs each pass, lanes past the last
// segment on zeros, so the shuffles always see the whole warp.
template <int LOGB>
__device__ __forceinline__ void fwht_rows_regs(float* ws, int n_seg, float c) {
    using S = FwhtShape<LOGB>;
    static_assert(S::W == 1, "one warp per segment at most");
    constexpr int SPW = 32 / S::TPS;  // segments per warp pass
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int ts = lane & (S::TPS - 1), sl = lane / S::TPS;
    for (int base = warp * SPW; base < n_seg; base += nwarps * SPW) {  // warp-uniform
        const int seg = base + sl;
        const bool active = seg < n_seg;
        float v[S::E];
        if (active) {
            load_contig<S::E>(ws + (size_t)seg * S::B + ts * S::E, v);
        } else {
#pragma unroll
            for (int i = 0; i < S::E; ++i) v[i] = 0.0f;
        }
        float out[1][S::R];
        fwht_segment<LOGB>(v, ts, lane, c, nullptr, out);
        if (active) store_contig<S::R>(ws + (size_t)seg * S::B + ts * S::R, out[0]);
    }
}

// b > 512: one barrier per stage over the whole CTA.
__device__ __forceinline__ void fwht_rows_smem(float* ws, int rows, int K, int logb, float c) {
    const int pairs = rows * K / 2;
    for (int st = 0; st < logb; ++st) {
        const int h = 1 << st;
        const bool last = st == logb - 1;
        for (int p = threadIdx.x; p < pairs; p += blockDim.x) {
            const int lo = ((p >> st) << (st + 1)) | (p & (h - 1));  // pairs never cross a block
            const float a = ws[lo], b = ws[lo + h];
            float u = __fadd_rn(a, b), v = __fsub_rn(a, b);
            if (last) {
                u = __fmul_rn(u, c);
                v = __fmul_rn(v, c);
            }
            ws[lo] = u;
            ws[lo + h] = v;
        }
        __syncthreads();
    }
}

__device__ __forceinline__ void fwht_rows_in_smem(float* ws, int rows, int K, int logb, float c) {
    const int n_seg = (rows * K) >> logb;
    switch (logb) {
        case 1: fwht_rows_regs<1>(ws, n_seg, c); break;
        case 2: fwht_rows_regs<2>(ws, n_seg, c); break;
        case 3: fwht_rows_regs<3>(ws, n_seg, c); break;
        case 4: fwht_rows_regs<4>(ws, n_seg, c); break;
        case 5: fwht_rows_regs<5>(ws, n_seg, c); break;
        case 6: fwht_rows_regs<6>(ws, n_seg, c); break;
        case 7: fwht_rows_regs<7>(ws, n_seg, c); break;
        case 8: fwht_rows_regs<8>(ws, n_seg, c); break;
        case 9: fwht_rows_regs<9>(ws, n_seg, c); break;
        default: fwht_rows_smem(ws, rows, K, logb, c); return;
    }
    __syncthreads();
}

// One CTA owns R <= 4 output rows, staged together in shared memory, so that R x G (row,
// candidate) pairs -- one per thread -- fill whole warps (G = 100 alone leaves a 128-thread CTA's
// last warp with 4 busy lanes, and the bottleneck, the conversion unit, is paid per warp).
// ROT: the rows are raw weights, rotated here first by 2^logb-point blocks (a1 and a2 in one
// pass).
template <int SET, bool ROT>
__global__ void __launch_bounds__(1024) quant_weights_kernel(const float* __restrict__ w, int64_t n_out, int64_t K,
                                                             int R, int G, double lo, double hi,
                                                             uint32_t* __restrict__ codes, float* __restrict__ scales,
                                                             int32_t* __restrict__ zeros, double* __restrict__ row_mse,
                                                             int logb, float c) {
    extern __shared__ __align__(16) float ws[];  // R rows of K floats
    __shared__ float cand[kQwMaxRows * kQwMaxG];
    __shared__ double mse[kQwMaxRows * kQwMaxG];
    __shared__ float red[kQwMaxRows][32];
    __shared__ float red_lo[kQwMaxRows][32];    // asymmetric: min(w, 0) partials
    __shared__ int8_t zc[kQwMaxRows * kQwMaxG];  // asymmetric: each candidate's zero point
    __shared__ int best_s[kQwMaxRows];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nthr = blockDim.x, nwarps = nthr >> 5;
    const int64_t row0 = (int64_t)blockIdx.x * R;
    const int rows = (int)min((int64_t)R, n_out - row0);

    // Stage the rows (rotating them when asked) and find each row's max |w|.
    if constexpr (ROT) {
        for (int r = 0; r < rows; ++r) {
            const float* wr = w + (row0 + r) * K;
            for (int64_t i = (int64_t)tid * 4; i < K; i += nthr * 4)
                if (QIFT_CK_RANGE((row0 + r) * K + i, 4, n_out * K))
                    *reinterpret_cast<float4*>(ws + r * K + i) = *reinterpret_cast<const float4*>(wr + i);
        }
        __syncthreads();
        fwht_rows_in_smem(ws, rows, (int)K, logb, c);
    }
    // (Asymmetric set: the row's max(w, 0) in m and min(w, 0) in mn instead.)
    float m[kQwMaxRows], mn[kQwMaxRows];
#pragma unroll
    for (int r = 0; r < kQwMaxRows; ++r) {
        m[r] = 0.0f;
        mn[r] = 0.0f;
        if (r < rows) {
            const float* wr = w + (row0 + r) * K;
            for (int64_t i = (int64_t)tid * 4; i < K; i += nthr * 4) {
                float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if constexpr (ROT) {
                    v = *reinterpret_cast<const float4*>(ws + r * K + i);
                } else {
                    if (QIFT_CK_RANGE((row0 + r) * K + i, 4, n_out * K)) v = *reinterpret_cast<const float4*>(wr + i);
                    *reinterpret_cast<float4*>(ws + r * K + i) = v;
                }
                if constexpr (SET == kSetAsym) {
                    m[r] = fmaxf(m[r], fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
                    mn[r] = fminf(mn[r], fminf(fminf(v.x, v.y), fminf(v.z, v.w)));
                } else {
                    m[r] = fmaxf(m[r], fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            m[r] = fmaxf(m[r], __shfl_xor_sync(0xffffffffu, m[r], o));
            if constexpr (SET == kSetAsym) mn[r] = fminf(mn[r], __shfl_xor_sync(0xffffffffu, mn[r], o));
        }
        if (lane == 0) {
            red[r][warp] = m[r];
            red_lo[r][warp] = mn[r];
        }
    }
    __syncthreads();
    if (tid < kQwMaxRows) {
        float v = 0.0f, u = 0.0f;
        for (int i = 0; i < nwarps; ++i) {
            v = fmaxf(v, red[tid][i]);
            u = fminf(u, red_lo[tid][i]);
        }
        red[tid][0] = v;
        red_lo[tid][0] = u;
    }
    __syncthreads();

    // Candidate scales, binary64 in the order lo + ((hi - lo) * k) / (G - 1), then * m / L.
    // Asymmetric set: s = (f * (max - min)) / 3, and the zero point z = rint(-(f * min) / s),
    // ties to even, clamped to [0, 3] (0 when s = 0).
    const double lambda = SET == kSetQift ? 1.5 : (SET == kSetPot ? 4.0 : (SET == kSetInt4 ? 7.0 : 2.0));
    for (int f = tid; f < rows * G; f += nthr) {
        const int r = f / G, g = f - r * G;
        const double fr = __dadd_rn(lo, __ddiv_rn(__dmul_rn(__dsub_rn(hi, lo), (double)g), (double)(G - 1)));
        if constexpr (SET == kSetAsym) {
            const double range = __dsub_rn((double)red[r][0], (double)red_lo[r][0]);
            const float sv = __double2float_rn(__ddiv_rn(__dmul_rn(fr, range), 3.0));
            int z = 0;
            if (sv > 0.0f) {
                z = __double2int_rn(__ddiv_rn(-__dmul_rn(fr, (double)red_lo[r][0]), (double)sv));
                z = z < 0 ? 0 : (z > 3 ? 3 : z);
            }
            cand[r * kQwMaxG + g] = sv;
            zc[r * kQwMaxG + g] = (int8_t)z;
        } else {
            cand[r * kQwMaxG + g] = __double2float_rn(__ddiv_rn(__dmul_rn(fr, (double)red[r][0]), lambda));
        }
    }
    __syncthreads();

    // MSE of every (row, candidate): sequential over the row, fp32 squared error widened to fp64.
    for (int f = tid; f < rows * G; f += nthr) {
        const int r = f / G, g = f - r * G;
        const Encoder<SET> enc(cand[r * kQwMaxG + g], SET == kSetAsym ? (int)zc[r * kQwMaxG + g] : 0);
        double acc = 0.0;
        const float4* w4 = reinterpret_cast<const float4*>(ws + r * K);
        for (int64_t i = 0; i < K / 4; ++i) {
            const float4 v = w4[i];
            acc = __dadd_rn(acc, (double)enc.sq_err(v.x));
            acc = __dadd_rn(acc, (double)enc.sq_err(v.y));
            acc = __dadd_rn(acc, (double)enc.sq_err(v.z));
            acc = __dadd_rn(acc, (double)enc.sq_err(v.w));
        }
        mse[r * kQwMaxG + g] = acc;
    }
    __syncthreads();

    // Argmin per row, first index on ties.
    if (tid < rows) {
        const double* mr = mse + tid * kQwMaxG;
        int b = 0;
        double bv = mr[0];
        for (int g = 1; g < G; ++g)
            if (mr[g] < bv) { bv = mr[g]; b = g; }
        best_s[tid] = b;
    }
    __syncthreads();

    // Encode and pack: word j holds the codes of inputs CPW*j .. CPW*j + CPW-1 -- 16 codes of 2
    // bits, least significant first, or (W4) 8 nibbles with byte i holding inputs i (low) and
    // i + 4 (high), so input p of the word sits at bit 8 (p % 4) + 4 (p / 4).
    constexpr int CPW = SET == kSetInt4 ? 8 : 16;
    auto shift = [](int p) { return SET == kSetInt4 ? 8 * (p & 3) + 4 * (p >> 2) : 2 * p; };
    for (int r = 0; r < rows; ++r) {
        const int b = best_s[r];
        const float sr = cand[r * kQwMaxG + b];
        const Encoder<SET> enc(sr, SET == kSetAsym ? (int)zc[r * kQwMaxG + b] : 0);
        uint32_t* crow = codes + (row0 + r) * (K / CPW);
        for (int64_t j = tid; j < K / CPW; j += nthr) {
            const float4* w4 = reinterpret_cast<const float4*>(ws + r * K + j * CPW);
            uint32_t word = 0;
#pragma unroll
            for (int v4 = 0; v4 < CPW / 4; ++v4) {
                const float4 v = w4[v4];
                word |= enc.code(v.x) << shift(4 * v4);
                word |= enc.code(v.y) << shift(4 * v4 + 1);
                word |= enc.code(v.z) << shift(4 * v4 + 2);
                word |= enc.code(v.w) << shift(4 * v4 + 3);
            }
            if (QIFT_CK_RANGE((row0 + r) * (K / CPW) + j, 1, n_out * (K / CPW))) crow[j] = word;
        }
        if (tid == 0 && QIFT_CK_RANGE(row0 + r, 1, n_out)) {
            scales[row0 + r] = SET == kSetQift ? __fmul_rn(sr, 0.5f) : sr;
            if constexpr (SET == kSetAsym) zeros[row0 + r] = zc[r * kQwMaxG + b];
            if (row_mse) row_mse[row0 + r] = __ddiv_rn(mse[r * kQwMaxG + b], (double)K);
        }
    }
}

template <int SET>
static cudaError_t launch_qw(const float* w, int64_t n_out, int64_t n_in, int G, double lo, double hi,
                             uint32_t* codes, float* scales, int32_t* zeros, double* row_mse, int block,
                             cudaStream_t s) {
    // As many rows per CTA as fit in ~100 KB of shared memory (so several CTAs share an SM).
    int R = (int)std::min<int64_t>(kQwMaxRows, std::max<int64_t>(1, (100 * 1024) / (n_in * 4)));
    const int threads = std::max(128, std::min(1024, (R * G + 31) / 32 * 32));
    const size_t smem = (size_t)R * n_in * sizeof(float);
    const int64_t grid = (n_out + R - 1) / R;
    if (block) {
        const cudaError_t e = ensure_smem(quant_weights_kernel<SET, true>, smem);
        if (e != cudaSuccess) return e;
        // Normalisation constant as in qift_rotate: binary64 1/sqrt(b) rounded once to binary32.
        const float c = (float)(1.0 / sqrt((double)block));
        quant_weights_kernel<SET, true><<<(unsigned)grid, threads, smem, s>>>(w, n_out, n_in, R, G, lo, hi, codes,
                                                                              scales, zeros, row_mse, ilog2(block), c);
        return cudaGetLastError();
    }
    const cudaError_t e = ensure_smem(quant_weights_kernel<SET, false>, smem);
    if (e != cudaSuccess) return e;
    quant_weights_kernel<SET, false><<<(unsigned)grid, threads, smem, s>>>(w, n_out, n_in, R, G, lo, hi, codes,
                                                                           scales, zeros, row_mse, 0, 1.0f);
    return cudaGetLastError();
}

cudaError_t launch_quantize_weights(const float* w, int64_t n_out, int64_t n_in, int set, int G, double lo,
                                    double hi, uint32_t* codes, float* scales, double* row_mse, cudaStream_t s,
                                    int block) {
    if (n_out == 0) return cudaSuccess;
    switch (set) {
        case kSetQift: return launch_qw<kSetQift>(w, n_out, n_in, G, lo, hi, codes, scales, nullptr, row_mse, block, s);
        case kSetPot: return launch_qw<kSetPot>(w, n_out, n_in, G, lo, hi, codes, scales, nullptr, row_mse, block, s);
        case kSetStd: return launch_qw<kSetStd>(w, n_out, n_in, G, lo, hi, codes, scales, nullptr, row_mse, block, s);
        case kSetInt4: return launch_qw<kSetInt4>(w, n_out, n_in, G, lo, hi, codes, scales, nullptr, row_mse, block, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_quantize_weights_asym(const float* w, int64_t n_out, int64_t n_in, int G, double lo, double hi,
                                         uint32_t* codes, float* scales, int32_t* zeros, double* row_mse,
                                         cudaStream_t s) {
    if (n_out == 0) return cudaSuccess;
    return launch_qw<kSetAsym>(w, n_out, n_in, G, lo, hi, codes, scales, zeros, row_mse, 0, s);
}

}  // namespace qift

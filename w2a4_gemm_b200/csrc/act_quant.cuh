// act_quant.cuh -- device pieces of the activation path shared by qift_quantize_acts and the
// fused decode kernel: block Walsh-Hadamard rotation of one token into shared memory (fp32
// stages, one rounding to fp16) with its max |x'|, and symmetric INT4 quantization.
//
// "Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
// Inference", Abstract: rotated W2A4 inference (4-bit activations).
#pragma once

#include "fwht.cuh"

namespace qift {

// Every function below runs on 256 threads: the whole CTA (Bar = CtaSync) or threads 0..255 of
// a larger one (Bar = GroupSync<256>).
constexpr int kActThreads = 256;

template <typename Bar = CtaSync>
__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    Bar::sync();
    if (warp == 0) {
        v = lane < (kActThreads / 32) ? red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[0] = v;
    }
    Bar::sync();
    const float m = red[0];
    Bar::sync();  // red may be reused right after
    return m;
}

// 4096-point rotation by one CTA: 4096 = 16 x 16 x 16, so three rounds of in-register 16-point
// butterflies (index bits 0-3, then 4-7, then 8-11) joined by two shared-memory transposes
// replace the warp-shuffle stages.  The stages still run in the order h = 1, 2, ..., 2048, so
// every output is the same sequence of fp32 operations.  The buffer is padded by 16 floats per
// 256 so that both transposes read conflict-free.
__host__ __device__ constexpr int tpad4096(int a) { return a + ((a >> 8) << 4); }
constexpr size_t kTbuf4096Bytes = (size_t)(tpad4096(4095) + 1) * sizeof(float);

// Shared memory the rotation needs besides the token itself (transpose buffer).
template <int LOGB>
__host__ __device__ constexpr size_t act_tbuf_bytes() {
    if constexpr (LOGB == 0) {
        return 0;
    } else if constexpr (LOGB == 12) {
        return kTbuf4096Bytes;
    } else {
        using S = FwhtShape<LOGB>;
        return S::W > 1 ? (size_t)(kActThreads / S::TPS) * S::B * sizeof(float) : 0;
    }
}

// R contiguous fp16 values (R even) from R/2 packed pairs.
template <int R>
__device__ __forceinline__ void store_half2s(__half* __restrict__ p, const __half2 (&h)[R / 2]) {
    if constexpr (R >= 8) {
#pragma unroll
        for (int i = 0; i < R / 2; i += 4) {
            uint4 t;
            t.x = *reinterpret_cast<const uint32_t*>(&h[i]);
            t.y = *reinterpret_cast<const uint32_t*>(&h[i + 1]);
            t.z = *reinterpret_cast<const uint32_t*>(&h[i + 2]);
            t.w = *reinterpret_cast<const uint32_t*>(&h[i + 3]);
            *reinterpret_cast<uint4*>(p + 2 * i) = t;
        }
    } else if constexpr (R == 4) {
        uint2 t;
        t.x = *reinterpret_cast<const uint32_t*>(&h[0]);
        t.y = *reinterpret_cast<const uint32_t*>(&h[1]);
        *reinterpret_cast<uint2*>(p) = t;
    } else {
        *reinterpret_cast<__half2*>(p) = h[0];
    }
}

// Rotate one token (K values at xt, fp16 or fp32, K % 16 == 0) into xs as fp16 and return
// max |x'|.  LOGB == 0: the token is already rotated (fp16 input only, copied as is).  `red`
// holds kActThreads/32 floats.
template <int LOGB, typename Bar = CtaSync, typename InT = __half>
__device__ __forceinline__ float rotate_token_f16(const InT* __restrict__ xt, int64_t K, float c, __half* xs,
                                                  float* tbuf, float* red) {
    static_assert(LOGB > 0 || sizeof(InT) == 2, "the copy path takes fp16 input");
    const int tid = threadIdx.x, lane = tid & 31;
    // max |x'| is taken on the fp16 values themselves, two at a time: a max does not round.
    __half2 amax2 = __float2half2_rn(0.0f);
    if constexpr (LOGB == 0) {
        for (int64_t i = (int64_t)tid * 8; i < K; i += kActThreads * 8) {
            const uint4 t = QIFT_CK_RANGE(i, 8, K) ? *reinterpret_cast<const uint4*>(xt + i) : make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(xs + i) = t;
            const __half2* h = reinterpret_cast<const __half2*>(&t);
#pragma unroll
            for (int j = 0; j < 4; ++j) amax2 = __hmax2(amax2, __habs2(h[j]));
        }
    } else if constexpr (LOGB == 12) {
        static_assert(kActThreads == 256, "one 16-value column per thread");
        const int lo = tid & 15, hi = tid >> 4;
        for (int64_t seg = 0; seg < K / 4096; ++seg) {
            float v[16];
            if (QIFT_CK_RANGE(seg * 4096 + tid * 16, 16, K)) {
                load_contig<16>(xt + seg * 4096 + tid * 16, v);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = 0.0f;
            }
            reg_stages<16>(v);  // h = 1 .. 8
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<float4*>(tbuf + tpad4096(16 * tid + i)) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            Bar::sync();
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = tbuf[tpad4096(lo + 16 * i + 256 * hi)];
            reg_stages<16>(v);  // h = 16 .. 128
#pragma unroll
            for (int i = 0; i < 16; ++i) tbuf[tpad4096(lo + 16 * i + 256 * hi)] = v[i];  // same slots as read
            Bar::sync();
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = tbuf[tpad4096(tid + 256 * i)];
            reg_stages<16>(v);  // h = 256 .. 2048
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                const __half2 h = __floats2half2_rn(__fmul_rn(v[i], c), __fmul_rn(v[i + 1], c));
                amax2 = __hmax2(amax2, __habs2(h));
                xs[seg * 4096 + tid + 256 * i] = __low2half(h);
                xs[seg * 4096 + tid + 256 * (i + 1)] = __high2half(h);
            }
            Bar::sync();  // tbuf is reused by the next segment
        }
    } else {
        using S = FwhtShape<LOGB>;
        constexpr int SPC = kActThreads / S::TPS;
        const int seg_local = tid >> S::LOGT;
        const int ts = tid & (S::TPS - 1);
        const int64_t nseg = K / S::B;
        for (int64_t p = 0; p < nseg; p += SPC) {
            const int64_t seg = p + seg_local;
            const bool active = seg < nseg;
            float v[S::E];
            if (active && QIFT_CK_RANGE(seg * S::B + ts * S::E, S::E, K)) {
                load_contig<S::E>(xt + seg * S::B + ts * S::E, v);
            } else {
#pragma unroll
                for (int i = 0; i < S::E; ++i) v[i] = 0.0f;
            }
            float out[S::W][S::R];
            fwht_segment<LOGB, Bar>(v, ts, lane, c, tbuf + (S::W > 1 ? seg_local * S::B : 0), out);
            if (active) {
#pragma unroll
                for (int j = 0; j < S::W; ++j) {
                    __half2 hv[S::R / 2];
#pragma unroll
                    for (int r = 0; r < S::R; r += 2) {
                        hv[r / 2] = __floats2half2_rn(out[j][r], out[j][r + 1]);
                        amax2 = __hmax2(amax2, __habs2(hv[r / 2]));
                    }
                    store_half2s<S::R>(xs + seg * S::B + ts * S::R + j * S::COL, hv);
                }
            }
            if constexpr (S::W > 1) Bar::sync();  // tbuf is reused by the next pass
        }
    }
    Bar::sync();
    const float2 a = __half22float2(amax2);
    return block_max<Bar>(fmaxf(a.x, a.y), red);
}

// Sixteen fp16 values -> sixteen INT4 codes in int8 bytes, natural order:
// clamp(rint_even(x * inv), -7, 7), one fp32 multiply per value.  inv = 7/m (IEEE division).
// rint is the magic-number add on the fp32 pipe: t = x * inv + 1.5 * 2^23 is exact and its
// low byte is the code in two's complement, so byte permutes gather the codes.  The clamp never
// binds: |x| <= m and inv <= (7/m)(1 + 2^-24), so |x * inv| < 7.5 and the rounded value is at
// most 7 in magnitude.
__device__ __forceinline__ uint4 quant16(const __half* xs16, float inv) {
    const uint4 a = *reinterpret_cast<const uint4*>(xs16);
    const uint4 b = *reinterpret_cast<const uint4*>(xs16 + 8);
    const __half2* ha = reinterpret_cast<const __half2*>(&a);
    const __half2* hb = reinterpret_cast<const __half2*>(&b);
    uint32_t packed[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const __half2* h = w < 2 ? ha + 2 * w : hb + 2 * (w - 2);
        const float2 f0 = __half22float2(h[0]);
        const float2 f1 = __half22float2(h[1]);
        const uint32_t t0 = __float_as_uint(__fadd_rn(__fmul_rn(f0.x, inv), 12582912.0f));
        const uint32_t t1 = __float_as_uint(__fadd_rn(__fmul_rn(f0.y, inv), 12582912.0f));
        const uint32_t t2 = __float_as_uint(__fadd_rn(__fmul_rn(f1.x, inv), 12582912.0f));
        const uint32_t t3 = __float_as_uint(__fadd_rn(__fmul_rn(f1.y, inv), 12582912.0f));
        packed[w] = prmt(prmt(t0, t1, 0x0040u), prmt(t2, t3, 0x0040u), 0x5410u);
    }
    return make_uint4(packed[0], packed[1], packed[2], packed[3]);
}

// Sixteen INT4 codes (int8 bytes, from quant16) -> eight bytes of two's-complement nibbles, the
// lower index in the low nibble.  Per word: keep the low nibbles, fold byte 2j+1's nibble onto
// byte 2j, then one byte permute gathers bytes 0 and 2 of two words.
__device__ __forceinline__ uint2 pack_int4_16(uint4 v) {
    const uint32_t a = v.x & 0x0F0F0F0Fu, b = v.y & 0x0F0F0F0Fu, c = v.z & 0x0F0F0F0Fu, d = v.w & 0x0F0F0F0Fu;
    return make_uint2(prmt(a | (a >> 4), b | (b >> 4), 0x6420u), prmt(c | (c >> 4), d | (d >> 4), 0x6420u));
}

}  // namespace qift

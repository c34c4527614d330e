// linear_gemv.cu -- qift_linear at decode batch sizes: an HBM-streaming W2A4 GEMV.
//
// "Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
// Inference", Abstract: "sign-and-shift decoded weight application" of the fixed 2-bit levels
// under rotated W2A4 inference.
//
// acc[t][n] = sum_k q[t][k] * L(code[n][k])  (int32),  y = ((float)acc * s_w[n]) * s_a[t].
//
// Each warp owns R output rows; lane l streams 16-byte groups of packed codes (64 weights)
// at word offsets 4l + 128j.  Every code load of the warp's rows is issued before any math so
// the whole weight tile is in flight at once.  A 32-bit word of 16 codes is decoded to int8
// with two masks, two shifts and four byte permutes against the set's level table (a Qift or
// power-of-two level is one table byte; for {+-1,+-4} the byte is the sign-and-shift result),
// and meets the matching activations with dp4a.  The activations of the lane's words are
// loaded once per chunk, permuted to the decode order, and reused across the R rows.
#include "common.cuh"
#include "internal.h"

namespace qift {

// Warps per CTA.  With two rows per warp, 8 warps (256 CTAs at 4096 x 4096, two per SM) measured
// 1.99 us per launch against 2.02 us for 4 warps and 2.10 us for 16, and the decode step with the
// activation quantizer ahead of it 4.2 against 4.4 us; 2 warps were slower still (2.29 us).
constexpr int kGemvWarps = 8;

template <typename OutT>
__device__ __forceinline__ void store_out(OutT* p, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_out<__half>(__half* p, float v) { *p = __float2half_rn(v); }

// TC tokens per CTA row of the grid (blockIdx.y picks the token chunk), R rows per warp,
// J 128-word slices per K chunk, VEC = codes rows are 16-byte aligned (K % 64 == 0).
template <int TC, int R, int J, bool VEC, typename OutT>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_kernel(const int8_t* __restrict__ q,
                                                               const float* __restrict__ s_a,
                                                               const uint32_t* __restrict__ codes,
                                                               const float* __restrict__ s_w, uint32_t lut,
                                                               int64_t T, int64_t N, int64_t K,
                                                               OutT* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t)blockIdx.x * kGemvWarps + (threadIdx.x >> 5);
    const int64_t row0 = warp * R;
    const int64_t t0 = (int64_t)blockIdx.y * TC;
    const int64_t KW = K / 16;
    int acc[R][TC];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int t = 0; t < TC; ++t) acc[r][t] = 0;

    // Codes of one K chunk (R rows x J slices x 4 words) straight into registers.
    uint4 cw[R][J];
    auto load_codes = [&](int64_t base) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int64_t n = row0 + r;
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int64_t wi = base + 4 * lane + 128 * j;
                uint4 c = make_uint4(0u, 0u, 0u, 0u);
                if (n < N && QIFT_CK_RANGE(n * KW + wi, wi + 4 <= KW ? 4 : KW - wi, N * KW)) {
                    const uint32_t* p = codes + n * KW + wi;
                    if (VEC && wi + 4 <= KW) {
                        c = ldg_stream_v4(p);
                    } else {
                        if (wi + 0 < KW) c.x = __ldg(p + 0);
                        if (wi + 1 < KW) c.y = __ldg(p + 1);
                        if (wi + 2 < KW) c.z = __ldg(p + 2);
                        if (wi + 3 < KW) c.w = __ldg(p + 3);
                    }
                }
                cw[r][j] = c;
            }
        }
    };
    // 1. The first chunk of codes is requested before waiting for the previous kernel on the
    //    stream (programmatic dependent launch): the weight stream overlaps its tail.  Only
    //    codes are read before the wait; activations, scales and y come after it.
    load_codes(0);
    griddep_launch_dependents();
    griddep_wait();
    // Scales are requested now, so their latency hides under the code stream.
    float sw[R], sa[TC];
#pragma unroll
    for (int r = 0; r < R; ++r) sw[r] = row0 + r < N ? __ldg(s_w + row0 + r) : 0.0f;
#pragma unroll
    for (int t = 0; t < TC; ++t) sa[t] = t0 + t < T ? __ldg(s_a + t0 + t) : 0.0f;

    for (int64_t base = 0; base < KW; base += 128 * J) {
        if (base > 0) load_codes(base);
        // 2. Activations of the lane's words, permuted to the decode order.
        uint32_t pa[TC][J][4][4];
#pragma unroll
        for (int t = 0; t < TC; ++t) {
#pragma unroll
            for (int j = 0; j < J; ++j) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int64_t wi = base + 4 * lane + 128 * j + u;
                    uint4 a = make_uint4(0u, 0u, 0u, 0u);
                    if (t0 + t < T && wi < KW && QIFT_CK_RANGE((t0 + t) * K + wi * 16, 16, T * K))
                        a = __ldg(reinterpret_cast<const uint4*>(q + (t0 + t) * K + wi * 16));
                    permute_acts(a, pa[t][j][u]);
                }
            }
        }
        // 3. Decode and accumulate.
#pragma unroll
        for (int r = 0; r < R; ++r) {
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const uint32_t words[4] = {cw[r][j].x, cw[r][j].y, cw[r][j].z, cw[r][j].w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint32_t d[4];
                    decode_word(words[u], lut, d);
#pragma unroll
                    for (int t = 0; t < TC; ++t) {
                        int a = acc[r][t];
                        a = dp4a(d[0], pa[t][j][u][0], a);
                        a = dp4a(d[1], pa[t][j][u][1], a);
                        a = dp4a(d[2], pa[t][j][u][2], a);
                        a = dp4a(d[3], pa[t][j][u][3], a);
                        acc[r][t] = a;
                    }
                }
            }
        }
    }
    // 4. Warp reduction and the fp32 epilogue.
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int t = 0; t < TC; ++t) {
            const int sum = __reduce_add_sync(0xffffffffu, acc[r][t]);
            const int64_t n = row0 + r, tt = t0 + t;
            if (lane == ((r * TC + t) & 31) && n < N && tt < T && QIFT_CK_RANGE(tt * N + n, 1, T * N)) {
                const float v = __fmul_rn(__fmul_rn((float)sum, sw[r]), sa[t]);
                store_out<OutT>(y + tt * N + n, v);
            }
        }
    }
}

// One token, n_in % 64 == 0: the codes of the first K chunk are loaded AND decoded to int8
// registers before the kernel waits for its predecessor, so after the wait only the
// activation token (staged once per CTA in shared memory, permuted to the decode order), the
// dp4a products, the warp reduction and the epilogue remain on the critical path.
// The staged token is laid out so that the warp's reads are conflict-free: word wi = base +
// 4 l + 128 j + u (lane l, slice j, word u of the lane's 16-byte code group) sits at slot
// base + 32 (4 j + u) + l, so each 16-byte read of a warp covers 512 contiguous bytes.  (Stored in
// word order, lane l's reads were 64 bytes apart: a 16-way bank conflict that cost ~0.5 us per
// launch at 4096 x 4096.)
// ONE: the row is a single chunk (n_in <= 2048 J), so no loop over chunks is compiled.
template <int R, int J, bool ONE, typename OutT>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv1_kernel(const int8_t* __restrict__ q,
                                                                const float* __restrict__ s_a,
                                                                const uint32_t* __restrict__ codes,
                                                                const float* __restrict__ s_w, uint32_t lut,
                                                                int64_t N, int64_t K, OutT* __restrict__ y) {
    extern __shared__ __align__(16) uint4 acts_s[];  // K/16 permuted 16-byte groups (chunk-padded)
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t)blockIdx.x * kGemvWarps + (threadIdx.x >> 5);
    const int64_t row0 = warp * R;
    const int64_t KW = K / 16;

    // All of a chunk's code loads are issued before any of them is decoded.
    uint4 cw[R][J];
    uint32_t dec[R][J][4][4];
    auto load_decode = [&](int64_t base) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int64_t wi = base + 4 * lane + 128 * j;
                cw[r][j] = (row0 + r < N && wi + 4 <= KW && QIFT_CK_RANGE((row0 + r) * KW + wi, 4, N * KW))
                               ? ldg_stream_v4(codes + (row0 + r) * KW + wi)
                               : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < J; ++j) {
                decode_word(cw[r][j].x, lut, dec[r][j][0]);
                decode_word(cw[r][j].y, lut, dec[r][j][1]);
                decode_word(cw[r][j].z, lut, dec[r][j][2]);
                decode_word(cw[r][j].w, lut, dec[r][j][3]);
            }
    };
    load_decode(0);
    griddep_launch_dependents();
    griddep_wait();

    float sw[R];
#pragma unroll
    for (int r = 0; r < R; ++r) sw[r] = row0 + r < N ? __ldg(s_w + row0 + r) : 0.0f;
    const float sa = __ldg(s_a);
    // Thread t reads word t (+ 128 per pass), coalesced, and stores it at its slot (a 4-way
    // bank conflict on the stores).  Measured slower: filling the slots in order with reads 64
    // bytes apart (2.34 against 2.02 us per launch at 4096 x 4096), and conflict-free stores
    // from a lane permutation inside each 32-word group (2.18 us).
    for (int i = threadIdx.x; i < (int)KW; i += kGemvWarps * 32) {
        uint32_t p[4];
        permute_acts(QIFT_CK_RANGE(16 * (int64_t)i, 16, K) ? __ldg(reinterpret_cast<const uint4*>(q) + i)
                                                            : make_uint4(0u, 0u, 0u, 0u),
                     p);
        const int in = i % (128 * J);  // word within its chunk: lane (in / 4) % 32, slice in / 128
        acts_s[i - in + 32 * (4 * (in >> 7) + (in & 3)) + ((in >> 2) & 31)] = make_uint4(p[0], p[1], p[2], p[3]);
    }
    // A partial last chunk leaves slots no word maps to; they are read only for words past the
    // row, which the reads below replace by zeros.
    __syncthreads();

    int acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0;
    for (int64_t base = 0; base < (ONE ? 1 : KW); base += 128 * J) {
        if (!ONE && base > 0) load_decode(base);
#pragma unroll
        for (int j = 0; j < J; ++j) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t wi = base + 4 * lane + 128 * j + u;
                const uint4 a = wi < KW ? acts_s[base + 32 * (4 * j + u) + lane] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    int v = acc[r];
                    v = dp4a(dec[r][j][u][0], a.x, v);
                    v = dp4a(dec[r][j][u][1], a.y, v);
                    v = dp4a(dec[r][j][u][2], a.z, v);
                    v = dp4a(dec[r][j][u][3], a.w, v);
                    acc[r] = v;
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int sum = __reduce_add_sync(0xffffffffu, acc[r]);
        if (lane == r && row0 + r < N && QIFT_CK_RANGE(row0 + r, 1, N))
            store_out<OutT>(y + row0 + r, __fmul_rn(__fmul_rn((float)sum, sw[r]), sa));
    }
}

template <int R, int J, bool ONE, typename OutT>
static cudaError_t launch_gemv1_t(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w,
                                uint32_t lut, int64_t N, int64_t K, OutT* y, cudaStream_t s) {
    const int64_t gx = ((N + R - 1) / R + kGemvWarps - 1) / kGemvWarps;
    if (gx > 0x7fffffff) return cudaErrorInvalidValue;
    const int64_t KW = K / 16, chunk = 128 * J;
    const size_t smem = (size_t)((KW + chunk - 1) / chunk * chunk) * 16;  // whole chunks of 16-byte groups
    cudaError_t e = ensure_smem(gemv1_kernel<R, J, ONE, OutT>, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)gx);
    cfg.blockDim = dim3(kGemvWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemv1_kernel<R, J, ONE, OutT>, q, s_a, codes, s_w, lut, N, K, y);
}

template <int R, int J, typename OutT>
static cudaError_t launch_gemv1(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w,
                                uint32_t lut, int64_t N, int64_t K, OutT* y, cudaStream_t s) {
    if (K <= 2048 * J) return launch_gemv1_t<R, J, true, OutT>(q, s_a, codes, s_w, lut, N, K, y, s);
    return launch_gemv1_t<R, J, false, OutT>(q, s_a, codes, s_w, lut, N, K, y, s);
}

template <int TC, int R, int J, typename OutT>
static cudaError_t launch_gemv_t(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w,
                                 uint32_t lut, int64_t T, int64_t N, int64_t K, OutT* y, cudaStream_t s) {
    const int64_t warps = (N + R - 1) / R;
    const int64_t gx = (warps + kGemvWarps - 1) / kGemvWarps;
    const int64_t gy = (T + TC - 1) / TC;
    if (gx > 0x7fffffff || gy > 65535) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)gx, (unsigned)gy);
    cfg.blockDim = dim3(kGemvWarps * 32);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    if ((K / 16) % 4 == 0)
        return cudaLaunchKernelEx(&cfg, gemv_kernel<TC, R, J, true, OutT>, q, s_a, codes, s_w, lut, T, N, K, y);
    return cudaLaunchKernelEx(&cfg, gemv_kernel<TC, R, J, false, OutT>, q, s_a, codes, s_w, lut, T, N, K, y);
}

template <typename OutT>
static cudaError_t dispatch_gemv(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w,
                                 uint32_t lut, int64_t T, int64_t N, int64_t K, OutT* y, cudaStream_t s) {
    if (T == 1 && K % 64 == 0) return launch_gemv1<2, 2, OutT>(q, s_a, codes, s_w, lut, N, K, y, s);
    if (T == 1) return launch_gemv_t<1, 4, 2, OutT>(q, s_a, codes, s_w, lut, T, N, K, y, s);
    if (T == 2) return launch_gemv_t<2, 4, 1, OutT>(q, s_a, codes, s_w, lut, T, N, K, y, s);
    return launch_gemv_t<4, 2, 1, OutT>(q, s_a, codes, s_w, lut, T, N, K, y, s);
}

bool linear_gemv_supported(int64_t T) { return T <= (int64_t)4 * 65535; }

cudaError_t launch_linear_gemv(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, int set,
                               int64_t T, int64_t N, int64_t K, void* y, bool f16, cudaStream_t s) {
    if (T == 0 || N == 0) return cudaSuccess;
    const uint32_t lut = level_lut(set);
    if (f16) return dispatch_gemv<__half>(q, s_a, codes, s_w, lut, T, N, K, static_cast<__half*>(y), s);
    return dispatch_gemv<float>(q, s_a, codes, s_w, lut, T, N, K, static_cast<float*>(y), s);
}

}  // namespace qift

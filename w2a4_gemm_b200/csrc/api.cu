// api.cu -- the extern "C" entry points of libqift.so: host-side validation and dispatch.
// Declarations, argument meaning, layouts and error behaviour are documented in qift.h.
#include <math.h>
#include <stdint.h>

#include <mutex>
#include <unordered_map>

#include "../../include/qift.h"
#include "../../include/qift_debug.h"
#include "internal.h"

namespace {

bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

constexpr int64_t kMaxInner = 32768;  // keeps |acc| < 2^24 and a token / row in shared memory

qift_status from_cuda(cudaError_t e) { return e == cudaSuccess ? QIFT_OK : QIFT_ERR_CUDA; }

bool valid_block(int64_t b) { return is_pow2(b) && b >= 2 && b <= 4096; }

}  // namespace

namespace qift {

// Debug pins (qift_debug.h), per host thread, so a pin set by one thread never changes the
// kernels another thread's calls launch.
static thread_local int g_linear_path = kPathAuto;
static thread_local bool g_pdl = true;
void debug_set_pdl(bool on) { g_pdl = on; }
bool pdl_enabled() { return g_pdl; }
void debug_set_linear_path(int path) { g_linear_path = path; }
int debug_linear_path() { return g_linear_path; }

cudaError_t ensure_smem_ptr(const void* kernel, size_t bytes) {
    static std::mutex mu;
    static std::unordered_map<uint64_t, size_t> granted;  // (kernel, device) -> bytes allowed
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t key = (reinterpret_cast<uintptr_t>(kernel) << 8) ^ (uint64_t)(dev & 0xff);
    std::lock_guard<std::mutex> lock(mu);
    auto it = granted.find(key);
    if (it != granted.end() && it->second >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) granted[key] = bytes;
    return e;
}

}  // namespace qift

extern "C" {

qift_status qift_rotate(const void* x, void* y, qift_dtype dt, int64_t rows, int64_t n, int32_t block,
                        void* stream) {
    if (dt != QIFT_F32 && dt != QIFT_F16) return QIFT_ERR_INVALID_ARG;
    if (rows < 0 || n < 0 || !valid_block(block) || n % block != 0) return QIFT_ERR_INVALID_ARG;
    if (rows == 0 || n == 0) return QIFT_OK;
    if (!x || !y || !aligned16(x) || !aligned16(y)) return QIFT_ERR_INVALID_ARG;
    const int64_t esz = dt == QIFT_F32 ? 4 : 2;
    if (rows > INT64_MAX / n / esz) return QIFT_ERR_INVALID_ARG;
    const uintptr_t bytes = (uintptr_t)(rows * n * esz);
    const uintptr_t xa = reinterpret_cast<uintptr_t>(x), ya = reinterpret_cast<uintptr_t>(y);
    if (xa != ya && xa < ya + bytes && ya < xa + bytes) return QIFT_ERR_INVALID_ARG;  // partial overlap
    return from_cuda(qift::launch_rotate(x, y, dt == QIFT_F16, rows, n, block, static_cast<cudaStream_t>(stream)));
}

qift_status qift_quantize_weights(const float* w_rot, int64_t n_out, int64_t n_in, qift_levelset set,
                                  int32_t grid_points, double lo, double hi, uint32_t* codes, float* scales,
                                  double* row_mse, void* stream) {
    if (set != QIFT_SET_QIFT && set != QIFT_SET_POT && set != QIFT_SET_STD && set != QIFT_SET_INT4)
        return QIFT_ERR_INVALID_ARG;
    if (n_out < 0 || n_in <= 0 || n_in % 16 != 0) return QIFT_ERR_INVALID_ARG;
    if (grid_points < 2 || grid_points > 256) return QIFT_ERR_INVALID_ARG;
    if (!(lo > 0.0) || !(hi >= lo) || !(hi <= 4.0)) return QIFT_ERR_INVALID_ARG;
    if (n_in > kMaxInner) return QIFT_ERR_UNSUPPORTED;
    if (n_out == 0) return QIFT_OK;
    if (!w_rot || !codes || !scales || !aligned16(w_rot) || !aligned16(codes) || !aligned4(scales))
        return QIFT_ERR_INVALID_ARG;
    if (row_mse && !aligned8(row_mse)) return QIFT_ERR_INVALID_ARG;
    if (n_out > 0x7fffffff) return QIFT_ERR_UNSUPPORTED;
    return from_cuda(qift::launch_quantize_weights(w_rot, n_out, n_in, (int)set, grid_points, lo, hi, codes, scales,
                                                   row_mse, static_cast<cudaStream_t>(stream)));
}

qift_status qift_quantize_weights_asym(const float* w_rot, int64_t n_out, int64_t n_in, int32_t grid_points,
                                       double lo, double hi, uint32_t* codes, float* scales, int32_t* zeros,
                                       double* row_mse, void* stream) {
    if (n_out < 0 || n_in <= 0 || n_in % 16 != 0) return QIFT_ERR_INVALID_ARG;
    if (grid_points < 2 || grid_points > 256) return QIFT_ERR_INVALID_ARG;
    if (!(lo > 0.0) || !(hi >= lo) || !(hi <= 4.0)) return QIFT_ERR_INVALID_ARG;
    if (n_in > kMaxInner) return QIFT_ERR_UNSUPPORTED;
    if (n_out == 0) return QIFT_OK;
    if (!w_rot || !codes || !scales || !zeros || !aligned16(w_rot) || !aligned16(codes) || !aligned4(scales) ||
        !aligned4(zeros))
        return QIFT_ERR_INVALID_ARG;
    if (row_mse && !aligned8(row_mse)) return QIFT_ERR_INVALID_ARG;
    if (n_out > 0x7fffffff) return QIFT_ERR_UNSUPPORTED;
    return from_cuda(qift::launch_quantize_weights_asym(w_rot, n_out, n_in, grid_points, lo, hi, codes, scales, zeros,
                                                        row_mse, static_cast<cudaStream_t>(stream)));
}

qift_status qift_rotate_quantize_weights(const float* w, int64_t n_out, int64_t n_in, int32_t block,
                                         qift_levelset set, int32_t grid_points, double lo, double hi,
                                         uint32_t* codes, float* scales, double* row_mse, void* stream) {
    if (set != QIFT_SET_QIFT && set != QIFT_SET_POT && set != QIFT_SET_STD && set != QIFT_SET_INT4)
        return QIFT_ERR_INVALID_ARG;
    if (n_out < 0 || n_in <= 0 || n_in % 16 != 0) return QIFT_ERR_INVALID_ARG;
    if (block != 0 && (!valid_block(block) || n_in % block != 0)) return QIFT_ERR_INVALID_ARG;
    if (grid_points < 2 || grid_points > 256) return QIFT_ERR_INVALID_ARG;
    if (!(lo > 0.0) || !(hi >= lo) || !(hi <= 4.0)) return QIFT_ERR_INVALID_ARG;
    if (n_in > kMaxInner) return QIFT_ERR_UNSUPPORTED;
    if (n_out == 0) return QIFT_OK;
    if (!w || !codes || !scales || !aligned16(w) || !aligned16(codes) || !aligned4(scales))
        return QIFT_ERR_INVALID_ARG;
    if (row_mse && !aligned8(row_mse)) return QIFT_ERR_INVALID_ARG;
    if (n_out > 0x7fffffff) return QIFT_ERR_UNSUPPORTED;
    return from_cuda(qift::launch_quantize_weights(w, n_out, n_in, (int)set, grid_points, lo, hi, codes, scales,
                                                   row_mse, static_cast<cudaStream_t>(stream), block));
}

qift_status qift_quantize_acts(const void* x, int64_t tokens, int64_t n_in, int32_t block, int8_t* q,
                               float* scales, void* stream) {
    if (tokens < 0 || n_in <= 0 || n_in % 16 != 0) return QIFT_ERR_INVALID_ARG;
    if (block != 0 && (!valid_block(block) || n_in % block != 0)) return QIFT_ERR_INVALID_ARG;
    if (n_in > kMaxInner) return QIFT_ERR_UNSUPPORTED;
    if (tokens == 0) return QIFT_OK;
    if (!x || !q || !scales || !aligned16(x) || !aligned16(q) || !aligned4(scales)) return QIFT_ERR_INVALID_ARG;
    if (tokens > 0x7fffffff) return QIFT_ERR_UNSUPPORTED;
    return from_cuda(
        qift::launch_quantize_acts(x, tokens, n_in, block, q, scales, static_cast<cudaStream_t>(stream)));
}

qift_status qift_quantize_kv(const void* x, int64_t tokens, int64_t n, int32_t block, uint8_t* packed,
                             float* scales, void* stream) {
    if (tokens < 0 || n <= 0 || n % 16 != 0) return QIFT_ERR_INVALID_ARG;
    if (block != 0 && (!valid_block(block) || n % block != 0)) return QIFT_ERR_INVALID_ARG;
    if (n > kMaxInner) return QIFT_ERR_UNSUPPORTED;
    if (tokens == 0) return QIFT_OK;
    if (!x || !packed || !scales || !aligned16(x) || !aligned16(packed) || !aligned4(scales))
        return QIFT_ERR_INVALID_ARG;
    if (tokens > 0x7fffffff) return QIFT_ERR_UNSUPPORTED;
    return from_cuda(qift::launch_quantize_kv(x, tokens, n, block, packed, scales, static_cast<cudaStream_t>(stream)));
}

qift_status qift_dequantize_kv(const uint8_t* packed, const float* scales, int64_t tokens, int64_t n, int32_t block,
                               void* out, void* stream) {
    if (tokens < 0 || n <= 0 || n % 16 != 0) return QIFT_ERR_INVALID_ARG;
    if (block != 0 && (!valid_block(block) || n % block != 0)) return QIFT_ERR_INVALID_ARG;
    if (n > 16384) return QIFT_ERR_UNSUPPORTED;
    if (tokens == 0) return QIFT_OK;
    if (!packed || !scales || !out || !aligned16(packed) || !aligned16(out) || !aligned4(scales))
        return QIFT_ERR_INVALID_ARG;
    if (tokens > 0x7fffffff) return QIFT_ERR_UNSUPPORTED;
    return from_cuda(
        qift::launch_dequantize_kv(packed, scales, tokens, n, block, out, static_cast<cudaStream_t>(stream)));
}

qift_status qift_linear(const int8_t* q_act, const float* act_scale, const uint32_t* codes, const float* w_scale,
                        qift_levelset set, int64_t tokens, int64_t n_out, int64_t n_in, void* y, qift_dtype out_dt,
                        void* stream) {
    if (set != QIFT_SET_QIFT && set != QIFT_SET_POT && set != QIFT_SET_STD && set != QIFT_SET_INT4)
        return QIFT_ERR_INVALID_ARG;
    if (out_dt != QIFT_F32 && out_dt != QIFT_F16) return QIFT_ERR_INVALID_ARG;
    if (tokens < 0 || n_out < 0 || n_in <= 0 || n_in % 16 != 0) return QIFT_ERR_INVALID_ARG;
    if (set == QIFT_SET_STD) return QIFT_ERR_UNSUPPORTED;
    if (n_in > kMaxInner) return QIFT_ERR_UNSUPPORTED;
    if (set == QIFT_SET_INT4 && !qift::linear_w4_supported(tokens == 0 ? 1 : tokens, n_in)) return QIFT_ERR_UNSUPPORTED;
    if (tokens == 0 || n_out == 0) return QIFT_OK;
    if (!q_act || !act_scale || !codes || !w_scale || !y) return QIFT_ERR_INVALID_ARG;
    if (!aligned16(q_act) || !aligned16(codes) || !aligned16(y) || !aligned4(act_scale) || !aligned4(w_scale))
        return QIFT_ERR_INVALID_ARG;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool f16 = out_dt == QIFT_F16;
    int path = qift::debug_linear_path();
    if (set == QIFT_SET_INT4) {
        // 4-bit weights: the tcgen05 pair GEMM from 17 tokens, the tensor-core skinny kernel for
        // 2..16, the CUDA-core GEMV for one; pinning "gemm_pair" or "skinny" forces that family,
        // any other pin the GEMV (which takes at most 16 tokens).
        if (path == qift::kPathAuto)
            path = tokens >= qift::kGemmMinTokens
                       ? qift::kPathGemmPair
                       : (tokens >= 2 && qift::linear_skinny_supported(tokens, n_out, n_in) ? qift::kPathSkinny
                                                                                            : qift::kPathGemv);
        if (path == qift::kPathGemmPair) {
            if (!qift::linear_gemm_supported(tokens, n_out, n_in)) return QIFT_ERR_UNSUPPORTED;
            return from_cuda(qift::launch_linear_gemm_pair(q_act, act_scale, codes, w_scale, (int)set, tokens, n_out,
                                                           n_in, y, f16, s));
        }
        if (path == qift::kPathSkinny) {
            if (!qift::linear_skinny_supported(tokens, n_out, n_in)) return QIFT_ERR_UNSUPPORTED;
            return from_cuda(qift::launch_linear_skinny(q_act, act_scale, codes, w_scale, (int)set, tokens, n_out,
                                                        n_in, y, f16, s));
        }
        if (tokens > 16) return QIFT_ERR_UNSUPPORTED;
        return from_cuda(qift::launch_linear_w4(q_act, act_scale, codes, w_scale, tokens, n_out, n_in, y, f16, s));
    }
    if (path == qift::kPathAuto) {
        if (tokens >= qift::kGemmMinTokens) {
            // Prefill sizes run on the tensor cores only.  The code matrix's rows must be 16-byte
            // multiples for the tensor-memory copies (n_in % 64 == 0); any other n_in is refused
            // rather than sent to the CUDA-core GEMV, whose cost grows with every token.
            if (!qift::linear_gemm_supported(tokens, n_out, n_in)) return QIFT_ERR_UNSUPPORTED;
            path = qift::kPathGemmPair;
        } else if (tokens >= 2 && qift::linear_skinny_supported(tokens, n_out, n_in))
            path = qift::kPathSkinny;
        else if (tokens == 1 && qift::linear_one_token_preferred(n_out, n_in))
            path = qift::kPathOneToken;
        else
            path = qift::kPathGemv;
    } else if ((path == qift::kPathGemmPair && !qift::linear_gemm_supported(tokens, n_out, n_in)) ||
               (path == qift::kPathGemv && !qift::linear_gemv_supported(tokens)) ||
               (path == qift::kPathSkinny && !qift::linear_skinny_supported(tokens, n_out, n_in)) ||
               (path == qift::kPathOneToken && (tokens != 1 || !qift::linear_one_token_supported(n_out, n_in)))) {
        return QIFT_ERR_UNSUPPORTED;
    }
    if (path == qift::kPathOneToken)
        return from_cuda(qift::launch_linear_one_token(q_act, act_scale, codes, w_scale, (int)set, n_out, n_in, y, f16,
                                                       s));
    if (path == qift::kPathGemmPair)
        return from_cuda(qift::launch_linear_gemm_pair(q_act, act_scale, codes, w_scale, (int)set, tokens, n_out,
                                                       n_in, y, f16, s));
    if (path == qift::kPathSkinny)
        return from_cuda(qift::launch_linear_skinny(q_act, act_scale, codes, w_scale, (int)set, tokens, n_out, n_in,
                                                    y, f16, s));
    return from_cuda(
        qift::launch_linear_gemv(q_act, act_scale, codes, w_scale, (int)set, tokens, n_out, n_in, y, f16, s));
}

qift_status qift_decode_linear(const void* x, int64_t tokens, int64_t n_in, int32_t block, const uint32_t* codes,
                               const float* w_scale, qift_levelset set, int64_t n_out, void* y, qift_dtype out_dt,
                               int8_t* q_out, float* act_scale_out, void* stream) {
    if (set != QIFT_SET_QIFT && set != QIFT_SET_POT && set != QIFT_SET_STD && set != QIFT_SET_INT4)
        return QIFT_ERR_INVALID_ARG;
    if (out_dt != QIFT_F32 && out_dt != QIFT_F16) return QIFT_ERR_INVALID_ARG;
    if (tokens < 0 || n_out < 0 || n_in <= 0 || n_in % 16 != 0) return QIFT_ERR_INVALID_ARG;
    if (block != 0 && (!valid_block(block) || n_in % block != 0)) return QIFT_ERR_INVALID_ARG;
    if (set == QIFT_SET_STD || tokens > 4 || n_in > 16384 || n_in % 64 != 0) return QIFT_ERR_UNSUPPORTED;
    if (tokens == 0 || n_out == 0) return QIFT_OK;
    if (!x || !codes || !w_scale || !y) return QIFT_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(y) || !aligned4(w_scale)) return QIFT_ERR_INVALID_ARG;
    if ((q_out && !aligned16(q_out)) || (act_scale_out && !aligned4(act_scale_out))) return QIFT_ERR_INVALID_ARG;
    if (n_out > 0x7fffffff / 2) return QIFT_ERR_UNSUPPORTED;
    const int path = qift::debug_linear_path();
    if (tokens == 1 && (path == qift::kPathAuto || path == qift::kPathOneToken) &&
        qift::decode_one_token_supported(n_out, n_in, block, (int)set))
        return from_cuda(qift::launch_decode_one_token(x, n_in, block, codes, w_scale, (int)set, n_out, y,
                                                       out_dt == QIFT_F16, q_out, act_scale_out,
                                                       static_cast<cudaStream_t>(stream)));
    return from_cuda(qift::launch_decode_linear(x, tokens, n_in, block, codes, w_scale, (int)set, n_out, y,
                                                out_dt == QIFT_F16, q_out, act_scale_out,
                                                static_cast<cudaStream_t>(stream)));
}

qift_status qift_device_error(void* stream, int32_t* detail) {
    if (detail) *detail = 0;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return QIFT_ERR_CUDA;
    int word = 0, word1 = 0;
    if (qift::read_and_clear_device_error(&word) != cudaSuccess) return QIFT_ERR_CUDA;
    if (qift::read_and_clear_one_token_error(&word1) != cudaSuccess) return QIFT_ERR_CUDA;
    word |= word1;
    if (detail) *detail = word;
    if (word & 0x100) return QIFT_ERR_CUDA;  // a failed bounds check (checked build only)
    return word ? QIFT_ERR_TIMEOUT : QIFT_OK;
}

qift_status qift_debug_check_line(int32_t* line) {
    if (!line) return QIFT_ERR_INVALID_ARG;
    int v = 0;
    if (qift::read_and_clear_check_line(&v) != cudaSuccess) return QIFT_ERR_CUDA;
    *line = v;
    return QIFT_OK;
}

int32_t qift_debug_checked_build(void) {
#ifdef QIFT_CHECK
    return 1;
#else
    return 0;
#endif
}

qift_status qift_debug_set_wait_limit(int64_t cycles) {
    qift::debug_set_gemm_wait_limit((long long)cycles);
    qift::debug_set_one_token_wait_limit((long long)cycles);
    return QIFT_OK;
}

qift_status qift_debug_set_linear_path(int32_t path) {
    if (path != qift::kPathAuto && path != qift::kPathGemv && path != qift::kPathSkinny &&
        path != qift::kPathGemmPair && path != qift::kPathOneToken)
        return QIFT_ERR_INVALID_ARG;
    qift::debug_set_linear_path(path);
    return QIFT_OK;
}

qift_status qift_debug_set_pdl(int32_t enable) {
    qift::debug_set_pdl(enable != 0);
    return QIFT_OK;
}

qift_status qift_debug_stall_next_gemm(void) {
    qift::debug_stall_next_gemm();
    return QIFT_OK;
}

qift_status qift_debug_stall_next_one_token(void) {
    qift::debug_stall_next_one_token();
    return QIFT_OK;
}

const char* qift_status_string(qift_status status) {
    switch (status) {
        case QIFT_OK: return "QIFT_OK";
        case QIFT_ERR_INVALID_ARG: return "QIFT_ERR_INVALID_ARG: an argument failed host-side validation";
        case QIFT_ERR_UNSUPPORTED: return "QIFT_ERR_UNSUPPORTED: valid request this build does not implement";
        case QIFT_ERR_CUDA: return "QIFT_ERR_CUDA: a CUDA launch or runtime call failed";
        case QIFT_ERR_TIMEOUT: return "QIFT_ERR_TIMEOUT: a bounded on-chip wait gave up";
        default: return "QIFT_UNKNOWN_STATUS";
    }
}

}  // extern "C"

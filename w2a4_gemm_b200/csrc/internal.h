// internal.h -- launchers shared between the C ABI (api.cu) and the kernel files.
// Arguments are validated by the caller; launchers only configure and launch.
#pragma once

#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace qift {

// The driver's cuTensorMapEncodeTiled (through the runtime's entry-point query, so the library
// links no libcuda); null if unavailable.
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device), so launches --
// including ones captured into CUDA graphs -- do not repeat the attribute call.
cudaError_t ensure_smem_ptr(const void* kernel, size_t bytes);

// Called for any dynamic size: the default 48 KB limit covers static plus dynamic shared memory,
// so a kernel with static buffers can pass it with less than 48 KB requested.
template <typename Kernel>
inline cudaError_t ensure_smem(Kernel kernel, size_t bytes) {
    if (bytes == 0) return cudaSuccess;
    return ensure_smem_ptr(reinterpret_cast<const void*>(kernel), bytes);
}

cudaError_t launch_rotate(const void* x, void* y, bool f16, int64_t rows, int64_t n, int block,
                          cudaStream_t s);

cudaError_t launch_quantize_acts(const void* x, int64_t tokens, int64_t n_in, int block, int8_t* q,
                                 float* scales, cudaStream_t s);

// KV4: the activation quantizer with the codes packed two per byte, and its inverse.
cudaError_t launch_quantize_kv(const void* x, int64_t tokens, int64_t n, int block, uint8_t* packed, float* scales,
                               cudaStream_t s);
cudaError_t launch_dequantize_kv(const uint8_t* packed, const float* scales, int64_t tokens, int64_t n, int block,
                                 void* out, cudaStream_t s);

// block > 0: w holds raw weights, rotated by W H_b^T in shared memory first (same bits as
// qift_rotate), so the offline pipeline reads each weight once and writes no fp32 temporary.
cudaError_t launch_quantize_weights(const float* w, int64_t n_out, int64_t n_in, int set, int grid_points,
                                    double lo, double hi, uint32_t* codes, float* scales, double* row_mse,
                                    cudaStream_t s, int block = 0);
// The asymmetric W2 baseline: the same search with a per-row zero point (zeros: int32 [n_out]).
cudaError_t launch_quantize_weights_asym(const float* w, int64_t n_out, int64_t n_in, int grid_points, double lo,
                                         double hi, uint32_t* codes, float* scales, int32_t* zeros, double* row_mse,
                                         cudaStream_t s);

// Decode-size linear: HBM-streaming GEMV (CUDA-core dp4a); its grid takes at most
// 4 * 65535 tokens.
bool linear_gemv_supported(int64_t tokens);
cudaError_t launch_linear_gemv(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w,
                               int set, int64_t tokens, int64_t n_out, int64_t n_in, void* y, bool f16,
                               cudaStream_t s);

// Small-batch linear (<= 16 tokens): mma.sync skinny GEMM, cluster split-K over DSMEM.
bool linear_skinny_supported(int64_t tokens, int64_t n_out, int64_t n_in);
cudaError_t launch_linear_skinny(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w,
                                 int set, int64_t tokens, int64_t n_out, int64_t n_in, void* y, bool f16,
                                 cudaStream_t s);

// One-launch decode step (1..4 tokens): rotation + INT4 + W2A4 GEMV, fused.
cudaError_t launch_decode_linear(const void* x, int64_t tokens, int64_t n_in, int block, const uint32_t* codes,
                                 const float* s_w, int set, int64_t n_out, void* y, bool f16, int8_t* q_out,
                                 float* sa_out, cudaStream_t s);

// Prefill-size linear: tcgen05 int8 tensor-core GEMM on CTA pairs (cta_group::2), the decoded
// weights as the A operand in tensor memory.
bool linear_gemm_supported(int64_t tokens, int64_t n_out, int64_t n_in);
cudaError_t launch_linear_gemm_pair(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w,
                                    int set, int64_t T, int64_t N, int64_t K, void* y, bool f16, cudaStream_t s);

// One token: qift_linear, and the fused decode step, on CTAs that bulk-copy their rows'
// codes into shared memory before waiting for the previous kernel (half an SM each).
bool linear_one_token_supported(int64_t n_out, int64_t n_in);
bool linear_one_token_preferred(int64_t n_out, int64_t n_in);  // over the warp-per-row GEMV
bool decode_one_token_supported(int64_t n_out, int64_t n_in, int block, int set);
cudaError_t launch_linear_one_token(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w,
                                    int set, int64_t n_out, int64_t n_in, void* y, bool f16, cudaStream_t s);
cudaError_t launch_decode_one_token(const void* x, int64_t n_in, int block, const uint32_t* codes, const float* s_w,
                                    int set, int64_t n_out, void* y, bool f16, int8_t* q_out, float* sa_out,
                                    cudaStream_t s);
void debug_set_one_token_wait_limit(long long cycles);
void debug_stall_next_one_token();
cudaError_t read_and_clear_one_token_error(int* word);

// 4-bit weights (QIFT_SET_INT4): which calls the library takes, and the CUDA-core W4A4 GEMV
// (1..16 tokens).
bool linear_w4_supported(int64_t tokens, int64_t n_in);
cudaError_t launch_linear_w4(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w,
                             int64_t tokens, int64_t n_out, int64_t n_in, void* y, bool f16, cudaStream_t s);

// Test hooks behind qift_debug.h (numbers 3 to 5 named GEMM forms that are no longer built).
enum LinearPath {
    kPathAuto = 0,
    kPathGemv = 1,
    kPathSkinny = 2,
    kPathGemmPair = 6,
    kPathOneToken = 7
};
void debug_set_linear_path(int path);
int debug_linear_path();
void debug_set_pdl(bool on);
bool pdl_enabled();  // programmatic dependent launch for the linear and decode kernels (default on)
void debug_set_gemm_wait_limit(long long cycles);
void debug_stall_next_gemm();

// Bounds-checked build: read and clear the source line of the first failed check (0: none, and
// always 0 in the normal build).
cudaError_t read_and_clear_check_line(int* line);

// Synchronous read-and-clear of the device error word set by bounded on-chip waits.
cudaError_t read_and_clear_device_error(int* word);

// Token count from which qift_linear uses the tensor-core GEMM instead of the GEMV.
constexpr int64_t kGemmMinTokens = 17;

}  // namespace qift

/*
 * qift_debug.h -- test hooks of libqift.so.  Not part of the computing interface: they exist
 * so a test can drive the bounded-wait failure path of the tensor-core GEMM on a real GPU
 * without faulting, trapping or hanging it.
 */
#ifndef QIFT_DEBUG_H_
#define QIFT_DEBUG_H_

#include <stdint.h>

#include "qift.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Give every on-chip wait of later tensor-core GEMM and one-token launches at most `cycles` SM
 * clock cycles before it gives up (default about 4e9, some two seconds).  cycles <= 0 restores
 * the default.  Per host thread: it applies to the launches that thread makes. */
qift_status qift_debug_set_wait_limit(int64_t cycles);

/* Make the next tensor-core GEMM launch (qift_linear with tokens >= 17) wait, in its MMA-issuing
 * thread, on a barrier that nothing ever arrives on.  That wait runs out after the wait limit,
 * the kernel abandons its tile, drains its copies, frees tensor memory and exits; the output is
 * left unspecified and qift_device_error() then reports QIFT_ERR_TIMEOUT.  One-shot, per host
 * thread. */
qift_status qift_debug_stall_next_gemm(void);

/* Make the next one-token launch (qift_linear or qift_decode_linear with tokens == 1) wait for
 * its staged codes on a barrier that nothing ever arrives on.  That wait runs out after the
 * wait limit; every CTA then waits for its own copies to land and exits without writing its
 * outputs, and qift_device_error() reports QIFT_ERR_TIMEOUT.  One-shot, per host thread. */
qift_status qift_debug_stall_next_one_token(void);

/* Turn programmatic dependent launch of the qift_linear and qift_decode_linear kernels on
 * (default) or off, to measure what the overlap with the previous kernel is worth.  Per host
 * thread. */
qift_status qift_debug_set_pdl(int32_t enable);

/* Pin the kernel family qift_linear uses: 0 = automatic (by batch size), 1 = CUDA-core GEMV
 * (warps stream their rows' codes into registers; at most 4 * 65535 tokens), 2 = tensor-core
 * skinny GEMM (tokens <= 16, n_in % 64 == 0), 6 = the tcgen05 GEMM on CTA pairs (two SMs per
 * tile, cta_group::2, decoded weights in tensor memory; n_in % 64 == 0), 7 = the one-token kernel
 * (tokens == 1, codes bulk-copied into shared memory).  Other values return
 * QIFT_ERR_INVALID_ARG.  A pinned family that cannot take a call makes it return
 * QIFT_ERR_UNSUPPORTED.  qift_decode_linear with one token uses the one-token kernel under 0 and
 * 7 and its warp-per-row kernel under any other pin.  All families give bit-identical results;
 * tests use this to cover each on the same inputs.  The pin is per host thread: it changes
 * only the calls that thread makes. */
qift_status qift_debug_set_linear_path(int32_t path);

/* 1 in the bounds-checked build of the library (compiled with -DQIFT_CHECK, for tests), 0 in
 * the normal build.  In the checked build every global index, bulk-copy range, tensor-map
 * coordinate and tensor-memory address a kernel computes is tested against the extent its
 * arguments imply; a failed test skips that access, sets bit 0x100 of the device error word
 * (qift_device_error() then returns QIFT_ERR_CUDA with that bit in *detail) and keeps the source
 * line of the first failure. */
int32_t qift_debug_checked_build(void);

/* Read and clear the source line of the first failed bounds check since the last call (0: none;
 * always 0 in the normal build).  Call after qift_device_error() has synchronised the stream. */
qift_status qift_debug_check_line(int32_t* line);

#ifdef __cplusplus
}
#endif

#endif /* QIFT_DEBUG_H_ */

/*
 * qift.h -- C ABI of libqift.so, the B200 (sm_100a) hot path of Qift W2A4 linear layers.
 *
 * Method: "Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4
 * LLM Inference" (Huang, Tsai, arXiv 2606.02823v1), Abstract.  Weights and activations are
 * Hadamard-rotated; each weight row keeps one scale and takes one of four fixed levels
 * ({+-0.5, +-1.5} s, i.e. {+-1, +-3} under the half scale t = s/2; or the power-of-two set
 * {+-1, +-4} t applied by sign and shift; the standard {-2,-1,0,+1} t is the baseline); the
 * linear multiplies 2-bit weights with 4-bit activations.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers owned by the caller; the library allocates nothing and
 *     keeps no pointer after the call returns.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  A call returns once its kernels are launched, not when they finish.
 *   - Arguments are validated on the host before anything is launched; a bad argument returns
 *     QIFT_ERR_INVALID_ARG (or QIFT_ERR_UNSUPPORTED for a valid request this build does not
 *     implement) and enqueues nothing.  A launch failure returns QIFT_ERR_CUDA.
 *   - Device pointers must be 16-byte aligned.  Sizes are element counts.
 *   - No call synchronises.  Kernels that wait on on-chip barriers give up after a bounded
 *     number of polls and record QIFT_ERR_TIMEOUT in a device error word;
 *     qift_device_error() reads and clears it.
 *   - NaN or Inf inputs give unspecified (but memory-safe) results.
 */
#ifndef QIFT_H_
#define QIFT_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QIFT_OK = 0,
    QIFT_ERR_INVALID_ARG = 1,
    QIFT_ERR_UNSUPPORTED = 2,
    QIFT_ERR_CUDA = 3,
    QIFT_ERR_TIMEOUT = 4
} qift_status;

/* Level sets.  The 2-bit codes 0..3 map to levels in increasing order (code 0 = most
 * negative).  QIFT_SET_INT4 is the 4-bit set of the Abstract's mixed W2/W4 layers: levels
 * {-7, ..., +7} * s stored as two's-complement nibbles, eight per 32-bit word. */
typedef enum {
    QIFT_SET_QIFT = 0, /* {-3, -1, +1, +3} * t, t = s/2  (= {-1.5, -0.5, +0.5, +1.5} * s) */
    QIFT_SET_POT = 1,  /* {-4, -1, +1, +4} * t  (power of two: sign and shift)             */
    QIFT_SET_STD = 2,  /* {-2, -1,  0, +1} * t  (standard W2 baseline)                     */
    QIFT_SET_INT4 = 3  /* {-7, ..., +7} * s      (4-bit weights, W4A4)                      */
} qift_levelset;

typedef enum { QIFT_F32 = 0, QIFT_F16 = 1 } qift_dtype;

/*
 * qift_rotate -- block-diagonal normalised Walsh-Hadamard rotation along the last axis.
 * Abstract: "Hadamard-rotated quantization pipeline" -- weights offline (W' = W H_b^T, fp32)
 * and activations online (x' = H_b x, fp16).
 *   x, y   : [rows][n] row-major, dtype dt (QIFT_F32 or QIFT_F16 = IEEE binary16 bits).
 *            y may equal x (in place); partial overlap is not allowed.
 *   block  : b, a power of two in [2, 4096]; n % b == 0.  Every length-b segment of a row is
 *            multiplied by H_b / sqrt(b), H_b the Sylvester Hadamard matrix.
 * Arithmetic: fp32 butterflies in stage order h = 1, 2, ..., b/2 ((u, v) -> (u+v, u-v)),
 * then one multiply by (float)(1/sqrt(b)); fp16 output rounds once to nearest even.
 */
qift_status qift_rotate(const void* x, void* y, qift_dtype dt, int64_t rows, int64_t n, int32_t block,
                        void* stream);

/*
 * qift_quantize_weights -- per-output-channel scale search, nearest-level encode, 2-bit pack.
 * Abstract: fixed two-bit code-to-level mapping with "the standard per-channel scale"
 * (zero-point-free, group-grid-free).
 *   w_rot      : fp32 [n_out][n_in], the rotated weights.  n_in % 16 == 0, n_in <= 32768.
 *   grid_points: G in [2, 256] candidate scales per row; 0 < lo <= hi <= 4:
 *                f_k = lo + ((hi - lo) * k) / (G - 1), s_k = (float)((f_k * max|w_row|) / L),
 *                in binary64, L = 1.5 (Qift, s-form levels +-0.5 s, +-1.5 s), 4 (PoT), 2 (std).
 *                The usual search is G = 100, lo = 0.2, hi = 1.0.
 *   codes      : u32 [n_out][n_in/16] out.  Code of input k sits in word k/16 at bits
 *                2*(k%16) and 2*(k%16)+1.  QIFT_SET_INT4: u32 [n_out][n_in/8]; the level of
 *                input k, as a two's-complement nibble, in word k/8 at bits
 *                8*(k%4) + 4*((k%8)/4) .. +3 (byte j: input j low, input j+4 high); L = 7; the
 *                nearest level compares |w| with the midpoints (j + 0.5) s.
 *   scales     : fp32 [n_out] out: t = s_best/2 for Qift, s_best for PoT and std, so the
 *                weight is level(code) * t with the integer levels of the set.
 *   row_mse    : fp64 [n_out] out, or NULL: the best candidate's mean squared error.
 * The MSE of candidate k is sum over the row, in index order, of (float)e^2 widened to fp64,
 * e = |w| - level (Qift/PoT, fp32) or w - level (std); ties in MSE go to the smaller k, ties
 * between two levels to the smaller magnitude, w >= 0 (and -0.0) to the positive side.
 */
qift_status qift_quantize_weights(const float* w_rot, int64_t n_out, int64_t n_in, qift_levelset set,
                                  int32_t grid_points, double lo, double hi, uint32_t* codes,
                                  float* scales, double* row_mse, void* stream);

/*
 * qift_rotate_quantize_weights -- the offline pipeline in one pass: qift_rotate of the weights
 * (fp32) followed by qift_quantize_weights, fused.  Abstract: "Hadamard-rotated quantization
 * pipeline".  The rotation runs on each CTA's rows in shared memory with the operations and
 * order of qift_rotate, so codes, scales and row_mse are bit-identical to the two calls; HBM sees
 * one fp32 read of W and no rotated temporary.
 *   w     : fp32 [n_out][n_in], the raw weights (not modified).
 *   block : Hadamard block b as in qift_rotate (n_in % b == 0); 0 = w is already rotated.
 *   other arguments as in qift_quantize_weights.
 */
qift_status qift_rotate_quantize_weights(const float* w, int64_t n_out, int64_t n_in, int32_t block,
                                         qift_levelset set, int32_t grid_points, double lo, double hi,
                                         uint32_t* codes, float* scales, double* row_mse, void* stream);

/*
 * qift_quantize_weights_asym -- the conventional asymmetric W2 baseline the Abstract compares the
 * no-zero sets against ("Conventional asymmetric W2"): per output channel a scale s and an
 * integer zero point z in [0, 3], weight (c - z) * s.  The page gives no formula; this is the
 * min-max affine quantizer with the range shrunk over the same candidate grid:
 *   candidate f (as in qift_quantize_weights): s = (f * (max(max w, 0) - min(min w, 0))) / 3 in
 *   binary64, one rounding to binary32; z = the nearest integer, ties to even, of
 *   -(f * min(min w, 0)) / s in binary64, clamped to [0, 3] (0 when s = 0);
 *   code c = clamp(rint(w / s) + z, 0, 3), w / s one binary32 division (c = z when s = 0);
 *   error e = w - (c - z) * s in binary32, e * e summed in binary64 in input order; the
 *   smallest sum wins, the earlier candidate on ties.
 *   w_rot, n_out, n_in, grid_points, lo, hi, codes (2-bit, packed as in qift_quantize_weights),
 *   row_mse, stream: as in qift_quantize_weights.
 *   scales : fp32 [n_out] out: s.        zeros : int32 [n_out] out: z (4-byte aligned).
 * The library has no linear for this set: it serves the reconstruction-error comparison.
 */
qift_status qift_quantize_weights_asym(const float* w_rot, int64_t n_out, int64_t n_in, int32_t grid_points,
                                       double lo, double hi, uint32_t* codes, float* scales, int32_t* zeros,
                                       double* row_mse, void* stream);

/*
 * qift_quantize_acts -- optional rotation + symmetric per-token INT4 quantization.
 * Abstract: the "A4" of rotated W2A4 inference.
 *   x      : fp16 (binary16 bits) [tokens][n_in], n_in % 16 == 0, n_in <= 32768.
 *   block  : 0 = x is already rotated; else as in qift_rotate (n_in % block == 0).
 *   q      : int8 [tokens][n_in] out, values in [-7, 7], one per byte.
 *   scales : fp32 [tokens] out, s_a = m / 7 with m = max |x'| of the token.
 * x' is the rotated token rounded once to fp16; q = clamp(rint(x' * (7/m)), -7, 7) with
 * round-half-even and one fp32 division for 7/m; an all-zero token gives q = 0, s_a = 0.
 * Launched as a programmatic dependent: it waits for the previous kernel on `stream` before
 * touching memory, then lets the following qift_linear start its weight stream early.
 */
qift_status qift_quantize_acts(const void* x, int64_t tokens, int64_t n_in, int32_t block, int8_t* q,
                               float* scales, void* stream);

/*
 * qift_quantize_kv / qift_dequantize_kv -- KV4: keys and values kept in 4 bits (the title's
 * "Rotated W2A4/KV4 LLM Inference").  The pages give no KV scheme; this one is the activation
 * path's: each token's K or V row is rotated by Hadamard blocks of `block` (the head dimension,
 * typically) and quantized to symmetric per-token INT4 exactly as qift_quantize_acts does, then
 * stored as two's-complement nibbles, two per byte, the lower index in the low nibble.
 *   x       : fp16 [tokens][n], n % 16 == 0, n <= 32768 (quantize) / 16384 (dequantize).
 *   block   : 0 = no rotation; else a power of two in [2, 4096] dividing n.
 *   packed  : u8 [tokens][n/2], 16-byte aligned.   scales: fp32 [tokens] (s = m / 7).
 *   out     : fp16 [tokens][n]: (float)q * s in binary32, rotated back (H_b / sqrt(b) is its own
 *             inverse) with qift_rotate's stages, rounded once to nearest even.
 * Both are programmatic dependents of the previous kernel on `stream` that read their inputs
 * only after it has finished.
 */
qift_status qift_quantize_kv(const void* x, int64_t tokens, int64_t n, int32_t block, uint8_t* packed,
                             float* scales, void* stream);
qift_status qift_dequantize_kv(const uint8_t* packed, const float* scales, int64_t tokens, int64_t n,
                               int32_t block, void* out, void* stream);

/*
 * qift_linear -- fused W2A4 linear: y[t][n] = ((float)acc[t][n] * w_scale[n]) * act_scale[t],
 * acc[t][n] = sum_k q_act[t][k] * level(code[n][k]) in int32.
 * Abstract: "sign-and-shift decoded weight application" of the fixed 2-bit levels.
 *   q_act     : int8 [tokens][n_in] from qift_quantize_acts.  act_scale: fp32 [tokens].
 *   codes     : u32 [n_out][n_in/16], w_scale: fp32 [n_out], from qift_quantize_weights.
 *   set       : QIFT_SET_QIFT or QIFT_SET_POT (QIFT_SET_STD -> QIFT_ERR_UNSUPPORTED), or
 *               QIFT_SET_INT4 (W4A4: codes u32 [n_out][n_in/8]; n_in % 64 == 0, else
 *               QIFT_ERR_UNSUPPORTED; acc = sum q * level, |acc| <= 7*7*n_in; one token on CUDA
 *               cores, 2..16 on the int8 tensor cores (mma.sync), 17 or more on the tcgen05 GEMM).
 *   y         : [tokens][n_out] out, out_dt QIFT_F32 or QIFT_F16 (round to nearest even).
 *   n_in      : multiple of 16, at most 32768 (so |acc| <= 7*4*n_in < 2^24 and (float)acc is
 *               exact).  tokens == 0 or n_out == 0 is a no-op.
 * Decode-size batches (tokens <= 16) run as an HBM-streaming GEMV; larger batches as an int8
 * tensor-core GEMM, which needs n_in % 64 == 0: tokens >= 17 with another n_in returns
 * QIFT_ERR_UNSUPPORTED (pad n_in to a multiple of 64 with zero activations -- any code in the
 * padded positions then contributes nothing).  All paths give bit-identical results.
 * Overlap: every kernel of this call (decode sizes and the prefill GEMM) is launched as a
 * programmatic dependent of the previous kernel on `stream` and may start reading the weights
 * -- `codes` and `w_scale`, nothing else --
 * before that kernel has finished; the values of q_act and act_scale are read, and y written,
 * only after it has completed (their cache lines may be prefetched into L2 before, which
 * changes no value).  So the kernel launched immediately before qift_linear on the same stream
 * must not write `codes` or `w_scale` (the usual order qift_quantize_weights ->
 * qift_quantize_acts -> qift_linear satisfies this: qift_quantize_acts waits for its
 * predecessor before it lets qift_linear start).
 */
qift_status qift_linear(const int8_t* q_act, const float* act_scale, const uint32_t* codes,
                        const float* w_scale, qift_levelset set, int64_t tokens, int64_t n_out,
                        int64_t n_in, void* y, qift_dtype out_dt, void* stream);

/*
 * qift_decode_linear -- one decode step in a single launch: qift_quantize_acts followed by
 * qift_linear, fused, for 1..4 tokens.  Same arithmetic and bit-identical results as the two
 * calls; it exists because at decode batch sizes the separate activation kernel and the hand-off
 * between the two launches cost more than the activation work itself.
 *   x           : fp16 [tokens][n_in], 1 <= tokens <= 4; n_in % 64 == 0 and n_in <= 16384
 *                 (other valid sizes return QIFT_ERR_UNSUPPORTED: use the two calls).
 *   block       : Hadamard block as in qift_quantize_acts (0 = x already rotated).
 *   codes, w_scale, set (QIFT or POT; INT4 -> QIFT_ERR_UNSUPPORTED), n_out, y, out_dt: as in
 *                 qift_linear.
 *   q_out       : int8 [tokens][n_in] or NULL -- receives the INT4 activations.
 *   act_scale_out: fp32 [tokens] or NULL -- receives s_a.
 * Like the decode GEMV it may read `codes` and `w_scale` before the kernel launched just before
 * it on the same stream has finished, so that kernel must not write them.
 */
qift_status qift_decode_linear(const void* x, int64_t tokens, int64_t n_in, int32_t block, const uint32_t* codes,
                               const float* w_scale, qift_levelset set, int64_t n_out, void* y, qift_dtype out_dt,
                               int8_t* q_out, float* act_scale_out, void* stream);

/* qift_device_error -- synchronise `stream`, then read and clear the device error word.
 * Returns QIFT_OK, QIFT_ERR_TIMEOUT (a bounded on-chip wait gave up; that call's output is
 * invalid) or QIFT_ERR_CUDA (a CUDA error, or -- in the bounds-checked test build only -- a failed
 * bounds check, bit 0x100 of the word).  *detail (may be NULL) receives the raw word.  The word is one per
 * device (the current one), not per stream or per call: a timeout of a kernel on any stream of
 * the device is reported to -- and cleared by -- whichever caller reads it first, so a caller
 * that runs work on several streams should synchronise them before reading it. */
qift_status qift_device_error(void* stream, int32_t* detail);

/* Human-readable name of a status.  Never NULL. */
const char* qift_status_string(qift_status status);

#ifdef __cplusplus
}
#endif

#endif /* QIFT_H_ */

// common.cuh -- small helpers shared by the Qift CUDA kernels (sm_100a only).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libqift is written for sm_100a (B200) only"
#endif

namespace qift {

// Bounds-checked build (-DQIFT_CHECK, a separate library for tests): QIFT_CK(cond) tests an
// index, copy range, tensor-map coordinate or tensor-memory address against the extent the
// kernel's own arguments imply.  A failed test sets bit 0x100 of the device error word, keeps
// the first failing source line, and yields false, so the guarded access is skipped: no trap,
// and no thread leaves code that others synchronise with.  In the normal build QIFT_CK(cond)
// is the constant true and cond is not evaluated.
// The recorded site is file_tag(__FILE__) * 100000 + __LINE__: the tag is an FNV-1a hash of
// the file's base name, modulo 1000.
__host__ __device__ constexpr uint32_t fnv1a_tail(const char* s, uint32_t h) {
    return *s ? fnv1a_tail(s + 1, (h ^ (uint32_t)(unsigned char)*s) * 16777619u) : h;
}
__host__ __device__ constexpr const char* base_name(const char* s, const char* last) {
    return *s ? base_name(s + 1, *s == '/' ? s + 1 : last) : last;
}
__host__ __device__ constexpr int file_tag(const char* path) {
    return (int)(fnv1a_tail(base_name(path, path), 2166136261u) % 1000u);
}
#ifdef QIFT_CHECK
extern __device__ int g_qift_error;
extern __device__ int g_qift_check_line;
__device__ __noinline__ inline bool check_fail(int site) {
    atomicOr(&g_qift_error, 0x100);
    atomicCAS(&g_qift_check_line, 0, site);
    return false;
}
#define QIFT_CK(cond) ((cond) || ::qift::check_fail(::qift::file_tag(__FILE__) * 100000 + __LINE__))
#else
#define QIFT_CK(cond) ((void)sizeof((cond) ? 1 : 0), true)  // unevaluated: no code, no unused-variable warning
#endif
// [off, off + len) inside [0, extent)
#define QIFT_CK_RANGE(off, len, extent) \
    QIFT_CK((int64_t)(off) >= 0 && (int64_t)(off) + (int64_t)(len) <= (int64_t)(extent))

constexpr int kSetQift = 0;
constexpr int kSetPot = 1;
constexpr int kSetStd = 2;
constexpr int kSetInt4 = 3;  // 4-bit weights {-7..7} * s as two's-complement nibbles, eight per word
constexpr int kSetAsym = 4;  // conventional asymmetric W2: (c - z) * s, integer zero point z per row

// Integer level table of a set packed as four signed bytes, byte c = level of code c, so that
// one byte permute (prmt) turns four 2-bit codes into four int8 weights.
//   Qift {-3,-1,+1,+3}: bytes FD FF 01 03.   PoT {-4,-1,+1,+4}: bytes FC FF 01 04.
__host__ __device__ constexpr uint32_t level_lut(int set) {
    return set == kSetPot ? 0x0401FFFCu : 0x0301FFFDu;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ int dp4a(uint32_t a, uint32_t b, int c) {
    return __dp4a((int)a, (int)b, c);
}

// Decode one packed word (16 codes, code k at bits 2k..2k+1) into 16 int8 weights held in
// four registers, in the order the activations are permuted to:
//   d0 = codes {0,2,4,6}, d1 = {8,10,12,14}, d2 = {1,3,5,7}, d3 = {9,11,13,15}.
// even = w & 0x33333333 holds code 2i in nibble i; odd = (w >> 2) & 0x33333333 holds 2i+1.
// prmt reads the low 16 bits of its selector as four nibbles, each picking one LUT byte.
__device__ __forceinline__ void decode_word(uint32_t w, uint32_t lut, uint32_t d[4]) {
    const uint32_t even = w & 0x33333333u;
    const uint32_t odd = (w >> 2) & 0x33333333u;
    d[0] = prmt(lut, 0u, even);
    d[1] = prmt(lut, 0u, even >> 16);
    d[2] = prmt(lut, 0u, odd);
    d[3] = prmt(lut, 0u, odd >> 16);
}

// Permute 16 int8 activations (natural order in four words) into the decode_word order.
__device__ __forceinline__ void permute_acts(uint4 a, uint32_t p[4]) {
    p[0] = prmt(a.x, a.y, 0x6420u);   // bytes 0,2 of x and 0,2 of y -> k = 0,2,4,6
    p[1] = prmt(a.z, a.w, 0x6420u);   // k = 8,10,12,14
    p[2] = prmt(a.x, a.y, 0x7531u);   // k = 1,3,5,7
    p[3] = prmt(a.z, a.w, 0x7531u);   // k = 9,11,13,15
}

// Decode one packed word into 16 int8 weights in natural input order: d[j] holds the weights
// of inputs 4j .. 4j+3.  Each byte of codes (four 2-bit fields) is spread to four nibbles --
// a byte permute places bytes 0/1 (or 2/3) of w 16 bits apart, then two shift-or-mask steps
// move every 2-bit field into its own nibble -- and one byte permute per four codes reads
// the level table.
__device__ __forceinline__ uint32_t spread_codes_to_nibbles(uint32_t two_bytes_16_apart) {
    uint32_t x = two_bytes_16_apart;
    x = (x | (x << 4)) & 0x0F0F0F0Fu;
    x = (x | (x << 2)) & 0x33333333u;
    return x;
}

__device__ __forceinline__ void decode_word_natural(uint32_t w, uint32_t lut, uint32_t d[4]) {
    const uint32_t lo = spread_codes_to_nibbles(prmt(w, 0u, 0x4140u));   // codes 0..7
    const uint32_t hi = spread_codes_to_nibbles(prmt(w, 0u, 0x4342u));   // codes 8..15
    d[0] = prmt(lut, 0u, lo);
    d[1] = prmt(lut, 0u, lo >> 16);
    d[2] = prmt(lut, 0u, hi);
    d[3] = prmt(lut, 0u, hi >> 16);
}

// 16-byte read-only global load that the compiler keeps in program order relative to other
// volatile asm (notably griddepcontrol.wait): used to put weight loads in flight before a
// kernel waits for its predecessor.
__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Ask L2 for the 128-byte lines of [p, p + bytes), one line per thread of the CTA (data that
// only this CTA reads).  A hint only -- see prefetch_l2_grid.
__device__ __forceinline__ void prefetch_l2_cta(const void* p, int64_t bytes) {
    const char* b = static_cast<const char*>(p);
    for (int64_t off = (int64_t)threadIdx.x * 128; off < bytes; off += (int64_t)blockDim.x * 128)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(b + off));
}

// Ask L2 for the 128-byte lines of [p, p + bytes) that every CTA reads, each line once across
// the grid: thread t of
// CTA b takes lines (b + t * G), (b + t * G) + G * blockDim, ...  Only a hint: L2 is where
// global writes become coherent, so a line fetched before the producer of p has finished is
// updated in place by its writes, and loads after griddep_wait() see them.
__device__ __forceinline__ void prefetch_l2_grid(const void* p, int64_t bytes) {
    const char* b = static_cast<const char*>(p);
    const int64_t G = gridDim.x, step = G * blockDim.x * 128;
    for (int64_t off = ((int64_t)blockIdx.x + (int64_t)threadIdx.x * G) * 128; off < bytes; off += step)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(b + off));
}

// Programmatic dependent launch.  wait: block until the kernels this launch depends on have
// completed and their writes are visible (a no-op without a programmatic dependency).
// launch_dependents: allow the next kernel on the stream to start launching.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// Barrier policies for device code that a whole CTA, or only its first N threads, runs.
struct CtaSync {
    __device__ __forceinline__ static void sync() { __syncthreads(); }
};
// Named barrier 1 over threads 0 .. N-1 (N a multiple of 32); the other threads must not use
// barrier 1 meanwhile.
template <int N>
struct GroupSync {
    __device__ __forceinline__ static void sync() { asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory"); }
};

__host__ __device__ constexpr int ilog2(int v) { return v <= 1 ? 0 : 1 + ilog2(v >> 1); }

}  // namespace qift

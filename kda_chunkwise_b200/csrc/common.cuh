// Shared device helpers and compile-time constants of the KDA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// Decay floor of the scaled-sigmoid mapping ("Kimi K3 · Lesson 3 of 14", eq. 5 passage).
constexpr float kGMin = -5.0f;
// Chunk of the chunkwise form and its 16-token tiles ("Kimi K3 · Lesson 3 of 14": with the
// floor at -5 a tile accumulates at most 80 of log-decay, so 1/Gamma <= e^80 fits fp32/bf16).
constexpr int kChunk = 64;
constexpr int kTile = 16;
constexpr int kTilesPerChunk = kChunk / kTile;

// Bits of the per-device error word.
constexpr unsigned kErrBadSeqlens = 1u;   // cu_seqlens not monotone / not ending at total_tokens
constexpr unsigned kErrSeqTooLong = 2u;   // a sequence longer than the max_seqlen given
constexpr unsigned kErrTimeout = 4u;      // a bounded wait gave up
constexpr unsigned kErrRange = 16u;       // a prefill state ended non-finite: some fp16 tensor-core
                                          //   operand (state, pseudo-values, values) left +-65504

__device__ __forceinline__ int64_t min64(int64_t x, int64_t y) { return x < y ? x : y; }

// Token span [s0, s1) of sequence n, clamped into [0, total] so that malformed cu_seqlens can
// never address memory outside the packed tensors.  Returns false if cu_seqlens was malformed.
__device__ __forceinline__ bool seq_span(const int32_t *cu, int n, int num_seqs, int64_t total,
                                         int64_t &s0, int64_t &s1) {
    const int64_t r0 = cu[n], r1 = cu[n + 1];
    s0 = r0 < 0 ? 0 : (r0 > total ? total : r0);
    s1 = r1 < s0 ? s0 : (r1 > total ? total : r1);
    return r0 == s0 && r1 == s1 && (n != 0 || r0 == 0) && (n != num_seqs - 1 || r1 == total);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t x) {
    return __uint_as_float(static_cast<uint32_t>(x) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// Stores one output element in the caller's storage type (fp32 or bf16).
__device__ __forceinline__ void store_out(void *out, int64_t off, bool f32, float x) {
    if (f32) static_cast<float *>(out)[off] = x;
    else static_cast<uint16_t *>(out)[off] = f32_to_bf16(x);
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

// sigmoid from the hardware exp2 and reciprocal approximations (about 2 ulp); saturates cleanly
// (1 / inf = 0, no NaN) for |x| -> inf.
__device__ __forceinline__ float sigmoid_fast(float x) {
    return rcp_approx(1.0f + ex2_approx(-1.4426950408889634f * x));
}

// Log-decay g = g_min * sigmoid(exp(A_h) * a), with e^{A_h} precomputed by the caller.
__device__ __forceinline__ float log_decay(float a, float expA) {
    return kGMin * sigmoid_fast(expA * a);
}

}  // namespace kda

// Per-device error word; set with atomicOr by kernels, read and cleared by kda_sync_check.
// (The library is one translation unit, so this is its only definition.)
__device__ unsigned int g_kda_error_word = 0u;

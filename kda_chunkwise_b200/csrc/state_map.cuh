// Affine state maps for context-parallel prefill.
//
// Over a segment of a sequence the recurrence is affine in its incoming state: the state after
// the segment is S_out = M S_in + B, where B is the state reached from S_in = 0 and M the state
// reached by the homogeneous recurrence (v = 0) from S_in = I (both d_k x d_k / d_k x d_v per
// head).  Segments held by different GPUs exchange (M, B), fold them in order to get their
// incoming states, and rerun with the right initial state.  (The pages fix only that the state
// is carried sequentially and has a fixed shape: "Kimi K3 · Lesson 3 of 14", CHUNKWISE diagram;
// "K3 Architecture Illustrated", FIG 22.)
//
// This kernel applies one map: S_out[u] = M[u] S_in[u] + B[u] for every (sequence, head) unit u,
// in fp32 on the CUDA cores (the maps are small: 2 d_k^2 d_v flops per unit).
#pragma once

#include "common.cuh"

namespace kda {

constexpr int kCombineRows = 16;   // output rows per CTA
constexpr int kCombineK = 32;      // k-slab of S_in staged in shared memory

struct CombineParams {
    const float *M, *S_in, *B;
    float *S_out;
};

// grid: (DK / kCombineRows, units); block: 256 threads = kCombineRows rows x 16 column groups
template <int DK, int DV>
__global__ void __launch_bounds__(256) state_combine_kernel(const CombineParams p) {
    constexpr int CPT = DV / 16;   // columns per thread
    __shared__ float sS[kCombineK][DV];
    __shared__ float sM[kCombineRows][kCombineK + 1];
    const int64_t u = blockIdx.y;
    const int r0 = blockIdx.x * kCombineRows;
    const int tid = threadIdx.x, row = tid / 16, cg = tid % 16;
    const float *M = p.M + u * DK * DK;
    const float *S = p.S_in + u * DK * DV;
    float acc[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) acc[j] = 0.f;
    for (int k0 = 0; k0 < DK; k0 += kCombineK) {
        for (int e = tid; e < kCombineK * DV; e += 256) sS[e / DV][e % DV] = S[(int64_t)(k0 + e / DV) * DV + e % DV];
        for (int e = tid; e < kCombineRows * kCombineK; e += 256)
            sM[e / kCombineK][e % kCombineK] = M[(int64_t)(r0 + e / kCombineK) * DK + k0 + e % kCombineK];
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < kCombineK; ++k) {
            const float m = sM[row][k];
#pragma unroll
            for (int j = 0; j < CPT; ++j) acc[j] = fmaf(m, sS[k][cg + 16 * j], acc[j]);
        }
        __syncthreads();
    }
    const int64_t base = u * DK * DV + (int64_t)(r0 + row) * DV;
#pragma unroll
    for (int j = 0; j < CPT; ++j) p.S_out[base + cg + 16 * j] = acc[j] + p.B[base + cg + 16 * j];
}

}  // namespace kda

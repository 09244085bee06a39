// Decode step: one token of the KDA recurrence for N independent (sequence, head) states.
//
// Per state (d_k x d_v fp32, row = key channel), with alpha = exp(g):
//   S' = Diag(alpha) S;  r = S'^T k;  p = S'^T (scale q);  u = beta (v - r)
//   S  = S' + k u^T;     o = S^T (scale q) = p + (k . scale q) u;  out = sigmoid(gate) o
// ("Review A · Sequence and depth", Free recall: fade, erase, write, then the read S^T q;
//  "K3 Architecture Illustrated", FIG 22: the decode state keeps a fixed shape.)
//
// The step is HBM-bound (0.87 FLOP per byte): every state is read once and written once.  One CTA
// owns one state; each warp streams whole 512-byte rows with 16-byte loads, holds its rows in
// registers across the two phases (column reductions r and p, then the rank-1 update), and the
// two column reductions meet in shared memory.  Reading and writing use streaming cache hints
// because a state is touched once per step.
#pragma once

#include "common.cuh"

namespace kda {

struct DecodeParams {
    const uint16_t *q, *k, *v, *a, *gate;
    const float *beta, *A_log;
    float *state;
    void *out;
    int H;
    bool out_f32;
    float scale;
};

__device__ __forceinline__ float4 f4_fma(float s, float4 x, float4 acc) {
    acc.x = fmaf(s, x.x, acc.x);
    acc.y = fmaf(s, x.y, acc.y);
    acc.z = fmaf(s, x.z, acc.z);
    acc.w = fmaf(s, x.w, acc.w);
    return acc;
}

constexpr int kDecodeThreads = 256;

template <int DK, int DV>
__global__ void __launch_bounds__(kDecodeThreads) decode_step_kernel(const DecodeParams p) {
    constexpr int kThreads = kDecodeThreads;
    constexpr int LPR = DV / 4;          // threads per state row, one float4 each
    constexpr int RPP = kThreads / LPR;  // rows covered by the block in one pass
    constexpr int NR = DK / RPP;         // rows held per thread
    static_assert(DK % RPP == 0, "row split");

    __shared__ float s_alpha[DK], s_k[DK], s_q[DK];
    __shared__ float4 s_red[2][RPP][LPR];
    __shared__ __align__(16) float s_u[DV];
    __shared__ float s_kq;

    const int64_t nh = blockIdx.x;
    const int h = static_cast<int>(nh % p.H);
    const int tid = threadIdx.x;
    const int cq = tid % LPR, rg = tid / LPR;

    float4 *St = reinterpret_cast<float4 *>(p.state + nh * (int64_t)(DK * DV));
    float4 S[NR];
#pragma unroll
    for (int m = 0; m < NR; ++m) S[m] = __ldcs(St + (rg + m * RPP) * LPR + cq);

    const float expA = expf(p.A_log[h]);
    for (int i = tid; i < DK; i += kThreads) {
        const int64_t off = nh * DK + i;
        s_alpha[i] = __expf(log_decay(bf16_to_f32(p.a[off]), expA));
        s_k[i] = bf16_to_f32(p.k[off]);
        s_q[i] = p.scale * bf16_to_f32(p.q[off]);
    }
    __syncthreads();
    if (tid < 32) {
        float acc = 0.f;
        for (int i = tid; i < DK; i += 32) acc = fmaf(s_k[i], s_q[i], acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (tid == 0) s_kq = acc;
    }

    float4 r = make_float4(0.f, 0.f, 0.f, 0.f), pq = r;
#pragma unroll
    for (int m = 0; m < NR; ++m) {
        const int row = rg + m * RPP;
        const float al = s_alpha[row];
        S[m].x *= al; S[m].y *= al; S[m].z *= al; S[m].w *= al;
        r = f4_fma(s_k[row], S[m], r);
        pq = f4_fma(s_q[row], S[m], pq);
    }
    s_red[0][rg][cq] = r;
    s_red[1][rg][cq] = pq;
    __syncthreads();

    if (tid < DV) {
        const float *red_r = reinterpret_cast<const float *>(&s_red[0][0][0]);
        const float *red_p = reinterpret_cast<const float *>(&s_red[1][0][0]);
        float rr = 0.f, pp = 0.f;
#pragma unroll 8
        for (int g = 0; g < RPP; ++g) {
            rr += red_r[g * DV + tid];
            pp += red_p[g * DV + tid];
        }
        const int64_t off = nh * DV + tid;
        const float u = p.beta[nh] * (bf16_to_f32(p.v[off]) - rr);
        s_u[tid] = u;
        float o = fmaf(s_kq, u, pp);
        if (p.gate) o *= sigmoid_fast(bf16_to_f32(p.gate[off]));
        store_out(p.out, off, p.out_f32, o);
    }
    __syncthreads();

    const float4 u4 = reinterpret_cast<const float4 *>(s_u)[cq];
#pragma unroll
    for (int m = 0; m < NR; ++m) {
        const int row = rg + m * RPP;
        const float kk = s_k[row];
        float4 s = S[m];
        s.x = fmaf(kk, u4.x, s.x);
        s.y = fmaf(kk, u4.y, s.y);
        s.z = fmaf(kk, u4.z, s.z);
        s.w = fmaf(kk, u4.w, s.w);
        __stcs(St + row * LPR + cq, s);
    }
}

}  // namespace kda

// Multi-token decode with rollback, for speculative decoding: verify K proposed tokens against
// every state, then advance each state by the number of tokens its sequence accepted.
//
// The pages only fix that the recurrent state needs rollback handling once proposals are
// rejected ("K3 Architecture Illustrated", "Speculative decoding changes the value of extra
// computation").  The plainest reading: after a verify pass over tokens 1..K, the state must
// become the state after exactly the accepted prefix 1..j.  The recurrence makes that cheap
// without storing K states: with alpha_t = exp(g_t) and the write vector
//   u_t = beta_t (v_t - (Diag(alpha_t) S_{t-1})^T k_t),      S_t = Diag(alpha_t) S_{t-1} + k_t u_t^T,
// the state after j tokens needs only S_0, the k_t and g_t (inputs) and the K write vectors u_t
// (d_v floats each).  So
//   verify: read S_0 once, run the K tokens in registers, write every output and u_t;
//           the state in memory is not touched;
//   commit: read S_0 once, apply the first j_n updates, write S_{j_n} once (j_n = 0 leaves the
//           state as it was and writes nothing).
// Both kernels are HBM-bound and use the layout of the single-token decode step (one CTA per
// state, whole 512-byte rows per warp with 16-byte streaming loads held in registers).  Every
// token's small inputs (and commit's write vectors) are staged in shared memory up front, so the
// K dependent token steps wait on no global load.
#pragma once

#include "common.cuh"
#include "decode.cuh"

namespace kda {

constexpr int kSpecMaxTokens = 16;
constexpr int kSpecThreads = kDecodeThreads;   // the same reduction order as the decode step
constexpr unsigned kErrBadAccepted = 8u;   // error-word bit: an accepted count outside [0, K]

struct SpecParams {
    const uint16_t *q, *k, *v, *a, *gate;   // [N, K, H, d]
    const float *beta, *A_log;              // [N, K, H], [H]
    const int32_t *accepted;                // [N]   (commit)
    float *state;                           // [N, H, d_k, d_v]
    float *u;                               // [N, H, K, d_v]
    void *out;                              // [N, K, H, d_v]
    int H, K;
    bool out_f32;
    float scale;
};

template <int DK, int DV>
__global__ void __launch_bounds__(kSpecThreads) spec_verify_kernel(const SpecParams p) {
    constexpr int kThreads = kSpecThreads;
    constexpr int LPR = DV / 4;          // threads per state row, one float4 each
    constexpr int RPP = kThreads / LPR;  // rows covered by the block in one pass
    constexpr int NR = DK / RPP;         // rows held per thread

    __shared__ float s_alpha[kSpecMaxTokens][DK], s_k[kSpecMaxTokens][DK], s_q[kSpecMaxTokens][DK];
    __shared__ float s_v[kSpecMaxTokens][DV], s_beta[kSpecMaxTokens];
    __shared__ uint16_t s_g[kSpecMaxTokens][DV];   // gate logits (bf16)
    __shared__ float4 s_red[2][RPP][LPR];
    __shared__ __align__(16) float s_u[DV];
    __shared__ float s_kq;

    const int64_t nh = blockIdx.x;
    const int64_t n = nh / p.H;
    const int h = static_cast<int>(nh % p.H);
    const int tid = threadIdx.x;
    const int cq = tid % LPR, rg = tid / LPR;

    const float4 *St = reinterpret_cast<const float4 *>(p.state + nh * (int64_t)(DK * DV));
    float4 S[NR];
#pragma unroll
    for (int m = 0; m < NR; ++m) S[m] = __ldcs(St + (rg + m * RPP) * LPR + cq);
    const float expA = expf(p.A_log[h]);
    for (int e = tid; e < p.K * DK; e += kThreads) {   // all K tokens' inputs, once
        const int t = e / DK, i = e % DK;
        const int64_t tok = (n * p.K + t) * p.H + h;   // row of token t of this sequence, head h
        s_alpha[t][i] = __expf(log_decay(bf16_to_f32(p.a[tok * DK + i]), expA));
        s_k[t][i] = bf16_to_f32(p.k[tok * DK + i]);
        s_q[t][i] = p.scale * bf16_to_f32(p.q[tok * DK + i]);
    }
    for (int e = tid; e < p.K * DV; e += kThreads) {
        const int t = e / DV, i = e % DV;
        const int64_t off = ((n * p.K + t) * p.H + h) * DV + i;
        s_v[t][i] = bf16_to_f32(p.v[off]);
        if (p.gate) s_g[t][i] = p.gate[off];
    }
    if (tid < p.K) s_beta[tid] = p.beta[(n * p.K + tid) * p.H + h];
    __syncthreads();

    for (int t = 0; t < p.K; ++t) {
        const int64_t tok = (n * p.K + t) * p.H + h;
        if (tid < 32) {
            float acc = 0.f;
            for (int i = tid; i < DK; i += 32) acc = fmaf(s_k[t][i], s_q[t][i], acc);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (tid == 0) s_kq = acc;
        }
        float4 r = make_float4(0.f, 0.f, 0.f, 0.f), pq = r;
#pragma unroll
        for (int m = 0; m < NR; ++m) {
            const int row = rg + m * RPP;
            const float al = s_alpha[t][row];
            S[m].x *= al; S[m].y *= al; S[m].z *= al; S[m].w *= al;
            r = f4_fma(s_k[t][row], S[m], r);
            pq = f4_fma(s_q[t][row], S[m], pq);
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
            const int64_t off = tok * DV + tid;
            const float u = s_beta[t] * (s_v[t][tid] - rr);
            s_u[tid] = u;
            p.u[(nh * p.K + t) * DV + tid] = u;
            float o = fmaf(s_kq, u, pp);
            if (p.gate) o *= sigmoid_fast(bf16_to_f32(s_g[t][tid]));
            store_out(p.out, off, p.out_f32, o);
        }
        __syncthreads();
        const float4 u4 = reinterpret_cast<const float4 *>(s_u)[cq];
#pragma unroll
        for (int m = 0; m < NR; ++m) {
            const float kk = s_k[t][rg + m * RPP];
            S[m].x = fmaf(kk, u4.x, S[m].x);
            S[m].y = fmaf(kk, u4.y, S[m].y);
            S[m].z = fmaf(kk, u4.z, S[m].z);
            S[m].w = fmaf(kk, u4.w, S[m].w);
        }
        // the next token overwrites s_u and s_red only after every thread is done here
        __syncthreads();
    }
}

template <int DK, int DV>
__global__ void __launch_bounds__(kSpecThreads) spec_commit_kernel(const SpecParams p) {
    constexpr int kThreads = kSpecThreads;
    constexpr int LPR = DV / 4;
    constexpr int RPP = kThreads / LPR;
    constexpr int NR = DK / RPP;

    __shared__ float s_alpha[kSpecMaxTokens][DK], s_k[kSpecMaxTokens][DK];
    __shared__ __align__(16) float s_uw[kSpecMaxTokens][DV];

    const int64_t nh = blockIdx.x;
    const int64_t n = nh / p.H;
    const int h = static_cast<int>(nh % p.H);
    const int tid = threadIdx.x;
    const int cq = tid % LPR, rg = tid / LPR;

    int j = p.accepted[n];
    if (j < 0 || j > p.K) {
        if (tid == 0 && h == 0) atomicOr(&g_kda_error_word, kErrBadAccepted);
        j = j < 0 ? 0 : p.K;
    }
    if (j == 0) return;   // nothing accepted: the state stays as it is

    const float expA = expf(p.A_log[h]);
    for (int e = tid; e < j * DK; e += kThreads) {
        const int t = e / DK, i = e % DK;
        const int64_t tok = (n * p.K + t) * p.H + h;
        s_alpha[t][i] = __expf(log_decay(bf16_to_f32(p.a[tok * DK + i]), expA));
        s_k[t][i] = bf16_to_f32(p.k[tok * DK + i]);
    }
    for (int e = tid; e < j * DV; e += kThreads) s_uw[e / DV][e % DV] = __ldcs(p.u + (nh * p.K + e / DV) * DV + e % DV);
    __syncthreads();

    float4 *St = reinterpret_cast<float4 *>(p.state + nh * (int64_t)(DK * DV));
    float4 S[NR];
#pragma unroll
    for (int m = 0; m < NR; ++m) S[m] = __ldcs(St + (rg + m * RPP) * LPR + cq);
    for (int t = 0; t < j; ++t) {
        const float4 u4 = reinterpret_cast<const float4 *>(s_uw[t])[cq];
#pragma unroll
        for (int m = 0; m < NR; ++m) {
            const int row = rg + m * RPP;
            const float al = s_alpha[t][row], kk = s_k[t][row];
            S[m].x = fmaf(kk, u4.x, al * S[m].x);
            S[m].y = fmaf(kk, u4.y, al * S[m].y);
            S[m].z = fmaf(kk, u4.z, al * S[m].z);
            S[m].w = fmaf(kk, u4.w, al * S[m].w);
        }
    }
#pragma unroll
    for (int m = 0; m < NR; ++m) __stcs(St + (rg + m * RPP) * LPR + cq, S[m]);
}

}  // namespace kda

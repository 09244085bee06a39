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
#include "mma_frag.cuh"
#include "async_copy.cuh"
#include "f32x2.cuh"

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

// Dynamic shared memory of the verify kernel: the next state (fp32, its global layout), the next
// unit's raw inputs (bf16 a, k, q [K][DK], v, gate [K][DV]; fp32 beta [K]) and the current unit's
// derived inputs ({alpha, alpha, k, k} [K][DK] as float4 and {scale q, scale q} [K][DK] as float2,
// each pair one operand of the paired fp32 instructions; v, sigmoid(gate) [K][DV], beta [K],
// k . scale q [K], fp32).
template <int DK, int DV>
struct SpecVerifySmem {
    __host__ __device__ static size_t raw_off() { return (size_t)DK * DV * 4; }
    __host__ __device__ static size_t beta_off(int K) { return raw_off() + (size_t)K * (3 * DK + 2 * DV) * 2; }
    __host__ __device__ static size_t derived_off(int K) { return beta_off(K) + (size_t)((K + 3) & ~3) * 4; }
    __host__ __device__ static size_t bytes(int K) { return derived_off(K) + (size_t)K * (6 * DK + 2 * DV + 2) * 4; }
};

// Persistent: a CTA takes units blockIdx.x, blockIdx.x + gridDim.x, ...; while it runs the K token
// steps of one unit, the next unit's state and inputs are copied into shared memory asynchronously,
// so the loads of HBM overlap the dependent token steps.
template <int DK, int DV>
__global__ void __launch_bounds__(kSpecThreads) spec_verify_kernel(const SpecParams p, int64_t units) {
    constexpr int kThreads = kSpecThreads;
    constexpr int LPR = DV / 4;          // threads per state row, one float4 each
    constexpr int RPP = kThreads / LPR;  // rows covered by the block in one pass
    constexpr int NR = DK / RPP;         // rows held per thread
    using SL = SpecVerifySmem<DK, DV>;

    extern __shared__ __align__(16) unsigned char spec_dyn[];
    const int K = p.K;
    const float4 *sS = reinterpret_cast<const float4 *>(spec_dyn);
    const uint16_t *r_a = reinterpret_cast<const uint16_t *>(spec_dyn + SL::raw_off());
    const uint16_t *r_k = r_a + K * DK, *r_q = r_k + K * DK, *r_v = r_q + K * DK, *r_g = r_v + K * DV;
    const float *r_beta = reinterpret_cast<const float *>(spec_dyn + SL::beta_off(K));
    float4 *s_ak = reinterpret_cast<float4 *>(spec_dyn + SL::derived_off(K));   // {alpha, alpha, k, k}
    float2 *s_qq = reinterpret_cast<float2 *>(s_ak + K * DK);                   // {scale q, scale q}
    float *s_v = reinterpret_cast<float *>(s_qq + K * DK), *s_sg = s_v + K * DV;
    float *s_b = s_sg + K * DV, *s_kqt = s_b + K;
    // per token: the row groups' partial column sums, then the sums ([r or p][column quad])
    __shared__ float4 s_red[2][RPP][LPR];
    __shared__ float4 s_sum[2][LPR];

    const int tid = threadIdx.x;
    const int cq = tid % LPR, rg = tid / LPR;
    auto issue = [&](int64_t nh) {   // asynchronous copy of unit nh's state and inputs
        const int64_t n = nh / p.H;
        const int h = static_cast<int>(nh % p.H);
        const uint32_t base = smem_u32(spec_dyn);
        const float *St = p.state + nh * (int64_t)(DK * DV);
        for (int e = tid; e < DK * DV / 4; e += kThreads) cp_async_16(base + e * 16, St + e * 4, 16);
        const uint32_t raw = base + (uint32_t)SL::raw_off();
        for (int e = tid; e < K * (3 * DK / 8); e += kThreads) {   // a, k, q rows: 16 bytes = 8 values
            const int which = e / (K * DK / 8), r = e % (K * DK / 8), t = r / (DK / 8), j = r % (DK / 8);
            const uint16_t *src = which == 0 ? p.a : (which == 1 ? p.k : p.q);
            cp_async_16(raw + ((which * K + t) * DK + j * 8) * 2, src + ((n * K + t) * p.H + h) * DK + j * 8, 16);
        }
        for (int e = tid; e < K * (DV / 8); e += kThreads) {
            const int t = e / (DV / 8), j = e % (DV / 8);
            const int64_t off = ((n * K + t) * p.H + h) * DV + j * 8;
            cp_async_16(raw + (3 * K * DK + t * DV + j * 8) * 2, p.v + off, 16);
            if (p.gate) cp_async_16(raw + (3 * K * DK + (K + t) * DV + j * 8) * 2, p.gate + off, 16);
        }
        const uint32_t rb = base + (uint32_t)SL::beta_off(K);
        for (int t = tid; t < K; t += kThreads) cp_async_4(rb + t * 4, p.beta + (n * K + t) * p.H + h);
        cp_async_commit();
    };

    int64_t nh = blockIdx.x;
    if (nh < units) issue(nh);
    for (; nh < units; nh += gridDim.x) {
        const int64_t n = nh / p.H;
        const int h = static_cast<int>(nh % p.H);
        cp_async_wait_all();
        __syncthreads();   // this unit's copies have landed (every thread's)
        ulonglong2 S[NR];   // this thread's four columns of each row, as two packed pairs
#pragma unroll
        for (int m = 0; m < NR; ++m) S[m] = reinterpret_cast<const ulonglong2 *>(sS)[(rg + m * RPP) * LPR + cq];
        const float expA = expf(p.A_log[h]);
        for (int e = tid; e < K * DK; e += kThreads) {
            const float al = __expf(log_decay(bf16_to_f32(r_a[e]), expA)), kv = bf16_to_f32(r_k[e]);
            const float qv = p.scale * bf16_to_f32(r_q[e]);
            s_ak[e] = make_float4(al, al, kv, kv);
            s_qq[e] = make_float2(qv, qv);
        }
        for (int e = tid; e < K * DV; e += kThreads) {
            s_v[e] = bf16_to_f32(r_v[e]);
            if (p.gate) s_sg[e] = sigmoid_fast(bf16_to_f32(r_g[e]));
        }
        for (int t = tid; t < K; t += kThreads) s_b[t] = r_beta[t];
        __syncthreads();
        for (int t = tid >> 5; t < K; t += kThreads / 32) {   // k . scale q per token, as the decode step
            const int lane = tid & 31;
            float acc = 0.f;
            for (int i = lane; i < DK; i += 32) acc = fmaf(s_ak[t * DK + i].z, s_qq[t * DK + i].x, acc);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) s_kqt[t] = acc;
        }   // the state and raw buffers are free for the next unit
        if (nh + gridDim.x < units) issue(nh + gridDim.x);

        for (int t = 0; t < K; ++t) {
            const int64_t tok = (n * K + t) * p.H + h;
            // the decode step's arithmetic, two columns per instruction (same roundings, same bits)
            ulonglong2 r = make_ulonglong2(0ull, 0ull), pq = r;
#pragma unroll
            for (int m = 0; m < NR; ++m) {
                const int row = rg + m * RPP;
                const ulonglong2 ak = reinterpret_cast<const ulonglong2 *>(s_ak)[t * DK + row];   // (alpha, alpha), (k, k)
                const f32x2 qq = reinterpret_cast<const f32x2 *>(s_qq)[t * DK + row];
                S[m].x = f2_mul(S[m].x, ak.x);
                S[m].y = f2_mul(S[m].y, ak.x);
                r.x = f2_fma(ak.y, S[m].x, r.x);
                r.y = f2_fma(ak.y, S[m].y, r.y);
                pq.x = f2_fma(qq, S[m].x, pq.x);
                pq.y = f2_fma(qq, S[m].y, pq.y);
            }
            reinterpret_cast<ulonglong2 &>(s_red[0][rg][cq]) = r;
            reinterpret_cast<ulonglong2 &>(s_red[1][rg][cq]) = pq;
            __syncthreads();   // (the k . q of every token is ready too)
            // the column sums, once per column quad (2 x LPR threads), in row-group order from zero
            // as the decode step adds them; then every thread reads its own
            if (tid < 2 * LPR) {
                const int w = tid / LPR, c4 = tid % LPR;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int g = 0; g < RPP; ++g) {
                    const float4 x = s_red[w][g][c4];
                    acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
                }
                s_sum[w][c4] = acc;
            }
            __syncthreads();
            const float4 rr = s_sum[0][cq], pp = s_sum[1][cq];
            const float bt = s_b[t];
            const float4 v4 = reinterpret_cast<const float4 *>(s_v + t * DV)[cq];
            const float4 u4 = make_float4(bt * (v4.x - rr.x), bt * (v4.y - rr.y), bt * (v4.z - rr.z), bt * (v4.w - rr.w));
            if (rg == 0) {   // the first row group holds every column once
                reinterpret_cast<float4 *>(p.u + (nh * K + t) * DV)[cq] = u4;
                const float kq = s_kqt[t];
                float o[4] = {fmaf(kq, u4.x, pp.x), fmaf(kq, u4.y, pp.y), fmaf(kq, u4.z, pp.z), fmaf(kq, u4.w, pp.w)};
                if (p.gate) {
                    const float4 sg = reinterpret_cast<const float4 *>(s_sg + t * DV)[cq];
                    o[0] *= sg.x; o[1] *= sg.y; o[2] *= sg.z; o[3] *= sg.w;
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) store_out(p.out, tok * DV + 4 * cq + c, p.out_f32, o[c]);
            }
            const f32x2 u01 = f2_pack(u4.x, u4.y), u23 = f2_pack(u4.z, u4.w);
#pragma unroll
            for (int m = 0; m < NR; ++m) {
                const f32x2 kk = reinterpret_cast<const f32x2 *>(s_ak)[2 * (t * DK + rg + m * RPP) + 1];   // (k, k)
                S[m].x = f2_fma(kk, u01, S[m].x);
                S[m].y = f2_fma(kk, u23, S[m].y);
            }
        }
        __syncthreads();   // the derived inputs are read by every thread before the next unit's
    }
    cp_async_wait_all();   // nothing is left in flight at exit
}

// Dynamic shared memory of the commit kernel: the next state (fp32, its global layout), the next
// unit's raw inputs (bf16 a, k [K][DK]; fp32 write vectors u [K][DV]) and the current unit's alpha
// and k [K][DK] and write vectors [K][DV] (fp32).
template <int DK, int DV>
struct SpecCommitSmem {
    __host__ __device__ static size_t raw_off() { return (size_t)DK * DV * 4; }
    __host__ __device__ static size_t u_off(int K) { return raw_off() + (size_t)K * 2 * DK * 2; }
    __host__ __device__ static size_t derived_off(int K) { return u_off(K) + (size_t)K * DV * 4; }
    __host__ __device__ static size_t bytes(int K) { return derived_off(K) + (size_t)K * (2 * DK + DV) * 4; }
};

// Persistent, like the verify pass: while one state takes its accepted updates and is written
// back, the next state that accepted anything (and its inputs) is copied into shared memory.
// States whose sequence accepted nothing are neither read nor written.
template <int DK, int DV>
__global__ void __launch_bounds__(kSpecThreads) spec_commit_kernel(const SpecParams p, int64_t units) {
    constexpr int kThreads = kSpecThreads;
    constexpr int LPR = DV / 4;
    constexpr int RPP = kThreads / LPR;
    constexpr int NR = DK / RPP;
    using SL = SpecCommitSmem<DK, DV>;

    extern __shared__ __align__(16) unsigned char spec_dyn[];
    const int K = p.K;
    const float4 *sS = reinterpret_cast<const float4 *>(spec_dyn);
    const uint16_t *r_a = reinterpret_cast<const uint16_t *>(spec_dyn + SL::raw_off()), *r_k = r_a + K * DK;
    const float *r_u = reinterpret_cast<const float *>(spec_dyn + SL::u_off(K));
    float *s_alpha = reinterpret_cast<float *>(spec_dyn + SL::derived_off(K)), *s_k = s_alpha + K * DK;
    float *s_u = s_k + K * DK;

    const int tid = threadIdx.x;
    const int cq = tid % LPR, rg = tid / LPR;
    auto accepted = [&](int64_t nh) {   // the accepted count of unit nh's sequence, clamped to [0, K]
        const int64_t n = nh / p.H;
        int j = p.accepted[n];
        if (j < 0 || j > K) {
            if (tid == 0 && nh % p.H == 0) atomicOr(&g_kda_error_word, kErrBadAccepted);
            j = j < 0 ? 0 : K;
        }
        return j;
    };
    auto issue = [&](int64_t nh, int j) {   // asynchronous copy of unit nh's state and first j tokens' inputs
        const int64_t n = nh / p.H;
        const int h = static_cast<int>(nh % p.H);
        const uint32_t base = smem_u32(spec_dyn);
        const float *St = p.state + nh * (int64_t)(DK * DV);
        for (int e = tid; e < DK * DV / 4; e += kThreads) cp_async_16(base + e * 16, St + e * 4, 16);
        const uint32_t raw = base + (uint32_t)SL::raw_off();
        for (int e = tid; e < j * (2 * DK / 8); e += kThreads) {   // a, k rows: 16 bytes = 8 values
            const int which = e / (j * DK / 8), r = e % (j * DK / 8), t = r / (DK / 8), c8 = r % (DK / 8);
            const uint16_t *src = which == 0 ? p.a : p.k;
            cp_async_16(raw + ((which * K + t) * DK + c8 * 8) * 2, src + ((n * K + t) * p.H + h) * DK + c8 * 8, 16);
        }
        const uint32_t ru = base + (uint32_t)SL::u_off(K);
        for (int e = tid; e < j * (DV / 4); e += kThreads)
            cp_async_16(ru + e * 16, p.u + (nh * K) * DV + e * 4, 16);
        cp_async_commit();
    };
    auto next_unit = [&](int64_t nh, int &j) {   // the first unit from nh on that accepted anything
        for (; nh < units; nh += gridDim.x)
            if ((j = accepted(nh)) > 0) return nh;
        return units;
    };

    int j = 0;
    int64_t nh = next_unit(blockIdx.x, j);
    if (nh < units) issue(nh, j);
    while (nh < units) {
        const int h = static_cast<int>(nh % p.H);
        cp_async_wait_all();
        __syncthreads();   // this unit's copies have landed (every thread's)
        float4 S[NR];
#pragma unroll
        for (int m = 0; m < NR; ++m) S[m] = sS[(rg + m * RPP) * LPR + cq];
        const float expA = expf(p.A_log[h]);
        for (int e = tid; e < j * DK; e += kThreads) {
            s_alpha[e] = __expf(log_decay(bf16_to_f32(r_a[e]), expA));
            s_k[e] = bf16_to_f32(r_k[e]);
        }
        for (int e = tid; e < j * DV / 4; e += kThreads)
            reinterpret_cast<float4 *>(s_u)[e] = reinterpret_cast<const float4 *>(r_u)[e];
        __syncthreads();   // the state and raw buffers are free for the next unit
        int j2 = 0;
        const int64_t nh2 = next_unit(nh + gridDim.x, j2);
        if (nh2 < units) issue(nh2, j2);
        for (int t = 0; t < j; ++t) {
            const float4 u4 = reinterpret_cast<const float4 *>(s_u + t * DV)[cq];
#pragma unroll
            for (int m = 0; m < NR; ++m) {
                const int row = rg + m * RPP;
                const float al = s_alpha[t * DK + row], kk = s_k[t * DK + row];
                S[m].x = fmaf(kk, u4.x, al * S[m].x);
                S[m].y = fmaf(kk, u4.y, al * S[m].y);
                S[m].z = fmaf(kk, u4.z, al * S[m].z);
                S[m].w = fmaf(kk, u4.w, al * S[m].w);
            }
        }
        float4 *St = reinterpret_cast<float4 *>(p.state + nh * (int64_t)(DK * DV));
#pragma unroll
        for (int m = 0; m < NR; ++m) __stcs(St + (rg + m * RPP) * LPR + cq, S[m]);
        __syncthreads();   // alpha, k and u are read by every thread before the next unit's
        nh = nh2;
        j = j2;
    }
    cp_async_wait_all();   // nothing is left in flight at exit
}

}  // namespace kda

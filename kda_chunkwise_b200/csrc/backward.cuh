// Backward pass of the KDA recurrence: gradients of q, k, v, the decay logits a, beta, the gate
// logits, A_log and the initial state, given the gradients of the outputs and of the final state.
//
// The pages describe only the forward pass; its gradient is the reverse-mode derivative of the
// token-by-token recurrence ("Review A · Sequence and depth", Free recall; "Kimi K3 · Lesson 3
// of 14", eq. 5 passage and the output gate).  Per token, with S = S_{t-1}, x = e^A a,
// alpha = e^{-5 sigmoid(x)}, S' = Diag(alpha) S, r = S'^T k, u = beta (v - r), S_t = S' + k u^T,
// o = S_t^T (scale q), out = sigmoid(gate) o, and dS the gradient of S_t:
//   do = dout sigmoid(gate);  dgate = dout o sigmoid'(gate);  dq = scale S_t do;  dS += scale q do^T
//   du = dS^T k;  dv = beta du;  dbeta = du . (v - r);  dr = -beta du;  dS' = dS + k dr^T
//   dk = dS u + S' dr;  dalpha_i = sum_j dS'_ij S_ij;  dS_{t-1} = Diag(alpha) dS'
//   dx = dalpha alpha (-5) sigmoid(x)(1 - sigmoid(x));  da = e^A dx;  dA_log += dx . x
//
// Execution: one CTA per (sequence, head), the state and its gradient in registers, the layout of
// the decode step (a warp holds whole 512-byte rows, so row sums are warp shuffles and column sums
// go through shared memory).  A forward pass stores the state at the start of every 64-token chunk
// (workspace); then, chunk by chunk in reverse, the chunk's 64 states are recomputed into a
// per-unit scratch (workspace) and the tokens are undone in reverse order.  The recurrence is
// sequential in time, so this runs at the latency of its token steps.
#pragma once

#include "common.cuh"
#include "decode.cuh"

namespace kda {

constexpr int kBwdThreads = 512;
constexpr int kBwdChunk = 64;

// dynamic shared memory: one chunk's inputs, staged with coalesced loads before its token steps
template <int DK, int DV>
struct BwdStage {
    static constexpr int kQ = 0;                            // bf16 [64][DK]
    static constexpr int kK = kQ + kBwdChunk * DK * 2;
    static constexpr int kA = kK + kBwdChunk * DK * 2;
    static constexpr int kV = kA + kBwdChunk * DK * 2;      // bf16 [64][DV]
    static constexpr int kG = kV + kBwdChunk * DV * 2;
    static constexpr int kD = kG + kBwdChunk * DV * 2;      // fp32 [64][DV] dout
    static constexpr int kB = kD + kBwdChunk * DV * 4;      // fp32 [64] beta
    static constexpr int kBytes = kB + kBwdChunk * 4;
};

struct BwdParams {
    const uint16_t *q, *k, *v, *a, *gate;   // packed [T, H, d], bf16
    const float *beta, *A_log;              // [T, H], [H]
    const int32_t *cu;
    const float *S0;                        // [N, H, d_k, d_v] or null
    const float *dout;                      // [T, H, d_v] fp32
    const float *dS_T;                      // [N, H, d_k, d_v] or null
    float *dq, *dk, *dv, *da, *dbeta, *dgate, *dA_log, *dS0;
    float *ckpt;                            // [sum_n ceil(len_n / 64)][H][d_k][d_v]
    float *scratch;                         // [N H][64][d_k][d_v]
    int64_t total_tokens;
    int num_seqs, H;
    float scale;
};

template <int DK, int DV>
__global__ void __launch_bounds__(kBwdThreads) kda_bwd_kernel(const BwdParams p) {
    constexpr int LPR = DV / 4;                // threads per state row (float4 each)
    constexpr int RPP = kBwdThreads / LPR;     // rows per pass
    constexpr int NR = DK / RPP;               // rows per thread
    __shared__ float s_k[DK], s_q[DK], s_al[DK], s_x[DK];
    __shared__ float s_vec[4][DV];             // u, v - r, do, du
    __shared__ float4 s_red[2][RPP][LPR];
    __shared__ float s_beta, s_dx_dot;
    __shared__ float s_db[DV / 32];

    using ST = BwdStage<DK, DV>;
    extern __shared__ __align__(16) unsigned char bsm[];
    const uint16_t *sq = reinterpret_cast<const uint16_t *>(bsm + ST::kQ);
    const uint16_t *sk = reinterpret_cast<const uint16_t *>(bsm + ST::kK);
    const uint16_t *sa = reinterpret_cast<const uint16_t *>(bsm + ST::kA);
    const uint16_t *sv = reinterpret_cast<const uint16_t *>(bsm + ST::kV);
    const uint16_t *sg = reinterpret_cast<const uint16_t *>(bsm + ST::kG);
    const float *sd = reinterpret_cast<const float *>(bsm + ST::kD);
    const float *sb = reinterpret_cast<const float *>(bsm + ST::kB);
    const int64_t unit = blockIdx.x;
    const int n = static_cast<int>(unit / p.H), h = static_cast<int>(unit % p.H);
    const int tid = threadIdx.x, cq = tid % LPR, rg = tid / LPR;
    int64_t s0, s1;
    if (!seq_span(p.cu, n, p.num_seqs, p.total_tokens, s0, s1)) {
        if (tid == 0) atomicOr(&g_kda_error_word, kErrBadSeqlens);
    }
    const int64_t len = s1 - s0;
    const int nck = static_cast<int>((len + kBwdChunk - 1) / kBwdChunk);
    int64_t ckbase = 0;   // checkpoints of the sequences before this one
    for (int m = 0; m < n; ++m) {
        int64_t a0, a1;
        seq_span(p.cu, m, p.num_seqs, p.total_tokens, a0, a1);
        ckbase += (a1 - a0 + kBwdChunk - 1) / kBwdChunk;
    }
    const int64_t H = p.H;
    const float expA = expf(p.A_log[h]);
    const size_t SZ = (size_t)DK * DV;
    float4 *scratch = reinterpret_cast<float4 *>(p.scratch + (size_t)unit * kBwdChunk * SZ);
    auto ck_ptr = [&](int c) { return reinterpret_cast<float4 *>(p.ckpt + ((size_t)(ckbase + c) * H + h) * SZ); };

    // a chunk's inputs (tokens tc .. tc + L - 1) into shared memory, 16 bytes per load
    auto stage = [&](int64_t tc, int L, bool grads) {
        auto copy_rows = [&](const void *src, int off, int row_bytes) {
            const int pieces = row_bytes / 16;
            for (int e = tid; e < L * pieces; e += kBwdThreads) {
                const int i = e / pieces, j = e % pieces;
                const uint4 *g = reinterpret_cast<const uint4 *>(static_cast<const char *>(src) +
                                                                 ((tc + i) * H + h) * (int64_t)row_bytes) + j;
                *reinterpret_cast<uint4 *>(bsm + off + i * row_bytes + j * 16) = __ldg(g);
            }
        };
        copy_rows(p.q, ST::kQ, DK * 2);
        copy_rows(p.k, ST::kK, DK * 2);
        copy_rows(p.a, ST::kA, DK * 2);
        copy_rows(p.v, ST::kV, DV * 2);
        if (grads) {
            if (p.gate) copy_rows(p.gate, ST::kG, DV * 2);
            copy_rows(p.dout, ST::kD, DV * 4);
        }
        for (int i = tid; i < L; i += kBwdThreads)
            reinterpret_cast<float *>(bsm + ST::kB)[i] = p.beta[(tc + i) * H + h];
    };
    // token i of the staged chunk: alpha and x per key channel, k, scale q, beta
    auto load_tok = [&](int i) {
        for (int c = tid; c < DK; c += kBwdThreads) {
            const float x = expA * bf16_to_f32(sa[i * DK + c]);
            s_x[c] = x;
            s_al[c] = __expf(kGMin * sigmoid_fast(x));
            s_k[c] = bf16_to_f32(sk[i * DK + c]);
            s_q[c] = p.scale * bf16_to_f32(sq[i * DK + c]);
        }
        if (tid == 0) s_beta = sb[i];
    };
    // column sums over the rows of two per-thread partial vectors (through shared memory)
    auto col_sums = [&](float4 a0, float4 a1, float &c0, float &c1) {
        s_red[0][rg][cq] = a0;
        s_red[1][rg][cq] = a1;
        __syncthreads();
        c0 = c1 = 0.f;
        if (tid < DV) {
            const float *r0 = reinterpret_cast<const float *>(&s_red[0][0][0]);
            const float *r1 = reinterpret_cast<const float *>(&s_red[1][0][0]);
#pragma unroll 4
            for (int g = 0; g < RPP; ++g) {
                c0 += r0[g * DV + tid];
                c1 += r1[g * DV + tid];
            }
        }
    };
    // forward step S <- Diag(alpha) S + k u^T, with u = beta (v - (Diag(alpha) S)^T k); the token's
    // inputs are in shared memory; u goes to s_vec[0] and v - r to s_vec[1]
    auto fwd_step = [&](float4 (&S)[NR], int i) {
        float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 0; m < NR; ++m) {
            const int row = rg + m * RPP;
            const float al = s_al[row];
            S[m].x *= al; S[m].y *= al; S[m].z *= al; S[m].w *= al;
            r = f4_fma(s_k[row], S[m], r);
        }
        float rc, unused;
        col_sums(r, r, rc, unused);
        if (tid < DV) {
            const float vmr = bf16_to_f32(sv[i * DV + tid]) - rc;
            s_vec[1][tid] = vmr;
            s_vec[0][tid] = s_beta * vmr;
        }
        __syncthreads();
        const float4 u4 = reinterpret_cast<const float4 *>(s_vec[0])[cq];
#pragma unroll
        for (int m = 0; m < NR; ++m) {
            const float kk = s_k[rg + m * RPP];
            S[m].x = fmaf(kk, u4.x, S[m].x); S[m].y = fmaf(kk, u4.y, S[m].y);
            S[m].z = fmaf(kk, u4.z, S[m].z); S[m].w = fmaf(kk, u4.w, S[m].w);
        }
    };

    // ---- forward pass: the state at the start of every chunk ---------------------------------
    float4 S[NR];
    const float4 *S0p = p.S0 ? reinterpret_cast<const float4 *>(p.S0 + (size_t)unit * SZ) : nullptr;
#pragma unroll
    for (int m = 0; m < NR; ++m) S[m] = S0p ? S0p[(rg + m * RPP) * LPR + cq] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < nck; ++c) {
        const int64_t tc = s0 + (int64_t)c * kBwdChunk;
        const int L = static_cast<int>(min64(kBwdChunk, s1 - tc));
        float4 *ck = ck_ptr(c);
#pragma unroll
        for (int m = 0; m < NR; ++m) ck[(rg + m * RPP) * LPR + cq] = S[m];
        stage(tc, L, false);
        __syncthreads();
        for (int i = 0; i < L; ++i) {
            load_tok(i);
            __syncthreads();
            fwd_step(S, i);
            __syncthreads();
        }
    }

    // ---- backward, chunk by chunk in reverse ----------------------------------------------------
    float4 dS[NR];
    const float4 *dST = p.dS_T ? reinterpret_cast<const float4 *>(p.dS_T + (size_t)unit * SZ) : nullptr;
#pragma unroll
    for (int m = 0; m < NR; ++m) dS[m] = dST ? dST[(rg + m * RPP) * LPR + cq] : make_float4(0.f, 0.f, 0.f, 0.f);
    float dA_acc = 0.f;
    for (int c = nck - 1; c >= 0; --c) {
        const int64_t tc = s0 + (int64_t)c * kBwdChunk;
        const int L = static_cast<int>(min64(kBwdChunk, s1 - tc));
        // recompute the chunk's states: scratch[i] = state before token tc + i
        const float4 *ck = ck_ptr(c);
#pragma unroll
        for (int m = 0; m < NR; ++m) S[m] = ck[(rg + m * RPP) * LPR + cq];
        stage(tc, L, true);
        __syncthreads();
        for (int i = 0; i < L; ++i) {
#pragma unroll
            for (int m = 0; m < NR; ++m) scratch[(size_t)i * (SZ / 4) + (rg + m * RPP) * LPR + cq] = S[m];
            if (i + 1 == L) break;   // the state after the last token is not needed
            load_tok(i);
            __syncthreads();
            fwd_step(S, i);
            __syncthreads();
        }
        // undo the chunk's tokens in reverse order
        for (int i = L - 1; i >= 0; --i) {
            const int64_t t = tc + i;
            const int64_t tv = (t * H + h) * DV;
            float4 Sp[NR];   // S' = Diag(alpha) S_{t-1}
#pragma unroll
            for (int m = 0; m < NR; ++m) Sp[m] = scratch[(size_t)i * (SZ / 4) + (rg + m * RPP) * LPR + cq];
            load_tok(i);
            __syncthreads();
            float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int m = 0; m < NR; ++m) {
                const int row = rg + m * RPP;
                const float al = s_al[row];
                Sp[m].x *= al; Sp[m].y *= al; Sp[m].z *= al; Sp[m].w *= al;
                r = f4_fma(s_k[row], Sp[m], r);
            }
            float rc, unused;
            col_sums(r, r, rc, unused);
            if (tid < DV) {
                const float vmr = bf16_to_f32(sv[i * DV + tid]) - rc;
                s_vec[1][tid] = vmr;
                s_vec[0][tid] = s_beta * vmr;
            }
            __syncthreads();
            // o = S_t^T (scale q) with S_t = S' + k u^T:  o = S'^T (scale q) + (k . scale q) u
            const float4 u4 = reinterpret_cast<const float4 *>(s_vec[0])[cq];
            float4 pq = make_float4(0.f, 0.f, 0.f, 0.f), du = pq;
#pragma unroll
            for (int m = 0; m < NR; ++m) {
                const int row = rg + m * RPP;
                const float kk = s_k[row], qq = s_q[row];
                float4 St = Sp[m];
                St.x = fmaf(kk, u4.x, St.x); St.y = fmaf(kk, u4.y, St.y);
                St.z = fmaf(kk, u4.z, St.z); St.w = fmaf(kk, u4.w, St.w);
                pq = f4_fma(qq, St, pq);
            }
            float oc;
            col_sums(pq, pq, oc, unused);
            if (tid < DV) {
                const float dout = sd[i * DV + tid];
                float dov = dout;
                if (p.gate) {
                    const float sgv = sigmoid_fast(bf16_to_f32(sg[i * DV + tid]));
                    p.dgate[tv + tid] = dout * oc * sgv * (1.f - sgv);
                    dov = dout * sgv;
                }
                s_vec[2][tid] = dov;
            }
            __syncthreads();
            // dS += (scale q) do^T; then du = dS^T k
            const float4 do4 = reinterpret_cast<const float4 *>(s_vec[2])[cq];
#pragma unroll
            for (int m = 0; m < NR; ++m) {
                const int row = rg + m * RPP;
                const float qq = s_q[row];
                dS[m].x = fmaf(qq, do4.x, dS[m].x); dS[m].y = fmaf(qq, do4.y, dS[m].y);
                dS[m].z = fmaf(qq, do4.z, dS[m].z); dS[m].w = fmaf(qq, do4.w, dS[m].w);
                du = f4_fma(s_k[row], dS[m], du);
            }
            float duc;
            col_sums(du, du, duc, unused);
            if (tid < DV) {
                s_vec[3][tid] = duc;
                p.dv[tv + tid] = s_beta * duc;
            }
            if (tid == 0) s_dx_dot = 0.f;
            __syncthreads();
            // row sums: dq = S_t do, dk = dS u + S' dr (dr = -beta du), dalpha = rowsum(dS' (.) S_{t-1});
            // then dS <- Diag(alpha) (dS + k dr^T)
            const float4 du4 = reinterpret_cast<const float4 *>(s_vec[3])[cq];
            const float bt = s_beta;
            float dbeta_part = 0.f;
            if (tid < DV) dbeta_part = s_vec[3][tid] * s_vec[1][tid];
#pragma unroll
            for (int m = 0; m < NR; ++m) {
                const int row = rg + m * RPP;
                const float kk = s_k[row], al = s_al[row];
                float4 St = Sp[m];
                St.x = fmaf(kk, u4.x, St.x); St.y = fmaf(kk, u4.y, St.y);
                St.z = fmaf(kk, u4.z, St.z); St.w = fmaf(kk, u4.w, St.w);
                float dqp = St.x * do4.x + St.y * do4.y + St.z * do4.z + St.w * do4.w;
                float dkp = dS[m].x * u4.x + dS[m].y * u4.y + dS[m].z * u4.z + dS[m].w * u4.w
                          - bt * (Sp[m].x * du4.x + Sp[m].y * du4.y + Sp[m].z * du4.z + Sp[m].w * du4.w);
                float4 dSp = dS[m];
                dSp.x -= bt * kk * du4.x; dSp.y -= bt * kk * du4.y;
                dSp.z -= bt * kk * du4.z; dSp.w -= bt * kk * du4.w;
                // dalpha_i = sum_j dS'_ij S_{t-1,ij} = sum_j dS'_ij S'_ij / alpha_i
                float dap = dSp.x * Sp[m].x + dSp.y * Sp[m].y + dSp.z * Sp[m].z + dSp.w * Sp[m].w;
#pragma unroll
                for (int o = LPR / 2; o > 0; o >>= 1) {
                    dqp += __shfl_xor_sync(0xffffffffu, dqp, o);
                    dkp += __shfl_xor_sync(0xffffffffu, dkp, o);
                    dap += __shfl_xor_sync(0xffffffffu, dap, o);
                }
                if (cq == 0) {
                    const int64_t tk = (t * H + h) * DK + row;
                    p.dq[tk] = p.scale * dqp;
                    p.dk[tk] = dkp;
                    const float x = s_x[row];
                    const float sx = sigmoid_fast(x);
                    // dalpha = dap / alpha; dg = dalpha alpha = dap
                    const float dx = dap * kGMin * sx * (1.f - sx);
                    p.da[tk] = dx * expA;
                    atomicAdd(&s_dx_dot, dx * x);
                }
                dS[m].x = al * dSp.x; dS[m].y = al * dSp.y; dS[m].z = al * dSp.z; dS[m].w = al * dSp.w;
            }
            // dbeta = du . (v - r)
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dbeta_part += __shfl_xor_sync(0xffffffffu, dbeta_part, o);
            if (tid < DV && (tid & 31) == 0) s_db[tid >> 5] = dbeta_part;
            __syncthreads();
            if (tid == 0) {
                float db = 0.f;
#pragma unroll
                for (int w = 0; w < DV / 32; ++w) db += s_db[w];
                p.dbeta[t * H + h] = db;
                dA_acc += s_dx_dot;
            }
            __syncthreads();
        }
    }
    if (tid == 0) atomicAdd(p.dA_log + h, dA_acc);
    if (p.dS0) {
        float4 *d0 = reinterpret_cast<float4 *>(p.dS0 + (size_t)unit * SZ);
#pragma unroll
        for (int m = 0; m < NR; ++m) d0[(rg + m * RPP) * LPR + cq] = dS[m];
    }
}

}  // namespace kda

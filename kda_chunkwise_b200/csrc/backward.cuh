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
// Every one of these steps acts on the value columns j of S and dS independently, except the row
// sums (dq, dk, dalpha) and the dot product of dbeta, which add up over the columns.  So a unit
// (sequence, head) runs on a cluster of d_v / 32 CTAs, each holding a d_k x 32 column slice of S and
// dS in registers; the row sums are kept per CTA for a whole 32-token chunk in shared memory and
// added over the cluster through distributed shared memory once per chunk (in a fixed order: the
// result does not depend on timing).  Per token a CTA needs the column sums over d_k rows only:
// warp shuffles plus one block barrier.  A forward pass stores the state at the start of every
// chunk (workspace); then, chunk by chunk in reverse, the chunk's states are recomputed into a
// per-CTA scratch (workspace) and the tokens are undone in reverse order.  The recurrence is
// sequential in time, so this runs at the latency of its token steps.
#pragma once

#include "common.cuh"
#include "decode.cuh"
#include "mma_frag.cuh"
#include "async_copy.cuh"

namespace kda {

constexpr int kBwdThreads = 256;
constexpr int kBwdChunk = 32;   // tokens per checkpoint / recompute chunk
constexpr int kBwdCols = 32;    // value columns per CTA

// Dynamic shared memory of one CTA: two buffers of a chunk's raw inputs (the next chunk's are
// copied in asynchronously while the current one runs), values derived from the current chunk, the
// chunk's per-CTA row sums, and the per-warp column sums of the current token (two buffers).
template <int DK>
struct BwdSmem {
    static constexpr int C = kBwdChunk, DC = kBwdCols;
    // raw buffer (offsets within one buffer)
    static constexpr int kRQ = 0;                         // bf16 [C][DK] q, then k, then a
    static constexpr int kRK = kRQ + C * DK * 2;
    static constexpr int kRA = kRK + C * DK * 2;
    static constexpr int kRV = kRA + C * DK * 2;          // bf16 [C][DC] v (this CTA's columns)
    static constexpr int kRG = kRV + C * DC * 2;          // bf16 [C][DC] gate logits
    static constexpr int kRD = kRG + C * DC * 2;          // f32 [C][DC] dout
    static constexpr int kRB = kRD + C * DC * 4;          // f32 [C] beta
    static constexpr int kRaw = kRB + C * 4;
    // derived values and sums
    static constexpr int kAl = 2 * kRaw;                  // f32 [C][DK] alpha
    static constexpr int kV = kAl + C * DK * 4;           // f32 [C][DC] v
    static constexpr int kDo = kV + C * DC * 4;           // f32 [C][DC] dout sigmoid(gate)
    static constexpr int kDg = kDo + C * DC * 4;          // f32 [C][DC] dout sigmoid'(gate)
    static constexpr int kQK = kDg + C * DC * 4;          // f32 [C] scale q . k
    static constexpr int kP = kQK + C * 4;                // f32 [C][3][DK] row sums: S_t do, dk, dg
    static constexpr int kPB = kP + C * 3 * DK * 4;       // f32 [C] dbeta (this CTA's columns)
    static constexpr int kRed = kPB + C * 4;              // f32 [2][3][8 warps][DC]
    static constexpr int kBytes = kRed + 2 * 3 * 8 * DC * 4;
};

struct BwdParams {
    const uint16_t *q, *k, *v, *a, *gate;   // packed [T, H, d], bf16
    const float *beta, *A_log;              // [T, H], [H]
    const int32_t *cu;
    const float *S0;                        // [N, H, d_k, d_v] or null
    const float *dout;                      // [T, H, d_v] fp32
    const float *dS_T;                      // [N, H, d_k, d_v] or null
    float *dq, *dk, *dv, *da, *dbeta, *dgate, *dA_log, *dS0;
    int64_t ck_records;                     // chunk records per head the workspace holds
    float *ckpt;                            // [sum_n ceil(len_n / 32)][H][d_v / 32][d_k x 32 slice]
    float *scratch;                         // [N H][d_v / 32][32 tokens][d_k x 32 slice]
    int64_t total_tokens;
    int num_seqs, H;
    float scale;
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}

__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];\n"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];\n" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

// The recomputed states S' (the scratch) are written and read back within a chunk: they are kept in
// L2 with an evict-last policy so that the streamed inputs and gradients do not push them out.
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;\n" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void st_keep(float4 *p, float4 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;\n" ::"l"(p), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w), "l"(pol)
                 : "memory");
}

__device__ __forceinline__ float4 ld_keep(const float4 *p, uint64_t pol) {
    float4 v;
    asm volatile("ld.global.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;\n"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p), "l"(pol)
                 : "memory");
    return v;
}

// drop a 128-byte line of scratch from L2 without writing it back (its contents are dead)
__device__ __forceinline__ void l2_discard(const void *p) {
    asm volatile("discard.global.L2 [%0], 128;\n" ::"l"(p) : "memory");
}

// streaming (evict-first) store of a gradient that is never read again here
__device__ __forceinline__ void st_stream(float *p, float4 v) { __stcs(reinterpret_cast<float4 *>(p), v); }

__device__ __forceinline__ float f4_dot(float4 a, float4 b) { return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w; }

__device__ __forceinline__ float4 f4_add(float4 a, float4 b) {
    return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

// sum over the 4 row groups of a warp (lanes l, l ^ 8, l ^ 16, l ^ 24 share a column quad)
__device__ __forceinline__ float4 warp_rows_sum(float4 x) {
#pragma unroll
    for (int o = 8; o < 32; o <<= 1) {
        x.x += __shfl_xor_sync(0xffffffffu, x.x, o);
        x.y += __shfl_xor_sync(0xffffffffu, x.y, o);
        x.z += __shfl_xor_sync(0xffffffffu, x.z, o);
        x.w += __shfl_xor_sync(0xffffffffu, x.w, o);
    }
    return x;
}

template <int DK, int DV>
__global__ void __launch_bounds__(kBwdThreads) kda_bwd_kernel(const BwdParams p) {
    constexpr int C = kBwdChunk, DC = kBwdCols, G = DV / DC;
    constexpr int NR = DK / 32;                 // rows per thread: rg + 32 m
    constexpr int NT = kBwdThreads;
    static_assert(NR == 2 || NR == 4, "d_k must be 64 or 128");
    using SM = BwdSmem<DK>;
    extern __shared__ __align__(16) unsigned char bsm[];
    float *sAl = reinterpret_cast<float *>(bsm + SM::kAl);
    float *sV = reinterpret_cast<float *>(bsm + SM::kV);
    float *sDo = reinterpret_cast<float *>(bsm + SM::kDo);
    float *sDg = reinterpret_cast<float *>(bsm + SM::kDg);
    float *sQK = reinterpret_cast<float *>(bsm + SM::kQK);
    float *sP = reinterpret_cast<float *>(bsm + SM::kP);
    float *sPB = reinterpret_cast<float *>(bsm + SM::kPB);
    float *sRed = reinterpret_cast<float *>(bsm + SM::kRed);

    const int rank = static_cast<int>(cluster_ctarank());
    const int64_t unit = blockIdx.x / G;
    const int n = static_cast<int>(unit / p.H), h = static_cast<int>(unit % p.H);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, cq = tid & 7, rg = tid >> 3;
    int64_t s0, s1;
    if (!seq_span(p.cu, n, p.num_seqs, p.total_tokens, s0, s1)) {
        if (tid == 0 && rank == 0) atomicOr(&g_kda_error_word, kErrBadSeqlens);
    }
    const int64_t len = s1 - s0;
    int64_t ckbase = 0;   // checkpoints of the sequences before this one
    for (int m = 0; m < n; ++m) {
        int64_t a0, a1;
        seq_span(p.cu, m, p.num_seqs, p.total_tokens, a0, a1);
        ckbase += (a1 - a0 + C - 1) / C;
    }
    // Well-formed cu_seqlens never need more checkpoints than the workspace holds; malformed ones
    // (flagged above) are cut short so that no checkpoint lands past it.
    const int64_t ck_room = p.ck_records - ckbase > 0 ? p.ck_records - ckbase : 0;
    const int nck = static_cast<int>(min64((len + C - 1) / C, ck_room));
    const int64_t H = p.H;
    const float expA = expf(p.A_log[h]);
    const size_t SZ = (size_t)DK * DV, SL = (size_t)DK * DC;
    const int col0 = rank * DC + 4 * cq;   // first of this thread's four value columns
    float4 *scratch = reinterpret_cast<float4 *>(p.scratch + (size_t)unit * C * SZ + (size_t)rank * C * SL);
    const uint64_t keep = l2_evict_last_policy();
    auto ck_ptr = [&](int c) {
        return reinterpret_cast<float4 *>(p.ckpt + ((size_t)(ckbase + c) * H + h) * SZ + (size_t)rank * SL);
    };

    // The work is a list of jobs: the forward pass over chunks 0 .. nck - 2, then the backward over
    // chunks nck - 1 .. 0.  The raw inputs of job j + 1 are copied in while job j runs.
    const int nfwd = nck > 0 ? nck - 1 : 0, njobs = nfwd + nck;
    auto job_chunk = [&](int j) { return j < nfwd ? j : nck - 1 - (j - nfwd); };
    auto issue = [&](int j, int rb) {   // asynchronous copy of job j's raw inputs into buffer rb
        const bool grads = j >= nfwd;
        const int64_t tc = s0 + (int64_t)job_chunk(j) * C;
        const int L = static_cast<int>(min64(C, s1 - tc));
        const uint32_t raw = smem_u32(bsm + rb * SM::kRaw);
        constexpr int PR = DK * 2 / 16;
        for (int e = tid; e < 3 * L * PR; e += NT) {
            const int which = e / (L * PR), r = e % (L * PR), i = r / PR, j16 = r % PR;
            const uint16_t *src = which == 0 ? p.q : (which == 1 ? p.k : p.a);
            cp_async_16(raw + SM::kRQ + which * (C * DK * 2) + i * (DK * 2) + j16 * 16,
                        src + ((tc + i) * H + h) * DK + j16 * 8, 16);
        }
        for (int e = tid; e < L * (DC / 8); e += NT) {
            const int i = e / (DC / 8), j16 = e % (DC / 8);
            cp_async_16(raw + SM::kRV + i * (DC * 2) + j16 * 16, p.v + ((tc + i) * H + h) * DV + rank * DC + j16 * 8, 16);
            if (grads && p.gate)
                cp_async_16(raw + SM::kRG + i * (DC * 2) + j16 * 16,
                            p.gate + ((tc + i) * H + h) * DV + rank * DC + j16 * 8, 16);
        }
        if (grads) {
            for (int e = tid; e < L * (DC / 4); e += NT) {
                const int i = e / (DC / 4), j16 = e % (DC / 4);
                cp_async_16(raw + SM::kRD + i * (DC * 4) + j16 * 16, p.dout + ((tc + i) * H + h) * DV + rank * DC + j16 * 4, 16);
            }
        }
        for (int i = tid; i < L; i += NT) cp_async_4(raw + SM::kRB + i * 4, p.beta + (tc + i) * H + h);
        cp_async_commit();
    };
    // job j's raw inputs have landed in buffer rb: alpha, v in fp32 (and with the gradients: dout
    // sigmoid(gate), dout sigmoid'(gate), scale q . k)
    auto derive = [&](int L, bool grads, int rb) {
        cp_async_wait_all();
        __syncthreads();   // every thread's copies have landed; the previous job's readers are done
        const unsigned char *raw = bsm + rb * SM::kRaw;
        const uint16_t *rq = reinterpret_cast<const uint16_t *>(raw + SM::kRQ);
        const uint16_t *rk = reinterpret_cast<const uint16_t *>(raw + SM::kRK);
        const uint16_t *ra = reinterpret_cast<const uint16_t *>(raw + SM::kRA);
        for (int e = tid; e < L * DK; e += NT) sAl[e] = __expf(kGMin * sigmoid_fast(expA * bf16_to_f32(ra[e])));
        const uint16_t *rv = reinterpret_cast<const uint16_t *>(raw + SM::kRV);
        for (int e = tid; e < L * DC; e += NT) sV[e] = bf16_to_f32(rv[e]);
        if (grads) {
            const float *rd = reinterpret_cast<const float *>(raw + SM::kRD);
            const uint16_t *rgt = reinterpret_cast<const uint16_t *>(raw + SM::kRG);
            for (int e = tid; e < L * DC; e += NT) {
                const float d = rd[e];
                if (p.gate) {
                    const float sg = sigmoid_fast(bf16_to_f32(rgt[e]));
                    sDo[e] = d * sg;
                    sDg[e] = d * sg * (1.f - sg);
                } else {
                    sDo[e] = d;
                }
            }
            for (int i = warp; i < L; i += NT / 32) {
                float s = 0.f;
                for (int c = lane; c < DK; c += 32) s += bf16_to_f32(rq[i * DK + c]) * bf16_to_f32(rk[i * DK + c]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                if (lane == 0) sQK[i] = p.scale * s;
            }
        }
        __syncthreads();
    };

    int buf = 0;   // which of the two column-sum buffers the next token uses
    // sum of the 8 warps' float4 partials of column quad cq (pairwise)
    auto red_sum = [&](const float *red) {
        const float4 *r4 = reinterpret_cast<const float4 *>(red);
        const float4 a0 = f4_add(r4[0 * DC / 4 + cq], r4[1 * DC / 4 + cq]);
        const float4 a1 = f4_add(r4[2 * DC / 4 + cq], r4[3 * DC / 4 + cq]);
        const float4 a2 = f4_add(r4[4 * DC / 4 + cq], r4[5 * DC / 4 + cq]);
        const float4 a3 = f4_add(r4[6 * DC / 4 + cq], r4[7 * DC / 4 + cq]);
        return f4_add(f4_add(a0, a1), f4_add(a2, a3));
    };
    // forward step of token i: S <- S' + k u^T, S' = Diag(alpha) S, u = beta (v - S'^T k); S' is
    // stored to `save` when given
    auto fwd_tok = [&](float4 (&S)[NR], const uint16_t *sK, const float *sB, int i, float4 *save) {
        float kk[NR];
        float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 0; m < NR; ++m) {
            const int row = rg + 32 * m;
            const float al = sAl[i * DK + row];
            kk[m] = bf16_to_f32(sK[i * DK + row]);
            S[m].x *= al; S[m].y *= al; S[m].z *= al; S[m].w *= al;
            if (save) st_keep(save + m * NT + tid, S[m], keep);
            r = f4_fma(kk[m], S[m], r);
        }
        r = warp_rows_sum(r);
        float *red = sRed + buf * (3 * 8 * DC);
        if (lane < 8) reinterpret_cast<float4 *>(red + warp * DC)[cq] = r;
        __syncthreads();
        const float4 rt = red_sum(red);
        buf ^= 1;
        const float b = sB[i];
        const float4 v = reinterpret_cast<const float4 *>(sV + i * DC)[cq];
        const float4 u = make_float4(b * (v.x - rt.x), b * (v.y - rt.y), b * (v.z - rt.z), b * (v.w - rt.w));
#pragma unroll
        for (int m = 0; m < NR; ++m) S[m] = f4_fma(kk[m], u, S[m]);
    };

    float4 S[NR], dS[NR];
    {
        const float *S0p = p.S0 ? p.S0 + (size_t)unit * SZ : nullptr;
        const float *dTp = p.dS_T ? p.dS_T + (size_t)unit * SZ : nullptr;
#pragma unroll
        for (int m = 0; m < NR; ++m) {
            const size_t o = (size_t)(rg + 32 * m) * DV + col0;
            S[m] = S0p ? *reinterpret_cast<const float4 *>(S0p + o) : make_float4(0.f, 0.f, 0.f, 0.f);
            dS[m] = dTp ? *reinterpret_cast<const float4 *>(dTp + o) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    float dA_acc = 0.f;
    const uint32_t pBase = smem_u32(sP), pbBase = smem_u32(sPB);
    if (njobs > 0) issue(0, 0);
    for (int j = 0; j < njobs; ++j) {
        const int rb = j & 1;
        const int c = job_chunk(j);
        const bool bwd = j >= nfwd;
        const int64_t tc = s0 + (int64_t)c * C;
        const int L = static_cast<int>(min64(C, s1 - tc));
        const unsigned char *raw = bsm + rb * SM::kRaw;
        const uint16_t *sQ = reinterpret_cast<const uint16_t *>(raw + SM::kRQ);
        const uint16_t *sK = reinterpret_cast<const uint16_t *>(raw + SM::kRK);
        const uint16_t *sA = reinterpret_cast<const uint16_t *>(raw + SM::kRA);
        const float *sB = reinterpret_cast<const float *>(raw + SM::kRB);
        if (!bwd) {   // forward: the state at the start of the chunk, then its tokens
            float4 *ck = ck_ptr(c);
#pragma unroll
            for (int m = 0; m < NR; ++m) ck[m * NT + tid] = S[m];
        } else if (c + 1 < nck) {
            const float4 *ck = ck_ptr(c);
#pragma unroll
            for (int m = 0; m < NR; ++m) S[m] = ck[m * NT + tid];
        }   // (the backward of the last chunk starts from the forward's state)
        derive(L, bwd, rb);
        if (j + 1 < njobs) issue(j + 1, rb ^ 1);
        if (!bwd) {
            for (int i = 0; i < C; ++i) fwd_tok(S, sK, sB, i, nullptr);
            continue;
        }
        // recompute the chunk: scratch[i] = S' of token tc + i (this thread's part; read back by it)
        for (int i = 0; i + 1 < L; ++i) fwd_tok(S, sK, sB, i, scratch + (size_t)i * NR * NT);
#pragma unroll
        for (int m = 0; m < NR; ++m) {
            const float al = sAl[(L - 1) * DK + rg + 32 * m];
            st_keep(scratch + (size_t)((L - 1) * NR + m) * NT + tid,
                    make_float4(al * S[m].x, al * S[m].y, al * S[m].z, al * S[m].w), keep);
        }
        // undo the chunk's tokens in reverse order; S' and the row inputs of token i - 1 are fetched
        // while token i runs
        float4 Spn[NR];
        float kkn[NR], qqn[NR], aln[NR];
#pragma unroll
        for (int m = 0; m < NR; ++m) {
            const int row = rg + 32 * m;
            Spn[m] = ld_keep(scratch + (size_t)((L - 1) * NR + m) * NT + tid, keep);
            kkn[m] = bf16_to_f32(sK[(L - 1) * DK + row]);
            qqn[m] = p.scale * bf16_to_f32(sQ[(L - 1) * DK + row]);
            aln[m] = sAl[(L - 1) * DK + row];
        }
        for (int i = L - 1; i >= 0; --i) {
            float4 Sp[NR];
            float kk[NR], qq[NR], al[NR];
#pragma unroll
            for (int m = 0; m < NR; ++m) { Sp[m] = Spn[m]; kk[m] = kkn[m]; qq[m] = qqn[m]; al[m] = aln[m]; }
            if (i > 0) {
#pragma unroll
                for (int m = 0; m < NR; ++m) {
                    const int row = rg + 32 * m;
                    Spn[m] = ld_keep(scratch + (size_t)((i - 1) * NR + m) * NT + tid, keep);
                    kkn[m] = bf16_to_f32(sK[(i - 1) * DK + row]);
                    qqn[m] = p.scale * bf16_to_f32(sQ[(i - 1) * DK + row]);
                    aln[m] = sAl[(i - 1) * DK + row];
                }
            }
            float4 r = make_float4(0.f, 0.f, 0.f, 0.f), pq = r, dko = r;
#pragma unroll
            for (int m = 0; m < NR; ++m) {
                r = f4_fma(kk[m], Sp[m], r);
                pq = f4_fma(qq[m], Sp[m], pq);
                dko = f4_fma(kk[m], dS[m], dko);
            }
            r = warp_rows_sum(r);
            pq = warp_rows_sum(pq);
            dko = warp_rows_sum(dko);
            float *red = sRed + buf * (3 * 8 * DC);
            if (lane < 8) {
                reinterpret_cast<float4 *>(red + warp * DC)[cq] = r;
                reinterpret_cast<float4 *>(red + (8 + warp) * DC)[cq] = pq;
                reinterpret_cast<float4 *>(red + (16 + warp) * DC)[cq] = dko;
            }
            __syncthreads();
            const float4 rt = red_sum(red), pqt = red_sum(red + 8 * DC), dkt = red_sum(red + 16 * DC);
            buf ^= 1;
            const float b = sB[i], qk = sQK[i];
            const float4 v = reinterpret_cast<const float4 *>(sV + i * DC)[cq];
            const float4 do4 = reinterpret_cast<const float4 *>(sDo + i * DC)[cq];
            const float4 vmr = make_float4(v.x - rt.x, v.y - rt.y, v.z - rt.z, v.w - rt.w);
            const float4 u = make_float4(b * vmr.x, b * vmr.y, b * vmr.z, b * vmr.w);
            // du = (dS + scale q do^T)^T k = dS^T k + (scale q . k) do
            const float4 du = f4_fma(qk, do4, dkt);
            if (tid < 8) {   // row group 0 of warp 0 holds every column of the CTA once
                const int64_t ov = ((tc + i) * H + h) * DV + col0;
                st_stream(p.dv + ov, make_float4(b * du.x, b * du.y, b * du.z, b * du.w));
                if (p.gate) {   // o = S_t^T (scale q) = S'^T (scale q) + (scale q . k) u
                    const float4 o = f4_fma(qk, u, pqt);
                    const float4 dg = reinterpret_cast<const float4 *>(sDg + i * DC)[cq];
                    st_stream(p.dgate + ov, make_float4(dg.x * o.x, dg.y * o.y, dg.z * o.z, dg.w * o.w));
                }
            }
            if (warp == 0) {   // dbeta over this CTA's columns
                float db = f4_dot(du, vmr);
                db += __shfl_xor_sync(0xffffffffu, db, 1);
                db += __shfl_xor_sync(0xffffffffu, db, 2);
                db += __shfl_xor_sync(0xffffffffu, db, 4);
                if (lane == 0) sPB[i] = db;
            }
            const float udo = f4_dot(u, do4);
            float vals[3 * NR];
#pragma unroll
            for (int m = 0; m < NR; ++m) {
                const float4 dSn = f4_fma(qq[m], do4, dS[m]);
                const float sdu = f4_dot(Sp[m], du);
                vals[3 * m + 0] = f4_dot(Sp[m], do4) + kk[m] * udo;         // (S_t do)_row
                vals[3 * m + 1] = f4_dot(dSn, u) - b * sdu;                 // dk_row
                vals[3 * m + 2] = f4_dot(dSn, Sp[m]) - b * kk[m] * sdu;     // dalpha_row alpha_row
                const float4 dSp = f4_fma(-b * kk[m], du, dSn);
                dS[m] = make_float4(al[m] * dSp.x, al[m] * dSp.y, al[m] * dSp.z, al[m] * dSp.w);
            }
            // sum the row values over the 8 lanes of a row (lanes differ in bits 0..2), leaving each
            // lane pair (quad for NR = 2) with the three sums of one row
            const int b4 = (lane >> 2) & 1;
            float w1[3 * NR / 2];
#pragma unroll
            for (int k2 = 0; k2 < 3 * NR / 2; ++k2) {
                const float send = b4 ? vals[k2] : vals[k2 + 3 * NR / 2];
                const float keep = b4 ? vals[k2 + 3 * NR / 2] : vals[k2];
                w1[k2] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
            }
            if constexpr (NR == 4) {
                const int b2 = (lane >> 1) & 1;
                float w2[3];
#pragma unroll
                for (int k2 = 0; k2 < 3; ++k2) {
                    const float send = b2 ? w1[k2] : w1[k2 + 3];
                    const float keep = b2 ? w1[k2 + 3] : w1[k2];
                    w2[k2] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                    w2[k2] += __shfl_xor_sync(0xffffffffu, w2[k2], 1);
                }
                if ((lane & 1) == 0) {
                    const int row = rg + 32 * (2 * b4 + b2);
#pragma unroll
                    for (int q3 = 0; q3 < 3; ++q3) sP[(i * 3 + q3) * DK + row] = w2[q3];
                }
            } else {
#pragma unroll
                for (int k2 = 0; k2 < 3; ++k2) {
                    w1[k2] += __shfl_xor_sync(0xffffffffu, w1[k2], 2);
                    w1[k2] += __shfl_xor_sync(0xffffffffu, w1[k2], 1);
                }
                if ((lane & 3) == 0) {
                    const int row = rg + 32 * b4;
#pragma unroll
                    for (int q3 = 0; q3 < 3; ++q3) sP[(i * 3 + q3) * DK + row] = w1[q3];
                }
            }
        }
        // add the row sums over the cluster: this CTA finishes tokens i = rank (mod G)
        cluster_sync();
        const int mine = (L - rank + G - 1) / G;
        for (int e = tid; e < mine * (DK / 4); e += NT) {
            const int i = rank + G * (e / (DK / 4)), c4 = 4 * (e % (DK / 4));
            float4 acc[3];
#pragma unroll
            for (int q3 = 0; q3 < 3; ++q3) acc[q3] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int g = 0; g < G; ++g) {
#pragma unroll
                for (int q3 = 0; q3 < 3; ++q3)
                    acc[q3] = f4_add(acc[q3], ld_cluster_f4(mapa_shared(pBase + ((i * 3 + q3) * DK + c4) * 4, g)));
            }
            const int64_t ok = ((tc + i) * H + h) * DK + c4;
            st_stream(p.dq + ok, make_float4(p.scale * acc[0].x, p.scale * acc[0].y, p.scale * acc[0].z, p.scale * acc[0].w));
            st_stream(p.dk + ok, acc[1]);
            const float dg[4] = {acc[2].x, acc[2].y, acc[2].z, acc[2].w};
            float da[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const float x = expA * bf16_to_f32(sA[i * DK + c4 + jj]);
                const float sx = sigmoid_fast(x);
                const float dx = dg[jj] * kGMin * sx * (1.f - sx);
                da[jj] = dx * expA;
                dA_acc = fmaf(dx, x, dA_acc);
            }
            st_stream(p.da + ok, make_float4(da[0], da[1], da[2], da[3]));
        }
        if (tid < mine) {
            const int i = rank + G * tid;
            float db = 0.f;
#pragma unroll
            for (int g = 0; g < G; ++g) db += ld_cluster_f32(mapa_shared(pbBase + i * 4, g));
            p.dbeta[(tc + i) * H + h] = db;
        }
        cluster_sync();   // every CTA is done reading the row sums before they are overwritten
    }
    // the scratch is dead: drop it from L2 rather than write it back (every read of it came before
    // the last cluster barrier, which every thread of this CTA has passed)
    if (nck > 0) {
        const char *sc = reinterpret_cast<const char *>(scratch);
        for (int i = tid; i < C * NR * NT * 16 / 128; i += NT) l2_discard(sc + (size_t)i * 128);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dA_acc += __shfl_xor_sync(0xffffffffu, dA_acc, o);
    if (lane == 0 && dA_acc != 0.f) atomicAdd(p.dA_log + h, dA_acc);
    if (p.dS0) {
        float *d0 = p.dS0 + (size_t)unit * SZ;
#pragma unroll
        for (int m = 0; m < NR; ++m) *reinterpret_cast<float4 *>(d0 + (size_t)(rg + 32 * m) * DV + col0) = dS[m];
    }
}

}  // namespace kda

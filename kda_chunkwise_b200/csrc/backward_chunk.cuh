// Backward pass of the KDA recurrence in chunkwise form (64-token chunks): the products on the tensor
// cores (tf32 with hi/lo operand splits, fp32-accurate), the rest in fp32 on the CUDA cores.
//
// Per chunk with incoming state S0, b the chunk-local running sum of g, Gamma = e^b, Gamma_C its last
// row, the forward is  Q^ = Gamma (.) scale q, K^ = Gamma (.) k, K- = (Gamma_C / Gamma) (.) k,
//   M = strict_lower(sum_c k_ic k_jc e^{b_ic - b_jc}),  A = lower_incl(sum_c sq_ic k_jc e^{b_ic - b_jc}),
//   X = (I + diag(beta) M)^-1,  T' = X diag(beta),  W = T' K^,  U = T' V - W S0,
//   O = Q^ S0 + A U,  S_C = Diag(Gamma_C) S0 + K-^T U
// ("Kimi K3 · Lesson 3 of 14", CHUNKWISE diagram), and its derivative, chunk by chunk in reverse:
//   dU = A^T dO + K- dS_C,  dS0 = Q^T dO + Diag(Gamma_C) dS_C - W^T dU   (the only thing carried
//   between chunks), then per chunk dA = lower_incl(dO U^T), dK- = U dS_C^T, dW = -dU S0^T,
//   dT' = dW K^T + dU V^T, dv = T'^T dU, dX = dT' diag(beta), dL = strict_lower(-X^T dX X^T),
//   dbeta, and the key / query / log-decay gradients with every 1/e^b inside a pair
//   E_ijc = e^{b_ic - b_jc}, i >= j (so nothing overflows):
//   dq = scale (e^b (dO S0^T) + sum_{j<=i} dA_ij k_j E_ij),  P = e^b (T'^T dW) + sum_{j<i} dM_ij k_j E_ij,
//   Q = sum_{i>=j} dA_ij sq_i E_ij + sum_{i>j} dM_ij k_i E_ij,  R = e^{b_C - b} dK-,  dM = diag(beta) dL,
//   dk = P + Q + R,  db = dq q + (P - Q - R) k (+ sum R k + dGamma_C Gamma_C on the last row),
//   dg = reverse running sum of db,  then g = -5 sigmoid(e^A a) gives da and dA_log.
// Four launches: per chunk the forward operands (chunk-parallel); per unit the states at the chunk
// starts (sequential over chunks, one CTA per 32 value columns); per unit the state gradients in
// reverse (the same); per chunk the rest (chunk-parallel).
#pragma once

#include "common.cuh"

namespace kda {

constexpr int kBcChunk = 64;
constexpr int kBcThreads = 256;
constexpr int kBcCols = 32;   // value columns per CTA of the two sequential passes

// Workspace record of one (chunk, head), fp32 offsets.  Slots are reused once their first content
// is no longer needed (the later uses are named).
template <int DK, int DV>
struct BcRec {
    static constexpr int C = kBcChunk;
    static constexpr size_t kB = 0;                   // [C][DK] b
    static constexpr size_t kW = kB + C * DK;         // [C][DK] W; later dW, then Q
    static constexpr size_t kU = kW + C * DK;         // [C][DV] T' V, then U; later dv
    static constexpr size_t kKb = kU + C * DV;        // [C][DK] K-; later dK-, then db
    static constexpr size_t kQh = kKb + C * DK;       // [C][DK] Q^; later dO S0^T, then dq
    static constexpr size_t kA = kQh + C * DK;        // [C][C] A; later X^T dX
    static constexpr size_t kX = kA + C * C;          // [C][C] X
    static constexpr size_t kM = kX + C * C;          // [C][C] M
    static constexpr size_t kGC = kM + C * C;         // [DK] Gamma_C
    static constexpr size_t kS0 = kGC + DK;           // [DK][DV] incoming state; later T'^T dW, then P
    static constexpr size_t kdS = kS0 + (size_t)DK * DV;   // [DK][DV] state gradient at the chunk's end
    static constexpr size_t kdU = kdS + (size_t)DK * DV;   // [C][DV]
    static constexpr size_t kdO = kdU + C * DV;       // [C][DV] dout sigmoid(gate); later V, zero padded
    static constexpr size_t kSize = kdO + C * DV;
};

// Shared-memory staging of bc_gemm: a k-slice of 16 of opA ([M][16 + 4]) and of opB ([16][N + 8]),
// padded so that the fragment reads below are free of bank conflicts.
constexpr int kBcKs = 16;
constexpr int kBcStageFloats = 128 * (kBcKs + 4) + kBcKs * (128 + 8);

__device__ __forceinline__ uint32_t bc_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;\n" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void bc_mma_tf32(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// C (M x N, row stride ldc) = alpha opA (M x K) opB (K x N) [+ C], by the whole CTA (8 warps) on the
// tensor cores: mma.sync m16n8k8 in tf32 on operands split as x = hi + lo (both tf32), summing
// lo*hi + hi*lo + hi*hi, which keeps fp32's accuracy to about 2^-21 of each product.  The operands
// (global or shared memory, any row strides) are staged 16 values of K at a time in `stage`
// (kBcStageFloats floats of shared memory) with coalesced loads.  Warp w takes row block
// w / (8 / (M / 16)) and a run of N / 8 / (8 / (M / 16)) column blocks of 8.
// opA(i, k) = TA ? A[k lda + i] : A[i lda + k];  opB(k, j) = TB ? B[j ldb + k] : B[k ldb + j].
// Contains CTA barriers: every thread calls it, and it begins with one, so the operands' writers
// need no barrier of their own before the call (the caller still needs one after it before C is
// read by other threads).
template <int M, int N, int K, bool TA, bool TB>
__device__ __forceinline__ void bc_gemm(const float *A, int lda, const float *B, int ldb, float *Cm, int ldc,
                                        float alpha, bool accumulate, float *stage) {
    constexpr int LA = kBcKs + 4, LB = N + 8;
    constexpr int TM = M / 16, TN = N / 8, WPM = 8 / TM, NPW = TN / WPM;
    static_assert(M % 16 == 0 && N % 8 == 0 && K % kBcKs == 0 && TM <= 8 && 8 % TM == 0 && TN % WPM == 0, "shape");
    static_assert(M * LA + kBcKs * LB <= kBcStageFloats, "stage");
    float *As = stage, *Bs = stage + M * LA;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
    const int mt = warp / WPM, nt0 = (warp % WPM) * NPW;
    float acc[NPW][4];
#pragma unroll
    for (int u = 0; u < NPW; ++u) acc[u][0] = acc[u][1] = acc[u][2] = acc[u][3] = 0.f;
    // the next k-slice is read into registers while the current one is multiplied, so the global
    // (L2) latency of the operands overlaps the products
    constexpr int EA = M * kBcKs, EB = kBcKs * N;
    constexpr int NA = (EA + kBcThreads - 1) / kBcThreads, NB = (EB + kBcThreads - 1) / kBcThreads;
    float ra[NA], rb[NB];
    auto fetch = [&](int k0) {
#pragma unroll
        for (int q = 0; q < NA; ++q) {
            const int e = threadIdx.x + q * kBcThreads;
            if (e < EA) ra[q] = TA ? A[(size_t)(k0 + e / M) * lda + e % M] : A[(size_t)(e / kBcKs) * lda + k0 + e % kBcKs];
        }
#pragma unroll
        for (int q = 0; q < NB; ++q) {
            const int e = threadIdx.x + q * kBcThreads;
            if (e < EB) rb[q] = TB ? B[(size_t)(e / kBcKs) * ldb + k0 + e % kBcKs] : B[(size_t)(k0 + e / N) * ldb + e % N];
        }
    };
    auto stage_slice = [&]() {
#pragma unroll
        for (int q = 0; q < NA; ++q) {
            const int e = threadIdx.x + q * kBcThreads;
            if (e < EA) {
                if (TA) As[(e % M) * LA + e / M] = ra[q];
                else As[(e / kBcKs) * LA + e % kBcKs] = ra[q];
            }
        }
#pragma unroll
        for (int q = 0; q < NB; ++q) {
            const int e = threadIdx.x + q * kBcThreads;
            if (e < EB) {
                if (TB) Bs[(e % kBcKs) * LB + e / kBcKs] = rb[q];
                else Bs[(e / N) * LB + e % N] = rb[q];
            }
        }
    };
    __syncthreads();   // on entry: the operands are written
    fetch(0);
    for (int k0 = 0; k0 < K; k0 += kBcKs) {
        if (k0 > 0) __syncthreads();   // the previous slice is consumed
        stage_slice();
        __syncthreads();
        if (k0 + kBcKs < K) fetch(k0 + kBcKs);
#pragma unroll
        for (int ks = 0; ks < kBcKs; ks += 8) {
            uint32_t ah[4], al[4];
            {
                const float *a = As + (16 * mt + g) * LA + ks + t4;
                const float av[4] = {a[0], a[8 * LA], a[4], a[8 * LA + 4]};
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    ah[r] = bc_tf32(av[r]);
                    al[r] = bc_tf32(av[r] - __uint_as_float(ah[r]));
                }
            }
#pragma unroll
            for (int u = 0; u < NPW; ++u) {
                const float *b = Bs + (ks + t4) * LB + 8 * (nt0 + u) + g;
                const float b0 = b[0], b1 = b[4 * LB];
                const uint32_t bh0 = bc_tf32(b0), bh1 = bc_tf32(b1);
                const uint32_t bl0 = bc_tf32(b0 - __uint_as_float(bh0)), bl1 = bc_tf32(b1 - __uint_as_float(bh1));
                bc_mma_tf32(acc[u], al, bh0, bh1);
                bc_mma_tf32(acc[u], ah, bl0, bl1);
                bc_mma_tf32(acc[u], ah, bh0, bh1);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < NPW; ++u) {
        const int r0 = 16 * mt + g, c0 = 8 * (nt0 + u) + 2 * t4;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const size_t o = (size_t)(r0 + 8 * (q >> 1)) * ldc + c0 + (q & 1);
            const float r = alpha * acc[u][q];
            Cm[o] = accumulate ? Cm[o] + r : r;
        }
    }
}

// Bulk prefetch of [ptr, ptr + bytes) into L2 (ptr and bytes multiples of 16), issued by one thread:
// the chunk records were written by an earlier kernel and have mostly left L2 by the time they are
// read, and the passes over chunks know which record comes next.
__device__ __forceinline__ void bc_prefetch_l2(const void *ptr, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(ptr), "r"(bytes) : "memory");
}

// The chunk with global index gc (over every sequence's chunks, in order): its sequence n, index c
// within the sequence and token span; false past the last chunk.
__device__ __forceinline__ bool bc_find(const BwdParams &p, int64_t gc, int &n, int &c, int64_t &t0, int &L) {
    int64_t base = 0;
    for (int m = 0; m < p.num_seqs; ++m) {
        int64_t s0, s1;
        seq_span(p.cu, m, p.num_seqs, p.total_tokens, s0, s1);
        const int64_t nc = (s1 - s0 + kBcChunk - 1) / kBcChunk;
        if (gc < base + nc) {
            n = m;
            c = static_cast<int>(gc - base);
            t0 = s0 + (int64_t)c * kBcChunk;
            L = static_cast<int>(min64(kBcChunk, s1 - t0));
            return true;
        }
        base += nc;
    }
    return false;
}

__device__ __forceinline__ int64_t bc_chunk_base(const BwdParams &p, int n) {
    int64_t base = 0;
    for (int m = 0; m < n; ++m) {
        int64_t s0, s1;
        seq_span(p.cu, m, p.num_seqs, p.total_tokens, s0, s1);
        base += (s1 - s0 + kBcChunk - 1) / kBcChunk;
    }
    return base;
}

// ---- 1. per chunk: the forward operands ------------------------------------------------------
template <int DK, int DV>
__global__ void __launch_bounds__(kBcThreads, 1) bc_prep_kernel(const BwdParams p) {
    constexpr int C = kBcChunk, NT = kBcThreads, LK = DK + 1, LV = DV + 1, LC = C + 1;
    using R = BcRec<DK, DV>;
    extern __shared__ __align__(16) float bcs[];
    float *sk = bcs;                 // [C][LK] k, later K^
    float *sq = sk + C * LK;         // [C][LK] scale q
    float *sb = sq + C * LK;         // [C][LK] b
    float *sv = sb + C * LK;         // [C][LV] v
    float *sX = sv + C * LV;         // [C][LC] X
    float *sL = sX + C * LC;         // [C][LC] M, then L, then T'
    float *sbeta = sL + C * LC;      // [C]
    float *sstage = sbeta + C;       // bc_gemm staging
    const int64_t gc = blockIdx.x / p.H;
    const int h = static_cast<int>(blockIdx.x % p.H);
    int n, c, L;
    int64_t t0;
    if (!bc_find(p, gc, n, c, t0, L)) return;
    float *rec = p.ckpt + (size_t)blockIdx.x * R::kSize;
    const int tid = threadIdx.x;
    const int64_t H = p.H;
    const float expA = expf(p.A_log[h]);
    for (int e = tid; e < C * DK; e += NT) {   // rows past the chunk: k = q = 0, g = 0
        const int i = e / DK, ch = e % DK;
        const bool in = i < L;
        const int64_t o = ((t0 + i) * H + h) * DK + ch;
        sk[i * LK + ch] = in ? bf16_to_f32(p.k[o]) : 0.f;
        sq[i * LK + ch] = in ? p.scale * bf16_to_f32(p.q[o]) : 0.f;
        sb[i * LK + ch] = in ? kGMin / (1.f + expf(-expA * bf16_to_f32(p.a[o]))) : 0.f;   // g for now
    }
    for (int e = tid; e < C * DV; e += NT) {
        const int i = e / DV, ch = e % DV;
        sv[i * LV + ch] = i < L ? bf16_to_f32(p.v[((t0 + i) * H + h) * DV + ch]) : 0.f;
    }
    for (int i = tid; i < C; i += NT) sbeta[i] = i < L ? p.beta[(t0 + i) * H + h] : 0.f;
    __syncthreads();
    for (int ch = tid; ch < DK; ch += NT) {   // b = running sum of g
        float s = 0.f;
        for (int i = 0; i < C; ++i) {
            s += sb[i * LK + ch];
            sb[i * LK + ch] = s;
        }
        rec[R::kGC + ch] = expf(s);
    }
    __syncthreads();
    for (int e = tid; e < C * DK; e += NT) {
        const int i = e / DK, ch = e % DK;
        rec[R::kB + e] = sb[i * LK + ch];
        const float kk = sk[i * LK + ch];
        rec[R::kKb + e] = kk * expf(sb[(C - 1) * LK + ch] - sb[i * LK + ch]);
        rec[R::kQh + e] = sq[i * LK + ch] * expf(sb[i * LK + ch]);
    }
    // M (strict lower) and A (lower, diagonal included), one (i, j) pair per thread at a time
    for (int e = tid; e < C * C; e += NT) {
        const int i = e / C, j = e % C;
        float m = 0.f, a = 0.f;
        if (j <= i) {
            for (int ch = 0; ch < DK; ++ch) {
                const float E = __expf(sb[i * LK + ch] - sb[j * LK + ch]);
                const float kj = sk[j * LK + ch] * E;
                a = fmaf(sq[i * LK + ch], kj, a);
                m = fmaf(sk[i * LK + ch], kj, m);
            }
            if (j == i) m = 0.f;
        }
        sL[i * LC + j] = m;
        rec[R::kM + e] = m;
        rec[R::kA + e] = a;
        sX[i * LC + j] = i == j ? 1.f : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += NT) {   // L = diag(beta) M
        const int i = e / C, j = e % C;
        sL[i * LC + j] *= sbeta[i];
    }
    __syncthreads();
    // X = (I + L)^-1, unit lower triangular: row by row, X_ij = -sum_{j<=m<i} L_im X_mj
    for (int i = 1; i < C; ++i) {
        if (tid < i) {
            const int j = tid;
            float s = 0.f;
            for (int m = j; m < i; ++m) s = fmaf(sL[i * LC + m], sX[m * LC + j], s);
            sX[i * LC + j] = -s;
        }
        __syncthreads();
    }
    for (int e = tid; e < C * C; e += NT) {   // X to the record; T' = X diag(beta) over L
        const int i = e / C, j = e % C;
        rec[R::kX + e] = sX[i * LC + j];
        sL[i * LC + j] = sX[i * LC + j] * sbeta[j];
    }
    for (int e = tid; e < C * DK; e += NT) {   // K^ = Gamma (.) k
        const int i = e / DK, ch = e % DK;
        sk[i * LK + ch] *= expf(sb[i * LK + ch]);
    }
    __syncthreads();
    bc_gemm<C, DK, C, false, false>(sL, LC, sk, LK, rec + R::kW, DK, 1.f, false, sstage);   // W = T' K^
    bc_gemm<C, DV, C, false, false>(sL, LC, sv, LV, rec + R::kU, DV, 1.f, false, sstage);   // T' V
}

// ---- 2. per unit and 32 value columns: the state at every chunk start, and U -----------------
template <int DK, int DV>
__global__ void __launch_bounds__(kBcThreads, 1) bc_state_kernel(const BwdParams p) {
    constexpr int C = kBcChunk, NT = kBcThreads, DC = kBcCols, G = DV / DC;
    using R = BcRec<DK, DV>;
    constexpr int LK = DK + 1;
    extern __shared__ __align__(16) float bcs[];
    float *sS = bcs;                 // [DK][DC]
    float *sU = sS + DK * DC;        // [C][DC]
    float *sT = sU + C * DC;         // [DK][DC]
    float *sW = sT + DK * DC;        // [C][LK] W of the chunk
    float *sKb = sW + C * LK;        // [C][LK] K- of the chunk
    float *sstage = sKb + C * LK;    // bc_gemm staging
    const int64_t unit = blockIdx.x / G;
    const int slice = static_cast<int>(blockIdx.x % G);
    const int n = static_cast<int>(unit / p.H), h = static_cast<int>(unit % p.H);
    int64_t s0, s1;
    if (!seq_span(p.cu, n, p.num_seqs, p.total_tokens, s0, s1) && threadIdx.x == 0 && slice == 0)
        atomicOr(&g_kda_error_word, kErrBadSeqlens);
    const int64_t base = bc_chunk_base(p, n);
    // malformed cu_seqlens (flagged above) are cut short: no record past the workspace's
    const int64_t room = p.ck_records - base > 0 ? p.ck_records - base : 0;
    const int nck = static_cast<int>(min64((s1 - s0 + C - 1) / C, room));
    const int tid = threadIdx.x, col0 = slice * DC;
    for (int e = tid; e < DK * DC; e += NT) {
        const int r = e / DC, cc = e % DC;
        sS[e] = p.S0 ? p.S0[(size_t)unit * DK * DV + (size_t)r * DV + col0 + cc] : 0.f;
    }
    __syncthreads();
    for (int c = 0; c < nck; ++c) {
        float *rec = p.ckpt + (size_t)((base + c) * p.H + h) * R::kSize;
        if (tid == 0 && c + 1 < nck) {   // the next chunk's W and T'V (adjacent), K- and Gamma_C
            const float *nx = rec + (size_t)p.H * R::kSize;
            bc_prefetch_l2(nx + R::kW, (uint32_t)(C * (DK + DV) * 4));
            bc_prefetch_l2(nx + R::kKb, (uint32_t)(C * DK * 4));
            bc_prefetch_l2(nx + R::kGC, (uint32_t)(DK * 4));
        }
        for (int e = tid; e < DK * DC; e += NT) {
            const int r = e / DC, cc = e % DC;
            rec[R::kS0 + (size_t)r * DV + col0 + cc] = sS[e];
        }
        for (int e = tid; e < C * DC; e += NT) {
            const int i = e / DC, cc = e % DC;
            sU[e] = rec[R::kU + (size_t)i * DV + col0 + cc];
        }
        for (int e = tid; e < C * DK; e += NT) {
            const int i = e / DK, ch = e % DK;
            sW[i * LK + ch] = rec[R::kW + e];
            sKb[i * LK + ch] = rec[R::kKb + e];
        }
        __syncthreads();
        bc_gemm<C, DC, DK, false, false>(sW, LK, sS, DC, sU, DC, -1.f, true, sstage);   // U = T'V - W S0
        __syncthreads();
        for (int e = tid; e < C * DC; e += NT) {
            const int i = e / DC, cc = e % DC;
            rec[R::kU + (size_t)i * DV + col0 + cc] = sU[e];
        }
        bc_gemm<DK, DC, C, true, false>(sKb, LK, sU, DC, sT, DC, 1.f, false, sstage);   // K-^T U
        __syncthreads();
        for (int e = tid; e < DK * DC; e += NT) sS[e] = fmaf(rec[R::kGC + e / DC], sS[e], sT[e]);
        __syncthreads();
    }
}

// ---- 3. per unit and 32 value columns, in reverse: the outputs' gate, dU and the state gradients
template <int DK, int DV>
__global__ void __launch_bounds__(kBcThreads, 1) bc_dstate_kernel(const BwdParams p) {
    constexpr int C = kBcChunk, NT = kBcThreads, DC = kBcCols, G = DV / DC;
    using R = BcRec<DK, DV>;
    constexpr int LK = DK + 1, LC = C + 1;
    extern __shared__ __align__(16) float bcs[];
    float *sdS = bcs;                // [DK][DC]
    float *sO = sdS + DK * DC;       // [C][DC] O, then dO
    float *sdU = sO + C * DC;        // [C][DC]
    float *sT = sdU + C * DC;        // [DK][DC]
    float *sQh = sT + DK * DC;       // [C][LK] the chunk's Q^, K-, W and A
    float *sKb = sQh + C * LK;
    float *sW = sKb + C * LK;
    float *sA = sW + C * LK;         // [C][LC]
    float *sstage = sA + C * LC;     // bc_gemm staging
    const int64_t unit = blockIdx.x / G;
    const int slice = static_cast<int>(blockIdx.x % G);
    const int n = static_cast<int>(unit / p.H), h = static_cast<int>(unit % p.H);
    int64_t s0, s1;
    if (!seq_span(p.cu, n, p.num_seqs, p.total_tokens, s0, s1) && threadIdx.x == 0 && slice == 0)
        atomicOr(&g_kda_error_word, kErrBadSeqlens);
    const int64_t base = bc_chunk_base(p, n);
    // malformed cu_seqlens (flagged above) are cut short: no record past the workspace's
    const int64_t room = p.ck_records - base > 0 ? p.ck_records - base : 0;
    const int nck = static_cast<int>(min64((s1 - s0 + C - 1) / C, room));
    const int64_t H = p.H;
    const int tid = threadIdx.x, col0 = slice * DC;
    for (int e = tid; e < DK * DC; e += NT) {
        const int r = e / DC, cc = e % DC;
        sdS[e] = p.dS_T ? p.dS_T[(size_t)unit * DK * DV + (size_t)r * DV + col0 + cc] : 0.f;
    }
    __syncthreads();
    for (int c = nck - 1; c >= 0; --c) {
        float *rec = p.ckpt + (size_t)((base + c) * H + h) * R::kSize;
        if (tid == 0 && c > 0) {   // the next chunk in reverse: W and U, K-, Q^ and A, Gamma_C and S0
            const float *nx = rec - (size_t)H * R::kSize;
            bc_prefetch_l2(nx + R::kW, (uint32_t)(C * (DK + DV) * 4));
            bc_prefetch_l2(nx + R::kKb, (uint32_t)((2 * C * DK + C * C) * 4));
            bc_prefetch_l2(nx + R::kGC, (uint32_t)((DK + DK * DV) * 4));
        }
        const int64_t t0 = s0 + (int64_t)c * C;
        const int L = static_cast<int>(min64(C, s1 - t0));
        for (int e = tid; e < C * DK; e += NT) {
            const int i = e / DK, ch = e % DK;
            sQh[i * LK + ch] = rec[R::kQh + e];
            sKb[i * LK + ch] = rec[R::kKb + e];
            sW[i * LK + ch] = rec[R::kW + e];
        }
        for (int e = tid; e < C * C; e += NT) sA[(e / C) * LC + e % C] = rec[R::kA + e];
        __syncthreads();
        // O = Q^ S0 + A U (pre-gate outputs of this chunk's columns)
        bc_gemm<C, DC, DK, false, false>(sQh, LK, rec + R::kS0 + col0, DV, sO, DC, 1.f, false, sstage);
        __syncthreads();
        bc_gemm<C, DC, C, false, false>(sA, LC, rec + R::kU + col0, DV, sO, DC, 1.f, true, sstage);
        __syncthreads();
        for (int e = tid; e < C * DC; e += NT) {   // dO = dout sigmoid(gate); dgate = dout O sigmoid'
            const int i = e / DC, cc = e % DC;
            float d = 0.f;
            if (i < L) {
                const int64_t o = ((t0 + i) * H + h) * DV + col0 + cc;
                d = p.dout[o];
                if (p.gate) {
                    const float sg = 1.f / (1.f + expf(-bf16_to_f32(p.gate[o])));
                    p.dgate[o] = d * sO[e] * sg * (1.f - sg);
                    d *= sg;
                }
            }
            sO[e] = d;
            rec[R::kdO + (size_t)i * DV + col0 + cc] = d;
        }
        for (int e = tid; e < DK * DC; e += NT) {
            const int r = e / DC, cc = e % DC;
            rec[R::kdS + (size_t)r * DV + col0 + cc] = sdS[e];
        }
        __syncthreads();
        // dU = A^T dO + K- dS_C
        bc_gemm<C, DC, C, true, false>(sA, LC, sO, DC, sdU, DC, 1.f, false, sstage);
        __syncthreads();
        bc_gemm<C, DC, DK, false, false>(sKb, LK, sdS, DC, sdU, DC, 1.f, true, sstage);
        __syncthreads();
        for (int e = tid; e < C * DC; e += NT) {
            const int i = e / DC, cc = e % DC;
            rec[R::kdU + (size_t)i * DV + col0 + cc] = sdU[e];
        }
        // dS0 = Q^T dO + Diag(Gamma_C) dS_C - W^T dU
        bc_gemm<DK, DC, C, true, false>(sQh, LK, sO, DC, sT, DC, 1.f, false, sstage);
        __syncthreads();
        bc_gemm<DK, DC, C, true, false>(sW, LK, sdU, DC, sT, DC, -1.f, true, sstage);
        __syncthreads();
        for (int e = tid; e < DK * DC; e += NT) sdS[e] = fmaf(rec[R::kGC + e / DC], sdS[e], sT[e]);
        __syncthreads();
    }
    if (p.dS0) {
        for (int e = tid; e < DK * DC; e += NT) {
            const int r = e / DC, cc = e % DC;
            p.dS0[(size_t)unit * DK * DV + (size_t)r * DV + col0 + cc] = sdS[e];
        }
    }
}

// ---- 4. per chunk: every input's gradient ------------------------------------------------------
template <int DK, int DV>
__global__ void __launch_bounds__(kBcThreads, 1) bc_grad_kernel(const BwdParams p) {
    constexpr int C = kBcChunk, NT = kBcThreads, LK = DK + 1, LC = C + 1;
    using R = BcRec<DK, DV>;
    extern __shared__ __align__(16) float bcs[];
    float *sk = bcs;                 // [C][LK] k
    float *sq = sk + C * LK;         // [C][LK] scale q
    float *sb = sq + C * LK;         // [C][LK] b
    float *sKh = sb + C * LK;        // [C][LK] K^
    float *sdA = sKh + C * LK;       // [C][LC] dA
    float *sX = sdA + C * LC;        // [C][LC] X
    float *sM = sX + C * LC;         // [C][LC] M, then dM
    float *sT = sM + C * LC;         // [C][LC] T', then dT', then dX, then dL
    float *sbeta = sT + C * LC;      // [C]
    float *sdb = sbeta + C;          // [C] dbeta
    float *sdGC = sdb + C;           // [DK]
    float *sred = sdGC + DK;         // [NT / 32]
    float *sstage = sred + NT / 32;  // bc_gemm staging
    const int64_t gc = blockIdx.x / p.H;
    const int h = static_cast<int>(blockIdx.x % p.H);
    int n, c, L;
    int64_t t0;
    if (!bc_find(p, gc, n, c, t0, L)) return;
    float *rec = p.ckpt + (size_t)blockIdx.x * R::kSize;
    const int tid = threadIdx.x;
    const int64_t H = p.H;
    if (tid == 0) bc_prefetch_l2(rec, (uint32_t)(R::kSize * 4));   // every slot of it is read below
    const float expA = expf(p.A_log[h]);
    for (int e = tid; e < C * DK; e += NT) {
        const int i = e / DK, ch = e % DK;
        const bool in = i < L;
        const int64_t o = ((t0 + i) * H + h) * DK + ch;
        const float kk = in ? bf16_to_f32(p.k[o]) : 0.f;
        const float bb = rec[R::kB + e];
        sk[i * LK + ch] = kk;
        sq[i * LK + ch] = in ? p.scale * bf16_to_f32(p.q[o]) : 0.f;
        sb[i * LK + ch] = bb;
        sKh[i * LK + ch] = kk * expf(bb);
    }
    for (int e = tid; e < C * C; e += NT) {
        const int i = e / C, j = e % C;
        sX[i * LC + j] = rec[R::kX + e];
        sM[i * LC + j] = rec[R::kM + e];
    }
    for (int i = tid; i < C; i += NT) sbeta[i] = i < L ? p.beta[(t0 + i) * H + h] : 0.f;
    for (int ch = tid >> 5; ch < DK; ch += NT / 32) {   // dGamma_C = rowsum(dS_C (.) S0), a warp per row
        float s = 0.f;
        for (int v = tid & 31; v < DV; v += 32)
            s = fmaf(rec[R::kdS + (size_t)ch * DV + v], rec[R::kS0 + (size_t)ch * DV + v], s);
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if ((tid & 31) == 0) sdGC[ch] = s;
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += NT) {   // T' = X diag(beta)
        const int i = e / C, j = e % C;
        sT[i * LC + j] = sX[i * LC + j] * sbeta[j];
    }
    // dA = lower_incl(dO U^T);  dO S0^T over Q^;  dK- = U dS_C^T over K-;  dW = -dU S0^T over W
    bc_gemm<C, C, DV, false, true>(rec + R::kdO, DV, rec + R::kU, DV, sdA, LC, 1.f, false, sstage);
    bc_gemm<C, DK, DV, false, true>(rec + R::kdO, DV, rec + R::kS0, DV, rec + R::kQh, DK, 1.f, false, sstage);
    bc_gemm<C, DK, DV, false, true>(rec + R::kU, DV, rec + R::kdS, DV, rec + R::kKb, DK, 1.f, false, sstage);
    bc_gemm<C, DK, DV, false, true>(rec + R::kdU, DV, rec + R::kS0, DV, rec + R::kW, DK, -1.f, false, sstage);
    __syncthreads();
    for (int e = tid; e < C * C; e += NT) {
        const int i = e / C, j = e % C;
        if (j > i) sdA[i * LC + j] = 0.f;
    }
    for (int e = tid; e < C * DV; e += NT) {   // V, zero padded, over dO (no longer needed)
        const int i = e / DV, ch = e % DV;
        rec[R::kdO + e] = i < L ? bf16_to_f32(p.v[((t0 + i) * H + h) * DV + ch]) : 0.f;
    }
    __syncthreads();
    // T'^T dW over S0 (no longer needed);  dv = T'^T dU over U
    bc_gemm<C, DK, C, true, false>(sT, LC, rec + R::kW, DK, rec + R::kS0, DK, 1.f, false, sstage);
    bc_gemm<C, DV, C, true, false>(sT, LC, rec + R::kdU, DV, rec + R::kU, DV, 1.f, false, sstage);
    __syncthreads();
    for (int e = tid; e < C * DV; e += NT) {
        const int i = e / DV, ch = e % DV;
        if (i < L) p.dv[((t0 + i) * H + h) * DV + ch] = rec[R::kU + e];
    }
    // dT' = dW K^T + dU V^T (over T', after the transposed use above)
    bc_gemm<C, C, DK, false, true>(rec + R::kW, DK, sKh, LK, sT, LC, 1.f, false, sstage);
    __syncthreads();
    bc_gemm<C, C, DV, false, true>(rec + R::kdU, DV, rec + R::kdO, DV, sT, LC, 1.f, true, sstage);
    __syncthreads();
    // dbeta_j = sum_i dT'_ij X_ij;  dX = dT' diag(beta)
    for (int j = tid; j < C; j += NT) {
        float s = 0.f;
        for (int i = 0; i < C; ++i) s = fmaf(sT[i * LC + j], sX[i * LC + j], s);
        sdb[j] = s;
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += NT) {
        const int i = e / C, j = e % C;
        sT[i * LC + j] *= sbeta[j];
    }
    __syncthreads();
    // dL = strict_lower(-X^T dX X^T): Y = X^T dX over A (no longer needed), then dL = -Y X^T over dX
    bc_gemm<C, C, C, true, false>(sX, LC, sT, LC, rec + R::kA, C, 1.f, false, sstage);
    __syncthreads();
    bc_gemm<C, C, C, false, true>(rec + R::kA, C, sX, LC, sT, LC, -1.f, false, sstage);
    __syncthreads();
    // dbeta_i += sum_{j<i} dL_ij M_ij;  dM = diag(beta) dL (strict lower)
    for (int i = tid; i < C; i += NT) {
        float s = 0.f;
        for (int j = 0; j < i; ++j) s = fmaf(sT[i * LC + j], sM[i * LC + j], s);
        sdb[i] += s;
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += NT) {
        const int i = e / C, j = e % C;
        sM[i * LC + j] = j < i ? sbeta[i] * sT[i * LC + j] : 0.f;
    }
    for (int i = tid; i < L; i += NT) p.dbeta[(t0 + i) * H + h] = sdb[i];
    __syncthreads();
    // the pairwise sums: NT / DK threads per key channel, each taking every (NT / DK)-th row
    constexpr int TPC = NT / DK;
    {
        const int ch = tid % DK, part = tid / DK;
        for (int i = part; i < C; i += TPC) {   // dq (over Q^'s slot) and P (over S0's slot)
            const float bi = sb[i * LK + ch];
            float aq = expf(bi) * rec[R::kQh + (size_t)i * DK + ch];
            float ap = expf(bi) * rec[R::kS0 + (size_t)i * DK + ch];
            for (int j = 0; j <= i; ++j) {
                const float E = __expf(bi - sb[j * LK + ch]);
                const float kE = sk[j * LK + ch] * E;
                aq = fmaf(sdA[i * LC + j], kE, aq);
                ap = fmaf(sM[i * LC + j], kE, ap);   // dM_ii = 0
            }
            rec[R::kQh + (size_t)i * DK + ch] = p.scale * aq;
            rec[R::kS0 + (size_t)i * DK + ch] = ap;
        }
        for (int j = part; j < C; j += TPC) {   // Q (over W's slot)
            const float bj = sb[j * LK + ch];
            float aQ = 0.f;
            for (int i = j; i < C; ++i) {
                const float E = __expf(sb[i * LK + ch] - bj);
                aQ = fmaf(sdA[i * LC + j] * sq[i * LK + ch] + sM[i * LC + j] * sk[i * LK + ch], E, aQ);
            }
            rec[R::kW + (size_t)j * DK + ch] = aQ;
        }
    }
    __syncthreads();   // every row of dq, P and Q is in place
    float dA_acc = 0.f;
    for (int ch = tid; ch < DK; ch += NT) {
        const float bC = sb[(C - 1) * LK + ch];
        float lastR = 0.f;
        // dk = P + Q + R, db = dq q + (P - Q - R) k over K-'s slot (dK-), the last row's extra terms
        for (int r = 0; r < C; ++r) {
            const size_t o = (size_t)r * DK + ch;
            const float kk = sk[r * LK + ch];
            const float Rr = expf(bC - sb[r * LK + ch]) * rec[R::kKb + o];
            const float P = rec[R::kS0 + o], Q = rec[R::kW + o], dq = rec[R::kQh + o];
            const float qq = p.scale != 0.f ? sq[r * LK + ch] / p.scale : 0.f;
            lastR = fmaf(Rr, kk, lastR);
            if (r < L) {
                const int64_t go = ((t0 + r) * H + h) * DK + ch;
                p.dk[go] = P + Q + Rr;
                p.dq[go] = dq;
            }
            rec[R::kKb + o] = dq * qq + (P - Q - Rr) * kk;
        }
        // dg = reverse running sum of db; g = -5 sigmoid(x), x = e^A a
        float run = lastR + sdGC[ch] * expf(bC);
        for (int r = C - 1; r >= 0; --r) {
            run += rec[R::kKb + (size_t)r * DK + ch];
            if (r < L) {
                const int64_t go = ((t0 + r) * H + h) * DK + ch;
                const float x = expA * bf16_to_f32(p.a[go]);
                const float sx = 1.f / (1.f + expf(-x));
                const float dx = run * kGMin * sx * (1.f - sx);
                p.da[go] = dx * expA;
                dA_acc = fmaf(dx, x, dA_acc);
            }
        }
    }
    // dA_log: this CTA's sum, added once
    for (int o = 16; o > 0; o >>= 1) dA_acc += __shfl_xor_sync(0xffffffffu, dA_acc, o);
    if ((tid & 31) == 0) sred[tid >> 5] = dA_acc;
    __syncthreads();
    if (tid == 0) {
        float s = 0.f;
        for (int w = 0; w < NT / 32; ++w) s += sred[w];
        atomicAdd(p.dA_log + h, s);
    }
}

template <int DK, int DV>
struct BcSmem {
    static constexpr int C = kBcChunk, LK = DK + 1, LV = DV + 1, LC = C + 1;
    static constexpr int kPrep = (3 * C * LK + C * LV + 2 * C * LC + C + kBcStageFloats) * 4;
    static constexpr int kState = (2 * DK * kBcCols + C * kBcCols + 2 * C * LK + kBcStageFloats) * 4;
    static constexpr int kDState = (2 * DK * kBcCols + 2 * C * kBcCols + 3 * C * LK + C * LC + kBcStageFloats) * 4;
    static constexpr int kGrad = (4 * C * LK + 4 * C * LC + 2 * C + DK + kBcThreads / 32 + kBcStageFloats) * 4;
};

}  // namespace kda

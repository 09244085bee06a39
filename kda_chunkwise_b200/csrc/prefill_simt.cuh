// Chunkwise prefill, CUDA-core (fp32 FMA) kernels.
//
// The chunkwise form ("Kimi K3 · Lesson 3 of 14", CHUNKWISE diagram): a sequence is cut into
// 64-token chunks; inside a chunk every position is computed at once, and the state passes
// sequentially from chunk to chunk.  Per chunk, with incoming state S0, chunk-local cumulative
// log-decay b_r = sum_{i<=r} g_i (per key channel) and Gamma_r = e^{b_r}:
//   Q^ = Gamma (.) (scale q)   K^ = Gamma (.) k   K- = (Gamma_C / Gamma) (.) k
//   L_ij = beta_i sum_c k_ic k_jc e^{b_ic - b_jc}   (j < i)
//   A_ij =        sum_c q_ic k_jc e^{b_ic - b_jc}   (j <= i)
//   (I + L) W = diag(beta) K^,  (I + L) U~ = diag(beta) V          (forward substitution)
//   U = U~ - W S0;   O = Q^ S0 + A U;   S_C = Diag(Gamma_C) S0 + K-^T U
// O = Q^ S0 + A U is the pages' "(Gamma (.) Q) S + A V~" with V~ = U.
//
// The 1/Gamma rescale ("each key rescaled by the reciprocal of its accumulated decay") is done
// per 16-token tile: for the rows of tile p the reference point is r_p = b just before tile p, so
// the row factor e^{b_i - r_p} lies in [e^-80, 1] and the column factor e^{r_p - b_j} lies in
// (0, e^80] for j <= end of tile p.  The g_min = -5 bound is what keeps e^80 finite in fp32/bf16,
// so the diagonal tiles need no special position-pair path.
//
// Two kernels per window of chunks: `prep` (chunk-parallel: gate, cumsum, rescale, Gram, solve)
// writes one record per (sequence, chunk, head) to the workspace; `state` walks the chunks of
// each (sequence, head, 32-column slab of d_v) in order, carrying S in shared memory.
#pragma once

#include "common.cuh"

namespace kda {

template <int DK, int DV>
struct ChunkRecord {
    // fp32 offsets inside one record
    static constexpr int kW = 0;                          // W   [64][DK]
    static constexpr int kU = kW + kChunk * DK;           // U~  [64][DV]
    static constexpr int kQ = kU + kChunk * DV;           // Q^  [64][DK]
    static constexpr int kKb = kQ + kChunk * DK;          // K-  [64][DK]
    static constexpr int kA = kKb + kChunk * DK;          // A   [64][64]
    static constexpr int kG = kA + kChunk * kChunk;       // Gamma_C [DK]
    static constexpr int kFloats = ((kG + DK) + 63) / 64 * 64;  // 256-byte multiple
};

struct PrepParams {
    const uint16_t *q, *k, *v, *a;
    const float *beta, *A_log;
    const int32_t *cu;
    float *rec;
    int64_t total_tokens;
    int num_seqs, H, chunk0, Wc;
    float scale;
};

template <int DK, int DV>
constexpr int prep_smem_bytes() {
    return 4 * (5 * kChunk * (DK + 1) + kChunk * DV + kChunk * (kChunk + 1) + kChunk);
}

template <int DK, int DV>
__global__ void __launch_bounds__(256) prep_simt_kernel(const PrepParams p) {
    using R = ChunkRecord<DK, DV>;
    constexpr int PK = DK + 1;
    extern __shared__ float sm[];
    float *sb = sm;                   // [64][PK] cumulative log-decay b
    float *sq = sb + kChunk * PK;     // [64][PK] scale*q, then scale*q*e^{b - r_tile}
    float *sk = sq + kChunk * PK;     // [64][PK] k
    float *skr = sk + kChunk * PK;    // [64][PK] k*e^{b - r_tile}      (row operand)
    float *skc = skr + kChunk * PK;   // [64][PK] k*e^{r_p - b}         (column operand)
    float *sv = skc + kChunk * PK;    // [64][DV]
    float *sL = sv + kChunk * DV;     // [64][65]
    float *sbeta = sL + kChunk * (kChunk + 1);

    const int h = blockIdx.y;
    const int n = blockIdx.x / p.Wc, cl = blockIdx.x % p.Wc;
    int64_t s0, s1;
    seq_span(p.cu, n, p.num_seqs, p.total_tokens, s0, s1);
    const int64_t t0 = s0 + (int64_t)(p.chunk0 + cl) * kChunk;
    if (t0 >= s1) return;
    const int L = static_cast<int>(min64(kChunk, s1 - t0));
    const int64_t H = p.H;
    float *rec = p.rec + ((int64_t)(n * p.Wc + cl) * H + h) * R::kFloats;
    const int tid = threadIdx.x;
    const float expA = expf(p.A_log[h]);

    for (int e = tid; e < kChunk * DK; e += 256) {
        const int i = e / DK, c = e % DK;
        float g = 0.f, qv = 0.f, kv = 0.f;
        if (i < L) {
            const int64_t off = ((t0 + i) * H + h) * DK + c;
            g = log_decay(bf16_to_f32(p.a[off]), expA);
            qv = p.scale * bf16_to_f32(p.q[off]);
            kv = bf16_to_f32(p.k[off]);
        }
        sb[i * PK + c] = g;
        sq[i * PK + c] = qv;
        sk[i * PK + c] = kv;
    }
    for (int e = tid; e < kChunk * DV; e += 256) {
        const int i = e / DV, c = e % DV;
        sv[e] = i < L ? bf16_to_f32(p.v[((t0 + i) * H + h) * DV + c]) : 0.f;
    }
    if (tid < kChunk) sbeta[tid] = tid < L ? p.beta[(t0 + tid) * H + h] : 0.f;
    __syncthreads();

    // chunk-local inclusive cumsum of the log-decay (padded rows carry g = 0)
    if (tid < DK) {
        float acc = 0.f;
        for (int i = 0; i < kChunk; ++i) {
            acc += sb[i * PK + tid];
            sb[i * PK + tid] = acc;
        }
    }
    __syncthreads();

    // Q^, K-, Gamma_C; then the tile-referenced row operands (same element set per thread)
    for (int e = tid; e < kChunk * DK; e += 256) {
        const int i = e / DK, c = e % DK;
        const float b = sb[i * PK + c], bC = sb[(kChunk - 1) * PK + c];
        const float qv = sq[i * PK + c], kv = sk[i * PK + c];
        rec[R::kQ + i * DK + c] = qv * __expf(b);
        rec[R::kKb + i * DK + c] = kv * __expf(bC - b);
        const int pt = i / kTile;
        const float ref = pt ? sb[(pt * kTile - 1) * PK + c] : 0.f;
        const float f = __expf(b - ref);
        sq[i * PK + c] = qv * f;
        skr[i * PK + c] = kv * f;
    }
    if (tid < DK) rec[R::kG + tid] = __expf(sb[(kChunk - 1) * PK + tid]);
    __syncthreads();

    // Gram rows tile by tile; columns rescaled by 1/Gamma relative to the row tile's reference
    for (int pt = 0; pt < kTilesPerChunk; ++pt) {
        const int ncols = kTile * (pt + 1);
        for (int e = tid; e < ncols * DK; e += 256) {
            const int j = e / DK, c = e % DK;
            const float ref = pt ? sb[(pt * kTile - 1) * PK + c] : 0.f;
            skc[j * PK + c] = sk[j * PK + c] * __expf(ref - sb[j * PK + c]);
        }
        __syncthreads();
        for (int e = tid; e < kTile * kChunk; e += 256) {
            const int i = pt * kTile + e / kChunk, j = e % kChunk;
            float aq = 0.f, ak = 0.f;
            if (j <= i) {
#pragma unroll 8
                for (int c = 0; c < DK; ++c) {
                    const float kc = skc[j * PK + c];
                    aq = fmaf(sq[i * PK + c], kc, aq);
                    ak = fmaf(skr[i * PK + c], kc, ak);
                }
            }
            rec[R::kA + i * kChunk + j] = aq;
            sL[i * (kChunk + 1) + j] = j < i ? sbeta[i] * ak : 0.f;
        }
        __syncthreads();
    }

    // forward substitution, one column of W (or U~) per thread, held in registers
    for (int col = tid; col < DK + DV; col += 256) {
        const bool isW = col < DK;
        const int c = isW ? col : col - DK;
        float x[kChunk];
#pragma unroll
        for (int i = 0; i < kChunk; ++i) {
            float rhs = isW ? sk[i * PK + c] * __expf(sb[i * PK + c]) : sv[i * DV + c];
            rhs *= sbeta[i];
#pragma unroll
            for (int j = 0; j < i; ++j) rhs = fmaf(-sL[i * (kChunk + 1) + j], x[j], rhs);
            x[i] = rhs;
        }
        float *dst = rec + (isW ? R::kW : R::kU);
        const int ld = isW ? DK : DV;
#pragma unroll
        for (int i = 0; i < kChunk; ++i) dst[i * ld + c] = x[i];
    }
}

struct StateParams {
    const float *rec;
    const uint16_t *gate;
    void *out;
    const int32_t *cu;
    const float *S_in;
    float *S_out;
    int64_t total_tokens;
    int num_seqs, H, chunk0, Wc, max_chunks, first_window;
    bool out_f32;
};

constexpr int kSlab = 32;  // d_v columns per state CTA

template <int DK, int DV>
constexpr int state_smem_bytes() {
    return 4 * (DK * kSlab + 3 * kChunk * (DK + 1) + kChunk * (kChunk + 1) +
                2 * kChunk * (kSlab + 1) + DK);
}

template <int DK, int DV>
__global__ void __launch_bounds__(256) state_simt_kernel(const StateParams p) {
    using R = ChunkRecord<DK, DV>;
    constexpr int PK = DK + 1, PS = kSlab + 1;
    extern __shared__ float sm[];
    float *sS = sm;                        // [DK][kSlab]
    float *sW = sS + DK * kSlab;           // [64][PK]
    float *sQ = sW + kChunk * PK;          // [64][PK]
    float *sKb = sQ + kChunk * PK;         // [64][PK]
    float *sA = sKb + kChunk * PK;         // [64][65]
    float *sUt = sA + kChunk * (kChunk + 1);  // [64][PS]
    float *sU = sUt + kChunk * PS;         // [64][PS]
    float *sg = sU + kChunk * PS;          // [DK]

    const int n = blockIdx.x, h = blockIdx.y, col0 = blockIdx.z * kSlab;
    const int tid = threadIdx.x;
    const int64_t H = p.H;
    int64_t s0, s1;
    const bool well_formed = seq_span(p.cu, n, p.num_seqs, p.total_tokens, s0, s1);
    const int64_t len = s1 - s0;
    const int64_t nchunks = (len + kChunk - 1) / kChunk;
    if (p.first_window && h == 0 && blockIdx.z == 0 && tid == 0) {
        if (!well_formed) atomicOr(&g_kda_error_word, kErrBadSeqlens);
        if (nchunks > p.max_chunks) atomicOr(&g_kda_error_word, kErrSeqTooLong);
    }
    const int c_begin = p.chunk0;
    const int c_end = static_cast<int>(min64(p.chunk0 + p.Wc, nchunks));
    if (c_begin >= c_end && !p.first_window) return;

    const size_t st_base = ((size_t)n * H + h) * DK * DV + col0;
    for (int e = tid; e < DK * kSlab; e += 256) {
        const int c = e / kSlab, j = e % kSlab;
        sS[e] = p.S_in ? p.S_in[st_base + (size_t)c * DV + j] : 0.f;
    }

    for (int ch = c_begin; ch < c_end; ++ch) {
        const float *rec = p.rec + ((int64_t)(n * p.Wc + (ch - p.chunk0)) * H + h) * R::kFloats;
        const int64_t t0 = s0 + (int64_t)ch * kChunk;
        const int L = static_cast<int>(min64(kChunk, s1 - t0));
        __syncthreads();  // previous chunk done with the staging buffers
        for (int e = tid; e < kChunk * DK; e += 256) {
            const int i = e / DK, c = e % DK;
            sW[i * PK + c] = rec[R::kW + e];
            sQ[i * PK + c] = rec[R::kQ + e];
            sKb[i * PK + c] = rec[R::kKb + e];
        }
        for (int e = tid; e < kChunk * kChunk; e += 256)
            sA[(e / kChunk) * (kChunk + 1) + e % kChunk] = rec[R::kA + e];
        for (int e = tid; e < kChunk * kSlab; e += 256) {
            const int i = e / kSlab, j = e % kSlab;
            sUt[i * PS + j] = rec[R::kU + i * DV + col0 + j];
        }
        for (int c = tid; c < DK; c += 256) sg[c] = rec[R::kG + c];
        __syncthreads();

        // U = U~ - W S
        for (int e = tid; e < kChunk * kSlab; e += 256) {
            const int i = e / kSlab, j = e % kSlab;
            float acc = sUt[i * PS + j];
#pragma unroll 8
            for (int c = 0; c < DK; ++c) acc = fmaf(-sW[i * PK + c], sS[c * kSlab + j], acc);
            sU[i * PS + j] = acc;
        }
        __syncthreads();

        // O = Q^ S + A U, gated, stored as bf16
        for (int e = tid; e < kChunk * kSlab; e += 256) {
            const int i = e / kSlab, j = e % kSlab;
            float acc = 0.f;
#pragma unroll 8
            for (int c = 0; c < DK; ++c) acc = fmaf(sQ[i * PK + c], sS[c * kSlab + j], acc);
            for (int jj = 0; jj <= i; ++jj) acc = fmaf(sA[i * (kChunk + 1) + jj], sU[jj * PS + j], acc);
            if (i < L) {
                const int64_t off = ((t0 + i) * H + h) * DV + col0 + j;
                if (p.gate) acc *= sigmoid_fast(bf16_to_f32(p.gate[off]));
                store_out(p.out, off, p.out_f32, acc);
            }
        }
        __syncthreads();

        // S = Diag(Gamma_C) S + K-^T U   (each element read and written by one thread)
        for (int e = tid; e < DK * kSlab; e += 256) {
            const int c = e / kSlab, j = e % kSlab;
            float acc = sg[c] * sS[e];
#pragma unroll 8
            for (int i = 0; i < kChunk; ++i) acc = fmaf(sKb[i * PK + c], sU[i * PS + j], acc);
            sS[e] = acc;
        }
    }
    __syncthreads();
    for (int e = tid; e < DK * kSlab; e += 256) {
        const int c = e / kSlab, j = e % kSlab;
        p.S_out[st_base + (size_t)c * DV + j] = sS[e];
    }
}

}  // namespace kda

// Fused chunkwise prefill: one persistent kernel, producer and consumer roles in every CTA.
//
// The chunkwise form ("Kimi K3 · Lesson 3 of 14", CHUNKWISE diagram): 64-token chunks, every
// position of a chunk computed at once with dense products, the state carried sequentially from
// chunk to chunk.  Per chunk, with incoming state S, chunk-local cumulative log-decay
// b_r = sum_{i<=r} g_i (per key channel) and Gamma_r = e^{b_r}:
//   Q^ = Gamma (.) (scale q)    K^ = Gamma (.) k    K- = (Gamma_C / Gamma) (.) k
//   L_ij = beta_i sum_c k_ic k_jc e^{b_ic - b_jc}  (j < i)      T' = (I + L)^-1 diag(beta)
//   A_ij =        sum_c q_ic k_jc e^{b_ic - b_jc}  (j <= i)     W = T' K^,  U~ = T' V
//   U = U~ - W S;   O = Q^ S + A U;   S <- Diag(Gamma_C) S + K-^T U;   out = sigmoid(gate) O
// O = Q^ S + A U is the pages' "(Gamma (.) Q) S + A V~".
//
// 1/Gamma rescale on 16-token tiles ("each key rescaled by the reciprocal of its accumulated
// decay").  With r_p = b just before tile p, every token carries a row factor e^{b_i - r_p} in
// [e^-80, 1] and a rescaled key K~_j = k_j e^{r_q - b_j} (q = its tile) in [1, e^80] |k|.  Gram
// block (p, q <= p) is  sum_c (q_ic e^{b_ic - r_p}) (K~_jc e^{r_p - r_q}):  the column factor
// e^{r_p - b_j} is <= e^80 on the diagonal block and <= 1 below it.  The g >= -5 floor is what
// caps it at e^80, finite in bf16, so diagonal blocks are dense tensor-core products like the
// rest.  Each factor is a product of terms each <= 1 or <= e^80, so an underflow only drops a
// term that is itself below e^-87.
//
// Precision.  The A = Q K^T Gram feeds the output directly and needs more than bf16 operands: its
// operands are split into bf16 hi + lo and accumulated as hi.hi + hi.lo + lo.hi (about 16 bits).
// The K K^T Gram (the solve's L) is plain bf16.  Everything on the value path (A, T', K^, V, W,
// U~, Q^, K-, the state and U) is fp16 with fp32 accumulation: 11 significant bits, ample range
// for unit keys and bounded values.  The state itself stays fp32 in registers.
//
// Work decomposition.  A unit is one (sequence, head).  Its d_v columns are split into G slabs
// of 32; the unit runs on a cluster of G CTAs (the cluster only guarantees the G CTAs run at the
// same time).  Every CTA has 16 warps:
//   consumer warps 0-7:  the sequential state pass for slab `rank` of the unit.
//   producer warps 8-15: the chunk-parallel work for chunks rank, rank + G, rank + 2G, ...,
//                        written as ready-to-use mma fragments into the unit's ring.
// The ring (2G slots per unit, in the workspace, small enough to stay in L2) carries chunk c in
// slot c % 2G; `full` and `empty` counters per slot order the hand-off (release/acquire at gpu
// scope).  Every wait is bounded: on timeout the waiting role records kErrTimeout and returns.
#pragma once

#include "common.cuh"
#include "mma_frag.cuh"

namespace kda {

constexpr int kSlab = 32;                 // d_v columns per consumer
constexpr int kRoleThreads = 256;         // threads per role
constexpr int kFusedThreads = 2 * kRoleThreads;
constexpr int kBarConsumer = 1, kBarProducer = 2;
constexpr float kLog2e = 1.4426950408889634f;

// Ring slot layout.  "Tile" = one 16x16 fp16 A-operand tile stored fragment-major: lane l's four
// 32-bit registers at byte 16 l, so a warp loads or stores a tile with one 16-byte access per lane.
template <int DK, int DV>
struct RingLayout {
    static constexpr int G = DV / kSlab;          // slabs = consumers = producers per unit
    static constexpr int R = 2 * G;               // slots per unit
    static constexpr int KT = DK / 16;            // d_k tiles
    static constexpr int kW = 0;                  // W tiles   (token tile m, d_k tile k): m*KT + k
    static constexpr int kQ = kW + 4 * KT * 512;  // Q^ tiles  (m, k): m*KT + k
    static constexpr int kKbT = kQ + 4 * KT * 512;  // K-^T tiles (d_k tile m, token tile k): m*4 + k
    static constexpr int kA = kKbT + KT * 4 * 512;  // A tiles (m, k <= m): m(m+1)/2 + k
    static constexpr int kU = kA + 10 * 512;      // U~: [token tile][slab][lane][16 fp16]
    static constexpr int kGam = kU + 4 * G * 32 * 32;  // Gamma_C fp32 [DK]
    static constexpr int kBytes = ((kGam + DK * 4) + 1023) / 1024 * 1024;
};

// Shared memory of one CTA (bytes).
template <int DK, int DV>
struct FusedSmem {
    // consumer
    static constexpr int kS = 0;                      // fp16 [DK][32] state operand
    static constexpr int kU = kS + DK * kSlab * 2;    // fp16 [64][32] U operand
    static constexpr int kCFlag = kU + 64 * kSlab * 2;  // int abort flag
    static constexpr int kProd = (kCFlag + 16 + 1023) / 1024 * 1024;
    // producer (all [64][*] operand tiles are swizzled row-major)
    static constexpr int kQhi = kProd;                // bf16 [64][DK] q, then hi of q e^{b - r}
    static constexpr int kQlo = kQhi + 64 * DK * 2;   // bf16 [64][DK] lo of q e^{b - r}
    static constexpr int kK = kQlo + 64 * DK * 2;     // bf16 [64][DK] k
    static constexpr int kV = kK + 64 * DK * 2;       // bf16 [64][DV] v
    static constexpr int kKr = kV + 64 * DV * 2;      // bf16 [64][DK] a, then k e^{b - r}
    static constexpr int kKh = kKr + 64 * DK * 2;     // fp16 [64][DK] K^
    static constexpr int kKb = kKh + 64 * DK * 2;     // fp16 [64][DK] K-
    static constexpr int kKt = kKb + 64 * DK * 2;     // fp32 [64][DK] K~ = k e^{r_q - b}
    static constexpr int kB = kKt + 64 * DK * 4;      // fp32 [64][DK] b; later L, T fp32 [64][65]
    static constexpr int kBBytes = (64 * DK * 4 > 2 * 64 * 65 * 4) ? 64 * DK * 4 : 2 * 64 * 65 * 4;
    static constexpr int kTb = kB + kBBytes;          // fp16 [64][64] T'
    static constexpr int kTmp = kTb + 64 * 64 * 2;    // fp32 [3][16][17] solve scratch
    static constexpr int kBeta = kTmp + 3 * 16 * 17 * 4;  // fp32 [64]
    static constexpr int kTot = kBeta + 64 * 4;       // fp32 [4][DK] cumsum part totals
    static constexpr int kRef = kTot + 4 * DK * 4;    // fp32 [4][DK] r_p
    static constexpr int kEP = kRef + 4 * DK * 4;     // fp32 [4][DK] e^{r_p}
    static constexpr int kTT = kEP + 4 * DK * 4;      // fp32 [4][DK] e^{r_{p+1} - r_p}
    static constexpr int kAbc = kTT + 4 * DK * 4;     // fp32 [4][DK] e^{b_C - r_{p+1}}
    static constexpr int kD = kAbc + 4 * DK * 4;      // fp32 [6][DK] e^{r_p - r_q}, q < p
    static constexpr int kPFlag = kD + 6 * DK * 4;    // int abort flag
    static constexpr int kBytes = kPFlag + 16;
};

// index of the pair (p, q < p) in the 6-entry decay table
__host__ __device__ constexpr int pair_index(int p, int q) { return p * (p - 1) / 2 + q; }

struct FusedParams {
    const uint16_t *q, *k, *v, *a, *gate;
    const float *beta, *A_log;
    const int32_t *cu;
    const float *S_in;
    float *S_out;
    void *out;
    int *flags;         // [units][R][2]: full, empty
    char *ring;         // [units][R][slot bytes]
    int64_t total_tokens;
    int num_seqs, H;
    int max_seqlen;              // 0: no bound to check
    float scale;
    bool out_f32;
    unsigned long long wait_ns;  // bound of every wait
};

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Spin (one thread) until *flag >= target, at most wait_ns.  Returns false on timeout.
__device__ __forceinline__ bool wait_at_least(const int *flag, int target, unsigned long long wait_ns) {
    if (ld_acquire_gpu(flag) >= target) return true;
    const unsigned long long t0 = globaltimer_ns();
    unsigned ns = 32;
    while (true) {
        __nanosleep(ns);
        if (ld_acquire_gpu(flag) >= target) return true;
        if (ns < 256) ns <<= 1;
        if (globaltimer_ns() - t0 > wait_ns) return false;
    }
}

// Role-wide bounded wait: thread 0 of the role spins, the role's barrier publishes the outcome.
__device__ __forceinline__ bool role_wait(const int *flag, int target, int role_tid, int bar_id,
                                          volatile int *abort_flag, unsigned long long wait_ns) {
    if (role_tid == 0) {
        const bool ok = wait_at_least(flag, target, wait_ns);
        if (!ok) atomicOr(&g_kda_error_word, kErrTimeout);
        *abort_flag = ok ? 0 : 1;
    }
    named_bar(bar_id, kRoleThreads);
    return *abort_flag == 0;
}

__device__ __forceinline__ float2 unpack_f16(uint32_t v) {
    const __half2 h = *reinterpret_cast<const __half2 *>(&v);
    return __half22float2(h);
}

// ---------------------------------------------------------------------------------------------
// Producer: chunk-parallel work for chunks rank, rank + G, ... of one unit.
// ---------------------------------------------------------------------------------------------
template <int DK, int DV>
__device__ __forceinline__ void fused_producer(const FusedParams &p, unsigned char *sm, int unit,
                                               int h, int rank, int64_t s0, int64_t s1,
                                               int nchunks) {
    using RL = RingLayout<DK, DV>;
    using SM = FusedSmem<DK, DV>;
    constexpr int G = RL::G, R = RL::R, KT = RL::KT;
    constexpr int RB = DK * 2;   // row bytes of the [64][DK] 16-bit operands
    constexpr int RBV = DV * 2;
    const int tid = threadIdx.x - kRoleThreads;
    const int warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;

    unsigned char *const sQhi = sm + SM::kQhi, *const sQlo = sm + SM::kQlo, *const sK = sm + SM::kK;
    unsigned char *const sKr = sm + SM::kKr, *const sKh = sm + SM::kKh, *const sKb = sm + SM::kKb;
    unsigned char *const sKt = sm + SM::kKt, *const sTb = sm + SM::kTb;
    unsigned char *const sBb = sm + SM::kB;
    float *const sL = reinterpret_cast<float *>(sm + SM::kB);   // [64][65] once b is dead
    float *const sT = sL + 64 * 65;                             // [64][65]
    float *const sTmp = reinterpret_cast<float *>(sm + SM::kTmp);
    float *const sbeta = reinterpret_cast<float *>(sm + SM::kBeta);
    float *const stot = reinterpret_cast<float *>(sm + SM::kTot);
    float *const sref = reinterpret_cast<float *>(sm + SM::kRef);
    float *const sEP = reinterpret_cast<float *>(sm + SM::kEP);
    float *const sTT = reinterpret_cast<float *>(sm + SM::kTT);
    float *const sAbc = reinterpret_cast<float *>(sm + SM::kAbc);
    float *const sD = reinterpret_cast<float *>(sm + SM::kD);
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(sm + SM::kPFlag);
    auto bval = [&](int t, int c) -> float & {   // b in the swizzled fp32 layout
        return *reinterpret_cast<float *>(sBb + swz_f32<DK>(t, c & ~1) + ((c & 1) << 2));
    };

    const int64_t H = p.H;
    const float expA = expf(p.A_log[h]);
    int *const flags = p.flags + (size_t)unit * R * 2;
    char *const ring = p.ring + (size_t)unit * R * RL::kBytes;
    const uint32_t aQhi = smem_u32(sQhi), aQlo = smem_u32(sQlo), aK = smem_u32(sK);
    const uint32_t aV = smem_u32(sm + SM::kV), aKr = smem_u32(sKr), aKh = smem_u32(sKh);
    const uint32_t aKb = smem_u32(sKb), aTb = smem_u32(sTb);

    for (int c = rank; c < nchunks; c += G) {
        const int slot = c % R;
        const int64_t t0 = s0 + (int64_t)c * kChunk;
        const int L = static_cast<int>(min64(kChunk, s1 - t0));

        // 1. q, k, a, v rows of the chunk into shared memory (rows >= L zero-filled), and beta
        {
            constexpr int CPR = DK / 8;  // 16-byte chunks per row
            for (int e = tid; e < 64 * CPR; e += kRoleThreads) {
                const int row = e / CPR, ch = e % CPR;
                const bool in = row < L;
                const int64_t off = ((t0 + (in ? row : 0)) * H + h) * DK + ch * 8;
                const uint32_t dst = swz<RB>(row, ch);
                cp_async_16(aQhi + dst, p.q + off, in ? 16 : 0);
                cp_async_16(aK + dst, p.k + off, in ? 16 : 0);
                cp_async_16(aKr + dst, p.a + off, in ? 16 : 0);
            }
            constexpr int CPRV = DV / 8;
            for (int e = tid; e < 64 * CPRV; e += kRoleThreads) {
                const int row = e / CPRV, ch = e % CPRV;
                const bool in = row < L;
                const int64_t off = ((t0 + (in ? row : 0)) * H + h) * DV + ch * 8;
                cp_async_16(aV + swz<RBV>(row, ch), p.v + off, in ? 16 : 0);
            }
            if (tid < 64) sbeta[tid] = tid < L ? p.beta[(t0 + tid) * H + h] : 0.f;
            cp_async_wait_all();
            named_bar(kBarProducer, kRoleThreads);
        }

        // 2. log-decay g and its chunk-local inclusive cumsum b (rows >= L carry g = 0)
        {
            constexpr int PARTS = kRoleThreads / DK;   // 2 for d_k = 128, 4 for 64
            constexpr int TPP = 64 / PARTS;
            const int ch = tid % DK, part = tid / DK;
            float acc = 0.f;
#pragma unroll 4
            for (int i = 0; i < TPP; ++i) {
                const int t = part * TPP + i;
                const uint16_t raw = *reinterpret_cast<const uint16_t *>(sKr + swz_elem<RB>(t, ch));
                acc += t < L ? log_decay(bf16_to_f32(raw), expA) : 0.f;
                bval(t, ch) = acc;
            }
            stot[part * DK + ch] = acc;
            named_bar(kBarProducer, kRoleThreads);
            if (part > 0) {
                float off = 0.f;
                for (int pp = 0; pp < part; ++pp) off += stot[pp * DK + ch];
                for (int i = 0; i < TPP; ++i) bval(part * TPP + i, ch) += off;
            }
            named_bar(kBarProducer, kRoleThreads);
        }

        // 2b. per-channel tile constants
        if (tid < DK) {
            const int ch = tid;
            float r[5];
            r[0] = 0.f;
            r[1] = bval(15, ch);
            r[2] = bval(31, ch);
            r[3] = bval(47, ch);
            r[4] = bval(63, ch);   // b_C
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
                sref[pp * DK + ch] = r[pp];
                sEP[pp * DK + ch] = ex2(r[pp] * kLog2e);
                sTT[pp * DK + ch] = ex2((r[pp + 1] - r[pp]) * kLog2e);
                sAbc[pp * DK + ch] = ex2((r[4] - r[pp + 1]) * kLog2e);
#pragma unroll
                for (int qq = 0; qq < pp; ++qq)
                    sD[pair_index(pp, qq) * DK + ch] = ex2((r[pp] - r[qq]) * kLog2e);
            }
        }
        named_bar(kBarProducer, kRoleThreads);

        // the slot must be free (chunk c - R consumed by all G consumers) before any ring write
        if (c >= R) {
            if (!role_wait(flags + slot * 2 + 1, G * (c / R), tid, kBarProducer, abort_flag,
                           p.wait_ns))
                return;
        }
        char *const slotp = ring + (size_t)slot * RL::kBytes;

        // 3. operands.  Each thread owns the A-fragment positions of KT/2 tiles of [64][DK]
        //    (rows 16m + g, +8; columns 16kd + 2t4, +1, +8, +9) and writes its Q^ fragments
        //    straight to the ring.
#pragma unroll 1
        for (int j = 0; j < KT / 2; ++j) {
            const int idx = warp * (KT / 2) + j;
            const int m = idx / KT, kd = idx % KT, pt = m;   // token tile = 16-token tile
            uint32_t qfrag[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int t = 16 * m + g + 8 * (e & 1);
                const int ch = 16 * kd + 2 * t4 + 8 * (e >> 1);
                const uint32_t off = swz_elem<RB>(t, ch);
                const float2 bb = *reinterpret_cast<const float2 *>(sBb + swz_f32<DK>(t, ch));
                const float2 rr = *reinterpret_cast<const float2 *>(sref + pt * DK + ch);
                const float x0 = (bb.x - rr.x) * kLog2e, x1 = (bb.y - rr.y) * kLog2e;
                const float rf0 = ex2(x0), rf1 = ex2(x1);      // e^{b - r_p} in [e^-80, 1]
                const float iv0 = ex2(-x0), iv1 = ex2(-x1);    // e^{r_p - b} in [1, e^80]
                float2 qv = unpack_bf16(*reinterpret_cast<const uint32_t *>(sQhi + off));
                const float2 kv = unpack_bf16(*reinterpret_cast<const uint32_t *>(sK + off));
                qv.x *= p.scale;
                qv.y *= p.scale;
                const float2 ep = *reinterpret_cast<const float2 *>(sEP + pt * DK + ch);
                const float2 tt = *reinterpret_cast<const float2 *>(sTT + pt * DK + ch);
                const float2 ab = *reinterpret_cast<const float2 *>(sAbc + pt * DK + ch);
                uint32_t hi, lo;
                split_bf16(qv.x * rf0, qv.y * rf1, hi, lo);
                *reinterpret_cast<uint32_t *>(sQhi + off) = hi;
                *reinterpret_cast<uint32_t *>(sQlo + off) = lo;
                *reinterpret_cast<uint32_t *>(sKr + off) = pack_bf16(kv.x * rf0, kv.y * rf1);
                *reinterpret_cast<float2 *>(sKt + swz_f32<DK>(t, ch)) = make_float2(kv.x * iv0, kv.y * iv1);
                *reinterpret_cast<uint32_t *>(sKh + off) = pack_f16(kv.x * ep.x * rf0, kv.y * ep.y * rf1);
                // K- = k e^{b_C - b} = k (e^{b_C - r_{p+1}}) (e^{r_{p+1} - r_p} e^{r_p - b}), each <= 1
                *reinterpret_cast<uint32_t *>(sKb + off) =
                    pack_f16(kv.x * ab.x * (tt.x * iv0), kv.y * ab.y * (tt.y * iv1));
                qfrag[e] = pack_f16(qv.x * ep.x * rf0, qv.y * ep.y * rf1);   // Q^ = q e^{b}
            }
            stg_v4(slotp + RL::kQ + idx * 512 + lane * 16, make_uint4(qfrag[0], qfrag[1], qfrag[2], qfrag[3]));
        }
        named_bar(kBarProducer, kRoleThreads);

        // 4a. Gram blocks (p, q <= p), one n8 half per job: A = mask(Q K^T) (split bf16) and
        //     L = beta * strict(K K^T) (bf16).  Column fragments are built in registers from K~
        //     times e^{r_p - r_q} and split into bf16 hi + lo.
#pragma unroll 1
        for (int job = warp; job < 20; job += 8) {
            const int blk = job >> 1, nt = job & 1;
            const int pb = blk >= 6 ? 3 : blk >= 3 ? 2 : blk >= 1 ? 1 : 0;
            const int qb = blk - pb * (pb + 1) / 2;
            const int jrow = 16 * qb + 8 * nt + g;   // column index j of this lane's B element
            const float *dcol = pb > qb ? sD + pair_index(pb, qb) * DK : nullptr;
            float aqk[4] = {0.f, 0.f, 0.f, 0.f}, akk[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
            for (int ks = 0; ks < KT; ++ks) {
                uint32_t ahi[4], alo[4], ak[4];
                ldsm_x4(ahi, ldsm_addr_a<RB>(aQhi, 16 * pb, 16 * ks, lane));
                ldsm_x4(alo, ldsm_addr_a<RB>(aQlo, 16 * pb, 16 * ks, lane));
                ldsm_x4(ak, ldsm_addr_a<RB>(aKr, 16 * pb, 16 * ks, lane));
                const int c0 = 16 * ks + 2 * t4;
                float2 k0 = *reinterpret_cast<const float2 *>(sKt + swz_f32<DK>(jrow, c0));
                float2 k1 = *reinterpret_cast<const float2 *>(sKt + swz_f32<DK>(jrow, c0 + 8));
                if (dcol) {
                    const float2 d0 = *reinterpret_cast<const float2 *>(dcol + c0);
                    const float2 d1 = *reinterpret_cast<const float2 *>(dcol + c0 + 8);
                    k0.x *= d0.x; k0.y *= d0.y; k1.x *= d1.x; k1.y *= d1.y;
                }
                uint32_t bh0, bl0, bh1, bl1;
                split_bf16(k0.x, k0.y, bh0, bl0);
                split_bf16(k1.x, k1.y, bh1, bl1);
                mma_bf16(aqk, ahi, bh0, bh1);
                mma_bf16(aqk, ahi, bl0, bl1);
                mma_bf16(aqk, alo, bh0, bh1);
                mma_bf16(akk, ak, bh0, bh1);
            }
            const int i0 = 16 * pb + g, i1 = i0 + 8;
            const int jc = 16 * qb + 8 * nt + 2 * t4;
            const bool diag = pb == qb;
            // A fragment half (columns 8 nt .. 8 nt + 7 of the 16x16 tile), fp16
            const float a0 = !diag || jc <= i0 ? aqk[0] : 0.f;
            const float a1 = !diag || jc + 1 <= i0 ? aqk[1] : 0.f;
            const float a2 = !diag || jc <= i1 ? aqk[2] : 0.f;
            const float a3 = !diag || jc + 1 <= i1 ? aqk[3] : 0.f;
            stg_v2(slotp + RL::kA + blk * 512 + lane * 16 + nt * 8, pack_f16(a0, a1), pack_f16(a2, a3));
            const float b0 = sbeta[i0], b1 = sbeta[i1];
            sL[i0 * 65 + jc] = !diag || jc < i0 ? b0 * akk[0] : 0.f;
            sL[i0 * 65 + jc + 1] = !diag || jc + 1 < i0 ? b0 * akk[1] : 0.f;
            sL[i1 * 65 + jc] = !diag || jc < i1 ? b1 * akk[2] : 0.f;
            sL[i1 * 65 + jc + 1] = !diag || jc + 1 < i1 ? b1 * akk[3] : 0.f;
        }
        // 4b. K-^T fragments and Gamma_C
        for (int idx = warp; idx < 4 * KT; idx += 8) {
            uint32_t fr[4];
            const int md = idx / 4, kt = idx % 4;   // K-^T tile (d_k tile md, token tile kt)
            ldsm_x4_t(fr, ldsm_addr_bn<RB>(aKb, 16 * kt, 16 * md, lane));
            stg_v4(slotp + RL::kKbT + idx * 512 + lane * 16, make_uint4(fr[0], fr[1], fr[2], fr[3]));
        }
        if (tid < DK)   // e^{b_C} = e^{r_3} e^{b_C - r_3}
            reinterpret_cast<float *>(slotp + RL::kGam)[tid] = sEP[3 * DK + tid] * sTT[3 * DK + tid];
        named_bar(kBarProducer, kRoleThreads);

        // 5. T = (I + L)^-1, blocked: diagonal 16x16 inverses, then off-diagonal blocks by level
        if (warp < 4 && lane < 16) {
            const int pb = warp, m = lane, o = 16 * pb;
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float v = i == m ? 1.f : 0.f;
#pragma unroll
                for (int j = 0; j < i; ++j) v = fmaf(-sL[(o + i) * 65 + o + j], x[j], v);
                x[i] = i >= m ? v : 0.f;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) sT[(o + i) * 65 + o + m] = x[i];
        }
        named_bar(kBarProducer, kRoleThreads);
        {
            const int ii = tid >> 4, jj = tid & 15;
#pragma unroll 1
            for (int d = 1; d < 4; ++d) {
                // M = sum_{m=q}^{p-1} L_pm T_mq for every block (p, q = p - d)
                for (int bq = 0; bq + d < 4; ++bq) {
                    const int pb = bq + d;
                    float acc = 0.f;
                    for (int mb = bq; mb < pb; ++mb)
#pragma unroll
                        for (int x = 0; x < 16; ++x)
                            acc = fmaf(sL[(16 * pb + ii) * 65 + 16 * mb + x],
                                       sT[(16 * mb + x) * 65 + 16 * bq + jj], acc);
                    sTmp[(bq * 16 + ii) * 17 + jj] = acc;
                }
                named_bar(kBarProducer, kRoleThreads);
                // T_pq = -D_p M
                for (int bq = 0; bq + d < 4; ++bq) {
                    const int pb = bq + d;
                    float acc = 0.f;
#pragma unroll
                    for (int x = 0; x < 16; ++x)
                        acc = fmaf(sT[(16 * pb + ii) * 65 + 16 * pb + x], sTmp[(bq * 16 + x) * 17 + jj],
                                   acc);
                    sT[(16 * pb + ii) * 65 + 16 * bq + jj] = -acc;
                }
                named_bar(kBarProducer, kRoleThreads);
            }
        }
        // T' = T diag(beta) as fp16 (lower triangle incl. diagonal; zero above)
        for (int e = tid; e < 64 * 32; e += kRoleThreads) {
            const int i = e >> 5, j = (e & 31) * 2;
            const float v0 = j <= i ? sT[i * 65 + j] * sbeta[j] : 0.f;
            const float v1 = j + 1 <= i ? sT[i * 65 + j + 1] * sbeta[j + 1] : 0.f;
            *reinterpret_cast<uint32_t *>(sTb + swz_elem<128>(i, j)) = pack_f16(v0, v1);
        }
        named_bar(kBarProducer, kRoleThreads);

        // 6. W = T' K^ and U~ = T' V: warp -> token tile m, column half hf
        {
            const int m = warp & 3, hf = warp >> 2;
            constexpr int WN = DK / 2, UN = DV / 2;   // columns per half
            float accW[WN / 8][4], accU[UN / 8][4];
#pragma unroll
            for (int i = 0; i < WN / 8; ++i) accW[i][0] = accW[i][1] = accW[i][2] = accW[i][3] = 0.f;
#pragma unroll
            for (int i = 0; i < UN / 8; ++i) accU[i][0] = accU[i][1] = accU[i][2] = accU[i][3] = 0.f;
#pragma unroll
            for (int kt = 0; kt < 4; ++kt) {
                if (kt <= m) {
                    uint32_t af[4];
                    ldsm_x4(af, ldsm_addr_a<128>(aTb, 16 * m, 16 * kt, lane));
#pragma unroll
                    for (int np = 0; np < WN / 16; ++np) {
                        uint32_t bf[4];
                        ldsm_x4_t(bf, ldsm_addr_bt<RB>(aKh, 16 * kt, hf * WN + 16 * np, lane));
                        mma_f16(accW[2 * np], af, bf[0], bf[1]);
                        mma_f16(accW[2 * np + 1], af, bf[2], bf[3]);
                    }
#pragma unroll
                    for (int np = 0; np < UN / 16; ++np) {
                        uint32_t bf[4];
                        ldsm_x4_t(bf, ldsm_addr_bt<RBV>(aV, 16 * kt, hf * UN + 16 * np, lane));
                        mma_f16(accU[2 * np], af, bf16x2_to_f16x2(bf[0]), bf16x2_to_f16x2(bf[1]));
                        mma_f16(accU[2 * np + 1], af, bf16x2_to_f16x2(bf[2]), bf16x2_to_f16x2(bf[3]));
                    }
                }
            }
#pragma unroll
            for (int np = 0; np < WN / 16; ++np) {
                const int kd = hf * (WN / 16) + np;
                uint4 fr;
                fr.x = pack_f16(accW[2 * np][0], accW[2 * np][1]);
                fr.y = pack_f16(accW[2 * np][2], accW[2 * np][3]);
                fr.z = pack_f16(accW[2 * np + 1][0], accW[2 * np + 1][1]);
                fr.w = pack_f16(accW[2 * np + 1][2], accW[2 * np + 1][3]);
                stg_v4(slotp + RL::kW + (m * KT + kd) * 512 + lane * 16, fr);
            }
#pragma unroll
            for (int sl = 0; sl < UN / kSlab; ++sl) {
                const int s = hf * (UN / kSlab) + sl;
                const float(*u)[4] = accU + 4 * sl;
                uint4 lo, hi;
                lo.x = pack_f16(u[0][0], u[0][1]);
                lo.y = pack_f16(u[0][2], u[0][3]);
                lo.z = pack_f16(u[1][0], u[1][1]);
                lo.w = pack_f16(u[1][2], u[1][3]);
                hi.x = pack_f16(u[2][0], u[2][1]);
                hi.y = pack_f16(u[2][2], u[2][3]);
                hi.z = pack_f16(u[3][0], u[3][1]);
                hi.w = pack_f16(u[3][2], u[3][3]);
                char *dst = slotp + RL::kU + ((m * G + s) * 32 + lane) * 32;
                stg_v4(dst, lo);
                stg_v4(dst + 16, hi);
            }
        }
        named_bar(kBarProducer, kRoleThreads);
        if (tid == 0) {
            __threadfence();
            st_release_gpu(flags + slot * 2, c + 1);
        }
    }
}

// ---------------------------------------------------------------------------------------------
// Consumer: the sequential state pass for slab `rank` (32 columns of d_v) of one unit.
// ---------------------------------------------------------------------------------------------
template <int DK, int DV>
__device__ __forceinline__ void fused_consumer(const FusedParams &p, unsigned char *sm, int unit,
                                               int n, int h, int rank, int64_t s0, int64_t s1,
                                               int nchunks) {
    using RL = RingLayout<DK, DV>;
    using SM = FusedSmem<DK, DV>;
    constexpr int G = RL::G, R = RL::R, KT = RL::KT;
    constexpr int SNT = DK / 32;   // n8 tiles of the state per warp
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    unsigned char *const sS = sm + SM::kS;
    unsigned char *const sU = sm + SM::kU;
    const uint32_t aS = smem_u32(sS), aU = smem_u32(sU);
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(sm + SM::kCFlag);
    const int64_t H = p.H;
    const int col0 = rank * kSlab;
    int *const flags = p.flags + (size_t)unit * R * 2;
    const char *const ring = p.ring + (size_t)unit * R * RL::kBytes;

    // state tile of this warp: d_k rows 16 md + (g, g+8), slab columns 8 (sn0 + j) + 2 t4 (+1)
    const int md = DK == 128 ? warp : (warp & 3);
    const int sn0 = DK == 128 ? 0 : 2 * (warp >> 2);
    const int r0 = 16 * md + g, r1 = r0 + 8;
    const size_t st_base = ((size_t)n * H + h) * DK * DV + col0;
    float S[SNT][4];
#pragma unroll
    for (int j = 0; j < SNT; ++j) {
        const int cc = 8 * (sn0 + j) + 2 * t4;
        if (p.S_in) {
            const float2 x0 = *reinterpret_cast<const float2 *>(p.S_in + st_base + (size_t)r0 * DV + cc);
            const float2 x1 = *reinterpret_cast<const float2 *>(p.S_in + st_base + (size_t)r1 * DV + cc);
            S[j][0] = x0.x; S[j][1] = x0.y; S[j][2] = x1.x; S[j][3] = x1.y;
        } else {
            S[j][0] = S[j][1] = S[j][2] = S[j][3] = 0.f;
        }
    }
    // output tile of this warp: token rows 16 m + (g, g+8), slab columns 16 ch + 8 j + 2 t4 (+1)
    const int m = warp & 3, ch = warp >> 2;

    for (int c = 0; c < nchunks; ++c) {
        // fp16 copy of the state: the B operand of W S and Q^ S
#pragma unroll
        for (int j = 0; j < SNT; ++j) {
            const int cc = 8 * (sn0 + j) + 2 * t4;
            *reinterpret_cast<uint32_t *>(sS + swz_elem<64>(r0, cc)) = pack_f16(S[j][0], S[j][1]);
            *reinterpret_cast<uint32_t *>(sS + swz_elem<64>(r1, cc)) = pack_f16(S[j][2], S[j][3]);
        }
        const int slot = c % R;
        if (!role_wait(flags + slot * 2, c + 1, tid, kBarConsumer, abort_flag, p.wait_ns)) return;
        const char *const slotp = ring + (size_t)slot * RL::kBytes;
        const int64_t t0 = s0 + (int64_t)c * kChunk;
        const int L = static_cast<int>(min64(kChunk, s1 - t0));

        uint4 Wf[KT], Af[4], Kf[4];
#pragma unroll
        for (int kd = 0; kd < KT; ++kd) Wf[kd] = ldg_cg_v4(slotp + RL::kW + (m * KT + kd) * 512 + lane * 16);
#pragma unroll
        for (int kt = 0; kt < 4; ++kt) {
            Af[kt] = kt <= m ? ldg_cg_v4(slotp + RL::kA + (m * (m + 1) / 2 + kt) * 512 + lane * 16)
                             : make_uint4(0, 0, 0, 0);
            Kf[kt] = ldg_cg_v4(slotp + RL::kKbT + (md * 4 + kt) * 512 + lane * 16);
        }
        const uint4 Uf = ldg_cg_v4(slotp + RL::kU + ((m * G + rank) * 32 + lane) * 32 + ch * 16);
        const float gam0 = __ldcg(reinterpret_cast<const float *>(slotp + RL::kGam) + r0);
        const float gam1 = __ldcg(reinterpret_cast<const float *>(slotp + RL::kGam) + r1);
        const int i0 = 16 * m + g, i1 = i0 + 8;

        // U = U~ - W S  (the chain), then O = Q^ S
        float accU[2][4], accO[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) accU[j][e] = accO[j][e] = 0.f;
#pragma unroll
        for (int kd = 0; kd < KT; ++kd) {
            uint32_t bf[4];
            ldsm_x4_t(bf, ldsm_addr_bt<64>(aS, 16 * kd, 16 * ch, lane));
            const uint32_t wa[4] = {Wf[kd].x, Wf[kd].y, Wf[kd].z, Wf[kd].w};
            mma_f16(accU[0], wa, bf[0], bf[1]);
            mma_f16(accU[1], wa, bf[2], bf[3]);
        }
        {
            const uint32_t uw[4] = {Uf.x, Uf.y, Uf.z, Uf.w};
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float2 ut0 = unpack_f16(uw[2 * j]), ut1 = unpack_f16(uw[2 * j + 1]);
                accU[j][0] = ut0.x - accU[j][0];
                accU[j][1] = ut0.y - accU[j][1];
                accU[j][2] = ut1.x - accU[j][2];
                accU[j][3] = ut1.y - accU[j][3];
                const int cc = 16 * ch + 8 * j + 2 * t4;
                *reinterpret_cast<uint32_t *>(sU + swz_elem<64>(i0, cc)) = pack_f16(accU[j][0], accU[j][1]);
                *reinterpret_cast<uint32_t *>(sU + swz_elem<64>(i1, cc)) = pack_f16(accU[j][2], accU[j][3]);
            }
        }
#pragma unroll
        for (int kd = 0; kd < KT; ++kd) {
            uint32_t bf[4];
            ldsm_x4_t(bf, ldsm_addr_bt<64>(aS, 16 * kd, 16 * ch, lane));
            const uint4 q4 = ldg_cg_v4(slotp + RL::kQ + (m * KT + kd) * 512 + lane * 16);
            const uint32_t qa[4] = {q4.x, q4.y, q4.z, q4.w};
            mma_f16(accO[0], qa, bf[0], bf[1]);
            mma_f16(accO[1], qa, bf[2], bf[3]);
        }
        uint32_t gt[2][2] = {{0u, 0u}, {0u, 0u}};
        if (p.gate) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int cc = col0 + 16 * ch + 8 * j + 2 * t4;
                if (i0 < L) gt[j][0] = *reinterpret_cast<const uint32_t *>(p.gate + ((t0 + i0) * H + h) * DV + cc);
                if (i1 < L) gt[j][1] = *reinterpret_cast<const uint32_t *>(p.gate + ((t0 + i1) * H + h) * DV + cc);
            }
        }
        named_bar(kBarConsumer, kRoleThreads);   // U complete in shared memory

        // S = Diag(Gamma_C) S + K-^T U   (the chain)
#pragma unroll
        for (int j = 0; j < SNT; ++j) {
            S[j][0] *= gam0; S[j][1] *= gam0; S[j][2] *= gam1; S[j][3] *= gam1;
        }
#pragma unroll
        for (int kt = 0; kt < 4; ++kt) {
            const uint32_t ka[4] = {Kf[kt].x, Kf[kt].y, Kf[kt].z, Kf[kt].w};
#pragma unroll
            for (int np = 0; np < SNT / 2; ++np) {
                uint32_t bf[4];
                ldsm_x4_t(bf, ldsm_addr_bt<64>(aU, 16 * kt, 8 * sn0 + 16 * np, lane));
                mma_f16(S[2 * np], ka, bf[0], bf[1]);
                mma_f16(S[2 * np + 1], ka, bf[2], bf[3]);
            }
        }
        // O += A U, gate, store
#pragma unroll
        for (int kt = 0; kt < 4; ++kt) {
            if (kt <= m) {
                uint32_t bf[4];
                ldsm_x4_t(bf, ldsm_addr_bt<64>(aU, 16 * kt, 16 * ch, lane));
                const uint32_t aa[4] = {Af[kt].x, Af[kt].y, Af[kt].z, Af[kt].w};
                mma_f16(accO[0], aa, bf[0], bf[1]);
                mma_f16(accO[1], aa, bf[2], bf[3]);
            }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int cc = col0 + 16 * ch + 8 * j + 2 * t4;
            float o0 = accO[j][0], o1 = accO[j][1], o2 = accO[j][2], o3 = accO[j][3];
            if (p.gate) {
                const float2 ga = unpack_bf16(gt[j][0]), gb = unpack_bf16(gt[j][1]);
                o0 *= sigmoid_fast(ga.x); o1 *= sigmoid_fast(ga.y);
                o2 *= sigmoid_fast(gb.x); o3 *= sigmoid_fast(gb.y);
            }
            if (i0 < L) {
                const int64_t off = ((t0 + i0) * H + h) * DV + cc;
                if (p.out_f32) *reinterpret_cast<float2 *>(static_cast<float *>(p.out) + off) = make_float2(o0, o1);
                else *reinterpret_cast<uint32_t *>(static_cast<uint16_t *>(p.out) + off) = pack_bf16(o0, o1);
            }
            if (i1 < L) {
                const int64_t off = ((t0 + i1) * H + h) * DV + cc;
                if (p.out_f32) *reinterpret_cast<float2 *>(static_cast<float *>(p.out) + off) = make_float2(o2, o3);
                else *reinterpret_cast<uint32_t *>(static_cast<uint16_t *>(p.out) + off) = pack_bf16(o2, o3);
            }
        }
        // every warp is done with this slot and with sS / sU before they are rewritten
        named_bar(kBarConsumer, kRoleThreads);
        if (tid == 0) red_release_add_gpu(flags + slot * 2 + 1, 1);
    }
    if (p.S_out) {
#pragma unroll
        for (int j = 0; j < SNT; ++j) {
            const int cc = 8 * (sn0 + j) + 2 * t4;
            *reinterpret_cast<float2 *>(p.S_out + st_base + (size_t)r0 * DV + cc) = make_float2(S[j][0], S[j][1]);
            *reinterpret_cast<float2 *>(p.S_out + st_base + (size_t)r1 * DV + cc) = make_float2(S[j][2], S[j][3]);
        }
    }
}

template <int DK, int DV>
__global__ void __launch_bounds__(kFusedThreads, 1) kda_prefill_fused_kernel(const FusedParams p) {
    constexpr int G = DV / kSlab;
    extern __shared__ __align__(1024) unsigned char fsmem[];
    const int unit = blockIdx.x / G, rank = blockIdx.x % G;
    const int n = unit / p.H, h = unit % p.H;
    int64_t s0, s1;
    const bool well_formed = seq_span(p.cu, n, p.num_seqs, p.total_tokens, s0, s1);
    if (h == 0 && rank == 0 && threadIdx.x == 0) {
        if (!well_formed) atomicOr(&g_kda_error_word, kErrBadSeqlens);
        if (p.max_seqlen > 0 && s1 - s0 > p.max_seqlen) atomicOr(&g_kda_error_word, kErrSeqTooLong);
    }
    const int nchunks = static_cast<int>((s1 - s0 + kChunk - 1) / kChunk);
    if (threadIdx.x < kRoleThreads)
        fused_consumer<DK, DV>(p, fsmem, unit, n, h, rank, s0, s1, nchunks);
    else
        fused_producer<DK, DV>(p, fsmem, unit, h, rank, s0, s1, nchunks);
}

}  // namespace kda

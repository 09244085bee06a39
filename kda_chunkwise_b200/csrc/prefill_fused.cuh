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
// of 32; the unit runs on a cluster of G CTAs (the cluster guarantees the G CTAs run at the same
// time and gives them each other's shared-memory barriers).  Every CTA has 16 warps:
//   consumer warps 0-7:  the sequential state pass for slab `rank` of the unit, on tcgen05: the
//                        chunk's A operands in tensor memory, S and U as fp16 B operands in
//                        shared memory, fp32 accumulators in tensor memory.
//   producer warps 8-15: the chunk-parallel work for chunks rank, rank + G, rank + 2G, ...
//                        (mma.sync tiles of 16), written into the unit's ring in the layout the
//                        consumer copies straight into tensor memory.
// The ring (2G slots per unit, in the workspace, small enough to stay in L2) carries chunk c in
// slot c % 2G.  Shared-memory mbarriers order the hand-off at cluster scope: every CTA has a
// `full` barrier per slot, on which the producing CTA arrives (remotely) once the chunk is in the
// ring; the producing CTA's `empty` barrier of the slot collects one arrival from each of the G
// consumers once they have read it.  Slot s is always produced by CTA s % G, so phase u of a
// slot's barriers belongs to chunk s + u 2G.  Every wait is bounded: on timeout the waiting role
// records kErrTimeout and returns; all threads then meet at a cluster barrier before exit, so no
// CTA leaves while another may still arrive on its barriers.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "mma_frag.cuh"
#include "gate_sigmoid.cuh"
#include "umma.cuh"

namespace kda {

constexpr int kSlab = 32;                 // d_v columns per consumer
constexpr int kRoleThreads = 256;         // threads per role
constexpr int kFusedThreads = 2 * kRoleThreads;
constexpr int kBarConsumer = 1, kBarProducer = 2;
constexpr float kLog2e = 1.4426950408889634f;

// Ring slot layout.  The consumer moves the tensor-core A operands of a chunk into tensor memory
// (TMEM), so the producer writes them as "TMEM images": [16-byte chunk j][TMEM lane][16 bytes],
// where chunk j of a lane holds its 32-bit columns 4j .. 4j + 3 and column c holds the fp16 pair
// (row, 2c), (row, 2c + 1).  A warp then reads 512 contiguous bytes per load, one 16-byte piece
// per lane.
template <int DK, int DV>
struct RingLayout {
    static constexpr int G = DV / kSlab;          // slabs = consumers = producers per unit
    static constexpr int R = 2 * G;               // slots per unit
    static constexpr int KT = DK / 16;            // d_k tiles
    static constexpr int kA1 = 0;                 // [W ; Q^]: lanes 0-63 W, 64-127 Q^ (K = d_k)
    static constexpr int kA2 = kA1 + DK / 8 * 128 * 16;  // K-^T: lanes = d_k rows (K = tokens)
    static constexpr int kA3 = kA2 + 8 * DK * 16;        // A: lanes 64-127 = token rows (K = tokens)
    static constexpr int kA4 = kA3 + 8 * 64 * 16;        // A - fp16(A), the same image
    static constexpr int kU = kA4 + 8 * 64 * 16;  // U~: [slab][half][chunk 2][row 64][8 fp16]
    static constexpr int kGam = kU + G * 2 * 2 * 64 * 16;  // Gamma_C fp32 [DK]
    static constexpr int kBytes = ((kGam + DK * 4) + 1023) / 1024 * 1024;
};

// Shared memory of one CTA (bytes).
template <int DK, int DV>
struct FusedSmem {
    using RL = RingLayout<DK, DV>;
    // consumer (B operands of the tensor-core products: 8 x 8 fp16 core matrices, MN-major)
    static constexpr int kB1 = 0;                     // S_c: K = d_k rows, N = 32 columns
    static constexpr int kB2 = kB1 + DK * kSlab * 2;  // U:   K = 64 tokens, N = 32 columns
    static constexpr int kB3 = kB2 + 64 * kSlab * 2;  // U - fp16(U), the same layout
    static constexpr int kFull = kB3 + 64 * kSlab * 2;  // u64 mbarrier [R]: chunk published
    static constexpr int kEmpty = kFull + 8 * RL::R;  // u64 mbarrier [R]: chunk consumed (the
                                                      //   producing CTA's copy is the one used)
    static constexpr int kM1 = kEmpty + 8 * RL::R;    // u64 mbarrier: [W; Q^] S complete
    static constexpr int kM2 = kM1 + 8;               // u64 mbarrier: K-^T U and A U complete
    static constexpr int kTmem = kM2 + 8;             // u32 TMEM base address
    static constexpr int kCFlag = kTmem + 8;          // int abort flag
    static constexpr int kProd = (kCFlag + 16 + 1023) / 1024 * 1024;
    // producer (all [64][*] operand tiles are swizzled row-major)
    static constexpr int kQhi = kProd;                // bf16 [64][DK] q, then hi of q e^{b - r}
    static constexpr int kQlo = kQhi + 64 * DK * 2;   // bf16 [64][DK] lo of q e^{b - r}
    static constexpr int kK = kQlo + 64 * DK * 2;     // bf16 [64][DK] k, then fp16 K-
    static constexpr int kV = kK + 64 * DK * 2;       // bf16 [64][DV] v
    static constexpr int kKr = kV + 64 * DV * 2;      // bf16 [64][DK] a, then k e^{b - r}
    static constexpr int kKh = kKr + 64 * DK * 2;     // fp16 [64][DK] K^
    static constexpr int kKt = kKh + 64 * DK * 2;     // fp32 [64][DK] K~
    static constexpr int kB = kKt + 64 * DK * 4;      // scratch of the later phases:
    static constexpr int kLd = kB;                    //   fp32 [4][16][17] diagonal blocks of L
    static constexpr int kLD = kLd + 4 * 16 * 17 * 4;   //   fp16 [64][64]: -L below the diagonal
                                                      //   blocks, (I + L_pp)^-1 on them
    static constexpr int kT = kLD + 64 * 64 * 2;      //   fp16 [64][64] T' = (I + L)^-1 diag(beta)
    static constexpr int kM = kT + 64 * 64 * 2;       //   fp16 [3][16][32] block-product scratch
    static constexpr int kQh = kT;                    //   fp16 [64][DK] Q^, copied to the ring
                                                      //   before T and M are written
    static constexpr int kBNeed = (kM + 3 * 16 * 64 > kQh + 64 * DK * 2 ? kM + 3 * 16 * 64 : kQh + 64 * DK * 2) - kB;
    static constexpr int kBBytes = (kBNeed + 15) / 16 * 16;
    static constexpr int kBeta = kB + kBBytes;        // fp32 [64]
    static constexpr int kTot = kBeta + 64 * 4;       // fp32 [2 * threads]: run totals of the decay sums
    static constexpr int kD = kTot + 2 * kRoleThreads * 4;   // fp32 [6][DK] e^{r_p - r_q}, q < p
    static constexpr int kPFlag = kD + 6 * DK * 4;    // int abort flag
    static constexpr int kBytes = kPFlag + 16;
    static_assert(kFull % 8 == 0, "mbarriers need 8-byte alignment");
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
    char *ring;         // [units][R][slot bytes]
    int64_t total_tokens;
    int num_seqs, H;
    int max_seqlen;              // 0: no bound to check
    float scale;
    bool out_f32;
    int stall_first_chunk;       // failure injection: never publish chunk 0
    unsigned long long wait_ns;  // bound of every wait
    // Segment maps (0: off).  Value columns [0, maps_cols) run the homogeneous recurrence from the
    // identity (v = 0, S_in = I, read from nowhere); columns [maps_cols, DV) take v from p.v, a
    // [T, H, DV - maps_cols] tensor, from S_in = 0.  The final state is then [M | B] of the tokens.
    int maps_cols;
};

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait until the phase with parity `parity` of a local mbarrier completes, at most wait_ns
// (hardware-suspended polls, %globaltimer bound).  Returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t addr, uint32_t parity,
                                                  unsigned long long wait_ns) {
    if (mbar_try(addr, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try(addr, parity))
        if (globaltimer_ns() - t0 > wait_ns) return false;
    return true;
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
    constexpr int RB = DK * 2;            // row bytes of the [64][DK] 16-bit operands
    constexpr int RBV = DV * 2;
    const int tid = threadIdx.x - kRoleThreads;
    const int warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;

    unsigned char *const sQhi = sm + SM::kQhi, *const sQlo = sm + SM::kQlo, *const sK = sm + SM::kK;
    unsigned char *const sKr = sm + SM::kKr, *const sKh = sm + SM::kKh, *const sKb = sm + SM::kK;
    unsigned char *const sKt = sm + SM::kKt, *const sV = sm + SM::kV;
    unsigned char *const sQh = sm + SM::kQh, *const sLD = sm + SM::kLD, *const sT = sm + SM::kT;
    unsigned char *const sM = sm + SM::kM;
    float *const sLd = reinterpret_cast<float *>(sm + SM::kLd);
    float *const sbeta = reinterpret_cast<float *>(sm + SM::kBeta);
    float *const stot = reinterpret_cast<float *>(sm + SM::kTot);
    float *const sD = reinterpret_cast<float *>(sm + SM::kD);
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(sm + SM::kPFlag);

    const int64_t H = p.H;
    const float expA = expf(p.A_log[h]);
    char *const ring = p.ring + (size_t)unit * R * RL::kBytes;
    const uint32_t aFull = smem_u32(sm + SM::kFull), aEmpty = smem_u32(sm + SM::kEmpty);
    const uint32_t aQhi = smem_u32(sQhi), aQlo = smem_u32(sQlo), aK = smem_u32(sK);
    const uint32_t aV = smem_u32(sV), aKr = smem_u32(sKr), aKh = smem_u32(sKh);
    const uint32_t aKb = smem_u32(sKb), aLD = smem_u32(sLD);
    const uint32_t aT = smem_u32(sT), aM = smem_u32(sM), aQh = smem_u32(sQh);

    // asynchronous input copies of one chunk: q, k, a as one commit group, v as another
    auto load_qka = [&](int cl) {
        const int64_t tl = s0 + (int64_t)cl * kChunk;
        const int Ll = static_cast<int>(min64(kChunk, s1 - tl));
        constexpr int CPR = DK / 8;  // 16-byte chunks per row
#pragma unroll
        for (int it = 0; it < 64 * CPR / kRoleThreads; ++it) {
            const int e = tid + it * kRoleThreads;
            const int row = e / CPR, ch = e % CPR;
            const bool in = row < Ll;
            const int64_t off = ((tl + (in ? row : 0)) * H + h) * DK + ch * 8;
            const uint32_t dst = swz<RB>(row, ch);
            cp_async_16(aQhi + dst, p.q + off, in ? 16 : 0);
            cp_async_16(aK + dst, p.k + off, in ? 16 : 0);
            cp_async_16(aKr + dst, p.a + off, in ? 16 : 0);
        }
        cp_async_commit();
    };
    auto load_v = [&](int cl) {
        const int64_t tl = s0 + (int64_t)cl * kChunk;
        const int Ll = static_cast<int>(min64(kChunk, s1 - tl));
        constexpr int CPRV = DV / 8;
#pragma unroll
        for (int it = 0; it < 64 * CPRV / kRoleThreads; ++it) {
            const int e = tid + it * kRoleThreads;
            const int row = e / CPRV, ch = e % CPRV;
            const bool in = row < Ll && ch * 8 >= p.maps_cols;   // the maps' homogeneous columns read 0
            const int vd = DV - p.maps_cols;                    // row length of p.v
            const int64_t off = in ? ((tl + row) * H + h) * vd + ch * 8 - p.maps_cols : 0;
            cp_async_16(aV + swz<RBV>(row, ch), p.v + off, in ? 16 : 0);
        }
        cp_async_commit();
    };

    // beta of a chunk (64 scattered floats), loaded a chunk ahead into registers
    auto load_beta = [&](int cl) -> float {
        if (tid >= 64 || cl >= nchunks) return 0.f;
        const int64_t tl = s0 + (int64_t)cl * kChunk;
        return tid < min64(kChunk, s1 - tl) ? __ldg(p.beta + (tl + tid) * H + h) : 0.f;
    };
    float beta_next = load_beta(rank);

    for (int c = rank; c < nchunks; c += G) {
        const int slot = c % R;
        const int64_t t0 = s0 + (int64_t)c * kChunk;
        const int L = static_cast<int>(min64(kChunk, s1 - t0));
        // 1. this chunk's q, k, a rows were requested at the end of the previous chunk's Gram
        //    phase and its v rows at the end of the previous chunk (the very first chunk
        //    requests them here), several microseconds ahead of use; rows >= L are zero-filled.
        {
            if (c == rank) {
                load_qka(c);
                load_v(c);
            }
            if (tid < 64) sbeta[tid] = beta_next;   // loaded one chunk ahead
            cp_async_wait_group<1>();   // q, k, a of this chunk (v may still be in flight)
            named_bar(kBarProducer, kRoleThreads);
        }
        beta_next = load_beta(c + G);

        // 2. log-decay g (in log2 units) and its running sum over each thread's run of tokens.
        //    Thread (part, channel pair cp) takes TPP consecutive tokens of channels 2cp, 2cp + 1:
        //    a whole 16-token tile (d_k = 128) or half of one (d_k = 64).  Rows >= L carry g = 0.
        constexpr int CP = DK / 2;                   // channel pairs
        constexpr int PARTS = kRoleThreads / CP;     // 4 (d_k = 128) or 8 (d_k = 64)
        constexpr int TPP = 64 / PARTS;              // tokens per run: 16 or 8
        constexpr int PPT = 16 / TPP;                // runs per 16-token tile: 1 or 2
        const int cp = tid % CP, part = tid / CP, ch = 2 * cp;
        const int pt = part / PPT;                   // tile of this run
        float2 l[TPP];
        {
            constexpr float kG2 = kGMin * kLog2e;
#pragma unroll
            for (int i = 0; i < TPP; ++i) {
                const int t = part * TPP + i;
                const float2 av = unpack_bf16(*reinterpret_cast<const uint32_t *>(sKr + swz_elem<RB>(t, ch)));
                float2 gg = make_float2(kG2 * sigmoid_fast(expA * av.x), kG2 * sigmoid_fast(expA * av.y));
                if (t >= L) gg = make_float2(0.f, 0.f);
                l[i] = i == 0 ? gg : make_float2(l[i - 1].x + gg.x, l[i - 1].y + gg.y);
            }
            *reinterpret_cast<float2 *>(stot + part * DK + ch) = l[TPP - 1];
        }
        // the slot must be free (chunk c - R consumed by all G consumers) before any ring write
        if (tid == 0) {
            bool ok = true;
            if (c >= R) {   // phase c / R - 1 of the slot's empty barrier: chunk c - R consumed
                ok = mbar_wait_bounded(aEmpty + 8 * slot, ((c / R) - 1) & 1, p.wait_ns);
                if (!ok) atomicOr(&g_kda_error_word, kErrTimeout);
            }
            *abort_flag = ok ? 0 : 1;
        }
        named_bar(kBarProducer, kRoleThreads);   // run totals visible
        if (*abort_flag) return;
        char *const slotp = ring + (size_t)slot * RL::kBytes;

        // 3. operands of every token of the run.  In log2 units, r_p = b before tile p, lo = the
        //    part of tile pt before this run; then per token
        //      e^{b - r_p} = 2^(l + lo) <= 1,   e^{r_p - b} = 2^-(l + lo) in [1, e^80],
        //    and Q r = scale q e^{b - r_p} (split bf16 hi + lo), K r = k e^{b - r_p} (bf16),
        //    K~ = k e^{r_p - b} (fp32), K^ = k e^{r_p} e^{b - r_p}, Q^ = scale q e^{r_p} e^{b - r_p},
        //    K- = k e^{b_C - r_{p+1}} (e^{r_{p+1} - r_p} e^{r_p - b}) (fp16; each factor <= 1).
        {
            float2 rp = make_float2(0.f, 0.f), lo = rp, tile = rp, bc = rp;
#pragma unroll
            for (int pp = 0; pp < PARTS; ++pp) {
                const float2 tv = *reinterpret_cast<const float2 *>(stot + pp * DK + ch);
                bc.x += tv.x; bc.y += tv.y;
                if (pp / PPT < pt) { rp.x += tv.x; rp.y += tv.y; }
                if (pp / PPT == pt) {
                    tile.x += tv.x; tile.y += tv.y;
                    if (pp < part) { lo.x += tv.x; lo.y += tv.y; }
                }
            }
            const float2 ep = make_float2(ex2(rp.x), ex2(rp.y));                    // e^{r_p}
            const float2 tt = make_float2(ex2(tile.x), ex2(tile.y));                // e^{r_{p+1} - r_p}
            const float2 ab = make_float2(ex2(bc.x - rp.x - tile.x), ex2(bc.y - rp.y - tile.y));   // e^{b_C - r_{p+1}}
            const float2 eps = make_float2(ep.x * p.scale, ep.y * p.scale);
            if (part == 0) {   // inter-tile decays e^{r_p - r_q} (q < p) and Gamma_C = e^{b_C}
                float2 r[4];
                r[0] = make_float2(0.f, 0.f);
#pragma unroll
                for (int pp = 1; pp < 4; ++pp) {
                    r[pp] = r[pp - 1];
#pragma unroll
                    for (int q2 = 0; q2 < PPT; ++q2) {
                        const float2 tv = *reinterpret_cast<const float2 *>(stot + ((pp - 1) * PPT + q2) * DK + ch);
                        r[pp].x += tv.x; r[pp].y += tv.y;
                    }
                }
#pragma unroll
                for (int pp = 1; pp < 4; ++pp)
#pragma unroll
                    for (int qq = 0; qq < pp; ++qq)
                        *reinterpret_cast<float2 *>(sD + pair_index(pp, qq) * DK + ch) =
                            make_float2(ex2(r[pp].x - r[qq].x), ex2(r[pp].y - r[qq].y));
                *reinterpret_cast<float2 *>(slotp + RL::kGam + ch * 4) = make_float2(ex2(bc.x), ex2(bc.y));
            }
#pragma unroll
            for (int i = 0; i < TPP; ++i) {
                const int t = part * TPP + i;
                const uint32_t off = swz_elem<RB>(t, ch);
                const float x0 = l[i].x + lo.x, x1 = l[i].y + lo.y;
                const float rf0 = ex2(x0), rf1 = ex2(x1);      // e^{b - r_p}
                const float iv0 = ex2(-x0), iv1 = ex2(-x1);    // e^{r_p - b}
                const float2 qv = unpack_bf16(*reinterpret_cast<const uint32_t *>(sQhi + off));
                const float2 kv = unpack_bf16(*reinterpret_cast<const uint32_t *>(sK + off));
                uint32_t hi, lo2;
                split_bf16(qv.x * p.scale * rf0, qv.y * p.scale * rf1, hi, lo2);
                *reinterpret_cast<uint32_t *>(sQhi + off) = hi;
                *reinterpret_cast<uint32_t *>(sQlo + off) = lo2;
                *reinterpret_cast<uint32_t *>(sKr + off) = pack_bf16(kv.x * rf0, kv.y * rf1);
                *reinterpret_cast<float2 *>(sKt + swz_f32<DK>(t, ch)) = make_float2(kv.x * iv0, kv.y * iv1);
                *reinterpret_cast<uint32_t *>(sKh + off) = pack_f16(kv.x * ep.x * rf0, kv.y * ep.y * rf1);
                *reinterpret_cast<uint32_t *>(sKb + off) = pack_f16(kv.x * ab.x * (tt.x * iv0), kv.y * ab.y * (tt.y * iv1));
                *reinterpret_cast<uint32_t *>(sQh + off) = pack_f16(qv.x * eps.x * rf0, qv.y * eps.y * rf1);
            }
        }
        named_bar(kBarProducer, kRoleThreads);

        // 4a. Gram blocks (p, q <= p), one block per job (both n8 halves share the A fragments):
        //     A = mask(Q K^T) (split bf16) and L = beta * strict(K K^T) (bf16).  Column fragments
        //     are built in registers from K~ times e^{r_p - r_q} and split into bf16 hi + lo.
#pragma unroll 1
        for (int blk = warp; blk < 10; blk += 8) {
            const int pb = blk >= 6 ? 3 : blk >= 3 ? 2 : blk >= 1 ? 1 : 0;
            const int qb = blk - pb * (pb + 1) / 2;
            const float *dcol = pb > qb ? sD + pair_index(pb, qb) * DK : nullptr;
            float ahh[2][4], ahl[2][4], alh[2][4], akk[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) ahh[nt][e] = ahl[nt][e] = alh[nt][e] = akk[nt][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KT; ++ks) {
                uint32_t ahi[4], alo[4], ak[4];
                ldsm_x4(ahi, ldsm_addr_a<RB>(aQhi, 16 * pb, 16 * ks, lane));
                ldsm_x4(alo, ldsm_addr_a<RB>(aQlo, 16 * pb, 16 * ks, lane));
                ldsm_x4(ak, ldsm_addr_a<RB>(aKr, 16 * pb, 16 * ks, lane));
                const int c0 = 16 * ks + 2 * t4;
                float2 d0 = make_float2(1.f, 1.f), d1 = d0;
                if (dcol) {
                    d0 = *reinterpret_cast<const float2 *>(dcol + c0);
                    d1 = *reinterpret_cast<const float2 *>(dcol + c0 + 8);
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int jrow = 16 * qb + 8 * nt + g;   // column j of this lane's B element
                    float2 k0 = *reinterpret_cast<const float2 *>(sKt + swz_f32<DK>(jrow, c0));
                    float2 k1 = *reinterpret_cast<const float2 *>(sKt + swz_f32<DK>(jrow, c0 + 8));
                    k0.x *= d0.x; k0.y *= d0.y; k1.x *= d1.x; k1.y *= d1.y;
                    uint32_t bh0, bl0, bh1, bl1;
                    split_bf16(k0.x, k0.y, bh0, bl0);
                    split_bf16(k1.x, k1.y, bh1, bl1);
                    mma_bf16(ahh[nt], ahi, bh0, bh1);
                    mma_bf16(ahl[nt], ahi, bl0, bl1);
                    mma_bf16(alh[nt], alo, bh0, bh1);
                    mma_bf16(akk[nt], ak, bh0, bh1);
                }
            }
            const int i0 = 16 * pb + g, i1 = i0 + 8;
            const bool diag = pb == qb;
            const float b0 = sbeta[i0], b1 = sbeta[i1];
            uint32_t afr[4], alo[4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int jc = 16 * qb + 8 * nt + 2 * t4;
                float aq[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) aq[e] = ahh[nt][e] + (ahl[nt][e] + alh[nt][e]);
                if (diag) {
                    if (jc > i0) aq[0] = 0.f;
                    if (jc + 1 > i0) aq[1] = 0.f;
                    if (jc > i1) aq[2] = 0.f;
                    if (jc + 1 > i1) aq[3] = 0.f;
                }
                // A as fp16 plus its fp16 rounding remainder (the output product uses both)
                afr[2 * nt] = pack_f16(aq[0], aq[1]);
                afr[2 * nt + 1] = pack_f16(aq[2], aq[3]);
                const float2 h0 = unpack_f16(afr[2 * nt]), h1 = unpack_f16(afr[2 * nt + 1]);
                alo[2 * nt] = pack_f16(aq[0] - h0.x, aq[1] - h0.y);
                alo[2 * nt + 1] = pack_f16(aq[2] - h1.x, aq[3] - h1.y);
                if (diag) {   // fp32 diagonal block for the 16x16 inverses
                    const int li = g, lj = 8 * nt + 2 * t4;
                    float *Ld = sLd + pb * 16 * 17;
                    Ld[li * 17 + lj] = lj < li ? b0 * akk[nt][0] : 0.f;
                    Ld[li * 17 + lj + 1] = lj + 1 < li ? b0 * akk[nt][1] : 0.f;
                    Ld[(li + 8) * 17 + lj] = lj < li + 8 ? b1 * akk[nt][2] : 0.f;
                    Ld[(li + 8) * 17 + lj + 1] = lj + 1 < li + 8 ? b1 * akk[nt][3] : 0.f;
                } else {      // -L below the diagonal blocks, fp16 A operand of the block products
                    *reinterpret_cast<uint32_t *>(sLD + swz_elem<128>(i0, jc)) = pack_f16(-b0 * akk[nt][0], -b0 * akk[nt][1]);
                    *reinterpret_cast<uint32_t *>(sLD + swz_elem<128>(i1, jc)) = pack_f16(-b1 * akk[nt][2], -b1 * akk[nt][3]);
                }
            }
            // A rows i0, i1 = lanes of the A image; columns 8qb + 4nt + t4 = chunk 2qb + nt
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                char *const b = slotp + RL::kA3 + ((2 * qb + nt) * 64 + i0) * 16 + t4 * 4;
                st_u32(b, afr[2 * nt]);
                st_u32(b + 8 * 16, afr[2 * nt + 1]);
                st_u32(b + (RL::kA4 - RL::kA3), alo[2 * nt]);
                st_u32(b + (RL::kA4 - RL::kA3) + 8 * 16, alo[2 * nt + 1]);
            }
        }
        if (warp >= 2) {   // zero blocks above the diagonal (the A image is read whole): one per warp
            const int ub = warp - 2;   // (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
            const int pb = ub < 3 ? 0 : ub < 5 ? 1 : 2, qb = ub < 3 ? ub + 1 : ub < 5 ? ub - 1 : 3;
            stg_v4(slotp + RL::kA3 + ((2 * qb + (lane >> 4)) * 64 + 16 * pb + (lane & 15)) * 16, make_uint4(0, 0, 0, 0));
            stg_v4(slotp + RL::kA4 + ((2 * qb + (lane >> 4)) * 64 + 16 * pb + (lane & 15)) * 16, make_uint4(0, 0, 0, 0));
        }
        // 4b. K-^T and Q^ to the ring, by warps 2-7 (warps 0 and 1 take two Gram blocks each).
        //     K-^T tile (d_k tile md, token tile kt) as an A fragment: register e of a lane is row
        //     16md + g (+8 for e odd), columns 8kt + t4 (+4 for e >= 2).
        for (int idx = warp - 2; idx >= 0 && idx < 4 * KT; idx += 6) {
            uint32_t fr[4];
            const int md = idx / 4, kt = idx % 4;
            ldsm_x4_t(fr, ldsm_addr_bn<RB>(aKb, 16 * kt, 16 * md, lane));
            char *const b = slotp + RL::kA2 + ((2 * kt) * DK + 16 * md + g) * 16 + t4 * 4;
            st_u32(b, fr[0]);
            st_u32(b + 8 * 16, fr[1]);
            st_u32(b + DK * 16, fr[2]);
            st_u32(b + DK * 16 + 8 * 16, fr[3]);
        }
        for (int e = tid - 64; e >= 0 && e < 64 * (DK / 8); e += kRoleThreads - 64) {   // Q^ row t -> lane 64 + t
            const int t = e & 63, j = e >> 6;
            stg_v4(slotp + RL::kA1 + (j * 128 + 64 + t) * 16, *reinterpret_cast<const uint4 *>(sQh + swz<RB>(t, j)));
        }
        named_bar(kBarProducer, kRoleThreads);
        // the q, k (now K-) and a (now K r) buffers are no longer read: request the next chunk's
        if (c + G < nchunks) load_qka(c + G);

        // 5. diagonal blocks D_p = (I + L_pp)^-1 by forward substitution (fp32), one column per lane,
        //    column-oriented: once x_j is final it is eliminated from every later row, so the
        //    dependent chain is 15 steps long; written as fp16 into the diagonal blocks of LD and T
        if (warp < 4 && lane < 16) {
            const int pb = warp, mcol = lane;
            const float *Ld = sLd + pb * 16 * 17;
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) x[i] = i == mcol ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < 15; ++j)
#pragma unroll
                for (int i = j + 1; i < 16; ++i) x[i] = fmaf(-Ld[i * 17 + j], x[j], x[i]);
            const float bcol = sbeta[16 * pb + mcol];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                *reinterpret_cast<__half *>(sLD + swz_elem<128>(16 * pb + i, 16 * pb + mcol)) = __float2half_rn(x[i]);
                *reinterpret_cast<__half *>(sT + swz_elem<128>(16 * pb + i, 16 * pb + mcol)) = __float2half_rn(x[i] * bcol);
            }
        }
        // this chunk's v rows (their group is older than the next chunk's q, k, a group)
        if (c + G < nchunks) cp_async_wait_group<1>();
        else cp_async_wait_group<0>();
        named_bar(kBarProducer, kRoleThreads);

        // 5b. off-diagonal blocks of T' = (I + L)^-1 diag(beta) by level d = p - q:
        //     T'_pq = D_p M,  M = sum_{m=q}^{p-1} (-L_pm) T'_mq   (16x16 tensor-core products);
        //     the recursion is linear in the columns of block column q, so starting it from the
        //     diagonal blocks D_q diag(beta_q) yields T' directly.
#pragma unroll 1
        for (int d = 1; d < 4; ++d) {
            if (warp < 4 - d) {
                const int qb = warp, pb = warp + d;
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                for (int mb = qb; mb < pb; ++mb) {
                    uint32_t af[4], bf[4];
                    ldsm_x4(af, ldsm_addr_a<128>(aLD, 16 * pb, 16 * mb, lane));   // -L_pm
                    ldsm_x4_t(bf, ldsm_addr_bt<128>(aT, 16 * mb, 16 * qb, lane));  // T_mq
                    mma_f16(acc[0], af, bf[0], bf[1]);
                    mma_f16(acc[1], af, bf[2], bf[3]);
                }
                const uint32_t aMw = aM + warp * 16 * 64;
                unsigned char *const sMw = sM + warp * 16 * 64;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int cc = 8 * j + 2 * t4;
                    *reinterpret_cast<uint32_t *>(sMw + swz_elem<64>(g, cc)) = pack_f16(acc[j][0], acc[j][1]);
                    *reinterpret_cast<uint32_t *>(sMw + swz_elem<64>(g + 8, cc)) = pack_f16(acc[j][2], acc[j][3]);
                }
                __syncwarp();
                float tq[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                {
                    uint32_t af[4], bf[4];
                    ldsm_x4(af, ldsm_addr_a<128>(aLD, 16 * pb, 16 * pb, lane));   // D_p
                    ldsm_x4_t(bf, ldsm_addr_bt<64>(aMw, 0, 0, lane));              // M
                    mma_f16(tq[0], af, bf[0], bf[1]);
                    mma_f16(tq[1], af, bf[2], bf[3]);
                }
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int cc = 16 * qb + 8 * j + 2 * t4;
                    *reinterpret_cast<uint32_t *>(sT + swz_elem<128>(16 * pb + g, cc)) = pack_f16(tq[j][0], tq[j][1]);
                    *reinterpret_cast<uint32_t *>(sT + swz_elem<128>(16 * pb + g + 8, cc)) = pack_f16(tq[j][2], tq[j][3]);
                }
            }
            named_bar(kBarProducer, kRoleThreads);
        }
        // 6. [W | U~] = T' [K^ | V].  Warp w owns 16-column units w and w + 8 of [W | U~]; the B
        //    fragments of a unit are loaded once per token tile and reused for every row tile.
        {
            constexpr int UW = DK / 16, UT = (DK + DV) / 16;
#pragma unroll 1
            for (int u = warp; u < UT; u += 8) {
                const bool isW = u < UW;
                const int vc = isW ? 16 * u : 16 * u - DK;    // column in K^ or V
                uint32_t bfr[4][4];
#pragma unroll
                for (int kt = 0; kt < 4; ++kt) {
                    if (isW) {
                        ldsm_x4_t(bfr[kt], ldsm_addr_bt<RB>(aKh, 16 * kt, vc, lane));
                    } else {
                        ldsm_x4_t(bfr[kt], ldsm_addr_bt<RBV>(aV, 16 * kt, vc, lane));
#pragma unroll
                        for (int e = 0; e < 4; ++e) bfr[kt][e] = bf16x2_to_f16x2(bfr[kt][e]);
                    }
                }
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                    for (int kt = 0; kt <= m; ++kt) {
                        uint32_t af[4];
                        ldsm_x4(af, ldsm_addr_a<128>(aT, 16 * m, 16 * kt, lane));
                        mma_f16(acc[0], af, bfr[kt][0], bfr[kt][1]);
                        mma_f16(acc[1], af, bfr[kt][2], bfr[kt][3]);
                    }
                    // rows 16m + g (+8); columns vc + 2t4 (+1) and vc + 8 + 2t4 (+1)
                    char *b;
                    int chunk_step;
                    if (isW) {   // [W; Q^] lanes 16m + g, columns 8u + t4 (chunk 2u) and + 4 (chunk 2u + 1)
                        b = slotp + RL::kA1 + ((2 * u) * 128 + 16 * m + g) * 16 + t4 * 4;
                        chunk_step = 128 * 16;
                    } else {     // U~ of slab vc / 32, half (vc / 16) % 2, chunks 0 and 1
                        b = slotp + RL::kU + ((((vc / kSlab) * 2 + ((vc >> 4) & 1)) * 2) * 64 + 16 * m + g) * 16 + t4 * 4;
                        chunk_step = 64 * 16;
                    }
                    st_u32(b, pack_f16(acc[0][0], acc[0][1]));
                    st_u32(b + 8 * 16, pack_f16(acc[0][2], acc[0][3]));
                    st_u32(b + chunk_step, pack_f16(acc[1][0], acc[1][1]));
                    st_u32(b + chunk_step + 8 * 16, pack_f16(acc[1][2], acc[1][3]));
                }
            }
        }
        named_bar(kBarProducer, kRoleThreads);
        if (c + G < nchunks) load_v(c + G);   // the v buffer is free now
        if (tid < G && !(c == 0 && p.stall_first_chunk))
            mbar_arrive_cluster(mapa_shared(aFull + 8 * slot, tid));   // publish to CTA tid
    }
}

// ---------------------------------------------------------------------------------------------
// Consumer: the sequential state pass for slab `rank` (32 columns of d_v) of one unit, on the
// 5th-generation tensor cores.
//
// Per chunk c, with S_c (fp32, in registers: thread (lane quadrant q, half) holds row 32q + lane,
// columns 16 half .. + 15; an fp16 copy in shared memory is the B operand):
//   D  = [W ; Q^] S_c            (M = 128: rows 0-63 W S_c, rows 64-127 Q^ S_c)     TMEM
//   U  = U~ - D[0:64]  -> shared memory (fp16, B operand)
//   D3 = K-^T U,   D[64:128] += A U   (there U and A each as fp16 value + remainder) TMEM
//   S_{c+1} = Diag(Gamma_C) S_c + D3;   out = sigmoid(gate) D[64:128]
// The A operands ([W; Q^], K-^T, A) of chunk c + 1 are fetched from the ring into registers while
// chunk c's products run and then stored into the other of two TMEM buffers; the ring slot is
// handed back as soon as that copy is done.  One thread issues the MMAs; every wait is bounded.
// ---------------------------------------------------------------------------------------------
template <int DK, int DV>
__device__ __forceinline__ void fused_consumer(const FusedParams &p, unsigned char *sm, uint32_t tmem, int unit,
                                               int n, int h, int rank, int64_t s0, int64_t s1, int nchunks) {
    using RL = RingLayout<DK, DV>;
    using SM = FusedSmem<DK, DV>;
    constexpr int G = RL::G, R = RL::R;
    constexpr int A1C = DK / 2;                        // TMEM columns of one [W; Q^] buffer
    constexpr uint32_t cD = 0, cD3 = 32, cA1 = 64, cA2 = cA1 + 2 * A1C, cA3 = cA2 + 64, cA4 = cA3 + 64;
    constexpr uint32_t kIdesc = umma_idesc_f16(128, kSlab);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, half = warp >> 2;
    const int row = 32 * q + lane;                     // this thread's TMEM lane
    const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
    const bool has_s = row < DK, has_u = row < 64, has_o = row >= 64;
    unsigned char *const sB1 = sm + SM::kB1, *const sB2 = sm + SM::kB2, *const sB3 = sm + SM::kB3;
    const uint32_t aB1 = smem_u32(sB1), aB2 = smem_u32(sB2), aB3 = smem_u32(sB3);
    const uint32_t aFull = smem_u32(sm + SM::kFull), aEmpty = smem_u32(sm + SM::kEmpty);
    const uint32_t aM1 = smem_u32(sm + SM::kM1), aM2 = smem_u32(sm + SM::kM2);
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(sm + SM::kCFlag);
    const int64_t H = p.H;
    const int col0 = rank * kSlab + 16 * half;         // this thread's first d_v column
    const char *const ring = p.ring + (size_t)unit * R * RL::kBytes;
    auto slot_of = [&](int c) { return ring + (size_t)(c % R) * RL::kBytes; };
    auto wait_bar = [&](uint32_t bar, uint32_t parity) {
        if (!mbar_wait_bounded(bar, parity, p.wait_ns)) {
            atomicOr(&g_kda_error_word, kErrTimeout);
            *abort_flag = 1;
        }
        __syncwarp();   // the warp-wide tcgen05 loads and stores that follow need a converged warp
    };
    // fp16 copy of 16 values of row k (columns 16 half ..) into a B operand (MN-major core matrices)
    auto store_b = [&](unsigned char *base, int k, const float (&x)[16]) {
#pragma unroll
        for (int g8 = 0; g8 < 2; ++g8) {
            const uint4 v = make_uint4(pack_f16(x[8 * g8 + 0], x[8 * g8 + 1]), pack_f16(x[8 * g8 + 2], x[8 * g8 + 3]),
                                       pack_f16(x[8 * g8 + 4], x[8 * g8 + 5]), pack_f16(x[8 * g8 + 6], x[8 * g8 + 7]));
            *reinterpret_cast<uint4 *>(base + (((k >> 3) * 4 + 2 * half + g8) * 64 + (k & 7) * 8) * 2) = v;
        }
    };
    // chunk cl's A operands: fetched from the ring into registers, then stored into TMEM buffer b
    // (each warp: its lane quadrant, its half of the columns)
    constexpr int NJ = A1C / 8;                        // 16-byte pieces of [W; Q^] per thread
    auto fetch_a12 = [&](int cl, uint4 (&x1)[NJ], uint4 (&x2)[4]) {
        const char *sp = slot_of(cl);
#pragma unroll
        for (int j = 0; j < NJ; ++j) x1[j] = ldg_cg_v4(sp + RL::kA1 + ((half * NJ + j) * 128 + row) * 16);
        if (has_s) {   // K-^T: lanes = d_k rows
#pragma unroll
            for (int j = 0; j < 4; ++j) x2[j] = ldg_cg_v4(sp + RL::kA2 + ((half * 4 + j) * DK + row) * 16);
        }
    };
    auto fetch_a3 = [&](int cl, uint4 (&x3)[4]) {   // A: lanes 64-127 = token rows (has_o threads)
        const char *sp = slot_of(cl);
#pragma unroll
        for (int j = 0; j < 4; ++j) x3[j] = ldg_cg_v4(sp + RL::kA3 + ((half * 4 + j) * 64 + row - 64) * 16);
    };
    auto st4 = [&](uint32_t taddr, const uint4 *x) {
        const uint32_t v[16] = {x[0].x, x[0].y, x[0].z, x[0].w, x[1].x, x[1].y, x[1].z, x[1].w,
                                x[2].x, x[2].y, x[2].z, x[2].w, x[3].x, x[3].y, x[3].z, x[3].w};
        tmem_st16(taddr, v);
    };
    // the remainder A - fp16(A) of chunk cl: straight from the ring into TMEM buffer b (has_o warps)
    auto copy_a4 = [&](int cl, int b) {
        const char *sp = slot_of(cl);
        uint4 x4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) x4[j] = ldg_cg_v4(sp + RL::kA4 + ((half * 4 + j) * 64 + row - 64) * 16);
        st4(tq + cA4 + b * 32 + 16 * half, x4);
    };
    auto put_a = [&](int b, const uint4 (&x1)[NJ], const uint4 (&x2)[4], const uint4 (&x3)[4]) {
#pragma unroll
        for (int part = 0; part < NJ / 4; ++part) st4(tq + cA1 + b * A1C + half * (A1C / 2) + 16 * part, x1 + 4 * part);
        if (has_s) st4(tq + cA2 + b * 32 + 16 * half, x2);
        if (has_o) st4(tq + cA3 + b * 32 + 16 * half, x3);
    };
    // per-thread operands kept in registers: U~ (rows 0-63), Gamma_C (state rows), gate logits
    // (output rows); each is reloaded for the next chunk right after its last use
    uint4 ut[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)}, gt[2] = {ut[0], ut[1]};
    float gam = 0.f;
    auto load_ut = [&](int cl) {
        const char *sp = slot_of(cl);
#pragma unroll
        for (int j = 0; j < 2; ++j) ut[j] = ldg_cg_v4(sp + RL::kU + ((((rank * 2 + half) * 2 + j) * 64) + row) * 16);
    };
    auto load_gam = [&](int cl) { return __ldcg(reinterpret_cast<const float *>(slot_of(cl) + RL::kGam) + row); };
    auto load_gate = [&](int cl) {
        gt[0] = gt[1] = make_uint4(0, 0, 0, 0);
        if (p.gate) {
            const int64_t tg = s0 + (int64_t)cl * kChunk + (row - 64);
            if (tg < s1) {
                const uint4 *gp = reinterpret_cast<const uint4 *>(p.gate + (tg * H + h) * DV + col0);
                gt[0] = __ldg(gp);
                gt[1] = __ldg(gp + 1);
            }
        }
    };

    // initial state; its fp16 copy is the first B operand
    const size_t st_base = ((size_t)n * H + h) * DK * DV;
    float S[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) S[j] = 0.f;
    if (has_s && p.maps_cols) {   // [I | 0]
#pragma unroll
        for (int j = 0; j < 16; ++j) S[j] = (col0 + j < p.maps_cols && col0 + j == row) ? 1.f : 0.f;
    } else if (has_s && p.S_in) {
        const float4 *sp = reinterpret_cast<const float4 *>(p.S_in + st_base + (size_t)row * DV + col0);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 x = sp[j];
            S[4 * j] = x.x; S[4 * j + 1] = x.y; S[4 * j + 2] = x.z; S[4 * j + 3] = x.w;
        }
    }
    if (has_s) store_b(sB1, row, S);

    uint4 x1[NJ], x2[4], x3[4];
    if (nchunks > 0) {   // chunk 0's operands
        wait_bar(aFull + 8 * 0, 0);
        fetch_a12(0, x1, x2);
        if (has_o) fetch_a3(0, x3);
        if (has_o) copy_a4(0, 0);
        if (has_u) load_ut(0);
        if (has_s) gam = load_gam(0);
        if (has_o) load_gate(0);
        put_a(0, x1, x2, x3);
        if (has_u) asm volatile("" ::"r"(ut[0].x), "r"(ut[1].x));   // arrived before slot 0 is handed back
        if (has_s) asm volatile("" ::"f"(gam));
    }
    fence_async_smem();
    tmem_wait_st();
    tc_fence_before();
    named_bar(kBarConsumer, kRoleThreads);
    tc_fence_after();
    if (*abort_flag) return;
    if (nchunks > 0 && tid == 0) mbar_arrive_relaxed_cluster(mapa_shared(aEmpty, 0));   // slot 0 copied

    for (int c = 0; c < nchunks; ++c) {
        const int buf = c & 1;
        const bool has_next = c + 1 < nchunks;
        const int64_t t0 = s0 + (int64_t)c * kChunk;
        const int L = static_cast<int>(min64(kChunk, s1 - t0));
        // 1. D = [W; Q^] S_c
        if (tid == 0) {
#pragma unroll
            for (int k = 0; k < DK / 16; ++k)
                umma_f16_ts(tmem + cD, tmem + cA1 + buf * A1C + 8 * k, umma_desc(aB1 + 1024 * k, 512, 128), kIdesc, k > 0);
            umma_commit(aM1);
        }
        // 2. chunk c+1's operands into registers; their L2 latency overlaps this chunk's products
        float gamn = 0.f;
        if (has_next) {
            wait_bar(aFull + 8 * ((c + 1) % R), ((c + 1) / R) & 1);
            fetch_a12(c + 1, x1, x2);
            if (has_s) gamn = load_gam(c + 1);
        }
        // 3. U = U~ - W S_c  (rows 0-63) -> B operand of the next products
        wait_bar(aM1, c & 1);
        tc_fence_after();
        if (has_u) {
            uint32_t d[16];
            tmem_ld16(tq + cD + 16 * half, d);
            tmem_wait_ld();
            float u[16], ulo[16];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const uint32_t w4[4] = {ut[j].x, ut[j].y, ut[j].z, ut[j].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 t = unpack_f16(w4[e]);
                    u[8 * j + 2 * e] = t.x - __uint_as_float(d[8 * j + 2 * e]);
                    u[8 * j + 2 * e + 1] = t.y - __uint_as_float(d[8 * j + 2 * e + 1]);
                }
            }
            // U enters the output product as fp16 U plus the fp16 rounding remainder U - fp16(U)
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
                const float2 hf = unpack_f16(pack_f16(u[e], u[e + 1]));
                ulo[e] = u[e] - hf.x;
                ulo[e + 1] = u[e + 1] - hf.y;
            }
            store_b(sB2, row, u);
            store_b(sB3, row, ulo);
            if (has_next) load_ut(c + 1);
        } else if (has_next) {
            fetch_a3(c + 1, x3);
            copy_a4(c + 1, buf ^ 1);   // that TMEM buffer's last reader, chunk c - 1, is complete
        }
        fence_async_smem();
        tmem_wait_st();
        tc_fence_before();
        named_bar(kBarConsumer, kRoleThreads);
        tc_fence_after();
        if (*abort_flag) return;
        // 4. D3 = K-^T U;  D[64:128] += A U
        if (tid == 0) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                umma_f16_ts(tmem + cD3, tmem + cA2 + buf * 32 + 8 * k, umma_desc(aB2 + 1024 * k, 512, 128), kIdesc, k > 0);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                umma_f16_ts(tmem + cD, tmem + cA3 + buf * 32 + 8 * k, umma_desc(aB2 + 1024 * k, 512, 128), kIdesc, 1);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                umma_f16_ts(tmem + cD, tmem + cA3 + buf * 32 + 8 * k, umma_desc(aB3 + 1024 * k, 512, 128), kIdesc, 1);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                umma_f16_ts(tmem + cD, tmem + cA4 + buf * 32 + 8 * k, umma_desc(aB2 + 1024 * k, 512, 128), kIdesc, 1);
            umma_commit(aM2);
        }
        // 5. chunk c+1's A operands into the other TMEM buffer (its last user, chunk c-1, is done)
        if (has_next) put_a(buf ^ 1, x1, x2, x3);
        // 6. S_{c+1} = Diag(Gamma_C) S_c + D3;  gated output rows
        wait_bar(aM2, c & 1);
        tc_fence_after();
        if (has_s) {
            uint32_t d[16];
            tmem_ld16(tq + cD3 + 16 * half, d);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) S[j] = fmaf(gam, S[j], __uint_as_float(d[j]));
            store_b(sB1, row, S);
        }
        if (has_o) {
            uint32_t d[16];
            tmem_ld16(tq + cD + 16 * half, d);
            tmem_wait_ld();
            const int i = row - 64;
            // gate and store, one copy per output type (the two never share registers)
            auto emit = [&](auto f32_tag) {
                constexpr bool F32 = decltype(f32_tag)::value;
                float o[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) o[j] = __uint_as_float(d[j]);
                if (p.gate) {
                    const uint32_t gw[8] = {gt[0].x, gt[0].y, gt[0].z, gt[0].w, gt[1].x, gt[1].y, gt[1].z, gt[1].w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float2 sg = F32 ? gate_sigmoid2_f32(gw[e]) : gate_sigmoid2(gw[e]);
                        o[2 * e] *= sg.x;
                        o[2 * e + 1] *= sg.y;
                    }
                }
                if (!p.out) return;   // no outputs wanted (the segment maps)
                const int64_t off = ((t0 + i) * H + h) * DV + col0;
                if constexpr (F32) {
                    float4 *op = reinterpret_cast<float4 *>(static_cast<float *>(p.out) + off);
#pragma unroll
                    for (int j = 0; j < 4; ++j) op[j] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
                } else {
                    uint4 *op = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.out) + off);
#pragma unroll
                    for (int j = 0; j < 2; ++j)
                        op[j] = make_uint4(pack_bf16(o[8 * j], o[8 * j + 1]), pack_bf16(o[8 * j + 2], o[8 * j + 3]),
                                           pack_bf16(o[8 * j + 4], o[8 * j + 5]), pack_bf16(o[8 * j + 6], o[8 * j + 7]));
                }
            };
            if (i < L) {
                if (p.out_f32) emit(std::true_type{});
                else emit(std::false_type{});
            }
            if (has_next) load_gate(c + 1);
        }
        // every value read from slot c+1 must have arrived before the slot is handed back
        if (has_next) {
            if (has_u) asm volatile("" ::"r"(ut[0].x), "r"(ut[1].x));
            if (has_s) asm volatile("" ::"f"(gamn));
        }
        fence_async_smem();
        tmem_wait_st();
        tc_fence_before();
        named_bar(kBarConsumer, kRoleThreads);
        tc_fence_after();
        if (*abort_flag) return;
        // 7. chunk c+1 now lives in TMEM and registers: hand its slot back to the producing CTA.
        //    Every value read from it has arrived, so no release ordering is needed.
        if (has_next && tid == 0)
            mbar_arrive_relaxed_cluster(mapa_shared(aEmpty + 8 * ((c + 1) % R), ((c + 1) % R) % G));
        gam = gamn;
    }
    if (has_s && p.S_out) {
        float4 *sp = reinterpret_cast<float4 *>(p.S_out + st_base + (size_t)row * DV + col0);
#pragma unroll
        for (int j = 0; j < 4; ++j) sp[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
    }
    // An fp16 operand that overflowed (state, pseudo-values, values beyond +-65504) becomes inf and
    // reaches the fp32 state, where no fade can remove it: a non-finite final state flags the unit.
    if (has_s) {
        bool bad = false;
#pragma unroll
        for (int j = 0; j < 16; ++j) bad |= !isfinite(S[j]);
        if (bad) atomicOr(&g_kda_error_word, kErrRange);
    }
}

template <int DK, int DV>
__global__ void __launch_bounds__(kFusedThreads, 1) kda_prefill_fused_kernel(const FusedParams p) {
    using SM = FusedSmem<DK, DV>;
    constexpr int G = DV / kSlab;
    constexpr uint32_t kTmemCols = 512;   // see the column map of the consumer
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
    // The cluster is G CTAs along x, so `rank` is this CTA's rank in it.
    if (threadIdx.x < RingLayout<DK, DV>::R) {
        mbar_init(smem_u32(fsmem + SM::kFull) + 8 * threadIdx.x, 1);
        mbar_init(smem_u32(fsmem + SM::kEmpty) + 8 * threadIdx.x, G);
    }
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(fsmem + SM::kM1), 1);
        mbar_init(smem_u32(fsmem + SM::kM2), 1);
        *reinterpret_cast<volatile int *>(fsmem + SM::kCFlag) = 0;
        *reinterpret_cast<volatile int *>(fsmem + SM::kPFlag) = 0;
    }
    if (threadIdx.x < 32) tmem_alloc(smem_u32(fsmem + SM::kTmem), kTmemCols);
    tc_fence_before();
    cluster_sync_after_init();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(fsmem + SM::kTmem);
    if (threadIdx.x < kRoleThreads)
        fused_consumer<DK, DV>(p, fsmem, tmem, unit, n, h, rank, s0, s1, nchunks);
    else
        fused_producer<DK, DV>(p, fsmem, unit, h, rank, s0, s1, nchunks);
    cp_async_wait_all();
    tc_fence_before();
    cluster_sync();   // no CTA exits while a peer may still arrive on its barriers
    tc_fence_after();
    if (threadIdx.x < 32) {
        __syncwarp();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace kda

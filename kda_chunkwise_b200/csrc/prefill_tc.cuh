// Per-unit chunkwise prefill on the 5th-generation tensor cores: one CTA per (sequence, head).
//
// The chunkwise form ("Kimi K3 · Lesson 3 of 14", CHUNKWISE diagram; "The mapping that changed"):
// per 64-token chunk with incoming state S, chunk-local cumulative log-decay b_r = sum_{i<=r} g_i
// (per key channel) and Gamma_r = e^{b_r},
//   Q^ = Gamma (.) (scale q)    K^ = Gamma (.) k    K- = (Gamma_C / Gamma) (.) k
//   A_ij = sum_c q_ic k_jc e^{b_ic - b_jc} (j <= i)   L_ij = beta_i sum_c k_ic k_jc e^{b_ic - b_jc} (j < i)
//   T' = (I + L)^-1 diag(beta),  W = T' K^,  U~ = T' V,  U = U~ - W S
//   O = Q^ S + A U  (the pages' "(Gamma (.) Q) S + A V~"),   S <- Diag(Gamma_C) S + K-^T U,
//   out = sigmoid(gate) (.) O.
// Every chunk is dense tensor-core work; only S crosses chunk boundaries.
//
// The 1/Gamma rescale on 16-token tiles ("each key rescaled by the reciprocal of its accumulated
// decay"): with r_p = b just before tile p, a token i of tile p carries the row factor
// f_i = e^{b_i - r_p} in [e^-80, 1] (the g >= -5 floor caps a tile's decay at 80) and the key
// factor 1/f_i in [1, e^80].  Gram block (p, q <= p) is sum_c (q_ic f_ic)(k_jc e^{r_p,c - b_jc}):
//   - diagonal blocks (q = p): the key factor reaches e^80, beyond fp16, so these 16 x 16 x d_k
//     products run on mma.sync m16n8k8 in tf32 (fp32 range, 11-bit significand), straight from the
//     registers of the threads that computed the factors;
//   - blocks below the diagonal: both factors are <= 1 and a factor that underflows belongs to a
//     term below e^-87, so fp16 operands lose nothing: one tcgen05 MMA (M = 128: the row-scaled
//     q and k rows of the four tiles, N = 96 rescaled keys, K = d_k) computes all of them.
// Everything on the value path (T', K^, V, W, Q^, K-, A, S, U) is fp16 with fp32 accumulation; U
// and A, whose rounding shows most in the largest outputs, enter the output product A U as an fp16
// value plus its fp16 rounding remainder (about 22 significant bits).  The state's master copy is fp32
// in tensor memory.
//
// Work per chunk (one CTA, 16 warps, the phases separated by CTA barriers):
//   0. TMA: q, k, v, a rows of the chunk (3-d tensor maps over [T, H, d], two 64-channel boxes per
//      tensor, 128-byte swizzle), each issued as soon as its buffer is free; a is double buffered.
//   1. pass 1 (thread = 2 channels x 8 tokens): g = -5 sigmoid(e^{A_h} a) in log2 units, the
//      within-tile running sum l, tile totals; tables e^{r_p}, e^{b_C - r_p}, e^{r_p' - r_p}, Gamma_C.
//      Chunk c + 1's pass 1 runs during chunk c's steps 5, 7 and 9 (while the tensor cores work).
//   2. pass 2 (warp = tile x channel half, lane = the two rows and 16 channels an MMA fragment
//      holds): f = 2^l, 1/f; the diagonal Gram blocks (mma.sync tf32); fp16 row-scaled q, k rows into
//      TMEM (tcgen05.st 16x256b, the fragment layout); rescaled keys of later tiles (fp16) into shared
//      memory; Q^, K^, K-, V converted in place over the input rows.
//   3. off-diagonal Gram MMA; meanwhile the fp16 copy of the state is written (B operand of step 7)
//      and the state scaled by Gamma_C in TMEM.
//   4. solve: 16 x 16 diagonal inverses by forward substitution, off-diagonal blocks of T' level by
//      level (mma.sync); A assembled from the diagonal and off-diagonal Gram blocks.
//   5. D[0:64] = [T'; 0] [K^ | V] = [W | U~]                         (tcgen05, N = 256, K = 64)
//   6. -W -> TMEM, beside Q^ (rows 64-127)
//   7. D[:, 128:256] += [-W; Q^] S   -> rows 0-63 U, rows 64-127 Q^ S  (tcgen05, A in TMEM)
//   8. U -> shared memory (fp16 value and remainder); its TMEM rows zeroed
//   9. S += K-^T U  (S pre-scaled by Gamma_C);  D[:, 128:256] += [A_hi; A_lo] U -> O in two parts
//  10. out = sigmoid(gate) O (gate logits read from global memory during step 9), staged in shared
//      memory, stored by TMA (row by row for a sequence's last chunk).
// Every wait on a TMA or MMA completion is bounded (%globaltimer); a timeout records kErrTimeout in
// the device error word and every thread leaves the chunk loop at the next barrier.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "mma_frag.cuh"
#include "gate_sigmoid.cuh"
#include "umma.cuh"

namespace kda {
namespace tc {

constexpr int kThreads = 512;
constexpr int kRankMax = 128;      // batches of at most this many sequences run longest first
constexpr int kMmaWarp = 6;        // tile 2 (pass 2), channel quarter 1 (Gram step), idle in the solve
constexpr int kTmaWarp = 10;       // tile 2 (pass 2), channel quarter 2 (Gram step), idle in the solve
constexpr int kD = 128;            // d_k = d_v of this kernel
constexpr float kLog2e = 1.4426950408889634f;

// ---- shared memory map (bytes; every operand tile 1024-aligned) ----------------------------------
constexpr int kQ = 0;              // q -> Q^            SW128 [2 atoms][64 rows][128 B]
constexpr int kK = 16384;          // k -> K^            ] together the B operand [K^ | V]
constexpr int kV = 32768;          // v -> V (fp16)      ]   (four 64-channel atoms, 8 KB apart)
constexpr int kA0 = 49152;         // a of even chunks -> K- (A operand of K-^T U, MN-major)
constexpr int kA1 = 65536;         // a of odd chunks  -> K-
constexpr int kLT0 = 81920;        // fp32 l table, rows 0-31 (16 KB): pass 1 -> pass 2
constexpr int kL = 98304;          // U (fp16, 16 KB) and A'' (16 KB); then the output staging
constexpr int kGB = 131072;        // fp16 rescaled keys of later tiles: K-major, no swizzle, 96 rows
constexpr int kT = kGB;            // T'' (after the Gram): SW128 [128][64], rows in slot order (below);
                                   //   after [W | U~], the remainder U - fp16(U) (B operand like U)
constexpr int kUlo = kGB;
constexpr int kAm = kL + 16384;    // A'' (after pass 2): SW128 [128][64]: fp16 A in the query slots, the
                                   //   remainder A - fp16(A) in the key slots
constexpr int kS = 155648;         // fp16 S: B operand, MN-major, no swizzle (K = d_k, N = d_v)
constexpr int kLD = 188416;        // fp16 [64][64] swizzled: -L below the diagonal blocks, D_p on them;
                                   //   before that rows 32-63 of the l table
constexpr int kLT1 = kLD;          // fp32 l table, rows 32-63 (16 KB, up to kLdf)
constexpr int kLdf = 204800;       // fp32 [4][16][17] diagonal blocks of L
constexpr int kTot = kLdf + 4 * 16 * 17 * 4;   // fp32 [8][128] half-tile totals of l
constexpr int kTE = kTot + 4096;   // fp32 [4][128] 2^{r_p}
constexpr int kTK = kTE + 2048;    // fp32 [4][128] 2^{b_C - r_p}
constexpr int kTD = kTK + 2048;    // fp32 [6][128] 2^{r_p' - r_p}, p < p'
constexpr int kGam = kTD + 3072;   // fp32 [128] Gamma_C
constexpr int kBeta = kGam + 512;  // fp32 [64]
constexpr int kBar = kBeta + 256;  // u64 mbarriers: q, kv, a0, a1, gate, mma
constexpr int kMisc = kBar + 64;   // u32 TMEM base, int abort flag
constexpr int kSmemBytes = kMisc + 16;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(kGB + 3 * 8192 <= kS && kGB + 96 * 256 <= kS, "GB region");

// ---- slot order of the 128 rows of the chunk's accumulators ---------------------------------------
// Token row i of the chunk (tile p = i / 16, r = i % 16) has two rows: its query slot 32 p + r
// (row-scaled q in the Gram, Q^ in the state products, the output O) and its key slot
// 32 p + 16 + r (row-scaled k in the Gram, then W, U~, U).  Every TMEM lane quadrant thus holds
// both slots of one tile, so the work on either kind of row is shared by all four schedulers.
__host__ __device__ constexpr int qslot(int i) { return 32 * (i >> 4) + (i & 15); }
__host__ __device__ constexpr int kslot(int i) { return 32 * (i >> 4) + 16 + (i & 15); }

// ---- value-channel order of every N = d_v operand and accumulator (V, U~, U, S, O) ---------------
// Within each block of 32 value channels, column n = 8b + 2t + e (b, t < 4, e < 2) holds channel
// 8t + 2b + e.  A 16x256b TMEM load gives lane (g, t) the columns 8b + 2t + e, b = 0..3: eight
// consecutive channels 8t .. 8t + 7, so the gate is read and the output written 16 bytes at a time.
__host__ __device__ constexpr int vperm(int n) { return 8 * ((n >> 1) & 3) + 2 * ((n >> 3) & 3) + (n & 1); }

// ---- tensor memory columns -----------------------------------------------------------------------
constexpr uint32_t cWU = 0;        // [W | U~] -> [. | U] (key slots), [. | O] (query slots); 256 columns
constexpr uint32_t cGA = 0;        // fp16 row-scaled rows (A operand of the off-diagonal Gram), 64 cols
constexpr uint32_t cGD = 64;       // off-diagonal Gram (fp32), 96 columns
constexpr uint32_t cS = 256;       // fp32 state (128 columns)
constexpr uint32_t cWQ = 384;      // fp16 -W (key slots) and Q^ (query slots), A operand of W S, Q^ S

// order of the off-diagonal key rows: tile p' uses rows off(p') .. off(p') + 16 p' - 1
__host__ __device__ constexpr int gb_off(int pp) { return pp == 1 ? 0 : pp == 2 ? 16 : 48; }
__host__ __device__ constexpr int td_index(int p, int pp) { return p == 0 ? pp - 1 : p == 1 ? pp + 1 : 5; }

struct Params {
    const uint16_t *gate;            // [T, H, 128] bf16 gate logits, or null
    const float *beta, *A_log;
    const int32_t *cu;
    const float *S_in;
    float *S_out;
    void *out;
    int64_t total_tokens;
    int num_seqs, H;
    int max_seqlen;
    float scale;
    bool out_f32, has_gate;
    unsigned long long wait_ns;
};

struct Maps {
    CUtensorMap q, k, v, a;
    CUtensorMap out;   // [T, H, 128] output: bf16 boxes of 64 channels, or fp32 boxes of 32 channels
};

// ---- small PTX helpers ---------------------------------------------------------------------------
__device__ __forceinline__ bool elect_one() {
    uint32_t p;
    asm volatile("{\n.reg .pred P;\nelect.sync _|P, 0xffffffff;\nselp.u32 %0, 1, 0, P;\n}\n" : "=r"(p));
    return p != 0;
}

__device__ __forceinline__ unsigned long long gtimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, unsigned long long ns) {
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = gtimer();
    while (!mbar_try(bar, parity))
        if (gtimer() - t0 > ns) return false;
    return true;
}

__device__ __forceinline__ void expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}

// one 64-channel x 64-token box of a [T, H, d] tensor (x = channel offset, 0 or 64)
__device__ __forceinline__ void tma_box(uint32_t dst, const CUtensorMap *map, int x, int h, int t, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(h), "r"(t), "r"(bar)
        : "memory");
}

// one box of the staged output tile -> global (bulk-group completion)
__device__ __forceinline__ void tma_store_box(const CUtensorMap *map, uint32_t src, int x, int h, int t) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];\n" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(x), "r"(h), "r"(t)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
// the shared-memory source of every committed store has been read / every store is complete
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory"); }

__device__ __forceinline__ void prefetch_map(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;\n" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_tf32(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// tcgen05.st 16x256b: lane (g, t) of the warp writes TMEM lanes base + g (r0, r1) and base + g + 8
// (r2, r3), columns 2t and 2t + 1 of the 8-column block at taddr -- the m16n8 fragment layout.
__device__ __forceinline__ void tmem_st_frag(uint32_t taddr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("tcgen05.st.sync.aligned.16x256b.x1.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(taddr), "r"(r0), "r"(r1), "r"(r2),
                 "r"(r3)
                 : "memory");
}

// tcgen05.ld / st 16x256b.x4: lane (g, t) of the warp holds TMEM lanes base + g (v[4b], v[4b + 1]) and
// base + g + 8 (v[4b + 2], v[4b + 3]), columns 8b + 2t and 8b + 2t + 1, b = 0..3
__device__ __forceinline__ void tmem_ld_frag4(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
          "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st_frag4(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// tcgen05.mma kind::f16 with both operands in shared memory, or A in tensor memory
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile("{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
                 "l"(a), "l"(b), "r"(idesc), "r"(acc)
                 : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile("{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
                 "r"(a), "l"(b), "r"(idesc), "r"(acc)
                 : "memory");
}

// shared-memory matrix descriptor: no swizzle (layout 0) or 128-byte swizzle (layout 2)
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}
// instruction descriptor, kind::f16: fp16 A and B, fp32 D, A/B major (0 = K, 1 = MN)
__host__ __device__ constexpr uint32_t idesc(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// byte offset of element (row, col) of a [rows][64]-element SW128 tile (2-byte elements)
__device__ __forceinline__ uint32_t sw128(int row, int col) {
    return row * 128 + ((((col >> 3) ^ row) & 7) << 4) + ((col & 7) << 1);
}
// element (token i, channel c) of a TMA-loaded [2 atoms][64][64] tile (also the bf16 output staging)
__device__ __forceinline__ uint32_t in_off(int i, int c) { return (c >> 6) * 8192 + sw128(i, c & 63); }
// element (token i, channel c) of the fp32 output staging: [4 atoms of 32 channels][64][128 B], SW128
__device__ __forceinline__ uint32_t out_off_f32(int i, int c) {
    return (c >> 5) * 8192 + i * 128 + ((((c >> 2) & 7) ^ (i & 7)) << 4) + ((c & 3) << 2);
}
// byte offset of element (k, n) of an MN-major, no-swizzle fp16 B operand with N = 128
__device__ __forceinline__ uint32_t bmn_off(int k, int n) { return (((k >> 3) * 16 + (n >> 3)) << 7) + ((k & 7) << 4) + ((n & 7) << 1); }
// fp32 l table [64][128] with its 16-byte chunks XOR-ed by 4 (row & 1): conflict-free for both passes;
// rows 0-31 at kLT0, rows 32-63 at kLT1
__device__ __forceinline__ uint32_t l_off(int i, int c) { return i * 512 + ((((c >> 2) ^ ((i & 1) << 2))) << 4) + ((c & 3) << 2); }
__device__ __forceinline__ uint32_t lt_addr(int i, int c) { return (i < 32 ? kLT0 : kLT1 - 32 * 512) + l_off(i, c); }

__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts32(uint32_t a, uint32_t v) { asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(a), "r"(v)); }
__device__ __forceinline__ void sts64(uint32_t a, uint32_t x, uint32_t y) {
    asm volatile("st.shared.v2.b32 [%0], {%1,%2};\n" ::"r"(a), "r"(x), "r"(y));
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w));
}

__device__ __forceinline__ void bar_all() { named_bar(1, kThreads); }

// ---------------------------------------------------------------------------------------------
// The solve: T' = (I + L)^-1 diag(beta), given the diagonal inverses D_p = (I + L_pp)^-1 (fp16, on
// the diagonal blocks of LD), T'_pp = D_p diag(beta_p) (on those of T') and the fp16 blocks -L_pm
// (m < p) in LD:  T'_pq = D_p sum_{m=q}^{p-1} (-L_pm) T'_mq  for p = q + 1, q + 2, ... as 16 x 16
// products; starting from D_q diag(beta_q) yields T' directly.  Column block q of T' needs only
// column block q, so warp (q, half) computes its 8 columns of blocks (q + 1, q) .. (3, q) in turn
// with no barrier.  The chain stays in registers: every -L_pm and D_p fragment is loaded up front,
// and a product's accumulator (rows g, g + 8, columns 2 t4, 2 t4 + 1) becomes the B fragment of the
// next product (rows 2 t4, 2 t4 + 1, column g) by an 8 x 8 register transpose.  T' is an SW128
// [64][64] tile (the MMA's A operand); its rows are the key slots of a 128-row tile whose query
// slots are zero.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x2_t(uint32_t (&r)[2], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n" : "=r"(r[0]), "=r"(r[1]) : "r"(addr));
}

__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
    return y;
}

template <int QB>
__device__ __forceinline__ void solve_column(uint32_t base, int half, int lane) {
    constexpr int NP = 3 - QB;   // blocks below the diagonal in column block QB
    const int g = lane >> 2, t4 = lane & 3;
    uint32_t lf[NP][NP][4], df[NP][4];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int pb = QB + 1 + p;
#pragma unroll
        for (int m = 0; m <= p; ++m) ldsm_x4(lf[p][m], ldsm_addr_a<128>(base + kLD, 16 * pb, 16 * (QB + m), lane));   // -L_pm
        ldsm_x4(df[p], ldsm_addr_a<128>(base + kLD, 16 * pb, 16 * pb, lane));                                          // D_p
    }
    uint32_t tf[NP + 1][2];   // B fragments of T'_mq, m = QB .. 3 (this warp's 8 columns)
    ldsm_x2_t(tf[0], base + kT + swz<128>(32 * QB + 16 + (lane & 15), 2 * QB + half));
    const int cc = 16 * QB + 8 * half + 2 * t4;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int pb = QB + 1 + p;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int m = 0; m <= p; ++m) mma_f16(acc, lf[p][m], tf[m][0], tf[m][1]);
        float tq[4] = {0.f, 0.f, 0.f, 0.f};
        mma_f16(tq, df[p], transpose8x8(pack_f16(acc[0], acc[1])), transpose8x8(pack_f16(acc[2], acc[3])));
        const uint32_t t0 = pack_f16(tq[0], tq[1]), t1 = pack_f16(tq[2], tq[3]);
        sts32(base + kT + sw128(32 * pb + 16 + g, cc), t0);
        sts32(base + kT + sw128(32 * pb + 24 + g, cc), t1);
        if (p + 1 < NP) {
            tf[p + 1][0] = transpose8x8(t0);
            tf[p + 1][1] = transpose8x8(t1);
        }
    }
}

__device__ __forceinline__ void solve(unsigned char *sm, int warp, int lane) {
    const uint32_t base = smem_u32(sm);
    const int half = warp & 1;
    switch (warp >> 1) {
        case 0: solve_column<0>(base, half, lane); break;
        case 1: solve_column<1>(base, half, lane); break;
        case 2: solve_column<2>(base, half, lane); break;
        default: break;
    }
}

__global__ void __launch_bounds__(kThreads, 1) kda_prefill_tc_kernel(const __grid_constant__ Maps maps, const Params p) {
    extern __shared__ __align__(1024) unsigned char sm[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Units in order of decreasing sequence length (ties by index) when the batch is small enough to
    // rank here: blocks start in index order, so the longest units start first and the last wave
    // holds the shortest.  Larger batches keep the packed order.
    const int h = blockIdx.x % p.H;
    int n = blockIdx.x / p.H;
    if (p.num_seqs <= kRankMax) {
        int64_t *len = reinterpret_cast<int64_t *>(sm + kL);
        int *pick = reinterpret_cast<int *>(sm + kL + 8 * kRankMax);
        if (tid < p.num_seqs) len[tid] = (int64_t)__ldg(p.cu + tid + 1) - __ldg(p.cu + tid);
        __syncthreads();
        if (tid < p.num_seqs) {
            const int64_t li = len[tid];
            int r = 0;
            for (int j = 0; j < p.num_seqs; ++j) r += (len[j] > li) || (len[j] == li && j < tid);
            if (r == n) *pick = tid;
        }
        __syncthreads();
        n = *pick;
    }
    const uint32_t base = smem_u32(sm);
    const uint32_t bQ = base + kBar, bKV = bQ + 8, bA0 = bQ + 16, bA1 = bQ + 24, bMma = bQ + 40;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kMisc + 4);

    int64_t s0, s1;
    const bool well_formed = seq_span(p.cu, n, p.num_seqs, p.total_tokens, s0, s1);
    if (h == 0 && tid == 0) {
        if (!well_formed) atomicOr(&g_kda_error_word, kErrBadSeqlens);
        if (p.max_seqlen > 0 && s1 - s0 > p.max_seqlen) atomicOr(&g_kda_error_word, kErrSeqTooLong);
    }
    const int nchunks = static_cast<int>((s1 - s0 + kChunk - 1) / kChunk);

    if (tid == 0) {
        for (int i = 0; i < 6; ++i) mbar_init(bQ + 8 * i, 1);
        *abort_flag = 0;
        prefetch_map(&maps.q); prefetch_map(&maps.k); prefetch_map(&maps.v); prefetch_map(&maps.a); prefetch_map(&maps.out);
    }
    if (warp == 0) tmem_alloc(base + kMisc, 512);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + kMisc);

    const float expA = expf(p.A_log[h]);
    const int64_t H = p.H;
    float *sbeta = reinterpret_cast<float *>(sm + kBeta);
    // One elected lane of warp kMmaWarp issues (and waits for) the tensor-core products, one of warp
    // kTmaWarp the TMA copies: warps with the least work of their own in pass 2, the Gram step and
    // the solve, so that the serial issue does not hold up a CTA barrier.
    const bool mma_lead = warp == kMmaWarp && elect_one();
    const bool tma_lead = warp == kTmaWarp && elect_one();
    uint32_t pend = 0, pend_par = 0;   // tma_lead only: loads in flight per barrier (q, kv, a0, a1) and their wait parity
    auto issued = [&](int i, uint32_t parity) { pend |= 1u << i; pend_par = (pend_par & ~(1u << i)) | (parity << i); };
    auto load_pair = [&](const CUtensorMap *map, uint32_t dst, uint32_t bar, int cl) {
        const int t = static_cast<int>(s0 + (int64_t)cl * kChunk);
        tma_box(dst, map, 0, h, t, bar);
        tma_box(dst + 8192, map, 64, h, t, bar);
    };
    if (tma_lead && nchunks > 0) {
        expect_tx(bA0, 16384); load_pair(&maps.a, base + kA0, bA0, 0); issued(2, 0);
        expect_tx(bQ, 16384); load_pair(&maps.q, base + kQ, bQ, 0); issued(0, 0);
        expect_tx(bKV, 32768); load_pair(&maps.k, base + kK, bKV, 0); load_pair(&maps.v, base + kV, bKV, 0); issued(1, 0);
    }
    auto load_beta = [&](int cl) -> float {
        if (tid >= 64 || cl >= nchunks) return 0.f;
        const int64_t tl = s0 + (int64_t)cl * kChunk;
        return tid < s1 - tl ? __ldg(p.beta + (tl + tid) * H + h) : 0.f;
    };
    float beta_next = load_beta(0);

    // epilogue mapping: TMEM lane quadrant q4 = warp % 4 (rows 32 q4 + lane), column quarter
    // cq = warp / 4 (columns 32 cq .. 32 cq + 31 of a 128-column matrix)
    const int q4 = warp & 3, cq = warp >> 2, row = 32 * q4 + lane;
    const uint32_t tq = tmem + ((uint32_t)(32 * q4) << 16);

    // initial state -> TMEM (fp32; step 3 writes its fp16 copy)
    {
        const size_t st_base = ((size_t)n * H + h) * kD * kD;
        float x[32];
        if (p.S_in) {
            const float4 *sp = reinterpret_cast<const float4 *>(p.S_in + st_base + (size_t)row * kD + 32 * cq);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 v = __ldg(sp + j);
                x[4 * j] = v.x; x[4 * j + 1] = v.y; x[4 * j + 2] = v.z; x[4 * j + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] = 0.f;
        }
        float xp[32];   // in the column order of the value channels
#pragma unroll
        for (int j = 0; j < 32; ++j) xp[j] = x[vperm(j)];
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            uint32_t v[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(xp[16 * part + e]);
            tmem_st16(tq + cS + 32 * cq + 16 * part, v);
        }
        tmem_wait_st();
    }

    uint32_t mma_phase = 0;
    auto mma_wait = [&]() {   // the issuing thread waits for the latest commit (bounded); the CTA
                              // barrier that follows every call releases the others
        if (mma_lead && !wait_bounded(bMma, mma_phase, p.wait_ns)) {
            atomicOr(&g_kda_error_word, kErrTimeout);
            *abort_flag = 1;
        }
        mma_phase ^= 1;
    };
    auto mma_sync = [&]() {   // ... then a CTA barrier, after which the flag is read by everyone
        mma_wait();
        tc_fence_before();
        bar_all();
        tc_fence_after();
    };
    auto in_wait = [&](uint32_t bar, uint32_t parity) {
        if (!wait_bounded(bar, parity, p.wait_ns)) { atomicOr(&g_kda_error_word, kErrTimeout); *abort_flag = 1; }
        else pend &= ~(1u << ((bar - bQ) >> 3));
    };
    auto sync_tc = [&]() {   // shared-memory and TMEM writes visible to the tensor core and all threads
        fence_async_smem();
        tmem_wait_st();
        tc_fence_before();
        bar_all();
        tc_fence_after();
    };
    // 32 consecutive fp32 TMEM columns of this thread's lane
    auto tld32 = [&](uint32_t taddr, uint32_t (&v)[32]) {
        uint32_t a[16], b[16];
        tmem_ld16(taddr, a);
        tmem_ld16(taddr + 16, b);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) { v[e] = a[e]; v[16 + e] = b[e]; }
    };
    // 32 fp32 values as fp16 into row k of an MN-major B operand (columns 32 cb ..)
    auto store_b32 = [&](uint32_t region, int k, int cb, const uint32_t (&v)[32]) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            sts128(region + bmn_off(k, 32 * cb + 8 * j),
                   make_uint4(pack_f16(__uint_as_float(v[8 * j]), __uint_as_float(v[8 * j + 1])),
                              pack_f16(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3])),
                              pack_f16(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5])),
                              pack_f16(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7]))));
    };

    // ---- 1. pass 1 of chunk cl, in two halves with a CTA barrier between them -----------------------
    //      thread = channel pair cp (channels 2cp, 2cp + 1) x half tile part (8 tokens).
    //      (a) g = -5 sigmoid(e^{A_h} a) in log2 units and the running sum over the part's 8 tokens;
    //          part totals to shared memory;  (b) the within-tile running sums l (the l table) and
    //      the tables of the tile references.  Chunk 0's pass 1 runs before the chunk loop; that of
    //      chunk c + 1 runs inside chunk c, while the tensor cores work on chunk c's products.
    const int p1_cp = tid & 63, p1_part = tid >> 6, p1_pt = p1_part >> 1, p1_c0 = 2 * p1_cp;
    float p1_lx[8], p1_ly[8], p1_sx = 0.f, p1_sy = 0.f;
    // (a) in two halves of four tokens (half 0 waits for the a tile), so that each half fits under
    // one tensor-core step
    auto pass1a = [&](int cl, int half) {
        const int64_t tl = s0 + (int64_t)cl * kChunk;
        const int Ll = static_cast<int>(min64(kChunk, s1 - tl));
        const uint32_t ab = (cl & 1) ? base + kA1 : base + kA0;
        if (half == 0) {
            in_wait((cl & 1) ? bA1 : bA0, (cl >> 1) & 1);
            p1_sx = p1_sy = 0.f;
        }
        constexpr float kG2 = kGMin * kLog2e;
#pragma unroll
        for (int i = 4 * half; i < 4 * half + 4; ++i) {
            const int t = 8 * p1_part + i;
            const float2 av = unpack_bf16(lds32(ab + in_off(t, p1_c0)));
            float gx = kG2 * sigmoid_fast(expA * av.x), gy = kG2 * sigmoid_fast(expA * av.y);
            if (t >= Ll) gx = gy = 0.f;
            p1_sx += gx; p1_sy += gy;
            p1_lx[i] = p1_sx; p1_ly[i] = p1_sy;
        }
        if (half == 1) {
            float *tot = reinterpret_cast<float *>(sm + kTot);   // [8 half tiles][128]
            *reinterpret_cast<float2 *>(tot + p1_part * 128 + p1_c0) = make_float2(p1_sx, p1_sy);
        }
    };
    auto pass1b = [&]() {
        const float *tot = reinterpret_cast<const float *>(sm + kTot);
        const int part = p1_part, pt = p1_pt, c0 = p1_c0;
        // within-tile running sum: the second half adds the first half's total
        const float2 off = (part & 1) ? *reinterpret_cast<const float2 *>(tot + (part - 1) * 128 + c0) : make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int t = 8 * part + i;
            *reinterpret_cast<float2 *>(sm + lt_addr(t, c0)) = make_float2(p1_lx[i] + off.x, p1_ly[i] + off.y);
        }
        if ((part & 1) == 0) {   // tables of tile pt, once per channel pair
            float2 T4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 x0 = *reinterpret_cast<const float2 *>(tot + (2 * q) * 128 + c0);
                const float2 x1 = *reinterpret_cast<const float2 *>(tot + (2 * q + 1) * 128 + c0);
                T4[q] = make_float2(x0.x + x1.x, x0.y + x1.y);
            }
            float2 R = make_float2(0.f, 0.f), BC = R;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (q < pt) { R.x += T4[q].x; R.y += T4[q].y; }
                BC.x += T4[q].x; BC.y += T4[q].y;
            }
            *reinterpret_cast<float2 *>(sm + kTE + (pt * 128 + c0) * 4) = make_float2(ex2(R.x), ex2(R.y));
            *reinterpret_cast<float2 *>(sm + kTK + (pt * 128 + c0) * 4) = make_float2(ex2(BC.x - R.x), ex2(BC.y - R.y));
            float2 Rn = R;
#pragma unroll
            for (int pp = 1; pp < 4; ++pp) {
                if (pp <= pt) continue;
                Rn.x += T4[pp - 1].x; Rn.y += T4[pp - 1].y;
                *reinterpret_cast<float2 *>(sm + kTD + (td_index(pt, pp) * 128 + c0) * 4) =
                    make_float2(ex2(Rn.x - R.x), ex2(Rn.y - R.y));
            }
            if (pt == 0) *reinterpret_cast<float2 *>(sm + kGam + c0 * 4) = make_float2(ex2(BC.x), ex2(BC.y));
        }
    };
    if (nchunks > 0) {
        pass1a(0, 0);
        pass1a(0, 1);
        bar_all();
        pass1b();
    }

    for (int c = 0; c < nchunks; ++c) {
        const int64_t t0 = s0 + (int64_t)c * kChunk;
        const int L = static_cast<int>(min64(kChunk, s1 - t0));
        const uint32_t aBuf = (c & 1) ? base + kA1 : base + kA0;
        if (tid < 64) sbeta[tid] = beta_next;
        beta_next = load_beta(c + 1);
        // the next chunk's a goes into the other buffer (its K- of chunk c-1 is consumed)
        if (tma_lead && c + 1 < nchunks) {
            const uint32_t nb = (c & 1) ? base + kA0 : base + kA1, nbar = (c & 1) ? bA0 : bA1;
            expect_tx(nbar, 16384);
            load_pair(&maps.a, nb, nbar, c + 1);
            issued((c & 1) ? 2 : 3, ((c + 1) >> 1) & 1);
        }
        in_wait(bQ, c & 1);
        in_wait(bKV, c & 1);
        if (tma_lead) bulk_wait_read();   // the previous chunk's output stores have read the staging area
        bar_all();
        if (*abort_flag) break;

        // ---- 2. pass 2: operands and the diagonal Gram blocks -------------------------------------
        //      warp = tile pt x channel quarter cq; lane (g, t4) = rows g, g + 8 of the tile and the
        //      channels 32 cq + 16 s + 4 t4 .. + 3 (s = 0, 1), the layout of the MMA fragments
        float qk[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        float kk[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const int pt = warp & 3;                        // tile (= TMEM lane quadrant of this warp)
        const int g = lane >> 2, t4 = lane & 3;
        {
            const int i0 = 16 * pt + g, i1 = i0 + 8;
            const bool in0 = i0 < L, in1 = i1 < L, partial = L < kChunk;
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const int cb = 32 * cq + 16 * s + 4 * t4;     // this lane's 4 channels cb .. cb + 3
                // rows i0 and i1 = i0 + 8 share their low three bits: row i1 is 8 rows (1 KB of a
                // swizzled input tile, 4 KB of the l table) after row i0
                const uint32_t oq0 = in_off(i0, cb), oq1 = oq0 + 1024;
                uint2 qr0 = lds64(base + kQ + oq0), qr1 = lds64(base + kQ + oq1);
                uint2 kr0 = lds64(base + kK + oq0), kr1 = lds64(base + kK + oq1);
                const uint32_t ol0 = lt_addr(i0, cb);   // rows i0 and i0 + 8 lie in the same half
                const float4 l0 = *reinterpret_cast<const float4 *>(sm + ol0);
                const float4 l1 = *reinterpret_cast<const float4 *>(sm + ol0 + 4096);
                const float4 te = *reinterpret_cast<const float4 *>(sm + kTE + (pt * 128 + cb) * 4);
                const float4 tk = *reinterpret_cast<const float4 *>(sm + kTK + (pt * 128 + cb) * 4);
                float qv[2][4], kv[2][4], lv[2][4];
                {
                    const float2 a0 = unpack_bf16(qr0.x), a1 = unpack_bf16(qr0.y), b0 = unpack_bf16(qr1.x), b1 = unpack_bf16(qr1.y);
                    qv[0][0] = a0.x; qv[0][1] = a0.y; qv[0][2] = a1.x; qv[0][3] = a1.y;
                    qv[1][0] = b0.x; qv[1][1] = b0.y; qv[1][2] = b1.x; qv[1][3] = b1.y;
                    const float2 c0 = unpack_bf16(kr0.x), c1 = unpack_bf16(kr0.y), d0 = unpack_bf16(kr1.x), d1 = unpack_bf16(kr1.y);
                    kv[0][0] = c0.x; kv[0][1] = c0.y; kv[0][2] = c1.x; kv[0][3] = c1.y;
                    kv[1][0] = d0.x; kv[1][1] = d0.y; kv[1][2] = d1.x; kv[1][3] = d1.y;
                    lv[0][0] = l0.x; lv[0][1] = l0.y; lv[0][2] = l0.z; lv[0][3] = l0.w;
                    lv[1][0] = l1.x; lv[1][1] = l1.y; lv[1][2] = l1.z; lv[1][3] = l1.w;
                }
                if (partial) {   // rows past the sequence's end are zero (warp-uniform branch)
                    if (!in0) { qv[0][0] = qv[0][1] = qv[0][2] = qv[0][3] = 0.f; kv[0][0] = kv[0][1] = kv[0][2] = kv[0][3] = 0.f; }
                    if (!in1) { qv[1][0] = qv[1][1] = qv[1][2] = qv[1][3] = 0.f; kv[1][0] = kv[1][1] = kv[1][2] = kv[1][3] = 0.f; }
                }
                const float tev[4] = {te.x, te.y, te.z, te.w}, tkv[4] = {tk.x, tk.y, tk.z, tk.w};
                float qr[2][4], kr[2][4], kt[2][4];   // row-scaled q, k (<= 1) and rescaled keys (>= 1)
#pragma unroll
                for (int r = 0; r < 2; ++r)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float f = ex2(lv[r][e]), fi = ex2(-lv[r][e]);
                        qr[r][e] = p.scale * qv[r][e] * f;
                        kr[r][e] = kv[r][e] * f;
                        kt[r][e] = kv[r][e] * fi;
                    }
                // diagonal Gram blocks, tf32: k-step u uses channels cb + 2u (slot t4) and cb + 2u + 1 (slot t4 + 4)
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int e0 = 2 * u, e1 = 2 * u + 1;
                    const uint32_t aq0 = to_tf32(qr[0][e0]), aq1 = to_tf32(qr[1][e0]), aq2 = to_tf32(qr[0][e1]), aq3 = to_tf32(qr[1][e1]);
                    const uint32_t ak0 = to_tf32(kr[0][e0]), ak1 = to_tf32(kr[1][e0]), ak2 = to_tf32(kr[0][e1]), ak3 = to_tf32(kr[1][e1]);
                    const uint32_t b00 = to_tf32(kt[0][e0]), b01 = to_tf32(kt[0][e1]), b10 = to_tf32(kt[1][e0]), b11 = to_tf32(kt[1][e1]);
                    mma_tf32(qk[0], aq0, aq1, aq2, aq3, b00, b01);
                    mma_tf32(qk[1], aq0, aq1, aq2, aq3, b10, b11);
                    mma_tf32(kk[0], ak0, ak1, ak2, ak3, b00, b01);
                    mma_tf32(kk[1], ak0, ak1, ak2, ak3, b10, b11);
                }
                // fp16 row-scaled q, k rows -> TMEM (Gram A operand; rows of tile pt: q at lanes 32pt..+15,
                // k at 32pt + 16..+31; column = channel pair)
                {
                    const uint32_t col = tmem + cGA + (uint32_t)(16 * cq + 8 * s);
                    tmem_st_frag(col + ((uint32_t)(32 * pt) << 16), pack_f16(qr[0][0], qr[0][1]), pack_f16(qr[0][2], qr[0][3]),
                                 pack_f16(qr[1][0], qr[1][1]), pack_f16(qr[1][2], qr[1][3]));
                    tmem_st_frag(col + ((uint32_t)(32 * pt + 16) << 16), pack_f16(kr[0][0], kr[0][1]), pack_f16(kr[0][2], kr[0][3]),
                                 pack_f16(kr[1][0], kr[1][1]), pack_f16(kr[1][2], kr[1][3]));
                }
                // rescaled keys for the later tiles' off-diagonal blocks: row gb_off(pp) + i
#pragma unroll
                for (int pp = 1; pp < 4; ++pp) {
                    if (pp <= pt) continue;
                    const float4 td = *reinterpret_cast<const float4 *>(sm + kTD + (td_index(pt, pp) * 128 + cb) * 4);
                    const float tdv[4] = {td.x, td.y, td.z, td.w};
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int nrow = gb_off(pp) + (r ? i1 : i0);
                        const uint32_t o = kGB + (nrow >> 3) * 2048 + (cb >> 3) * 128 + (nrow & 7) * 16 + (cb & 7) * 2;
                        sts64(base + o, pack_f16(kt[r][0] * tdv[0], kt[r][1] * tdv[1]), pack_f16(kt[r][2] * tdv[2], kt[r][3] * tdv[3]));
                    }
                }
                // Q^ = q^ e^{r_p} (above, into TMEM); in place: K^ = k^ e^{r_p}, V -> fp16; K- = K~ e^{b_C - r_p}
                // into the a buffer
                tmem_st_frag(tmem + cWQ + (uint32_t)(16 * cq + 8 * s) + ((uint32_t)(32 * pt) << 16),
                             pack_f16(qr[0][0] * tev[0], qr[0][1] * tev[1]), pack_f16(qr[0][2] * tev[2], qr[0][3] * tev[3]),
                             pack_f16(qr[1][0] * tev[0], qr[1][1] * tev[1]), pack_f16(qr[1][2] * tev[2], qr[1][3] * tev[3]));
                sts64(base + kK + oq0, pack_f16(kr[0][0] * tev[0], kr[0][1] * tev[1]), pack_f16(kr[0][2] * tev[2], kr[0][3] * tev[3]));
                sts64(base + kK + oq1, pack_f16(kr[1][0] * tev[0], kr[1][1] * tev[1]), pack_f16(kr[1][2] * tev[2], kr[1][3] * tev[3]));
                sts64(aBuf + oq0, pack_f16(kt[0][0] * tkv[0], kt[0][1] * tkv[1]), pack_f16(kt[0][2] * tkv[2], kt[0][3] * tkv[3]));
                sts64(aBuf + oq1, pack_f16(kt[1][0] * tkv[0], kt[1][1] * tkv[1]), pack_f16(kt[1][2] * tkv[2], kt[1][3] * tkv[3]));
            }
            // V -> fp16 in the value-channel column order (rows past the end -> 0), by the warps of
            // the last tile: they have no rescaled keys to write for later tiles, so this evens out the
            // schedulers' work.  Lane = rows lane and lane + 32 of channel block cq; output chunk b
            // (columns 8b .. 8b + 7) takes word b of each of the four source chunks.
            if (pt == 3) {
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int i = lane + 32 * rr;
                    uint4 src[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) src[j] = lds128(base + kV + in_off(i, 32 * cq + 8 * j));
                    if (partial && i >= L) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) src[j] = make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        const uint32_t w0 = b == 0 ? src[0].x : b == 1 ? src[0].y : b == 2 ? src[0].z : src[0].w;
                        const uint32_t w1 = b == 0 ? src[1].x : b == 1 ? src[1].y : b == 2 ? src[1].z : src[1].w;
                        const uint32_t w2 = b == 0 ? src[2].x : b == 1 ? src[2].y : b == 2 ? src[2].z : src[2].w;
                        const uint32_t w3 = b == 0 ? src[3].x : b == 1 ? src[3].y : b == 2 ? src[3].z : src[3].w;
                        sts128(base + kV + in_off(i, 32 * cq + 8 * b),
                               make_uint4(bf16x2_to_f16x2(w0), bf16x2_to_f16x2(w1), bf16x2_to_f16x2(w2), bf16x2_to_f16x2(w3)));
                    }
                }
            }
        }
        // the four channel quarters' diagonal partial sums: quarters 1-3 put theirs into the output
        // staging area (free from the end of the previous chunk to step 8), quarter 0 adds them in a
        // fixed order, (x0 + x2) + (x1 + x3)
        float *xch = reinterpret_cast<float *>(sm + kL);   // [3][4 tiles][16][32]
        if (cq >= 1) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                xch[(((cq - 1) * 4 + pt) * 16 + e) * 32 + lane] = qk[e >> 2][e & 3];
                xch[(((cq - 1) * 4 + pt) * 16 + 8 + e) * 32 + lane] = kk[e >> 2][e & 3];
            }
        }
        sync_tc();
        if (*abort_flag) break;

        // ---- 3. off-diagonal Gram (TMEM A rows x rescaled keys) ----------------------------------
        if (warp == kMmaWarp) {
            if (mma_lead) {
                constexpr uint32_t id = idesc(128, 96, 0, 0);
                const uint64_t dg = sdesc(base + kGB, 128, 2048, 0);
#pragma unroll
                for (int k = 0; k < kD / 16; ++k)
                    mma_ts(tmem + cGD, tmem + cGA + 8 * k, dg + 16 * k, id, k > 0);
                umma_commit(bMma);
            }
            __syncwarp();
        }
        // every thread is past pass 2: the q buffer is free for the next chunk's q
        if (tma_lead && c + 1 < nchunks) {
            expect_tx(bQ, 16384);
            load_pair(&maps.q, base + kQ, bQ, c + 1);
            issued(0, (c + 1) & 1);
        }
        if (cq == 0) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int i0 = ((0 * 4 + pt) * 16 + e) * 32 + lane, i1 = i0 + 4 * 16 * 32, i2 = i1 + 4 * 16 * 32;
                qk[e >> 2][e & 3] = (qk[e >> 2][e & 3] + xch[i1]) + (xch[i0] + xch[i2]);
                kk[e >> 2][e & 3] = (kk[e >> 2][e & 3] + xch[i1 + 256]) + (xch[i0 + 256] + xch[i2 + 256]);
            }
        }
        // meanwhile: the diagonal blocks of L (fp32) and their inverses D_p = (I + L_pp)^-1, by
        // column-oriented forward substitution, one column per lane of warp pt (kept in registers
        // until the Gram MMA has released the tiles they are written to);
        // S <- Gamma_C S (fp32, in TMEM)
        float dinv[16];
        if (cq == 0) {
            const float *sb = reinterpret_cast<const float *>(sm + kBeta);
            float *Ldp = reinterpret_cast<float *>(sm + kLdf) + pt * 16 * 17;
            const float bi0 = sb[16 * pt + g], bi1 = sb[16 * pt + g + 8];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int j = 8 * nt + 2 * t4, r0 = g, r1 = g + 8;
                Ldp[r0 * 17 + j] = j < r0 ? bi0 * kk[nt][0] : 0.f;
                Ldp[r0 * 17 + j + 1] = j + 1 < r0 ? bi0 * kk[nt][1] : 0.f;
                Ldp[r1 * 17 + j] = j < r1 ? bi1 * kk[nt][2] : 0.f;
                Ldp[r1 * 17 + j + 1] = j + 1 < r1 ? bi1 * kk[nt][3] : 0.f;
            }
            __syncwarp();
            const int mcol = lane & 15;
#pragma unroll
            for (int i = 0; i < 16; ++i) dinv[i] = i == mcol ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < 15; ++j)
#pragma unroll
                for (int i = j + 1; i < 16; ++i) dinv[i] = fmaf(-Ldp[i * 17 + j], dinv[j], dinv[i]);
            // D_p into its tile (free since pass 2); T'_pp = D_p diag(beta_p) in fp32 over L_pp, for
            // step 4 to round into T'' (the Gram product still reads the rescaled keys under T'')
            __syncwarp();
            if (lane < 16) {
                const float bcol = sb[16 * pt + lane];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    *reinterpret_cast<__half *>(sm + kLD + sw128(16 * pt + i, 16 * pt + lane)) = __float2half_rn(dinv[i]);
                    Ldp[i * 17 + lane] = dinv[i] * bcol;
                }
            }
        }
        // the state, 32 columns at a time: fp16 copy of S_c (the B operand of step 7), then
        // S <- Gamma_C S; quarter 1 also takes quarter 0's columns (those warps invert)
        if (cq != 0) {
            const float gam = reinterpret_cast<const float *>(sm + kGam)[row];
#pragma unroll 1
            for (int cb = cq == 1 ? 0 : cq; cb <= cq; ++cb) {
                uint32_t v[32];
                tld32(tq + cS + 32 * cb, v);
                store_b32(base + kS, row, cb, v);
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(gam * __uint_as_float(v[e]));
                uint32_t a[16], b[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) { a[e] = v[e]; b[e] = v[16 + e]; }
                tmem_st16(tq + cS + 32 * cb, a);
                tmem_st16(tq + cS + 32 * cb + 16, b);
            }
        }
        mma_wait();
        tmem_wait_st();
        tc_fence_before();
        bar_all();
        tc_fence_after();
        if (*abort_flag) break;

        // ---- 4. solve inputs: A rows (tile pt) and -L rows from the Gram, diagonal blocks ----------
        {
            const float *sb = reinterpret_cast<const float *>(sm + kBeta);
            // off-diagonal block blk (< pt) of tile pt's rows from TMEM: lanes 32pt + r (q rows: A and
            // its remainder) and 32pt + 16 + r (k rows: -L), all lanes of the warp
            auto offdiag = [&](int blk) {
                const int r = lane & 15;
                const bool krow = lane >= 16;
                const int i = 16 * pt + r;
                const float sg = krow ? -sb[i] : 1.f;
                uint32_t v[16];
                tmem_ld16(tmem + ((uint32_t)(32 * pt) << 16) + cGD + gb_off(pt) + 16 * blk, v);
                tmem_wait_ld();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float x0 = sg * __uint_as_float(v[8 * hh + 2 * e]), x1 = sg * __uint_as_float(v[8 * hh + 2 * e + 1]);
                        hi[e] = pack_f16(x0, x1);
                        const float2 hf = unpack_f16(hi[e]);
                        lo[e] = pack_f16(x0 - hf.x, x1 - hf.y);
                    }
                    if (krow) {
                        sts128(base + kLD + sw128(i, 16 * blk + 8 * hh), make_uint4(hi[0], hi[1], hi[2], hi[3]));
                    } else {
                        sts128(base + kAm + sw128(qslot(i), 16 * blk + 8 * hh), make_uint4(hi[0], hi[1], hi[2], hi[3]));
                        sts128(base + kAm + sw128(kslot(i), 16 * blk + 8 * hh), make_uint4(lo[0], lo[1], lo[2], lo[3]));
                    }
                }
            };
            const int split = (pt + 1) >> 1;   // quarter 1 takes blocks [0, split), quarter 0 the rest
            if (cq == 0) {
                // diagonal blocks of A from the fragments (j <= i): fp16 A in the query slots, the
                // rounding remainder A - fp16(A) (fp16) in the key slots
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int j = 8 * nt + 2 * t4;   // column within the tile
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int r = g + 8 * hh;
                        const float x0 = j <= r ? qk[nt][2 * hh] : 0.f, x1 = j + 1 <= r ? qk[nt][2 * hh + 1] : 0.f;
                        const uint32_t hi = pack_f16(x0, x1);
                        const float2 hf = unpack_f16(hi);
                        sts32(base + kAm + sw128(32 * pt + r, 16 * pt + j), hi);
                        sts32(base + kAm + sw128(32 * pt + 16 + r, 16 * pt + j), pack_f16(x0 - hf.x, x1 - hf.y));
                    }
                }
                for (int blk = split; blk < pt; ++blk) offdiag(blk);
            } else if (cq == 1) {
                for (int blk = 0; blk < split; ++blk) offdiag(blk);
                if (lane < 16) {   // A and its remainder: zeros right of the diagonal block
                    const int i = 16 * pt + lane;
                    for (int cc = 16 * (pt + 1); cc < 64; cc += 8) {
                        sts128(base + kAm + sw128(qslot(i), cc), make_uint4(0, 0, 0, 0));
                        sts128(base + kAm + sw128(kslot(i), cc), make_uint4(0, 0, 0, 0));
                    }
                }
            } else {
                // T'' (over the rescaled keys, consumed by the Gram): zero query slots (4 tiles x 16
                // rows x 8 chunks of 16 bytes) and zero blocks above the diagonal in the key slots,
                // (0, 1..3), (1, 2..3), (2, 3) (16 rows x 2 chunks each)
                for (int e = tid - 256; e < 512 + 192; e += 256) {
                    if (e < 512) {
                        sts128(base + kT + (32 * (e >> 7) + ((e >> 3) & 15)) * 128 + 16 * (e & 7), make_uint4(0, 0, 0, 0));
                    } else {
                        const int ub = (e - 512) >> 5, r = ((e - 512) >> 1) & 15, hh = e & 1;
                        const int pb = ub < 3 ? 0 : ub < 5 ? 1 : 2, qb = ub < 3 ? ub + 1 : ub < 5 ? ub - 1 : 3;
                        sts128(base + kT + sw128(32 * pb + 16 + r, 16 * qb + 8 * hh), make_uint4(0, 0, 0, 0));
                    }
                }
                // the diagonal blocks T'_pp (fp32 from step 3) rounded into their key slots
                const float *Ldf = reinterpret_cast<const float *>(sm + kLdf);
                for (int e = tid - 256; e < 4 * 256; e += 256) {
                    const int pb = e >> 8, i = (e >> 4) & 15, j = e & 15;
                    *reinterpret_cast<__half *>(sm + kT + sw128(kslot(16 * pb + i), 16 * pb + j)) =
                        __float2half_rn(Ldf[(pb * 16 + i) * 17 + j]);
                }
            }
        }
        bar_all();
        solve(sm, warp, lane);
        sync_tc();   // T' visible to the tensor core

        // ---- 5. [W | U~] = [T'; 0] [K^ | V] ---------------------------------------------------------
        if (warp == kMmaWarp) {
            if (mma_lead) {
                constexpr uint32_t id = idesc(128, 256, 0, 1);
                // descriptors advance along K by adding the 16-byte start offset (no carry: every
                // shared-memory address here is below 2^18)
                const uint64_t dt = sdesc(base + kT, 16, 1024, 2), dk = sdesc(base + kK, 8192, 1024, 2);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_ss(tmem + cWU, dt + 2 * k, dk + 128 * k, id, k > 0);
                umma_commit(bMma);
            }
            __syncwarp();
        }
        if (c + 1 < nchunks) pass1a(c + 1, 0);   // the next chunk's pass 1 (a), first four tokens
        mma_sync();
        if (*abort_flag) break;
        // ---- 6. -W -> TMEM rows 0-63 of [-W; Q^] ----------------------------------------------------
        {
            uint32_t v[32], w[16];
            tld32(tq + cWU + 32 * cq, v);
            tmem_ld16(tq + cWQ + 16 * cq, w);
            tmem_wait_ld();
            if (lane >= 16) {   // key slot: -W;  query slot: Q^ stays
#pragma unroll
                for (int e = 0; e < 16; ++e) w[e] = pack_f16(-__uint_as_float(v[2 * e]), -__uint_as_float(v[2 * e + 1]));
            }
            tmem_st16(tq + cWQ + 16 * cq, w);
        }
        sync_tc();
        // ---- 7. D[:, 128:256] += [-W; Q^] S --------------------------------------------------------
        if (warp == kMmaWarp) {
            if (mma_lead) {
                constexpr uint32_t id = idesc(128, 128, 0, 1);
                const uint64_t ds = sdesc(base + kS, 2048, 128, 0);
#pragma unroll
                for (int k = 0; k < kD / 16; ++k)
                    mma_ts(tmem + cWU + 128, tmem + cWQ + 8 * k, ds + 256 * k, id, 1);
                umma_commit(bMma);
            }
            __syncwarp();
        }
        // the k, v buffers were read by step 5 (complete): the next chunk's k, v
        if (tma_lead && c + 1 < nchunks) {
            expect_tx(bKV, 32768);
            load_pair(&maps.k, base + kK, bKV, c + 1);
            load_pair(&maps.v, base + kV, bKV, c + 1);
            issued(1, (c + 1) & 1);
        }
        if (c + 1 < nchunks) pass1a(c + 1, 1);   // the next chunk's pass 1 (a), last four tokens
        mma_sync();
        if (*abort_flag) break;
        // ---- 8. U (key slots) -> shared memory (fp16, MN-major B operand) ----------------------------
        //      as fp16 U plus its rounding remainder U - fp16(U) (into the T'' tile, free since step 5);
        //      lane (g, t4) holds tokens 16 q4 + g, + 8 and columns 32 cq + 8 b + 2 t4, + 1 (16x256b).
        //      The key slots are then zeroed: step 9 accumulates A_lo U there.
        {
            const uint32_t ta = tq + (16u << 16) + cWU + 128 + 32 * cq;
            uint32_t u16[16];
            tmem_ld_frag4(ta, u16);
            tmem_wait_ld();
            {
                uint32_t z[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) z[e] = 0u;
                tmem_st_frag4(ta, z);
            }
#pragma unroll
            for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const float x0 = __uint_as_float(u16[4 * b + 2 * rr]), x1 = __uint_as_float(u16[4 * b + 2 * rr + 1]);
                    const uint32_t hi = pack_f16(x0, x1);
                    const float2 hf = unpack_f16(hi);
                    const uint32_t o = bmn_off(16 * q4 + g + 8 * rr, 32 * cq + 8 * b + 2 * t4);
                    sts32(base + kL + o, hi);
                    sts32(base + kUlo + o, pack_f16(x0 - hf.x, x1 - hf.y));
                }
        }
        sync_tc();
        // ---- 9. S += K-^T U;  D[:, 128:256] += A'' U  (the query slots become O) ---------------------
        //      U and A each enter the output as fp16 value + fp16 remainder: A'' holds A_hi in the
        //      query slots and A_lo in the key slots, so A'' (U_hi + U_lo) leaves Q^ S + A_hi U in the
        //      query slots and A_lo U in the (zeroed) key slots; the epilogue adds the two (the
        //      state's K-^T U takes U_hi only: its rounding there does not show)
        if (warp == kMmaWarp) {
            if (mma_lead) {
                constexpr uint32_t id = idesc(128, 128, 1, 1), id2 = idesc(128, 128, 0, 1);
                const uint64_t da = sdesc(aBuf, 8192, 1024, 2), du = sdesc(base + kL, 2048, 128, 0);
                const uint64_t dm = sdesc(base + kAm, 16, 1024, 2), dl = sdesc(base + kUlo, 2048, 128, 0);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_ss(tmem + cS, da + 128 * k, du + 256 * k, id, 1);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_ss(tmem + cWU + 128, dm + 2 * k, du + 256 * k, id2, 1);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_ss(tmem + cWU + 128, dm + 2 * k, dl + 256 * k, id2, 1);
                umma_commit(bMma);
            }
            __syncwarp();
        }
        if (c + 1 < nchunks) pass1b();         // the next chunk's pass 1, second half
        // meanwhile: this thread's gate logits, tokens 16 q4 + g and + 8, channels 32 cq + 8 t4 .. + 7
        uint4 gpre[2];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int i = 16 * q4 + g + 8 * rr;
            gpre[rr] = (p.has_gate && i < L)
                ? __ldg(reinterpret_cast<const uint4 *>(p.gate + ((t0 + i) * H + h) * kD + 32 * cq + 8 * t4))
                : make_uint4(0, 0, 0, 0);
        }
        mma_sync();
        if (*abort_flag) break;
        // ---- 10. new S (fp16 copy); gated output rows -----------------------------------------------
        {
            // tokens 16 q4 + g and + 8 (lane (g, t4)), columns 32 cq + 8b + 2t4 + e = channels
            // 32 cq + 8 t4 + 2b + e: query slots (Q^ S + A_hi U) plus key slots (A_lo U)
            uint32_t oq[16], ok[16];
            tmem_ld_frag4(tq + cWU + 128 + 32 * cq, oq);
            tmem_ld_frag4(tq + (16u << 16) + cWU + 128 + 32 * cq, ok);
            tmem_wait_ld();
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int i = 16 * q4 + g + 8 * rr, cc = 32 * cq + 8 * t4;
                const uint32_t gw[4] = {gpre[rr].x, gpre[rr].y, gpre[rr].z, gpre[rr].w};
                float o[8];
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    o[2 * b] = __uint_as_float(oq[4 * b + 2 * rr]) + __uint_as_float(ok[4 * b + 2 * rr]);
                    o[2 * b + 1] = __uint_as_float(oq[4 * b + 2 * rr + 1]) + __uint_as_float(ok[4 * b + 2 * rr + 1]);
                    if (p.has_gate) {
                        const float2 sg = p.out_f32 ? gate_sigmoid2_f32(gw[b]) : gate_sigmoid2(gw[b]);
                        o[2 * b] *= sg.x;
                        o[2 * b + 1] *= sg.y;
                    }
                }
                if (p.out_f32) {
                    sts128(base + kL + out_off_f32(i, cc), make_uint4(__float_as_uint(o[0]), __float_as_uint(o[1]),
                                                                      __float_as_uint(o[2]), __float_as_uint(o[3])));
                    sts128(base + kL + out_off_f32(i, cc + 4), make_uint4(__float_as_uint(o[4]), __float_as_uint(o[5]),
                                                                          __float_as_uint(o[6]), __float_as_uint(o[7])));
                } else {
                    sts128(base + kL + in_off(i, cc), make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]),
                                                                 pack_bf16(o[4], o[5]), pack_bf16(o[6], o[7])));
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        bar_all();
        tc_fence_after();
        if (L == kChunk) {
            // a whole chunk: TMA stores of the staged tile (the staging area is next written in the
            // next chunk's pass 2, after the issuing thread has waited for these reads)
            if (tma_lead) {
                if (p.out_f32) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) tma_store_box(&maps.out, base + kL + 8192 * j, 32 * j, h, (int)t0);
                } else {
                    tma_store_box(&maps.out, base + kL, 0, h, (int)t0);
                    tma_store_box(&maps.out, base + kL + 8192, 64, h, (int)t0);
                }
                bulk_commit();
            }
        } else {
            // rows < L of the staged output -> global, 16 bytes per thread and step
            if (p.out_f32) {
                float *outp = static_cast<float *>(p.out);
                for (int e = tid; e < 64 * 32; e += kThreads) {
                    const int i = e >> 5, chk = e & 31;
                    if (i < L)
                        *reinterpret_cast<uint4 *>(outp + ((t0 + i) * H + h) * kD + 4 * chk) = lds128(base + kL + out_off_f32(i, 4 * chk));
                }
            } else {
                uint16_t *outp = static_cast<uint16_t *>(p.out);
                for (int e = tid; e < 64 * 16; e += kThreads) {
                    const int i = e >> 4, chk = e & 15;
                    if (i < L)
                        *reinterpret_cast<uint4 *>(outp + ((t0 + i) * H + h) * kD + 8 * chk) = lds128(base + kL + in_off(i, 8 * chk));
                }
            }
            bar_all();   // the staging area is next written in the next chunk's pass 2
        }
    }

    if (tma_lead) bulk_wait_all();
    // copies and products issued but never waited for complete before the CTA leaves (bounded)
    if (*abort_flag && tma_lead) {
        for (int i = 0; i < 4; ++i)
            if (pend >> i & 1) wait_bounded(bQ + 8 * i, pend_par >> i & 1, p.wait_ns);
    }
    if (*abort_flag && mma_lead) wait_bounded(bMma, mma_phase ^ 1, p.wait_ns);
    // final state (fp32, from TMEM).  An fp16 operand that overflowed (state, pseudo-values, values
    // beyond +-65504) becomes inf and reaches the fp32 state, where no fade can remove it: a
    // non-finite final state flags the unit.
    if (!*abort_flag) {
        uint32_t v[32];
        tld32(tq + cS + 32 * cq, v);
        bool bad = false;
#pragma unroll
        for (int j = 0; j < 32; ++j) bad |= !isfinite(__uint_as_float(v[j]));
        if (bad) atomicOr(&g_kda_error_word, kErrRange);
        if (p.S_out) {
            const size_t st_base = ((size_t)n * H + h) * kD * kD;
            float x[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) x[vperm(j)] = __uint_as_float(v[j]);
            float4 *sp = reinterpret_cast<float4 *>(p.S_out + st_base + (size_t)row * kD + 32 * cq);
#pragma unroll
            for (int j = 0; j < 8; ++j) sp[j] = make_float4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace tc
}  // namespace kda

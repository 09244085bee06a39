// Warp-level tensor-core helpers: bf16 m16n8k16 MMA with fp32 accumulation, ldmatrix loads from
// swizzled shared memory, and the fragment layouts the prefill kernel relies on.
//
// Fragment layouts of mma.m16n8k16 (bf16 or fp16 inputs) (g = lane / 4, t = lane % 4):
//   A (16x16, row major): a[0] = (g, 2t..2t+1)   a[1] = (g+8, 2t..)   a[2] = (g, 2t+8..)
//                         a[3] = (g+8, 2t+8..)
//   B (16x8):             b[0] = (k 2t..2t+1, n g)   b[1] = (k 2t+8.., n g)
//   C (16x8, fp32):       c[0..1] = (g, 2t..2t+1)   c[2..3] = (g+8, 2t..2t+1)
// Two adjacent C tiles (columns 0-7 and 8-15) converted to bf16 are exactly an A fragment of the
// 16x16 tile they cover; the kernels use that to feed one product's result into the next.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace kda {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

__device__ __forceinline__ float2 unpack_bf16(uint32_t v) {
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&v);
    return __bfloat1622float2(b);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

__device__ __forceinline__ float2 unpack_f16(uint32_t v) {
    const __half2 h = *reinterpret_cast<const __half2 *>(&v);
    return __half22float2(h);
}

// bf16 pair -> fp16 pair (exact for values inside the fp16 range)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
    const float2 f = unpack_bf16(v);
    return pack_f16(f.x, f.y);
}

// Split x into bf16 hi + lo with hi + lo = x to about 2^-16 relative.
__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const float2 hf = __bfloat1622float2(h);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = pack_bf16(x0 - hf.x, x1 - hf.y);
}

// The MMAs are plain (non-volatile) asm: they only read and write registers, so the compiler may
// schedule them around the (volatile) shared-memory fragment loads.
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                        uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a row-major tile whose rows are
// `row_bytes` long (a multiple of 64), with the chunk index XOR-swizzled so that the eight rows an
// ldmatrix reads at one logical chunk fall in eight different bank groups.
template <int ROW_BYTES>
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
    static_assert(ROW_BYTES % 64 == 0, "row size");
    if constexpr (ROW_BYTES >= 128) {
        return row * ROW_BYTES + ((chunk ^ (row & 7)) << 4);
    } else {  // 64-byte rows: two rows share a 128-byte line
        return row * ROW_BYTES + ((chunk ^ ((row >> 1) & 3)) << 4);
    }
}

// Byte offset of element (row, col) (2-byte elements) in the same swizzled layout.
template <int ROW_BYTES>
__device__ __forceinline__ uint32_t swz_elem(int row, int col) {
    return swz<ROW_BYTES>(row, col >> 3) + ((col & 7) << 1);
}

// Address that lane `lane` passes to ldmatrix.x4 for the 16x16 tile at (row0, col0) of a swizzled
// bf16 matrix: matrices 0..3 are (rows +0, cols +0), (rows +8, cols +0), (rows +0, cols +8),
// (rows +8, cols +8).  Non-transposed this yields the A fragment of the tile; transposed, on a
// [k][n] matrix, it yields the B fragments of the two n8 tiles (b0,b1 of n-tile 0 in r[0], r[1];
// of n-tile 1 in r[2], r[3]).
template <int ROW_BYTES>
__device__ __forceinline__ uint32_t ldsm_addr_a(uint32_t base, int row0, int col0, int lane) {
    const int mi = lane >> 3, r = lane & 7;
    return base + swz<ROW_BYTES>(row0 + r + ((mi & 1) << 3), (col0 >> 3) + (mi >> 1));
}

// For transposed B loads from a [k][n] matrix the second x4 matrix must be the k+8 half of the same
// n-tile: matrices are (k +0, n +0), (k +8, n +0), (k +0, n +8), (k +8, n +8), which is the same
// addressing as ldsm_addr_a with rows = k and cols = n.
template <int ROW_BYTES>
__device__ __forceinline__ uint32_t ldsm_addr_bt(uint32_t base, int k0, int n0, int lane) {
    return ldsm_addr_a<ROW_BYTES>(base, k0, n0, lane);
}

// For non-transposed B loads from an [n][k] matrix (k contiguous): matrices (n +0, k +0) -> b0 of
// n-tile 0, (n +0, k +8) -> b1 of n-tile 0, (n +8, k +0) -> b0 of n-tile 1, (n +8, k +8) -> b1.
template <int ROW_BYTES>
__device__ __forceinline__ uint32_t ldsm_addr_bn(uint32_t base, int n0, int k0, int lane) {
    const int mi = lane >> 3, r = lane & 7;
    return base + swz<ROW_BYTES>(n0 + r + ((mi >> 1) << 3), (k0 >> 3) + (mi & 1));
}

// Byte offset of the fp32 pair (row, col), col even, in a [rows][ROW_FLOATS] fp32 matrix whose
// 16-byte chunks are XOR-swizzled so that 8 rows x 4 consecutive pairs cost two wavefronts.
template <int ROW_FLOATS>
__device__ __forceinline__ uint32_t swz_f32(int row, int col) {
    const int chunk = (col >> 2) ^ ((row & 3) << 1);
    return row * ROW_FLOATS * 4 + (chunk << 4) + ((col & 3) << 2);
}

__device__ __forceinline__ void named_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(nthreads) : "memory");
}

// 16-byte load through L2 only (never a stale L1 line: ring slots are rewritten between uses).
__device__ __forceinline__ uint4 ldg_cg_v4(const void *p) {
    return __ldcg(reinterpret_cast<const uint4 *>(p));
}

__device__ __forceinline__ void st_u32(void *p, uint32_t x) {
    asm volatile("st.global.u32 [%0], %1;\n" ::"l"(p), "r"(x) : "memory");
}

__device__ __forceinline__ void stg_v4(void *p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// 16-byte asynchronous global->shared copy; bytes beyond src_bytes (0 or 16) are zero-filled.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}

// ---- mbarriers and the cluster ------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t addr, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(addr), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the cluster, then synchronise all threads of the cluster.
__device__ __forceinline__ void cluster_sync_after_init() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// Synchronise all threads of the cluster; safe for threads that reach it on diverged paths.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release;\nbarrier.cluster.wait.acquire;\n" ::: "memory");
}

// Address of the same shared-memory offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// Arrive (release, cluster scope) on an mbarrier that may live in another CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];\n" ::"r"(cluster_addr) : "memory");
}

// Arrive (relaxed, cluster scope): for a hand-back after which nothing written needs ordering.
__device__ __forceinline__ void mbar_arrive_relaxed_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];\n" ::"r"(cluster_addr) : "memory");
}

// Wait (acquire, cluster scope) for the phase with parity `parity` of a local mbarrier, letting the
// hardware suspend the thread for a bounded, implementation-defined time; true once the phase has
// completed, false if the suspension ended first.
__device__ __forceinline__ bool mbar_try(uint32_t addr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(addr), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;\n" ::: "memory");
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace kda

// libkda: C ABI entry points (declared in include/kda.h), argument validation and launches.
// The whole library is this one translation unit; kernels live in the included headers.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <mutex>
#include <cstring>
#include <string>
#include <vector>

#include "kda.h"
#include "common.cuh"
#include "decode.cuh"
#include "prefill_fused.cuh"
#include "prefill_tc.cuh"
#include "speculative.cuh"
#include "preprocess.cuh"
#include "state_map.cuh"
#include "backward.cuh"
#include "backward_chunk.cuh"

namespace {

thread_local std::string t_last_error;
std::atomic<uint64_t> g_launches{0};

kda_status fail(kda_status s, const std::string &msg) {
    t_last_error = msg;
    return s;
}

kda_status cuda_fail(cudaError_t e, const char *where) {
    return fail(KDA_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool supported_dim(int d) { return d == 64 || d == 128; }

// Workspace of the chunkwise path: per-unit rings of chunk records.
size_t ring_slot_bytes(int d_k, int d_v) {
    if (d_k == 128 && d_v == 128) return kda::RingLayout<128, 128>::kBytes;
    if (d_k == 128 && d_v == 64) return kda::RingLayout<128, 64>::kBytes;
    if (d_k == 64 && d_v == 128) return kda::RingLayout<64, 128>::kBytes;
    return kda::RingLayout<64, 64>::kBytes;
}

int ring_slots(int d_v) { return 2 * (d_v / kda::kSlab); }

size_t ring_bytes(int64_t units, int d_k, int d_v) {
    return (size_t)units * ring_slots(d_v) * ring_slot_bytes(d_k, d_v);
}

bool sizes_ok(int64_t total_tokens, int32_t num_seqs, int32_t max_seqlen, int32_t H) {
    return total_tokens >= 0 && num_seqs >= 0 && max_seqlen >= 0 && H > 0;
}

constexpr unsigned long long kWaitNs = 4000000000ull;   // bound of every device-side wait (4 s)

// failure injection (kda_inject_stall): withhold chunk 0, shorten the wait bound
std::atomic<int> g_inject_stall{0};
std::atomic<unsigned long long> g_inject_wait_ns{kWaitNs};

template <int DK, int DV>
kda_status launch_prefill(const kda::FusedParams &p, int64_t units, cudaStream_t stream) {
    constexpr int G = DV / kda::kSlab;
    const int smem = kda::FusedSmem<DK, DV>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kda::kda_prefill_fused_kernel<DK, DV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefill)");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(units * G));
    cfg.blockDim = dim3(kda::kFusedThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kda::kda_prefill_fused_kernel<DK, DV>, p);
    if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return KDA_OK;
}


// ---- the per-unit tensor-core prefill (d_k = d_v = 128) -----------------------------------------

// Which prefill kernel kda_chunk_fwd runs: 0 = chosen from the shapes, 1 = cluster kernel with the
// L2 ring, 2 = one CTA per unit (set by kda_set_prefill_path; for tests and measurements).
std::atomic<int> g_prefill_path{0};

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// 3-d map over a [T, H, 128] bf16 (or fp32) tensor: boxes of 128 bytes of channels (64 bf16, 32
// fp32) x 1 head x 64 tokens, 128-byte swizzle (the layout of the kernel's shared-memory tiles);
// loaded rows past T read as zeros, stored rows past T are dropped.
bool encode_thd(CUtensorMap *map, const void *ptr, int64_t T, int H, bool f32 = false) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t es = f32 ? 4 : 2;
    const cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {128 * es, (cuuint64_t)H * 128 * es};
    const cuuint32_t box[3] = {(cuuint32_t)(128 / es), 1, 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr),
               dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sm_count() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return sms;
}

// Clusters of the d = 128 cluster kernel (four CTAs each) that fit on the device at once: 33 on a
// 148-SM B200 (a cluster must sit inside one GPC; a probe launch confirms 33 run together and 36
// take two waves).  Queried once per process, on the device current at the first call (the GPUs of
// one node are alike); without a device (or if the query fails) the B200 figure scaled by the SM
// count.
int64_t prefill_cluster_capacity() {
    static std::atomic<int> cached{0};
    int c = cached.load(std::memory_order_relaxed);
    if (c > 0) return c;
    constexpr int G = 128 / kda::kSlab;
    const int smem = kda::FusedSmem<128, 128>::kBytes;
    int n = 0;
    if (cudaFuncSetAttribute(kda::kda_prefill_fused_kernel<128, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(G);
        cfg.blockDim = dim3(kda::kFusedThreads);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = G;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, kda::kda_prefill_fused_kernel<128, 128>, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();   // a failed query leaves no sticky error behind
    if (n <= 0) n = std::max(1, device_sm_count() * 33 / 148);
    cached.store(n, std::memory_order_relaxed);
    return n;
}

// The per-unit kernel keeps each unit on one SM (no workspace, no traffic between SMs); the
// cluster kernel spreads a unit's chunks over four SMs and runs a unit about 2.4 times faster
// (B200, d = 128: ~3.4 against ~8.3 us per 64-token chunk), but only C units run at once (C =
// prefill_cluster_capacity(), 33 on B200) against one unit per SM for the per-unit kernel.  So the
// cluster kernel wins while its units need at most two waves (units <= 2 C), the per-unit kernel
// from there on (measured on equal-length batches: 64 units 0.44 against 0.54 ms, 74 units 0.65
// against 0.54 ms).  `path` overrides the process-wide setting when non-zero.
bool use_tc_prefill(int64_t units, int d_k, int d_v, int path = 0) {
    if (d_k != 128 || d_v != 128) return false;
    if (g_inject_stall.load(std::memory_order_relaxed)) return false;   // the injection targets the cluster kernel
    const int forced = path ? path : g_prefill_path.load(std::memory_order_relaxed);
    if (forced) return forced == 2;
    return units > 2 * prefill_cluster_capacity();
}

kda_status launch_prefill_tc(const void *q, const void *k, const void *v, const void *a,
                             const kda::tc::Params &p, int64_t units, cudaStream_t stream) {
    kda::tc::Maps maps;
    if (!encode_thd(&maps.q, q, p.total_tokens, p.H) || !encode_thd(&maps.k, k, p.total_tokens, p.H) ||
        !encode_thd(&maps.v, v, p.total_tokens, p.H) || !encode_thd(&maps.a, a, p.total_tokens, p.H) ||
        !encode_thd(&maps.out, p.out, p.total_tokens, p.H, p.out_f32))
        return fail(KDA_ERR_CUDA, "kda_chunk_fwd: cuTensorMapEncodeTiled failed");
    cudaError_t e = cudaFuncSetAttribute(kda::tc::kda_prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kda::tc::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefill_tc)");
    kda::tc::kda_prefill_tc_kernel<<<(unsigned)units, kda::tc::kThreads, kda::tc::kSmemBytes, stream>>>(maps, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "prefill_tc launch");
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return KDA_OK;
}

template <int DK, int DV>
kda_status launch_decode(const kda::DecodeParams &p, int64_t units, cudaStream_t stream) {
    kda::decode_step_kernel<DK, DV><<<(unsigned)units, kda::kDecodeThreads, 0, stream>>>(p);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, "decode_step launch");
}

template <int DK, int DV>
kda_status launch_spec(const kda::SpecParams &p, int64_t units, bool commit, cudaStream_t stream) {
    if (commit) {
        // persistent: as many CTAs as fit on the device at once (at most one per unit)
        const size_t smem = kda::SpecCommitSmem<DK, DV>::bytes(p.K);
        cudaError_t e = cudaFuncSetAttribute(kda::spec_commit_kernel<DK, DV>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode_commit)");
        int dev = 0, sms = 0, per_sm = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kda::spec_commit_kernel<DK, DV>,
                                                               kda::kSpecThreads, smem)) != cudaSuccess)
            return cuda_fail(e, "decode_commit occupancy");
        if (per_sm < 1) return fail(KDA_ERR_UNSUPPORTED, "kda_decode_commit: kernel does not fit on an SM");
        const int64_t grid = units < (int64_t)per_sm * sms ? units : (int64_t)per_sm * sms;
        kda::spec_commit_kernel<DK, DV><<<(unsigned)grid, kda::kSpecThreads, smem, stream>>>(p, units);
    } else {
        // persistent: as many CTAs as fit on the device at once (at most one per unit)
        const size_t smem = kda::SpecVerifySmem<DK, DV>::bytes(p.K);
        cudaError_t e = cudaFuncSetAttribute(kda::spec_verify_kernel<DK, DV>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode_verify)");
        int dev = 0, sms = 0, per_sm = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kda::spec_verify_kernel<DK, DV>,
                                                               kda::kSpecThreads, smem)) != cudaSuccess)
            return cuda_fail(e, "decode_verify occupancy");
        if (per_sm < 1) return fail(KDA_ERR_UNSUPPORTED, "kda_decode_verify: kernel does not fit on an SM");
        const int64_t grid = units < (int64_t)per_sm * sms ? units : (int64_t)per_sm * sms;
        kda::spec_verify_kernel<DK, DV><<<(unsigned)grid, kda::kSpecThreads, smem, stream>>>(p, units);
    }
    g_launches.fetch_add(1, std::memory_order_relaxed);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, commit ? "decode_commit launch" : "decode_verify launch");
}

kda_status dispatch_spec(const kda::SpecParams &p, int64_t units, int d_k, int d_v, bool commit, cudaStream_t st) {
    if (d_k == 128 && d_v == 128) return launch_spec<128, 128>(p, units, commit, st);
    if (d_k == 128 && d_v == 64) return launch_spec<128, 64>(p, units, commit, st);
    if (d_k == 64 && d_v == 128) return launch_spec<64, 128>(p, units, commit, st);
    return launch_spec<64, 64>(p, units, commit, st);
}

template <int DK, int DV>
kda_status launch_bwd(const kda::BwdParams &p, int64_t units, cudaStream_t stream) {
    constexpr int G = DV / kda::kBwdCols;   // CTAs per unit: one per 32 value columns
    const int smem = kda::BwdSmem<DK>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kda::kda_bwd_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(chunk_bwd)");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(units * G));
    cfg.blockDim = dim3(kda::kBwdThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kda::kda_bwd_kernel<DK, DV>, p);
    if (e != cudaSuccess) return cuda_fail(e, "chunk_bwd launch");
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return KDA_OK;
}

// Built-in scratch for kda_chunk_fwd_noalloc (callers that cannot allocate).  Host code must not
// use this name as an address: it is a host-side stand-in; the device address comes from
// cudaGetSymbolAddress, looked up once per device below.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

}  // namespace

static __device__ __align__(256) unsigned char g_kda_static_scratch[kStaticScratchBytes];

namespace {

kda_status static_scratch_address(void **ptr) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd_noalloc: cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices)
        return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_fwd_noalloc: device ordinal out of range");
    // Looked up on every call (it allocates nothing and is cheap), so a device reset or a new context
    // on the device never leaves a stale address behind.
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_kda_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd_noalloc: cudaGetSymbolAddress");
    *ptr = p;
    return KDA_OK;
}

}  // namespace

extern "C" {

const char *kda_status_string(kda_status s) {
    switch (s) {
        case KDA_OK: return "ok";
        case KDA_ERR_INVALID_ARG: return "invalid argument";
        case KDA_ERR_UNSUPPORTED: return "unsupported configuration";
        case KDA_ERR_CUDA: return "CUDA error";
        case KDA_ERR_TIMEOUT: return "device-side wait timed out";
        case KDA_ERR_RANGE: return "value outside the fp16 operand range";
    }
    return "unknown status";
}

const char *kda_last_error(void) { return t_last_error.c_str(); }

uint64_t kda_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

size_t kda_chunk_fwd_workspace_min(int64_t total_tokens, int32_t num_seqs, int32_t max_seqlen,
                                   int32_t H, int32_t d_k, int32_t d_v) {
    if (!sizes_ok(total_tokens, num_seqs, max_seqlen, H) || !supported_dim(d_k) || !supported_dim(d_v))
        return 0;
    const int64_t units = (int64_t)num_seqs * H;
    if (use_tc_prefill(units, d_k, d_v)) return 0;
    return ring_bytes(units, d_k, d_v);
}

size_t kda_chunk_fwd_workspace_size(int64_t total_tokens, int32_t num_seqs, int32_t max_seqlen,
                                    int32_t H, int32_t d_k, int32_t d_v) {
    return kda_chunk_fwd_workspace_min(total_tokens, num_seqs, max_seqlen, H, d_k, d_v);
}

}  // extern "C"

namespace {

// kda_chunk_fwd with an optional choice of prefill kernel (0: the process-wide setting)
kda_status chunk_fwd_impl(const void *q, const void *k, const void *v, const void *a,
                          const float *beta, const void *gate, const float *A_log,
                          const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                          int32_t max_seqlen, int32_t H, int32_t d_k, int32_t d_v, float scale,
                          const float *initial_state, float *final_state, void *out,
                          kda_dtype out_dtype, void *workspace, size_t workspace_bytes,
                          void *stream, int path) {
    if (!sizes_ok(total_tokens, num_seqs, max_seqlen, H))
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: negative size or H <= 0");
    if (!supported_dim(d_k) || !supported_dim(d_v))
        return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_fwd: d_k and d_v must be 64 or 128");
    if (num_seqs == 0) {
        if (total_tokens != 0) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: tokens without sequences");
        return KDA_OK;
    }
    if (!cu_seqlens || !A_log) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: NULL cu_seqlens or A_log");
    if (total_tokens > 0 && (!q || !k || !v || !a || !beta || !out))
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: NULL q/k/v/a/beta/out");
    if (out_dtype != KDA_DTYPE_BF16 && out_dtype != KDA_DTYPE_F32)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: out_dtype must be KDA_DTYPE_BF16 or KDA_DTYPE_F32");
    const void *ptrs[] = {q, k, v, a, gate, initial_state, final_state, out, workspace};
    for (const void *ptr : ptrs)
        if (ptr && !aligned(ptr, 16)) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: tensor pointer not 16-byte aligned");
    const void *ptrs4[] = {beta, A_log, cu_seqlens};
    for (const void *ptr : ptrs4)
        if (ptr && !aligned(ptr, 4)) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: beta/A_log/cu_seqlens not 4-byte aligned");
    const size_t need = use_tc_prefill((int64_t)num_seqs * H, d_k, d_v, path) ? 0 : ring_bytes((int64_t)num_seqs * H, d_k, d_v);
    if (need > 0 && !workspace) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: NULL workspace");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: workspace not 256-byte aligned");
    if (workspace_bytes < need)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: workspace too small (need " +
                                             std::to_string(need) + " bytes)");

    const int64_t units = (int64_t)num_seqs * H;
    if (units * (d_v / kda::kSlab) > 0x7fffffffLL)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: num_seqs * H too large");
    if (total_tokens > 0x7fffffc0LL)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: total_tokens too large");
    if (use_tc_prefill(units, d_k, d_v, path) && total_tokens > 0) {
        kda::tc::Params tp{};
        tp.beta = beta;
        tp.A_log = A_log;
        tp.cu = cu_seqlens;
        tp.S_in = initial_state;
        tp.S_out = final_state;
        tp.out = out;
        tp.total_tokens = total_tokens;
        tp.num_seqs = num_seqs;
        tp.H = H;
        tp.max_seqlen = max_seqlen;
        tp.scale = scale;
        tp.out_f32 = out_dtype == KDA_DTYPE_F32;
        tp.has_gate = gate != nullptr;
        tp.gate = static_cast<const uint16_t *>(gate);
        tp.wait_ns = kWaitNs;
        return launch_prefill_tc(q, k, v, a, tp, units, static_cast<cudaStream_t>(stream));
    }
    char *ws = static_cast<char *>(workspace);
    kda::FusedParams p{};
    p.q = static_cast<const uint16_t *>(q);
    p.k = static_cast<const uint16_t *>(k);
    p.v = static_cast<const uint16_t *>(v);
    p.a = static_cast<const uint16_t *>(a);
    p.gate = static_cast<const uint16_t *>(gate);
    p.beta = beta;
    p.A_log = A_log;
    p.cu = cu_seqlens;
    p.S_in = initial_state;
    p.S_out = final_state;
    p.out = out;
    p.ring = ws;
    p.total_tokens = total_tokens;
    p.num_seqs = num_seqs;
    p.H = H;
    p.max_seqlen = max_seqlen;
    p.scale = scale;
    p.out_f32 = out_dtype == KDA_DTYPE_F32;
    p.stall_first_chunk = g_inject_stall.load(std::memory_order_relaxed);
    p.wait_ns = p.stall_first_chunk ? g_inject_wait_ns.load(std::memory_order_relaxed) : kWaitNs;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d_k == 128 && d_v == 128) return launch_prefill<128, 128>(p, units, st);
    if (d_k == 128 && d_v == 64) return launch_prefill<128, 64>(p, units, st);
    if (d_k == 64 && d_v == 128) return launch_prefill<64, 128>(p, units, st);
    return launch_prefill<64, 64>(p, units, st);
}

}  // namespace

extern "C" {

kda_status kda_chunk_fwd(const void *q, const void *k, const void *v, const void *a,
                         const float *beta, const void *gate, const float *A_log,
                         const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                         int32_t max_seqlen, int32_t H, int32_t d_k, int32_t d_v, float scale,
                         const float *initial_state, float *final_state, void *out,
                         kda_dtype out_dtype, void *workspace, size_t workspace_bytes,
                         void *stream) {
    return chunk_fwd_impl(q, k, v, a, beta, gate, A_log, cu_seqlens, num_seqs, total_tokens, max_seqlen, H, d_k, d_v,
                          scale, initial_state, final_state, out, out_dtype, workspace, workspace_bytes, stream, 0);
}

kda_status kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *a,
                                 const float *beta, const void *gate, const float *A_log,
                                 const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                                 int32_t max_seqlen, int32_t H, int32_t d_k, int32_t d_v,
                                 float scale, const float *initial_state, float *final_state,
                                 void *out, kda_dtype out_dtype, void *stream) {
    // With the kernel left to the shapes, sizes whose cluster-kernel records would not fit run the
    // per-unit kernel, which needs no scratch (d_k = d_v = 128); any other need beyond the array is
    // rejected.
    int path = 0;
    if (g_prefill_path.load(std::memory_order_relaxed) == 0 && sizes_ok(total_tokens, num_seqs, max_seqlen, H) &&
        kda_chunk_fwd_workspace_min(total_tokens, num_seqs, max_seqlen, H, d_k, d_v) > kStaticScratchBytes &&
        use_tc_prefill((int64_t)num_seqs * H, d_k, d_v, 2))
        path = 2;
    const size_t need = use_tc_prefill((int64_t)num_seqs * H, d_k, d_v, path) || !sizes_ok(total_tokens, num_seqs, max_seqlen, H)
                            ? 0
                            : kda_chunk_fwd_workspace_min(total_tokens, num_seqs, max_seqlen, H, d_k, d_v);
    if (need > kStaticScratchBytes)
        return fail(KDA_ERR_INVALID_ARG,
                    "kda_chunk_fwd_noalloc: these sizes need " + std::to_string(need) +
                        " bytes of scratch, more than the " + std::to_string(kStaticScratchBytes) +
                        " built into the library; call kda_chunk_fwd with a workspace instead");
    void *scratch = nullptr;
    const kda_status st = static_scratch_address(&scratch);
    if (st != KDA_OK) return st;
    return chunk_fwd_impl(q, k, v, a, beta, gate, A_log, cu_seqlens, num_seqs, total_tokens, max_seqlen, H, d_k, d_v,
                          scale, initial_state, final_state, out, out_dtype, scratch, kStaticScratchBytes, stream, path);
}

kda_status kda_decode_step(const void *q, const void *k, const void *v, const void *a,
                           const float *beta, const void *gate, const float *A_log, float *state,
                           void *out, kda_dtype out_dtype, int32_t N, int32_t H, int32_t d_k,
                           int32_t d_v, float scale, void *stream) {
    if (N < 0 || H <= 0) return fail(KDA_ERR_INVALID_ARG, "kda_decode_step: N < 0 or H <= 0");
    if (!supported_dim(d_k) || !supported_dim(d_v))
        return fail(KDA_ERR_UNSUPPORTED, "kda_decode_step: d_k and d_v must be 64 or 128");
    if (N == 0) return KDA_OK;
    if (!q || !k || !v || !a || !beta || !A_log || !state || !out)
        return fail(KDA_ERR_INVALID_ARG, "kda_decode_step: NULL required pointer");
    if (out_dtype != KDA_DTYPE_BF16 && out_dtype != KDA_DTYPE_F32)
        return fail(KDA_ERR_INVALID_ARG, "kda_decode_step: out_dtype must be KDA_DTYPE_BF16 or KDA_DTYPE_F32");
    const void *ptrs[] = {q, k, v, a, gate, state, out};
    for (const void *ptr : ptrs)
        if (ptr && !aligned(ptr, 16)) return fail(KDA_ERR_INVALID_ARG, "kda_decode_step: tensor pointer not 16-byte aligned");
    const void *ptrs4[] = {beta, A_log};
    for (const void *ptr : ptrs4)
        if (ptr && !aligned(ptr, 4)) return fail(KDA_ERR_INVALID_ARG, "kda_decode_step: beta/A_log not 4-byte aligned");
    const int64_t units = (int64_t)N * H;
    if (units > 0x7fffffffLL) return fail(KDA_ERR_INVALID_ARG, "kda_decode_step: N*H too large");
    kda::DecodeParams p{};
    p.q = static_cast<const uint16_t *>(q);
    p.k = static_cast<const uint16_t *>(k);
    p.v = static_cast<const uint16_t *>(v);
    p.a = static_cast<const uint16_t *>(a);
    p.gate = static_cast<const uint16_t *>(gate);
    p.beta = beta;
    p.A_log = A_log;
    p.state = state;
    p.out = out;
    p.out_f32 = out_dtype == KDA_DTYPE_F32;
    p.H = H;
    p.scale = scale;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d_k == 128 && d_v == 128) return launch_decode<128, 128>(p, units, st);
    if (d_k == 128 && d_v == 64) return launch_decode<128, 64>(p, units, st);
    if (d_k == 64 && d_v == 128) return launch_decode<64, 128>(p, units, st);
    return launch_decode<64, 64>(p, units, st);
}

kda_status kda_set_prefill_path(int32_t path) {
    if (path < 0 || path > 2) return fail(KDA_ERR_INVALID_ARG, "kda_set_prefill_path: path must be 0, 1 or 2");
    g_prefill_path.store(path, std::memory_order_relaxed);
    return KDA_OK;
}

int32_t kda_prefill_path(int64_t num_units, int32_t d_k, int32_t d_v) {
    return use_tc_prefill(num_units, d_k, d_v) ? 2 : 1;
}

kda_status kda_inject_stall(int32_t enable, uint64_t wait_limit_ns) {
    if (!enable) {
        g_inject_stall.store(0);
        return KDA_OK;
    }
    if (wait_limit_ns < 1000000ull || wait_limit_ns > kWaitNs)
        return fail(KDA_ERR_INVALID_ARG, "kda_inject_stall: wait_limit_ns must be in [1e6, 4e9]");
    g_inject_wait_ns.store(wait_limit_ns);
    g_inject_stall.store(1);
    return KDA_OK;
}

kda_status kda_decode_verify(const void *q, const void *k, const void *v, const void *a, const float *beta,
                             const void *gate, const float *A_log, const float *state, float *u, void *out,
                             kda_dtype out_dtype, int32_t N, int32_t K, int32_t H, int32_t d_k, int32_t d_v,
                             float scale, void *stream) {
    if (N < 0 || H <= 0) return fail(KDA_ERR_INVALID_ARG, "kda_decode_verify: N < 0 or H <= 0");
    if (K < 1 || K > kda::kSpecMaxTokens)
        return fail(KDA_ERR_INVALID_ARG, "kda_decode_verify: K must be in [1, 16]");
    if (!supported_dim(d_k) || !supported_dim(d_v))
        return fail(KDA_ERR_UNSUPPORTED, "kda_decode_verify: d_k and d_v must be 64 or 128");
    if (N == 0) return KDA_OK;
    if (!q || !k || !v || !a || !beta || !A_log || !state || !u || !out)
        return fail(KDA_ERR_INVALID_ARG, "kda_decode_verify: NULL required pointer");
    if (out_dtype != KDA_DTYPE_BF16 && out_dtype != KDA_DTYPE_F32)
        return fail(KDA_ERR_INVALID_ARG, "kda_decode_verify: out_dtype must be KDA_DTYPE_BF16 or KDA_DTYPE_F32");
    const void *ptrs[] = {q, k, v, a, gate, state, u, out};
    for (const void *ptr : ptrs)
        if (ptr && !aligned(ptr, 16)) return fail(KDA_ERR_INVALID_ARG, "kda_decode_verify: tensor pointer not 16-byte aligned");
    const void *ptrs4[] = {beta, A_log};
    for (const void *ptr : ptrs4)
        if (!aligned(ptr, 4)) return fail(KDA_ERR_INVALID_ARG, "kda_decode_verify: beta/A_log not 4-byte aligned");
    const int64_t units = (int64_t)N * H;
    if (units > 0x7fffffffLL) return fail(KDA_ERR_INVALID_ARG, "kda_decode_verify: N*H too large");
    kda::SpecParams p{};
    p.q = static_cast<const uint16_t *>(q);
    p.k = static_cast<const uint16_t *>(k);
    p.v = static_cast<const uint16_t *>(v);
    p.a = static_cast<const uint16_t *>(a);
    p.gate = static_cast<const uint16_t *>(gate);
    p.beta = beta;
    p.A_log = A_log;
    p.state = const_cast<float *>(state);   // read only by the verify kernel
    p.u = u;
    p.out = out;
    p.H = H;
    p.K = K;
    p.out_f32 = out_dtype == KDA_DTYPE_F32;
    p.scale = scale;
    return dispatch_spec(p, units, d_k, d_v, false, static_cast<cudaStream_t>(stream));
}

kda_status kda_decode_commit(const void *k, const void *a, const float *A_log, const int32_t *accepted,
                             const float *u, float *state, int32_t N, int32_t K, int32_t H, int32_t d_k,
                             int32_t d_v, void *stream) {
    if (N < 0 || H <= 0) return fail(KDA_ERR_INVALID_ARG, "kda_decode_commit: N < 0 or H <= 0");
    if (K < 1 || K > kda::kSpecMaxTokens)
        return fail(KDA_ERR_INVALID_ARG, "kda_decode_commit: K must be in [1, 16]");
    if (!supported_dim(d_k) || !supported_dim(d_v))
        return fail(KDA_ERR_UNSUPPORTED, "kda_decode_commit: d_k and d_v must be 64 or 128");
    if (N == 0) return KDA_OK;
    if (!k || !a || !A_log || !accepted || !u || !state)
        return fail(KDA_ERR_INVALID_ARG, "kda_decode_commit: NULL required pointer");
    const void *ptrs[] = {k, a, u, state};
    for (const void *ptr : ptrs)
        if (!aligned(ptr, 16)) return fail(KDA_ERR_INVALID_ARG, "kda_decode_commit: tensor pointer not 16-byte aligned");
    if (!aligned(A_log, 4) || !aligned(accepted, 4))
        return fail(KDA_ERR_INVALID_ARG, "kda_decode_commit: A_log/accepted not 4-byte aligned");
    const int64_t units = (int64_t)N * H;
    if (units > 0x7fffffffLL) return fail(KDA_ERR_INVALID_ARG, "kda_decode_commit: N*H too large");
    kda::SpecParams p{};
    p.k = static_cast<const uint16_t *>(k);
    p.a = static_cast<const uint16_t *>(a);
    p.A_log = A_log;
    p.accepted = accepted;
    p.u = const_cast<float *>(u);   // read only by the commit kernel
    p.state = state;
    p.H = H;
    p.K = K;
    return dispatch_spec(p, units, d_k, d_v, true, static_cast<cudaStream_t>(stream));
}

kda_status kda_short_conv(const void *x, const float *w, const int32_t *cu_seqlens, int32_t num_seqs,
                          int64_t total_tokens, int32_t H, int32_t d, int32_t width, int32_t l2norm, void *y,
                          void *stream) {
    if (total_tokens < 0 || num_seqs < 0 || H <= 0)
        return fail(KDA_ERR_INVALID_ARG, "kda_short_conv: negative size or H <= 0");
    if (!supported_dim(d)) return fail(KDA_ERR_UNSUPPORTED, "kda_short_conv: d must be 64 or 128");
    if (width < 1 || width > kda::kConvMaxWidth) return fail(KDA_ERR_INVALID_ARG, "kda_short_conv: width must be in [1, 4]");
    if (total_tokens == 0) return KDA_OK;
    if (num_seqs == 0) return fail(KDA_ERR_INVALID_ARG, "kda_short_conv: tokens without sequences");
    if (!x || !w || !cu_seqlens || !y) return fail(KDA_ERR_INVALID_ARG, "kda_short_conv: NULL required pointer");
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(w, 4) || !aligned(cu_seqlens, 4))
        return fail(KDA_ERR_INVALID_ARG, "kda_short_conv: misaligned pointer");
    kda::ConvParams p{};
    p.x = static_cast<const uint16_t *>(x);
    p.w = w;
    p.cu = cu_seqlens;
    p.y = static_cast<uint16_t *>(y);
    p.total_tokens = total_tokens;
    p.num_seqs = num_seqs;
    p.H = H;
    p.width = width;
    p.l2norm = l2norm != 0;
    const int64_t groups = (int64_t)H * (d / 8);
    const int64_t cblocks = (groups + kda::kPrepThreads - 1) / kda::kPrepThreads;
    if (cblocks > 65535) return fail(KDA_ERR_INVALID_ARG, "kda_short_conv: H * d too large");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    auto kern = d == 128 ? kda::short_conv_kernel<128> : kda::short_conv_kernel<64>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kda::kConvSmem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(short_conv)");
    // one run of consecutive tokens per CTA, as many CTAs as the device holds at once
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kda::kPrepThreads, kda::kConvSmem)) != cudaSuccess)
        return cuda_fail(e, "short_conv occupancy");
    if (per_sm < 1) return fail(KDA_ERR_UNSUPPORTED, "kda_short_conv: kernel does not fit on an SM");
    const int64_t want = std::max<int64_t>(1, (int64_t)sms * per_sm / cblocks);
    const int64_t run_len = std::max<int64_t>(kda::kConvAhead, (total_tokens + want - 1) / want);
    const int64_t runs = (total_tokens + run_len - 1) / run_len;
    const dim3 grid((unsigned)runs, (unsigned)cblocks);
    kern<<<grid, kda::kPrepThreads, kda::kConvSmem, st>>>(p, run_len);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    e = cudaGetLastError();
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, "short_conv launch");
}

kda_status kda_output_norm_gate(const float *o, const void *gate, const float *w, int64_t total_tokens, int32_t H,
                                int32_t d_v, float eps, void *out, kda_dtype out_dtype, void *stream) {
    if (total_tokens < 0 || H <= 0) return fail(KDA_ERR_INVALID_ARG, "kda_output_norm_gate: negative size or H <= 0");
    if (!supported_dim(d_v)) return fail(KDA_ERR_UNSUPPORTED, "kda_output_norm_gate: d_v must be 64 or 128");
    if (!(eps >= 0.f)) return fail(KDA_ERR_INVALID_ARG, "kda_output_norm_gate: eps must be >= 0");
    if (out_dtype != KDA_DTYPE_BF16 && out_dtype != KDA_DTYPE_F32)
        return fail(KDA_ERR_INVALID_ARG, "kda_output_norm_gate: out_dtype must be KDA_DTYPE_BF16 or KDA_DTYPE_F32");
    if (total_tokens == 0) return KDA_OK;
    if (!o || !w || !out) return fail(KDA_ERR_INVALID_ARG, "kda_output_norm_gate: NULL required pointer");
    if (!aligned(o, 16) || !aligned(out, 16) || (gate && !aligned(gate, 16)) || !aligned(w, 4))
        return fail(KDA_ERR_INVALID_ARG, "kda_output_norm_gate: misaligned pointer");
    kda::NormGateParams p{};
    p.o = o;
    p.gate = static_cast<const uint16_t *>(gate);
    p.w = w;
    p.out = out;
    p.rows = total_tokens * H;
    p.eps = eps;
    p.out_f32 = out_dtype == KDA_DTYPE_F32;
    const int64_t threads = p.rows * (d_v / 8);
    const int64_t blocks = (threads + kda::kPrepThreads - 1) / kda::kPrepThreads;
    if (blocks > 0x7fffffffLL) return fail(KDA_ERR_INVALID_ARG, "kda_output_norm_gate: too many rows");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d_v == 128) kda::norm_gate_kernel<128><<<(unsigned)blocks, kda::kPrepThreads, 0, st>>>(p);
    else kda::norm_gate_kernel<64><<<(unsigned)blocks, kda::kPrepThreads, 0, st>>>(p);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, "norm_gate launch");
}

size_t kda_segment_maps_workspace_size(int64_t total_tokens, int32_t num_seqs, int32_t H, int32_t d) {
    if (!sizes_ok(total_tokens, num_seqs, 0, H) || !supported_dim(d)) return 0;
    const int64_t units = (int64_t)num_seqs * H;
    const size_t slot = d == 128 ? kda::RingLayout<128, 256>::kBytes : kda::RingLayout<64, 128>::kBytes;
    const size_t ring = ((size_t)units * ring_slots(2 * d) * slot + 255) / 256 * 256;
    return ring + (size_t)units * d * 2 * d * 4;   // then the final states [M | B]
}

kda_status kda_segment_maps(const void *q, const void *k, const void *v, const void *a, const float *beta,
                            const float *A_log, const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                            int32_t max_seqlen, int32_t H, int32_t d, float scale, float *M, float *B,
                            void *workspace, size_t workspace_bytes, void *stream) {
    if (!sizes_ok(total_tokens, num_seqs, max_seqlen, H))
        return fail(KDA_ERR_INVALID_ARG, "kda_segment_maps: negative size or H <= 0");
    if (!supported_dim(d)) return fail(KDA_ERR_UNSUPPORTED, "kda_segment_maps: d must be 64 or 128");
    if (num_seqs == 0) {
        if (total_tokens != 0) return fail(KDA_ERR_INVALID_ARG, "kda_segment_maps: tokens without sequences");
        return KDA_OK;
    }
    if (!cu_seqlens || !A_log || !M || !B || !workspace)
        return fail(KDA_ERR_INVALID_ARG, "kda_segment_maps: NULL cu_seqlens, A_log, M, B or workspace");
    if (total_tokens > 0 && (!q || !k || !v || !a || !beta))
        return fail(KDA_ERR_INVALID_ARG, "kda_segment_maps: NULL q/k/v/a/beta");
    const void *ptrs[] = {q, k, v, a, M, B};
    for (const void *ptr : ptrs)
        if (ptr && !aligned(ptr, 16)) return fail(KDA_ERR_INVALID_ARG, "kda_segment_maps: tensor pointer not 16-byte aligned");
    const void *ptrs4[] = {beta, A_log, cu_seqlens};
    for (const void *ptr : ptrs4)
        if (ptr && !aligned(ptr, 4)) return fail(KDA_ERR_INVALID_ARG, "kda_segment_maps: beta/A_log/cu_seqlens not 4-byte aligned");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(KDA_ERR_INVALID_ARG, "kda_segment_maps: workspace not 256-byte aligned");
    const size_t need = kda_segment_maps_workspace_size(total_tokens, num_seqs, H, d);
    if (workspace_bytes < need)
        return fail(KDA_ERR_INVALID_ARG, "kda_segment_maps: workspace too small (need " + std::to_string(need) + " bytes)");
    const int64_t units = (int64_t)num_seqs * H;
    if (units * (2 * d / kda::kSlab) > 0x7fffffffLL) return fail(KDA_ERR_INVALID_ARG, "kda_segment_maps: num_seqs * H too large");
    if (total_tokens > 0x7fffffc0LL) return fail(KDA_ERR_INVALID_ARG, "kda_segment_maps: total_tokens too large");
    // one pass of the cluster kernel over value columns [0 | v] from [I | 0]: the final state is [M | B]
    const size_t slot = d == 128 ? kda::RingLayout<128, 256>::kBytes : kda::RingLayout<64, 128>::kBytes;
    const size_t ring = ((size_t)units * ring_slots(2 * d) * slot + 255) / 256 * 256;
    char *ws = static_cast<char *>(workspace);
    float *SMB = reinterpret_cast<float *>(ws + ring);
    kda::FusedParams p{};
    p.q = static_cast<const uint16_t *>(q);
    p.k = static_cast<const uint16_t *>(k);
    p.v = static_cast<const uint16_t *>(v);
    p.a = static_cast<const uint16_t *>(a);
    p.beta = beta;
    p.A_log = A_log;
    p.cu = cu_seqlens;
    p.S_out = SMB;
    p.ring = ws;
    p.total_tokens = total_tokens;
    p.num_seqs = num_seqs;
    p.H = H;
    p.max_seqlen = max_seqlen;
    p.scale = scale;
    p.wait_ns = kWaitNs;
    p.maps_cols = d;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const kda_status s = d == 128 ? launch_prefill<128, 256>(p, units, st) : launch_prefill<64, 128>(p, units, st);
    if (s != KDA_OK) return s;
    // [M | B] rows -> M and B
    const size_t rows = (size_t)units * d, wb = (size_t)d * 4;
    cudaError_t e = cudaMemcpy2DAsync(M, wb, SMB, 2 * wb, wb, rows, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = cudaMemcpy2DAsync(B, wb, SMB + d, 2 * wb, wb, rows, cudaMemcpyDeviceToDevice, st);
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, "kda_segment_maps: copy of the maps");
}

kda_status kda_state_combine(const float *M, const float *S_in, const float *B, float *S_out, int32_t units,
                             int32_t d_k, int32_t d_v, void *stream) {
    if (units < 0) return fail(KDA_ERR_INVALID_ARG, "kda_state_combine: units < 0");
    if (!supported_dim(d_k) || !supported_dim(d_v))
        return fail(KDA_ERR_UNSUPPORTED, "kda_state_combine: d_k and d_v must be 64 or 128");
    if (units == 0) return KDA_OK;
    if (!M || !S_in || !B || !S_out) return fail(KDA_ERR_INVALID_ARG, "kda_state_combine: NULL pointer");
    if (!aligned(M, 16) || !aligned(S_in, 16) || !aligned(B, 16) || !aligned(S_out, 16))
        return fail(KDA_ERR_INVALID_ARG, "kda_state_combine: pointer not 16-byte aligned");
    const size_t state_bytes = (size_t)units * d_k * d_v * 4;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(S_in), b0 = reinterpret_cast<uintptr_t>(S_out);
    if (a0 < b0 + state_bytes && b0 < a0 + state_bytes)
        return fail(KDA_ERR_INVALID_ARG, "kda_state_combine: S_out overlaps S_in");
    if (units > 65535) return fail(KDA_ERR_INVALID_ARG, "kda_state_combine: more than 65535 units per call");
    kda::CombineParams p{M, S_in, B, S_out};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const dim3 grid((unsigned)(d_k / kda::kCombineRows), (unsigned)units);
    if (d_k == 128 && d_v == 128) kda::state_combine_kernel<128, 128><<<grid, 256, 0, st>>>(p);
    else if (d_k == 128 && d_v == 64) kda::state_combine_kernel<128, 64><<<grid, 256, 0, st>>>(p);
    else if (d_k == 64 && d_v == 128) kda::state_combine_kernel<64, 128><<<grid, 256, 0, st>>>(p);
    else kda::state_combine_kernel<64, 64><<<grid, 256, 0, st>>>(p);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, "state_combine launch");
}

size_t kda_chunk_bwd_workspace_size(int64_t total_tokens, int32_t num_seqs, int32_t H, int32_t d_k, int32_t d_v) {
    if (total_tokens < 0 || num_seqs < 0 || H <= 0 || !supported_dim(d_k) || !supported_dim(d_v)) return 0;
    const size_t state = (size_t)d_k * d_v * 4;
    const size_t ckpts = (size_t)(total_tokens / kda::kBwdChunk + num_seqs) * H;   // >= sum ceil(len / 32)
    const size_t scratch = (size_t)num_seqs * H * kda::kBwdChunk;
    return (ckpts + scratch) * state;
}

kda_status kda_chunk_bwd(const void *q, const void *k, const void *v, const void *a, const float *beta,
                         const void *gate, const float *A_log, const int32_t *cu_seqlens, int32_t num_seqs,
                         int64_t total_tokens, int32_t H, int32_t d_k, int32_t d_v, float scale,
                         const float *initial_state, const float *dout, const float *dfinal_state, float *dq,
                         float *dk, float *dv, float *da, float *dbeta, float *dgate, float *dA_log,
                         float *dinitial_state, void *workspace, size_t workspace_bytes, void *stream) {
    if (total_tokens < 0 || num_seqs < 0 || H <= 0) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd: negative size or H <= 0");
    if (!supported_dim(d_k) || !supported_dim(d_v))
        return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_bwd: d_k and d_v must be 64 or 128");
    if (num_seqs == 0) {
        if (total_tokens != 0) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd: tokens without sequences");
        return KDA_OK;
    }
    if (!cu_seqlens || !A_log || !dA_log) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd: NULL cu_seqlens, A_log or dA_log");
    if (total_tokens > 0 && (!q || !k || !v || !a || !beta || !dout || !dq || !dk || !dv || !da || !dbeta))
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd: NULL input or gradient pointer");
    if (gate && !dgate) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd: gate given without dgate");
    const void *ptrs[] = {q, k, v, a, gate, initial_state, dout, dfinal_state, dq, dk, dv, da, dgate,
                          dinitial_state, workspace};
    for (const void *ptr : ptrs)
        if (ptr && !aligned(ptr, 16)) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd: tensor pointer not 16-byte aligned");
    const void *ptrs4[] = {beta, A_log, cu_seqlens, dbeta, dA_log};
    for (const void *ptr : ptrs4)
        if (ptr && !aligned(ptr, 4)) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd: scalar array not 4-byte aligned");
    const size_t need = kda_chunk_bwd_workspace_size(total_tokens, num_seqs, H, d_k, d_v);
    if (!workspace || workspace_bytes < need)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd: workspace missing or too small (need " + std::to_string(need) + " bytes)");
    const int64_t units = (int64_t)num_seqs * H;
    if (units * (d_v / kda::kBwdCols) > 0x7fffffffLL) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd: num_seqs * H too large");
    kda::BwdParams p{};
    p.ck_records = total_tokens / kda::kBwdChunk + num_seqs;
    p.q = static_cast<const uint16_t *>(q);
    p.k = static_cast<const uint16_t *>(k);
    p.v = static_cast<const uint16_t *>(v);
    p.a = static_cast<const uint16_t *>(a);
    p.gate = static_cast<const uint16_t *>(gate);
    p.beta = beta;
    p.A_log = A_log;
    p.cu = cu_seqlens;
    p.S0 = initial_state;
    p.dout = dout;
    p.dS_T = dfinal_state;
    p.dq = dq; p.dk = dk; p.dv = dv; p.da = da; p.dbeta = dbeta; p.dgate = dgate;
    p.dA_log = dA_log;
    p.dS0 = dinitial_state;
    const size_t state = (size_t)d_k * d_v;
    p.ckpt = static_cast<float *>(workspace);
    p.scratch = p.ckpt + (size_t)(total_tokens / kda::kBwdChunk + num_seqs) * H * state;
    p.total_tokens = total_tokens;
    p.num_seqs = num_seqs;
    p.H = H;
    p.scale = scale;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(dA_log, 0, sizeof(float) * H, st);   // the kernel accumulates into it
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(dA_log)");
    if (d_k == 128 && d_v == 128) return launch_bwd<128, 128>(p, units, st);
    if (d_k == 128 && d_v == 64) return launch_bwd<128, 64>(p, units, st);
    if (d_k == 64 && d_v == 128) return launch_bwd<64, 128>(p, units, st);
    return launch_bwd<64, 64>(p, units, st);
}

kda_status kda_sync_check(void *stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kda_sync_check: stream");
    unsigned word = 0;
    e = cudaMemcpyFromSymbol(&word, g_kda_error_word, sizeof(word));
    if (e != cudaSuccess) return cuda_fail(e, "kda_sync_check: read error word");
    if (word) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_kda_error_word, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e, "kda_sync_check: clear error word");
    }
    if (word & kda::kErrTimeout) return fail(KDA_ERR_TIMEOUT, "a bounded device-side wait gave up");
    if (word & kda::kErrBadSeqlens)
        return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is not monotone from 0 to total_tokens");
    if (word & kda::kErrSeqTooLong)
        return fail(KDA_ERR_INVALID_ARG, "a sequence is longer than max_seqlen");
    if (word & kda::kErrBadAccepted)
        return fail(KDA_ERR_INVALID_ARG, "an accepted count is outside [0, K] (it was clamped)");
    if (word & kda::kErrRange)
        return fail(KDA_ERR_RANGE, "a prefill state ended non-finite: a value, state or pseudo-value left the "
                                   "+-65504 range of the fp16 tensor-core operands; outputs and final states are not valid");
    return KDA_OK;
}

}  // extern "C"

// ---- prefill with host buffers: pieces along the token axis, copies overlapped with compute ------

namespace {

constexpr int kHostSlots = 2;             // staging slots: piece p uses slot p % 2
constexpr int64_t kHostPieceDefault = 2048;

struct HostPiece {
    int64_t a, e;       // packed tokens [a, e)
    int32_t n_lo, n_hi; // sequences taking part (inclusive)
    bool carry;         // sequence n_hi continues into the next piece
};

// Cuts the packed batch into pieces of about `piece` tokens.  A cut inside a sequence falls on a
// 64-token chunk boundary of that sequence, so each piece runs exactly the chunks the whole call
// would.  Sequence n takes part in the piece where it starts (an empty one at the very end, in the
// last piece) and in every piece it continues into.
// A cut at or below token e (0 < e < T) on a 64-token chunk boundary of the sequence containing e;
// -1 if cu_seqlens does not cover e.
int64_t chunk_cut(const int32_t *cu, int32_t N, int64_t e) {
    int32_t m = 0;
    while (m < N && cu[m + 1] <= e) ++m;
    if (m >= N) return -1;
    return cu[m] + ((e - cu[m]) / kda::kChunk) * kda::kChunk;
}

bool plan_pieces(const int32_t *cu, int32_t N, int64_t T, int64_t piece, std::vector<HostPiece> &out) {
    out.clear();
    std::vector<int64_t> cuts{0};
    for (int64_t a = 0; a < T;) {
        int64_t e = std::min<int64_t>(a + piece, T);
        if (e < T) {
            e = chunk_cut(cu, N, e);
            if (e <= a) return false;   // not reached for piece >= 64: a is a boundary of its own
        } else if (T - a >= 4 * kda::kChunk) {
            // the last piece is cut 3 : 1, so that little is left to copy out after the last prefill
            const int64_t m = chunk_cut(cu, N, a + 3 * (T - a) / 4);
            if (m > a && m < T) cuts.push_back(m);
        }
        cuts.push_back(e);
        a = e;
    }
    if (T == 0) cuts.push_back(0);   // one empty piece: the zero-length sequences' states
    for (size_t i = 0; i + 1 < cuts.size(); ++i) {
        const int64_t a = cuts[i], e = cuts[i + 1];
        int32_t lo = 0;   // first sequence not finished before a (empty ones starting at a included)
        while (lo < N && cu[lo + 1] <= a && cu[lo] < a) ++lo;
        int32_t hi = lo;  // last sequence starting before e (every remaining one in the last piece)
        while (hi + 1 < N && (e == T || cu[hi + 1] < e)) ++hi;
        if (lo >= N) return false;
        out.push_back({a, e, lo, hi, e < T && cu[hi + 1] > e});
    }
    return true;
}

struct HostLayout {
    size_t in_bytes, out_bytes, slot_bytes, ws_bytes, cu_bytes, state_bytes, total;
    int64_t max_tokens;
};

HostLayout host_layout(const std::vector<HostPiece> &pieces, int32_t N, int32_t H, int d_k, int d_v, bool f32_out) {
    HostLayout L{};
    int64_t max_tok = 0;
    size_t ws = 0, cu_count = 0;
    for (const HostPiece &pc : pieces) {
        max_tok = std::max(max_tok, pc.e - pc.a);
        ws = std::max(ws, kda_chunk_fwd_workspace_min(pc.e - pc.a, pc.n_hi - pc.n_lo + 1, 0, H, d_k, d_v));
        cu_count += (size_t)(pc.n_hi - pc.n_lo + 2);
    }
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t th = (size_t)max_tok * H;
    // q, k, a, v, gate (bf16), beta (fp32): each region rounded up so every pointer stays aligned
    L.in_bytes = 3 * up(th * d_k * 2) + 2 * up(th * d_v * 2) + up(th * 4);
    L.out_bytes = up(th * d_v * (f32_out ? 4 : 2));
    L.slot_bytes = L.in_bytes + L.out_bytes;
    L.ws_bytes = up(ws);
    L.cu_bytes = up(cu_count * 4 + (size_t)H * 4);
    L.state_bytes = up((size_t)N * H * d_k * d_v * 4);
    L.total = kHostSlots * L.slot_bytes + L.ws_bytes + L.cu_bytes + 2 * L.state_bytes;
    L.max_tokens = max_tok;
    return L;
}

}  // namespace

size_t kda_chunk_fwd_host_buffer_size(const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens, int32_t H,
                                      int32_t d_k, int32_t d_v, kda_dtype out_dtype, int64_t piece_tokens) {
    if (!cu_seqlens || num_seqs <= 0 || total_tokens < 0 || H <= 0 || !supported_dim(d_k) || !supported_dim(d_v))
        return 0;
    if (piece_tokens == 0) piece_tokens = kHostPieceDefault;
    if (piece_tokens < kda::kChunk) return 0;
    std::vector<HostPiece> pieces;
    if (!plan_pieces(cu_seqlens, num_seqs, total_tokens, piece_tokens, pieces)) return 0;
    return host_layout(pieces, num_seqs, H, d_k, d_v, out_dtype == KDA_DTYPE_F32).total;
}

kda_status kda_chunk_fwd_host(const void *q, const void *k, const void *v, const void *a, const float *beta,
                              const void *gate, const float *A_log, const int32_t *cu_seqlens, int32_t num_seqs,
                              int64_t total_tokens, int32_t H, int32_t d_k, int32_t d_v, float scale,
                              const float *initial_state, float *final_state, void *out, kda_dtype out_dtype,
                              int64_t piece_tokens, void *device_buffer, size_t device_buffer_bytes, void *stream) {
    if (total_tokens < 0 || num_seqs < 0 || H <= 0) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: negative size or H <= 0");
    if (!supported_dim(d_k) || !supported_dim(d_v))
        return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_fwd_host: d_k and d_v must be 64 or 128");
    if (num_seqs == 0) {
        if (total_tokens != 0) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: tokens without sequences");
        return KDA_OK;
    }
    if (!cu_seqlens || !A_log) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: NULL cu_seqlens or A_log");
    if (total_tokens > 0 && (!q || !k || !v || !a || !beta || !out))
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: NULL q/k/v/a/beta/out");
    if (out_dtype != KDA_DTYPE_BF16 && out_dtype != KDA_DTYPE_F32)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: out_dtype must be KDA_DTYPE_BF16 or KDA_DTYPE_F32");
    if (piece_tokens == 0) piece_tokens = kHostPieceDefault;
    if (piece_tokens < kda::kChunk) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: piece_tokens below 64");
    // cu_seqlens is read here on the host: it must be well formed
    if (cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != total_tokens)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: cu_seqlens must run from 0 to total_tokens");
    for (int32_t n = 0; n < num_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: cu_seqlens not monotone");
    std::vector<HostPiece> pieces;
    if (!plan_pieces(cu_seqlens, num_seqs, total_tokens, piece_tokens, pieces))
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: could not cut the batch into pieces");
    const bool f32_out = out_dtype == KDA_DTYPE_F32;
    const HostLayout L = host_layout(pieces, num_seqs, H, d_k, d_v, f32_out);
    if (!device_buffer || device_buffer_bytes < L.total)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: device buffer missing or too small (need " +
                                             std::to_string(L.total) + " bytes)");
    if ((reinterpret_cast<uintptr_t>(device_buffer) & 255u) != 0)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: device buffer not 256-byte aligned");

    // device buffer: [slot 0 | slot 1 | workspace | cu arrays + A_log | S in | S out]
    char *base = static_cast<char *>(device_buffer);
    char *ws = base + kHostSlots * L.slot_bytes;
    int32_t *d_cu = reinterpret_cast<int32_t *>(ws + L.ws_bytes);
    float *d_S = reinterpret_cast<float *>(ws + L.ws_bytes + L.cu_bytes);
    float *d_T = reinterpret_cast<float *>(reinterpret_cast<char *>(d_S) + L.state_bytes);
    // host copy of every piece's cu_seqlens, then A_log
    std::vector<int32_t> h_cu;
    std::vector<size_t> cu_off;
    for (const HostPiece &pc : pieces) {
        cu_off.push_back(h_cu.size());
        for (int32_t n = pc.n_lo; n <= pc.n_hi + 1; ++n)
            h_cu.push_back((int32_t)(std::min<int64_t>(std::max<int64_t>(cu_seqlens[n], pc.a), pc.e) - pc.a));
    }
    const size_t alog_off = h_cu.size();
    h_cu.resize(h_cu.size() + H);
    std::memcpy(h_cu.data() + alog_off, A_log, (size_t)H * 4);
    const float *d_Alog = reinterpret_cast<const float *>(d_cu + alog_off);

    cudaStream_t cs = static_cast<cudaStream_t>(stream);   // compute (the caller's stream)
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev_start = nullptr, ev_in[kHostSlots] = {}, ev_comp[kHostSlots] = {}, ev_out[kHostSlots] = {};
    cudaError_t e = cudaSuccess;
    auto cleanup = [&]() {
        for (int i = 0; i < kHostSlots; ++i) {
            if (ev_in[i]) cudaEventDestroy(ev_in[i]);
            if (ev_comp[i]) cudaEventDestroy(ev_comp[i]);
            if (ev_out[i]) cudaEventDestroy(ev_out[i]);
        }
        if (ev_start) cudaEventDestroy(ev_start);
        if (s_in) cudaStreamDestroy(s_in);      // released once their work completes
        if (s_out) cudaStreamDestroy(s_out);
    };
#define KDA_HOST_TRY(call, where)               \
    do {                                        \
        if ((e = (call)) != cudaSuccess) {      \
            cleanup();                          \
            return cuda_fail(e, where);         \
        }                                       \
    } while (0)
    KDA_HOST_TRY(cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking), "kda_chunk_fwd_host: stream");
    KDA_HOST_TRY(cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking), "kda_chunk_fwd_host: stream");
    KDA_HOST_TRY(cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming), "kda_chunk_fwd_host: event");
    for (int i = 0; i < kHostSlots; ++i) {
        KDA_HOST_TRY(cudaEventCreateWithFlags(&ev_in[i], cudaEventDisableTiming), "kda_chunk_fwd_host: event");
        KDA_HOST_TRY(cudaEventCreateWithFlags(&ev_comp[i], cudaEventDisableTiming), "kda_chunk_fwd_host: event");
        KDA_HOST_TRY(cudaEventCreateWithFlags(&ev_out[i], cudaEventDisableTiming), "kda_chunk_fwd_host: event");
    }
    // everything after what the caller queued before this call
    KDA_HOST_TRY(cudaEventRecord(ev_start, cs), "kda_chunk_fwd_host: record");
    KDA_HOST_TRY(cudaStreamWaitEvent(s_in, ev_start, 0), "kda_chunk_fwd_host: wait");
    KDA_HOST_TRY(cudaStreamWaitEvent(s_out, ev_start, 0), "kda_chunk_fwd_host: wait");
    KDA_HOST_TRY(cudaMemcpyAsync(d_cu, h_cu.data(), h_cu.size() * 4, cudaMemcpyHostToDevice, s_in), "kda_chunk_fwd_host: cu copy");
    const size_t state_bytes = (size_t)num_seqs * H * d_k * d_v * 4;
    if (initial_state)
        KDA_HOST_TRY(cudaMemcpyAsync(d_S, initial_state, state_bytes, cudaMemcpyHostToDevice, s_in), "kda_chunk_fwd_host: state copy");
    else
        KDA_HOST_TRY(cudaMemsetAsync(d_S, 0, state_bytes, s_in), "kda_chunk_fwd_host: state clear");

    const size_t SZ = (size_t)d_k * d_v;
    const size_t osz = f32_out ? 4 : 2;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t th_max = (size_t)L.max_tokens * H;
    for (size_t pi = 0; pi < pieces.size(); ++pi) {
        const HostPiece &pc = pieces[pi];
        const int slot = (int)(pi % kHostSlots);
        char *sb = base + slot * L.slot_bytes;
        char *dq = sb, *dk = dq + up(th_max * d_k * 2), *da = dk + up(th_max * d_k * 2);
        char *dv = da + up(th_max * d_k * 2), *dg = dv + up(th_max * d_v * 2);
        char *db = dg + up(th_max * d_v * 2), *dout = sb + L.in_bytes;
        const int64_t tok = pc.e - pc.a;
        const size_t rk = (size_t)H * d_k * 2, rv = (size_t)H * d_v * 2;
        // inputs of this piece into its slot, once the piece two back has consumed the slot
        if (pi >= kHostSlots) KDA_HOST_TRY(cudaStreamWaitEvent(s_in, ev_comp[slot], 0), "kda_chunk_fwd_host: wait");
        if (tok > 0) {
            KDA_HOST_TRY(cudaMemcpyAsync(dq, static_cast<const char *>(q) + pc.a * rk, tok * rk, cudaMemcpyHostToDevice, s_in), "kda_chunk_fwd_host: copy");
            KDA_HOST_TRY(cudaMemcpyAsync(dk, static_cast<const char *>(k) + pc.a * rk, tok * rk, cudaMemcpyHostToDevice, s_in), "kda_chunk_fwd_host: copy");
            KDA_HOST_TRY(cudaMemcpyAsync(da, static_cast<const char *>(a) + pc.a * rk, tok * rk, cudaMemcpyHostToDevice, s_in), "kda_chunk_fwd_host: copy");
            KDA_HOST_TRY(cudaMemcpyAsync(dv, static_cast<const char *>(v) + pc.a * rv, tok * rv, cudaMemcpyHostToDevice, s_in), "kda_chunk_fwd_host: copy");
            if (gate)
                KDA_HOST_TRY(cudaMemcpyAsync(dg, static_cast<const char *>(gate) + pc.a * rv, tok * rv, cudaMemcpyHostToDevice, s_in), "kda_chunk_fwd_host: copy");
            KDA_HOST_TRY(cudaMemcpyAsync(db, beta + pc.a * H, tok * H * 4, cudaMemcpyHostToDevice, s_in), "kda_chunk_fwd_host: copy");
        }
        KDA_HOST_TRY(cudaEventRecord(ev_in[slot], s_in), "kda_chunk_fwd_host: record");
        // the prefill of the piece, once its inputs are in and the piece two back has been copied out
        KDA_HOST_TRY(cudaStreamWaitEvent(cs, ev_in[slot], 0), "kda_chunk_fwd_host: wait");
        if (pi >= kHostSlots) KDA_HOST_TRY(cudaStreamWaitEvent(cs, ev_out[slot], 0), "kda_chunk_fwd_host: wait");
        const int32_t ns = pc.n_hi - pc.n_lo + 1;
        const kda_status st = kda_chunk_fwd(dq, dk, dv, da, reinterpret_cast<const float *>(db), gate ? dg : nullptr, d_Alog,
                                            d_cu + cu_off[pi], ns, tok, 0, H, d_k, d_v, scale, d_S + (size_t)pc.n_lo * H * SZ,
                                            d_T + (size_t)pc.n_lo * H * SZ, dout, out_dtype, ws, L.ws_bytes, cs);
        if (st != KDA_OK) {
            cleanup();
            return st;
        }
        if (pc.carry)   // the sequence continuing into the next piece starts there from this state
            KDA_HOST_TRY(cudaMemcpyAsync(d_S + (size_t)pc.n_hi * H * SZ, d_T + (size_t)pc.n_hi * H * SZ, H * SZ * 4,
                                         cudaMemcpyDeviceToDevice, cs), "kda_chunk_fwd_host: carry");
        KDA_HOST_TRY(cudaEventRecord(ev_comp[slot], cs), "kda_chunk_fwd_host: record");
        // the piece's outputs back to the host
        KDA_HOST_TRY(cudaStreamWaitEvent(s_out, ev_comp[slot], 0), "kda_chunk_fwd_host: wait");
        if (tok > 0)
            KDA_HOST_TRY(cudaMemcpyAsync(static_cast<char *>(out) + pc.a * H * d_v * osz, dout, tok * H * d_v * osz,
                                         cudaMemcpyDeviceToHost, s_out), "kda_chunk_fwd_host: copy out");
        KDA_HOST_TRY(cudaEventRecord(ev_out[slot], s_out), "kda_chunk_fwd_host: record");
    }
    if (final_state) {
        KDA_HOST_TRY(cudaStreamWaitEvent(s_out, ev_comp[(pieces.size() - 1) % kHostSlots], 0), "kda_chunk_fwd_host: wait");
        KDA_HOST_TRY(cudaMemcpyAsync(final_state, d_T, state_bytes, cudaMemcpyDeviceToHost, s_out), "kda_chunk_fwd_host: state out");
    }
    // the caller's stream reaches the end of the call once the last copy out is done
    KDA_HOST_TRY(cudaEventRecord(ev_out[0], s_out), "kda_chunk_fwd_host: record");
    KDA_HOST_TRY(cudaStreamWaitEvent(cs, ev_out[0], 0), "kda_chunk_fwd_host: wait");
#undef KDA_HOST_TRY
    cleanup();
    return KDA_OK;
}

// ---- the backward in chunkwise form ------------------------------------------------------------

namespace {

template <int DK, int DV>
kda_status launch_bwd_chunkwise(const kda::BwdParams &p, int64_t units, int64_t records, cudaStream_t st) {
    using SM = kda::BcSmem<DK, DV>;
    constexpr int G = DV / kda::kBcCols;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(kda::bc_prep_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kPrep)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(kda::bc_state_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kState)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(kda::bc_dstate_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kDState)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(kda::bc_grad_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kGrad)) != cudaSuccess)
        return cuda_fail(e, "cudaFuncSetAttribute(chunk_bwd_chunkwise)");
    kda::bc_prep_kernel<DK, DV><<<(unsigned)records, kda::kBcThreads, SM::kPrep, st>>>(p);
    kda::bc_state_kernel<DK, DV><<<(unsigned)(units * G), kda::kBcThreads, SM::kState, st>>>(p);
    kda::bc_dstate_kernel<DK, DV><<<(unsigned)(units * G), kda::kBcThreads, SM::kDState, st>>>(p);
    kda::bc_grad_kernel<DK, DV><<<(unsigned)records, kda::kBcThreads, SM::kGrad, st>>>(p);
    g_launches.fetch_add(4, std::memory_order_relaxed);
    e = cudaGetLastError();
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, "chunk_bwd_chunkwise launch");
}

size_t bc_record_floats(int d_k, int d_v) {
    if (d_k == 128 && d_v == 128) return kda::BcRec<128, 128>::kSize;
    if (d_k == 128 && d_v == 64) return kda::BcRec<128, 64>::kSize;
    if (d_k == 64 && d_v == 128) return kda::BcRec<64, 128>::kSize;
    return kda::BcRec<64, 64>::kSize;
}

}  // namespace

size_t kda_chunk_bwd_chunkwise_workspace_size(int64_t total_tokens, int32_t num_seqs, int32_t H, int32_t d_k,
                                              int32_t d_v) {
    if (total_tokens < 0 || num_seqs < 0 || H <= 0 || !supported_dim(d_k) || !supported_dim(d_v)) return 0;
    const size_t records = (size_t)(total_tokens / kda::kBcChunk + num_seqs) * H;   // >= sum ceil(len / 64) H
    return records * bc_record_floats(d_k, d_v) * 4;
}

kda_status kda_chunk_bwd_chunkwise(const void *q, const void *k, const void *v, const void *a, const float *beta,
                                   const void *gate, const float *A_log, const int32_t *cu_seqlens, int32_t num_seqs,
                                   int64_t total_tokens, int32_t H, int32_t d_k, int32_t d_v, float scale,
                                   const float *initial_state, const float *dout, const float *dfinal_state,
                                   float *dq, float *dk, float *dv, float *da, float *dbeta, float *dgate,
                                   float *dA_log, float *dinitial_state, void *workspace, size_t workspace_bytes,
                                   void *stream) {
    if (total_tokens < 0 || num_seqs < 0 || H <= 0) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd_chunkwise: negative size or H <= 0");
    if (!supported_dim(d_k) || !supported_dim(d_v))
        return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_bwd_chunkwise: d_k and d_v must be 64 or 128");
    if (num_seqs == 0) {
        if (total_tokens != 0) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd_chunkwise: tokens without sequences");
        return KDA_OK;
    }
    if (!cu_seqlens || !A_log || !dA_log) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd_chunkwise: NULL cu_seqlens, A_log or dA_log");
    if (total_tokens > 0 && (!q || !k || !v || !a || !beta || !dout || !dq || !dk || !dv || !da || !dbeta))
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd_chunkwise: NULL input or gradient pointer");
    if (gate && !dgate) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd_chunkwise: gate given without dgate");
    const void *ptrs[] = {q, k, v, a, gate, initial_state, dout, dfinal_state, dq, dk, dv, da, dgate,
                          dinitial_state, workspace};
    for (const void *ptr : ptrs)
        if (ptr && !aligned(ptr, 16)) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd_chunkwise: tensor pointer not 16-byte aligned");
    const void *ptrs4[] = {beta, A_log, cu_seqlens, dbeta, dA_log};
    for (const void *ptr : ptrs4)
        if (ptr && !aligned(ptr, 4)) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd_chunkwise: scalar array not 4-byte aligned");
    const size_t need = kda_chunk_bwd_chunkwise_workspace_size(total_tokens, num_seqs, H, d_k, d_v);
    if (!workspace || workspace_bytes < need)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd_chunkwise: workspace missing or too small (need " + std::to_string(need) + " bytes)");
    const int64_t units = (int64_t)num_seqs * H;
    const int64_t records = (total_tokens / kda::kBcChunk + num_seqs) * (int64_t)H;
    if (records > 0x7fffffffLL || units * (d_v / kda::kBcCols) > 0x7fffffffLL)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd_chunkwise: too many chunks or units");
    kda::BwdParams p{};
    p.ck_records = total_tokens / kda::kBcChunk + num_seqs;
    p.q = static_cast<const uint16_t *>(q);
    p.k = static_cast<const uint16_t *>(k);
    p.v = static_cast<const uint16_t *>(v);
    p.a = static_cast<const uint16_t *>(a);
    p.gate = static_cast<const uint16_t *>(gate);
    p.beta = beta;
    p.A_log = A_log;
    p.cu = cu_seqlens;
    p.S0 = initial_state;
    p.dout = dout;
    p.dS_T = dfinal_state;
    p.dq = dq; p.dk = dk; p.dv = dv; p.da = da; p.dbeta = dbeta; p.dgate = dgate;
    p.dA_log = dA_log;
    p.dS0 = dinitial_state;
    p.ckpt = static_cast<float *>(workspace);
    p.scratch = nullptr;
    p.total_tokens = total_tokens;
    p.num_seqs = num_seqs;
    p.H = H;
    p.scale = scale;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(dA_log, 0, sizeof(float) * H, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(dA_log)");
    if (d_k == 128 && d_v == 128) return launch_bwd_chunkwise<128, 128>(p, units, records, st);
    if (d_k == 128 && d_v == 64) return launch_bwd_chunkwise<128, 64>(p, units, records, st);
    if (d_k == 64 && d_v == 128) return launch_bwd_chunkwise<64, 128>(p, units, records, st);
    return launch_bwd_chunkwise<64, 64>(p, units, records, st);
}

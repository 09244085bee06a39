// libkda: C ABI entry points (declared in include/kda.h), argument validation and launches.
// The whole library is this one translation unit; kernels live in the included headers.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <mutex>
#include <cstring>
#include <string>

#include "kda.h"
#include "common.cuh"
#include "decode.cuh"
#include "prefill_simt.cuh"

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

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace of the chunkwise path: [running state | chunk records of one window].
size_t record_bytes(int d_k, int d_v) {
    const size_t floats = (size_t)kda::kChunk * (3 * d_k + d_v) + kda::kChunk * kda::kChunk + d_k;
    return round_up(floats * 4, 256);
}

size_t state_bytes(int32_t num_seqs, int32_t H, int d_k, int d_v) {
    return round_up((size_t)num_seqs * H * d_k * d_v * 4, 256);
}

int64_t max_chunks_of(int64_t total_tokens, int32_t max_seqlen) {
    const int64_t L = max_seqlen > 0 ? std::min<int64_t>(max_seqlen, total_tokens) : total_tokens;
    return (L + kda::kChunk - 1) / kda::kChunk;
}

bool sizes_ok(int64_t total_tokens, int32_t num_seqs, int32_t max_seqlen, int32_t H) {
    return total_tokens >= 0 && num_seqs >= 0 && max_seqlen >= 0 && H > 0;
}

constexpr size_t kDefaultWindowBudget = size_t(1) << 30;  // bytes of chunk records per window

template <int DK, int DV>
kda_status launch_chunk_fwd(const kda::PrepParams &pp0, const kda::StateParams &sp0,
                            int64_t windows, cudaStream_t stream) {
    const int prep_smem = kda::prep_smem_bytes<DK, DV>();
    const int state_smem = kda::state_smem_bytes<DK, DV>();
    cudaError_t e = cudaFuncSetAttribute(kda::prep_simt_kernel<DK, DV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, prep_smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prep)");
    e = cudaFuncSetAttribute(kda::state_simt_kernel<DK, DV>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, state_smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(state)");
    const int num_seqs = sp0.num_seqs;
    for (int64_t w = 0; w < windows; ++w) {
        kda::PrepParams pp = pp0;
        kda::StateParams sp = sp0;
        pp.chunk0 = sp.chunk0 = static_cast<int>(w * pp0.Wc);
        sp.first_window = w == 0;
        if (w > 0) sp.S_in = sp.S_out;
        if (sp0.max_chunks > 0) {
            dim3 grid((unsigned)(num_seqs * pp.Wc), (unsigned)pp.H);
            kda::prep_simt_kernel<DK, DV><<<grid, 256, prep_smem, stream>>>(pp);
            g_launches.fetch_add(1, std::memory_order_relaxed);
        }
        dim3 sgrid((unsigned)num_seqs, (unsigned)sp.H, DV / kda::kSlab);
        kda::state_simt_kernel<DK, DV><<<sgrid, 256, state_smem, stream>>>(sp);
        g_launches.fetch_add(1, std::memory_order_relaxed);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "chunk_fwd launch");
    }
    return KDA_OK;
}

template <int DK, int DV>
kda_status launch_decode(const kda::DecodeParams &p, int64_t units, cudaStream_t stream) {
    kda::decode_step_kernel<DK, DV><<<(unsigned)units, 256, 0, stream>>>(p);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, "decode_step launch");
}

// Built-in scratch for kda_chunk_fwd_noalloc (callers that cannot allocate).  Host code must not
// use this name as an address: it is a host-side stand-in; the device address comes from
// cudaGetSymbolAddress, looked up once per device below.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {};

}  // namespace

static __device__ __align__(256) unsigned char g_kda_static_scratch[kStaticScratchBytes];

namespace {

kda_status static_scratch_address(void **ptr) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd_noalloc: cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices)
        return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_fwd_noalloc: device ordinal out of range");
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_kda_static_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd_noalloc: cudaGetSymbolAddress");
        g_scratch_ptr[dev] = p;
    }
    *ptr = g_scratch_ptr[dev];
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
    }
    return "unknown status";
}

const char *kda_last_error(void) { return t_last_error.c_str(); }

uint64_t kda_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

size_t kda_chunk_fwd_workspace_min(int64_t total_tokens, int32_t num_seqs, int32_t max_seqlen,
                                   int32_t H, int32_t d_k, int32_t d_v) {
    if (!sizes_ok(total_tokens, num_seqs, max_seqlen, H) || !supported_dim(d_k) || !supported_dim(d_v))
        return 0;
    return state_bytes(num_seqs, H, d_k, d_v) + (size_t)num_seqs * H * record_bytes(d_k, d_v);
}

size_t kda_chunk_fwd_workspace_size(int64_t total_tokens, int32_t num_seqs, int32_t max_seqlen,
                                    int32_t H, int32_t d_k, int32_t d_v) {
    if (!sizes_ok(total_tokens, num_seqs, max_seqlen, H) || !supported_dim(d_k) || !supported_dim(d_v))
        return 0;
    const size_t per_row = (size_t)num_seqs * H * record_bytes(d_k, d_v);
    const int64_t max_chunks = std::max<int64_t>(1, max_chunks_of(total_tokens, max_seqlen));
    int64_t wc = per_row ? (int64_t)(kDefaultWindowBudget / per_row) : 1;
    wc = std::max<int64_t>(1, std::min<int64_t>(wc, max_chunks));
    return state_bytes(num_seqs, H, d_k, d_v) + per_row * (size_t)wc;
}

kda_status kda_chunk_fwd(const void *q, const void *k, const void *v, const void *a,
                         const float *beta, const void *gate, const float *A_log,
                         const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                         int32_t max_seqlen, int32_t H, int32_t d_k, int32_t d_v, float scale,
                         const float *initial_state, float *final_state, void *out,
                         kda_dtype out_dtype, void *workspace, size_t workspace_bytes,
                         void *stream) {
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
    if (!workspace) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: NULL workspace");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: workspace not 256-byte aligned");
    const size_t need = kda_chunk_fwd_workspace_min(total_tokens, num_seqs, max_seqlen, H, d_k, d_v);
    if (workspace_bytes < need)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: workspace too small (need " +
                                             std::to_string(need) + " bytes)");

    const int64_t max_chunks = max_chunks_of(total_tokens, max_seqlen);
    const size_t sbytes = state_bytes(num_seqs, H, d_k, d_v);
    const size_t per_row = (size_t)num_seqs * H * record_bytes(d_k, d_v);
    int64_t wc = (int64_t)((workspace_bytes - sbytes) / per_row);
    wc = std::max<int64_t>(1, std::min<int64_t>(wc, std::max<int64_t>(1, max_chunks)));
    wc = std::min<int64_t>(wc, (int64_t)(0x7fffffff / num_seqs));
    const int64_t windows = std::max<int64_t>(1, (max_chunks + wc - 1) / wc);

    char *ws = static_cast<char *>(workspace);
    float *run = final_state ? final_state : reinterpret_cast<float *>(ws);
    kda::PrepParams pp{};
    pp.q = static_cast<const uint16_t *>(q);
    pp.k = static_cast<const uint16_t *>(k);
    pp.v = static_cast<const uint16_t *>(v);
    pp.a = static_cast<const uint16_t *>(a);
    pp.beta = beta;
    pp.A_log = A_log;
    pp.cu = cu_seqlens;
    pp.rec = reinterpret_cast<float *>(ws + sbytes);
    pp.total_tokens = total_tokens;
    pp.num_seqs = num_seqs;
    pp.H = H;
    pp.Wc = (int)wc;
    pp.scale = scale;
    kda::StateParams sp{};
    sp.rec = pp.rec;
    sp.gate = static_cast<const uint16_t *>(gate);
    sp.out = out;
    sp.out_f32 = out_dtype == KDA_DTYPE_F32;
    sp.cu = cu_seqlens;
    sp.S_in = initial_state;
    sp.S_out = run;
    sp.total_tokens = total_tokens;
    sp.num_seqs = num_seqs;
    sp.H = H;
    sp.Wc = (int)wc;
    sp.max_chunks = (int)std::min<int64_t>(max_chunks, 0x7fffffff);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d_k == 128 && d_v == 128) return launch_chunk_fwd<128, 128>(pp, sp, windows, st);
    if (d_k == 128 && d_v == 64) return launch_chunk_fwd<128, 64>(pp, sp, windows, st);
    if (d_k == 64 && d_v == 128) return launch_chunk_fwd<64, 128>(pp, sp, windows, st);
    return launch_chunk_fwd<64, 64>(pp, sp, windows, st);
}

kda_status kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *a,
                                 const float *beta, const void *gate, const float *A_log,
                                 const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                                 int32_t max_seqlen, int32_t H, int32_t d_k, int32_t d_v,
                                 float scale, const float *initial_state, float *final_state,
                                 void *out, kda_dtype out_dtype, void *stream) {
    const size_t need = kda_chunk_fwd_workspace_min(total_tokens, num_seqs, max_seqlen, H, d_k, d_v);
    if (need > kStaticScratchBytes)
        return fail(KDA_ERR_INVALID_ARG,
                    "kda_chunk_fwd_noalloc: these sizes need " + std::to_string(need) +
                        " bytes of scratch, more than the " + std::to_string(kStaticScratchBytes) +
                        " built into the library; call kda_chunk_fwd with a workspace instead");
    void *scratch = nullptr;
    const kda_status st = static_scratch_address(&scratch);
    if (st != KDA_OK) return st;
    return kda_chunk_fwd(q, k, v, a, beta, gate, A_log, cu_seqlens, num_seqs, total_tokens,
                         max_seqlen, H, d_k, d_v, scale, initial_state, final_state, out,
                         out_dtype, scratch, kStaticScratchBytes, stream);
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
    return KDA_OK;
}

}  // extern "C"

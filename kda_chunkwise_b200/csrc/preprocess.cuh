// The two pieces of the KDA module around the recurrence that the pages name without giving their
// form ("K3 Architecture Illustrated", FIG 21: the actual module also has short convolution,
// normalisation and output gating; §"Why can K3's MLA use NoPE?": short convolution depends on
// input order).  Plainest readings:
//   short convolution: causal depthwise convolution over time within each sequence,
//       y_t[c] = sum_{j < W} w[h][c][j] x_{t - (W-1) + j}[c]      (x before the sequence start = 0)
//     with W <= 4 taps per channel, optionally followed by L2 normalisation of each (token, head)
//     row (the recurrence expects unit q and k);
//   pre-gate normalisation: RMS normalisation of each (token, head) output row with a per-channel
//     gain, then the sigmoid output gate:  out = sigmoid(gate) (.) o / sqrt(mean(o^2) + eps) (.) w.
// Both are HBM-bound streaming kernels: each thread owns 8 consecutive channels (a 16-byte piece of
// a row), and the row reductions are shuffles among the d/8 lanes that hold one (token, head).
#pragma once

#include "common.cuh"
#include "mma_frag.cuh"
#include "f32x2.cuh"

namespace kda {

constexpr int kConvMaxWidth = 4;
constexpr int kConvAhead = 16;        // input rows in flight per thread (a power of two)
constexpr int kPrepThreads = 256;
constexpr int kConvSmem = kConvAhead * kPrepThreads * 16;

struct ConvParams {
    const uint16_t *x;        // [T, H, d] bf16
    const float *w;           // [H, d, W]
    const int32_t *cu;        // [num_seqs + 1]
    uint16_t *y;              // [T, H, d] bf16
    int64_t total_tokens;
    int num_seqs, H, width;
    bool l2norm;
};

// first token of the sequence containing token t (cu_seqlens searched once per run)
__device__ __forceinline__ int seq_of(const int32_t *cu, int num_seqs, int64_t t) {
    int lo = 0, hi = num_seqs;   // invariant: cu[lo] <= t < cu[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cu[mid] <= t) lo = mid;
        else hi = mid;
    }
    return lo;
}

__device__ __forceinline__ void load8(const uint16_t *p, float (&v)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = bf16_to_f32(static_cast<uint16_t>(w4[i] & 0xFFFFu));
        v[2 * i + 1] = bf16_to_f32(static_cast<uint16_t>(w4[i] >> 16));
    }
}

__device__ __forceinline__ uint4 pack8_bf16(const float (&v)[8]) {
    uint32_t w4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w4[i] = (uint32_t)f32_to_bf16(v[2 * i]) | ((uint32_t)f32_to_bf16(v[2 * i + 1]) << 16);
    return make_uint4(w4[0], w4[1], w4[2], w4[3]);
}

// grid: x = runs of consecutive tokens (as many as fill the device once), y = blocks of
// kPrepThreads column groups (8 channels each, H d / 8 per token row).  A thread owns one column
// group for the whole run: its 8 channels' taps and the last W - 1 input rows stay in registers
// (each input is converted once), and its next kConvAhead input rows are always in flight --
// asynchronous 16-byte copies into a ring in shared memory that only this thread reads, so no
// barrier is needed and no registers are held for the rows in flight.
template <int D>
__global__ void __launch_bounds__(kPrepThreads) short_conv_kernel(const ConvParams p, int64_t run_len) {
    extern __shared__ __align__(16) uint4 conv_ring[];   // [kConvAhead][kPrepThreads]
    constexpr int LPH = D / 8;                        // lanes per (token, head) row
    const int64_t groups = (int64_t)p.H * LPH;        // 8-channel groups per token row
    const int64_t g = (int64_t)blockIdx.y * kPrepThreads + threadIdx.x;
    const bool active = g < groups;                   // whole (token, head) rows share a warp
    const int h = static_cast<int>(g / LPH);
    const int c0 = static_cast<int>(g % LPH) * 8;
    const int64_t t_begin = (int64_t)blockIdx.x * run_len;
    if (t_begin >= p.total_tokens) return;
    const int64_t t_end = min64(t_begin + run_len, p.total_tokens);
    const int W = p.width;
    const uint16_t *xcol = p.x + (int64_t)h * D + c0;   // row t at xcol + t H D
    const int64_t rstride = (int64_t)p.H * D;

    // the first kConvAhead rows of the run in flight (one commit group per row, empty past the end)
    const uint32_t ring = smem_u32(conv_ring) + threadIdx.x * 16;
#pragma unroll 1
    for (int i = 0; i < kConvAhead; ++i) {
        if (active && t_begin + i < t_end) cp_async_16(ring + i * kPrepThreads * 16, xcol + (t_begin + i) * rstride, 16);
        cp_async_commit();
    }

    // taps: slot k of the window holds x_{t-3+k}; the tap of x_{t-(W-1)+j} sits on slot 4 - W + j
    float wt[8][kConvMaxWidth - 1], wcur[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const float *wc = p.w + ((int64_t)h * D + c0 + c) * W;
#pragma unroll
        for (int k = 0; k < kConvMaxWidth - 1; ++k) {
            const int j = k - (kConvMaxWidth - W);
            wt[c][k] = (active && j >= 0) ? wc[j] : 0.f;
        }
        wcur[c] = active ? wc[W - 1] : 0.f;
    }
    const int k0 = kConvMaxWidth - W;   // first window slot with a tap
    // the same taps as channel pairs (2q, 2q + 1), for the paired fp32 instructions
    f32x2 wt2[4][kConvMaxWidth - 1], wcur2[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        wcur2[q] = f2_pack(wcur[2 * q], wcur[2 * q + 1]);
#pragma unroll
        for (int k = 0; k < kConvMaxWidth - 1; ++k) wt2[q][k] = f2_pack(wt[2 * q][k], wt[2 * q + 1][k]);
    }

    int s = seq_of(p.cu, p.num_seqs, t_begin);
    int64_t s_start = p.cu[s], s_end = p.cu[s + 1];
    // the window before the run: rows t_begin - 3 .. t_begin - 1 of the same sequence, else zero
    f32x2 win[kConvMaxWidth - 1][4];   // channel pairs
#pragma unroll
    for (int k = 0; k < kConvMaxWidth - 1; ++k) {
        const int64_t tk = t_begin - (kConvMaxWidth - 1) + k;
        float w8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (active && k >= k0 && tk >= s_start) load8(xcol + tk * rstride, w8);
#pragma unroll
        for (int q = 0; q < 4; ++q) win[k][q] = f2_pack(w8[2 * q], w8[2 * q + 1]);
    }

    const uint16_t *src = xcol + (t_begin + kConvAhead) * rstride;   // the next row to request
    uint16_t *dst = p.y + t_begin * rstride + (int64_t)h * D + c0;
    int slot = 0;
#pragma unroll 4
    for (int64_t t = t_begin; t < t_end; ++t) {
        cp_async_wait_group<kConvAhead - 1>();   // row t has landed
        const uint4 u = conv_ring[slot * kPrepThreads + threadIdx.x];
        // row t + kConvAhead into the slot just read (this thread's own slot: read, then refilled)
        if (active && t + kConvAhead < t_end) cp_async_16(ring + slot * (kPrepThreads * 16), src, 16);
        cp_async_commit();
        src += rstride;
        slot = (slot + 1) & (kConvAhead - 1);
        if (t >= s_end) {   // a new sequence starts here: its history is zero
            while (t >= s_end && s + 1 < p.num_seqs) { ++s; s_start = p.cu[s]; s_end = p.cu[s + 1]; }
            if (t >= s_end && threadIdx.x == 0) atomicOr(&g_kda_error_word, kErrBadSeqlens);
#pragma unroll
            for (int k = 0; k < kConvMaxWidth - 1; ++k)
#pragma unroll
                for (int q = 0; q < 4; ++q) win[k][q] = 0ull;
        }
        // the row's 8 channels as pairs (a bf16 pair widens to two fp32 by moving each half up)
        f32x2 xv[4];
        {
            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) xv[q] = f2_pack(__uint_as_float(w4[q] << 16), __uint_as_float(w4[q] & 0xFFFF0000u));
        }
        // y = w_cur x_t + sum of the window's taps, in the window's order (two channels per instruction)
        float y[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            f32x2 acc = f2_mul(wcur2[q], xv[q]);
#pragma unroll
            for (int k = 0; k < kConvMaxWidth - 1; ++k)
                if (k >= k0) acc = f2_fma(wt2[q][k], win[k][q], acc);
            f2_unpack(acc, y[2 * q], y[2 * q + 1]);
        }
        if (p.l2norm) {
            float ss = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) ss = fmaf(y[c], y[c], ss);
#pragma unroll
            for (int o = LPH / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            const float inv = rsqrtf(ss + 1e-12f);
#pragma unroll
            for (int c = 0; c < 8; ++c) y[c] *= inv;
        }
        if (active) *reinterpret_cast<uint4 *>(dst) = pack8_bf16(y);
        dst += rstride;
        // slide the window
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            win[0][q] = win[1][q];
            win[1][q] = win[2][q];
            win[2][q] = xv[q];
        }
    }
    cp_async_wait_all();   // nothing left in flight at exit
}

struct NormGateParams {
    const float *o;           // [T, H, d] fp32
    const uint16_t *gate;     // [T, H, d] bf16 or null
    const float *w;           // [d]
    void *out;                // [T, H, d] bf16 or fp32
    int64_t rows;             // T * H
    float eps;
    bool out_f32;
};

template <int D>
__global__ void __launch_bounds__(kPrepThreads) norm_gate_kernel(const NormGateParams p) {
    constexpr int LPH = D / 8;
    const int64_t g = (int64_t)blockIdx.x * kPrepThreads + threadIdx.x;
    const int64_t row = g / LPH;
    const int c0 = static_cast<int>(g % LPH) * 8;
    const bool active = row < p.rows;
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (active) {
        const float4 *src = reinterpret_cast<const float4 *>(p.o + row * D + c0);
        const float4 a = __ldcs(src), b = __ldcs(src + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) ss = fmaf(v[c], v[c], ss);
#pragma unroll
    for (int o = LPH / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(ss / D + p.eps);
    if (!active) return;
    float gt[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (p.gate) load8(p.gate + row * D + c0, gt);
    float y[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        y[c] = v[c] * inv * __ldg(p.w + c0 + c);
        if (p.gate) y[c] *= sigmoid_fast(gt[c]);
    }
    if (p.out_f32) {
        float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.out) + row * D + c0);
        dst[0] = make_float4(y[0], y[1], y[2], y[3]);
        dst[1] = make_float4(y[4], y[5], y[6], y[7]);
    } else {
        *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.out) + row * D + c0) = pack8_bf16(y);
    }
}

}  // namespace kda

// Output gate of the prefill kernels: sigmoid of a pair of bf16 gate logits, in the precision the
// output is stored in.
#pragma once

#include "mma_frag.cuh"

namespace kda {

// sigmoid of a pair of bf16 gate logits as 1/2 + tanh(x/2)/2, the tanh on the fp16x2 unit: one
// MUFU operation per pair instead of four (exp2 and reciprocal per value).  Absolute error at most
// 2.5e-4 over all bf16 logits: an eighth of the bf16 rounding (2^-9 relative) of an ungated output
// value, so it is used only where the gated output is stored in bf16.  x beyond the fp16 range
// saturates to 0 or 1 as the sigmoid does.
__device__ __forceinline__ float2 gate_sigmoid2(uint32_t g) {
    const float2 x = unpack_bf16(g);
    uint32_t t;
    asm("tanh.approx.f16x2 %0, %1;\n" : "=r"(t) : "r"(pack_f16(0.5f * x.x, 0.5f * x.y)));
    const float2 tf = unpack_f16(t);
    return make_float2(fmaf(0.5f, tf.x, 0.5f), fmaf(0.5f, tf.y, 0.5f));
}

// The same sigmoid to fp32 accuracy, for fp32 outputs: 1 / (1 + 2^(-x log2 e)) with the hardware
// exp2 and reciprocal approximations (relative error about 2^-21 over the whole range; x far below
// zero makes the power inf and the result 0, the sigmoid's limit).
__device__ __forceinline__ float2 gate_sigmoid2_f32(uint32_t g) {
    const float2 x = unpack_bf16(g);
    float e0, e1, r0, r1;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(e0) : "f"(-1.4426950408889634f * x.x));
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(e1) : "f"(-1.4426950408889634f * x.y));
    asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(r0) : "f"(1.0f + e0));
    asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(r1) : "f"(1.0f + e1));
    return make_float2(r0, r1);
}

}  // namespace kda

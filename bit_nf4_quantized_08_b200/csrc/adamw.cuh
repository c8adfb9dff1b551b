// adamw.cuh -- the optimizer step of the adapters and paged optimizer state.
//
// Only the LoRA matrices A and B train (QLoRA paper digest, sec. 4 steps:
// Adam updates L1 and L2 only; the frozen 4-bit weight gets no update).  One
// launch updates every adapter parameter of a block, laid out as one flat
// fp32 master copy with its fp32 first and second moments and its fp32
// gradient (the dA and dB the backward writes), and refreshes the bf16 copy
// that the linear calls read.  The update is decoupled weight decay (AdamW):
//   p  <- p * (1 - lr * wd)
//   m  <- b1 m + (1 - b1) g            v <- b2 v + (1 - b2) g^2
//   p  <- p - (lr / (1 - b1^t)) * m / (sqrt(v) / sqrt(1 - b2^t) + eps)
// in fp32, in that order.  It is bound by HBM bytes: 16 B read (p, m, v, g)
// and 14 B written (p, m, v, bf16 p) per parameter.  Grid-stride loop over
// 4-element vectors, 16-byte loads and stores.
//
// Paged state (blog note sec. 4 and tutorial "paged optimizers": optimizer
// states in unified memory move to host RAM when the GPU runs short and back
// when they are needed): the moments may live in managed memory; the kernel
// reads them through the same pointers, and the driver migrates the pages on
// demand or ahead of time on a prefetch.
#pragma once

#include "common.cuh"

namespace qlora {

struct AdamWParams {
    float* p;            // fp32 master parameters [n]
    float* m;            // fp32 first moment [n]
    float* v;            // fp32 second moment [n]
    const float* g;      // fp32 gradient [n]
    uint16_t* p_bf16;    // bf16 copy of the parameters [n] (written), may be null
    int64_t n;
    float lr, b1, b2, eps, decay;  // decay = 1 - lr * weight_decay
    float step_size;     // lr / (1 - b1^t)
    float rsqrt_bc2;     // 1 / sqrt(1 - b2^t)
    float grad_scale;
};

__device__ __forceinline__ float adamw_one(float p, float& m, float& v, float g, const AdamWParams& a) {
    g = __fmul_rn(g, a.grad_scale);
    p = __fmul_rn(p, a.decay);
    m = __fadd_rn(__fmul_rn(a.b1, m), __fmul_rn(1.0f - a.b1, g));
    v = __fadd_rn(__fmul_rn(a.b2, v), __fmul_rn(__fmul_rn(1.0f - a.b2, g), g));
    const float denom = __fadd_rn(__fmul_rn(__fsqrt_rn(v), a.rsqrt_bc2), a.eps);
    return __fsub_rn(p, __fmul_rn(a.step_size, __fdiv_rn(m, denom)));
}

__global__ void __launch_bounds__(256) k_adamw(const __grid_constant__ AdamWParams a) {
    const int64_t nv = a.n / 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += stride) {
        float4 p = __ldcs(reinterpret_cast<const float4*>(a.p) + i);
        float4 m = __ldcs(reinterpret_cast<const float4*>(a.m) + i);
        float4 v = __ldcs(reinterpret_cast<const float4*>(a.v) + i);
        const float4 g = __ldcs(reinterpret_cast<const float4*>(a.g) + i);
        p.x = adamw_one(p.x, m.x, v.x, g.x, a);
        p.y = adamw_one(p.y, m.y, v.y, g.y, a);
        p.z = adamw_one(p.z, m.z, v.z, g.z, a);
        p.w = adamw_one(p.w, m.w, v.w, g.w, a);
        __stcs(reinterpret_cast<float4*>(a.p) + i, p);
        __stcs(reinterpret_cast<float4*>(a.m) + i, m);
        __stcs(reinterpret_cast<float4*>(a.v) + i, v);
        if (a.p_bf16)
            __stcs(reinterpret_cast<uint2*>(a.p_bf16) + i, make_uint2(pack_bf16x2(p.x, p.y), pack_bf16x2(p.z, p.w)));
    }
    // tail (n % 4 elements)
    for (int64_t i = nv * 4 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < a.n; i += stride) {
        float m = a.m[i], v = a.v[i];
        const float p = adamw_one(a.p[i], m, v, a.g[i], a);
        a.p[i] = p;
        a.m[i] = m;
        a.v[i] = v;
        if (a.p_bf16) a.p_bf16[i] = (uint16_t)(pack_bf16x2(p, 0.0f) & 0xFFFFu);
    }
}

}  // namespace qlora

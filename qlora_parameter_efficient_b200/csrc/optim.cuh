// optim.cuh -- the adapter optimizer step: AdamW with an fp32 master copy and fp32 moments.
//
// "Low-Rank Adaptation (LoRA) and QLoRA: Mathematical Foundations...", section "The Memory
// Bottleneck of Full Parameter Fine-Tuning": AdamW keeps, per trainable parameter, an fp32
// master copy, the first moment m and the second moment v; with the base frozen only the
// adapter parameters carry them.  The pages print no update rule; this is the published
// decoupled-weight-decay AdamW, with the gradient first multiplied by grad_scale (the
// reciprocal of the number of accumulated micro-batches):
//   g' = grad_scale g;  m = b1 m + (1 - b1) g';  v = b2 v + (1 - b2) g'^2
//   w  = w (1 - lr wd) - lr (m / bc1) / (sqrt(v / bc2) + eps),   bc = 1 - b^t
// in fp32 (bc1, bc2 formed on the host in double).  A bf16 parameter is the round-to-nearest-
// even copy of the updated master.  The state may live in unified memory ("paged
// optimizers": "Large Language Model Fine-tuning and LoRA", section "Paged optimizers"): the
// kernel only reads and writes it, the driver migrates its pages.
//
// One element per thread-iteration, 4 consecutive elements per thread as 16-byte vectors when
// every array is 16-byte aligned and n is a multiple of 4; the kernel streams 30 bytes per bf16
// parameter (grad, master, m, v read; master, m, v, parameter written) and is HBM-bound.
#pragma once

#include "common.cuh"

namespace qlora {

struct AdamArgs {
    int64_t n;
    float lr, beta1, beta2, eps, wd, grad_scale;
    float bc1, bc2;                  // 1 - beta^t
};

__device__ __forceinline__ void adam_update(float& w, float& m, float& v, float g, const AdamArgs& a) {
    g *= a.grad_scale;
    m = a.beta1 * m + (1.f - a.beta1) * g;
    v = a.beta2 * v + (1.f - a.beta2) * g * g;
    const float mhat = m / a.bc1;
    const float denom = sqrtf(v / a.bc2) + a.eps;
    w = w * (1.f - a.lr * a.wd) - a.lr * mhat / denom;
}

// TP: float (param is the master, updated in place) or __nv_bfloat16 (master separate).
template <typename TP, bool VEC>
__global__ void __launch_bounds__(256) k_adamw(TP* __restrict__ param, float* __restrict__ master,
                                               const float* __restrict__ grad, float* __restrict__ m,
                                               float* __restrict__ v, AdamArgs a) {
    griddep_enter();
    float* wsrc = sizeof(TP) == 4 ? reinterpret_cast<float*>(param) : master;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    if constexpr (VEC) {
        for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < a.n / 4; q += stride) {
            float4 w4 = reinterpret_cast<const float4*>(wsrc)[q];
            float4 m4 = reinterpret_cast<const float4*>(m)[q];
            float4 v4 = reinterpret_cast<const float4*>(v)[q];
            const float4 g4 = reinterpret_cast<const float4*>(grad)[q];
            adam_update(w4.x, m4.x, v4.x, g4.x, a);
            adam_update(w4.y, m4.y, v4.y, g4.y, a);
            adam_update(w4.z, m4.z, v4.z, g4.z, a);
            adam_update(w4.w, m4.w, v4.w, g4.w, a);
            reinterpret_cast<float4*>(wsrc)[q] = w4;
            reinterpret_cast<float4*>(m)[q] = m4;
            reinterpret_cast<float4*>(v)[q] = v4;
            if constexpr (sizeof(TP) == 2) {
                uint2 p;
                p.x = pack_bf16x2(w4.x, w4.y);
                p.y = pack_bf16x2(w4.z, w4.w);
                reinterpret_cast<uint2*>(param)[q] = p;
            }
        }
    } else {
        for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < a.n; i += stride) {
            float w = wsrc[i], mm = m[i], vv = v[i];
            adam_update(w, mm, vv, grad[i], a);
            wsrc[i] = w;
            m[i] = mm;
            v[i] = vv;
            if constexpr (sizeof(TP) == 2) param[i] = __float2bfloat16_rn(w);
        }
    }
}

}  // namespace qlora

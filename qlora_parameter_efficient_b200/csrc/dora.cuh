// dora.cuh -- the DoRA backward's element-wise and small kernels (the two weight passes reuse the
// fused NF4 GEMM with the adapter rows as tokens, the rest of the backward is the LoRA one), and
// the scale pass of the forward that keeps the pre-scale output Z for the backward.
//
// DoRA with one magnitude per output row ("Large Language Model Fine-tuning and LoRA", section
// "Choosing what to adapt: targets and rank"; "Low-Rank Adaptation (LoRA) and QLoRA:
// Mathematical Foundations...", section "Advanced Variants: DoRA and LoRA+"): V = W^ + s B A,
// n_j = ||V[j, :]||, c_j = m_j / n_j, Z = X V^T and H = Z diag(c).  The backward is the chain
// rule through every factor, the norm included:
//   dZ = dH diag(c);  dc_j = sum_t dH[t, j] Z[t, j];  dm_j = dc_j / n_j;  e_j = -dc_j m_j / n_j^3
//   dX, dA, dB = the LoRA backward of dZ, plus the norm's term through V = W^ + s B A:
//   dB += s diag(e) (W^ A^T + s B (A A^T)),   dA += s (B^T diag(e) W^ + s (B^T diag(e) B) A)
// A row of norm 0 contributes nothing (c = e = dm = 0).
#pragma once

#include "common.cuh"

namespace qlora {

constexpr int kDoraChunks = 32;     // token chunks of the column reduction

// dZ = bf16(dH c) and per-chunk partials of dc_j = sum_t dH[t, j] Z[t, j] (fp32, tokens in order
// within a chunk).  Thread: two adjacent columns; CTA y: token chunk y.
__global__ void __launch_bounds__(256) k_dora_colred(const __nv_bfloat16* __restrict__ dH,
                                                     const __nv_bfloat16* __restrict__ Z,
                                                     const float* __restrict__ magnitude,
                                                     const float* __restrict__ norms, int64_t T,
                                                     int64_t d, __nv_bfloat16* __restrict__ dZ,
                                                     float* __restrict__ part) {
    griddep_enter();
    const int64_t j = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x);
    if (j >= d) return;
    const bool two = j + 1 < d;
    const bool pairs = (d & 1) == 0;                  // rows of whole bf16 pairs (4-byte aligned)
    const int64_t t0 = (T * blockIdx.y) / gridDim.y, t1 = (T * (blockIdx.y + 1)) / gridDim.y;
    const float n0 = norms[j], n1 = two ? norms[j + 1] : 0.f;
    const float c0 = n0 > 0.f ? magnitude[j] / n0 : 0.f;
    const float c1 = n1 > 0.f ? magnitude[j + 1] / n1 : 0.f;
    float a0 = 0.f, a1 = 0.f;
#pragma unroll 4
    for (int64_t t = t0; t < t1; ++t) {
        float2 gv, zv;
        if (pairs) {
            gv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dH + t * d + j));
            zv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(Z + t * d + j));
        } else {
            gv = make_float2(__bfloat162float(dH[t * d + j]), two ? __bfloat162float(dH[t * d + j + 1]) : 0.f);
            zv = make_float2(__bfloat162float(Z[t * d + j]), two ? __bfloat162float(Z[t * d + j + 1]) : 0.f);
        }
        a0 = fmaf(gv.x, zv.x, a0);
        a1 = fmaf(gv.y, zv.y, a1);
        if (pairs) {
            *reinterpret_cast<__nv_bfloat162*>(dZ + t * d + j) = __floats2bfloat162_rn(gv.x * c0, gv.y * c1);
        } else {
            dZ[t * d + j] = __float2bfloat16_rn(gv.x * c0);
            if (two) dZ[t * d + j + 1] = __float2bfloat16_rn(gv.y * c1);
        }
    }
    part[blockIdx.y * d + j] = a0;
    if (two) part[blockIdx.y * d + j + 1] = a1;
}

// dc (chunks in order), dm = dc / n and e = -dc m / n^3 (0 for a row of norm 0)
__global__ void k_dora_coef(const float* __restrict__ part, int chunks, int64_t d,
                            const float* __restrict__ magnitude, const float* __restrict__ norms,
                            float* __restrict__ dm, float* __restrict__ e) {
    griddep_enter();
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < d;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float dc = 0.f;
        for (int c = 0; c < chunks; ++c) dc += part[c * d + j];
        const float n = norms[j];
        dm[j] = n > 0.f ? dc / n : 0.f;
        e[j] = n > 0.f ? -dc * magnitude[j] / (n * n * n) : 0.f;
    }
}

// Ge[i][j] = bf16(B[j][i] e_j): the rows B^T diag(e) that the dX-form GEMM multiplies by W^ (row
// stride ld >= d, a multiple of 8 so that the GEMM's tensor map can read it; columns past d are
// zero)
__global__ void k_dora_ge(const __nv_bfloat16* __restrict__ B, const float* __restrict__ e, int r,
                          int64_t d, int64_t ld, __nv_bfloat16* __restrict__ ge) {
    griddep_enter();
    for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < r * ld;
         x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t i = x / ld, j = x % ld;
        ge[x] = __float2bfloat16_rn(j < d ? __bfloat162float(B[j * r + i]) * e[j] : 0.f);
    }
}

// The r x r Gram products AAt[i][l] = sum_k A[i][k] A[l][k] (which = 0) and
// BeB[i][l] = sum_j B[j][i] e_j B[j][l] (which = 1), fp32; one CTA per (i, l), a fixed-order
// tree over its 256 threads.
__global__ void __launch_bounds__(256) k_dora_gram(const __nv_bfloat16* __restrict__ A,
                                                   const __nv_bfloat16* __restrict__ B,
                                                   const float* __restrict__ e, int r, int64_t d,
                                                   int64_t k, float* __restrict__ aat,
                                                   float* __restrict__ beb) {
    griddep_enter();
    __shared__ float red[256];
    const int i = blockIdx.x / r, l = blockIdx.x % r;
    const int which = blockIdx.y;
    float acc = 0.f;
    if (which == 0) {
        for (int64_t c = threadIdx.x; c < k; c += blockDim.x)
            acc = fmaf(__bfloat162float(A[i * k + c]), __bfloat162float(A[l * k + c]), acc);
    } else {
        for (int64_t j = threadIdx.x; j < d; j += blockDim.x)
            acc = fmaf(__bfloat162float(B[j * r + i]) * e[j], __bfloat162float(B[j * r + l]), acc);
    }
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) (which == 0 ? aat : beb)[i * r + l] = red[0];
}

// dB[j][i] += s e_j (P[i][j] + s sum_l B[j][l] AAt[l][i]),  P = A W^T (r x d, bf16)
__global__ void k_dora_add_db(const __nv_bfloat16* __restrict__ P, const __nv_bfloat16* __restrict__ B,
                              const float* __restrict__ aat, const float* __restrict__ e, int r,
                              int64_t d, float s, float* __restrict__ dB) {
    griddep_enter();
    for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < d * r;
         x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t j = x / r;
        const int i = static_cast<int>(x % r);
        float v = 0.f;
        for (int l = 0; l < r; ++l) v = fmaf(__bfloat162float(B[j * r + l]), aat[l * r + i], v);
        dB[x] += s * e[j] * (__bfloat162float(P[i * d + j]) + s * v);
    }
}

// dA[i][c] += s (Q[i][c] + s sum_l BeB[i][l] A[l][c]),  Q = B^T diag(e) W^ (r x k, bf16)
__global__ void k_dora_add_da(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ A,
                              const float* __restrict__ beb, int r, int64_t k, float s,
                              float* __restrict__ dA) {
    griddep_enter();
    for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < r * k;
         x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int i = static_cast<int>(x / k);
        const int64_t c = x % k;
        float v = 0.f;
        for (int l = 0; l < r; ++l) v = fmaf(beb[i * r + l], __bfloat162float(A[l * k + c]), v);
        dA[x] += s * (__bfloat162float(Q[x]) + s * v);
    }
}

// H[t, j] = bf16(Z[t, j] c_j), c_j = m_j / n_j (0 where n_j = 0): the DoRA output from the saved
// pre-scale output.  Eight elements per thread when rows are whole 16-byte units, else one.
__global__ void k_dora_apply(const __nv_bfloat16* __restrict__ Z, const float* __restrict__ magnitude,
                             const float* __restrict__ norms, int64_t T, int64_t d,
                             __nv_bfloat16* __restrict__ H) {
    griddep_enter();
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    auto coef = [&](int64_t j) {
        const float n = norms[j];
        return n > 0.f ? magnitude[j] / n : 0.f;
    };
    if ((d & 7) == 0) {
        const int64_t n8 = T * d / 8;
        for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
            const int64_t j0 = (i * 8) % d;
            const uint4 z = reinterpret_cast<const uint4*>(Z)[i];
            const uint32_t zw[4] = {z.x, z.y, z.z, z.w};
            uint32_t hw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                __nv_bfloat162 v;
                *reinterpret_cast<uint32_t*>(&v) = zw[e];
                const float2 f = __bfloat1622float2(v);
                const __nv_bfloat162 h = __floats2bfloat162_rn(f.x * coef(j0 + 2 * e), f.y * coef(j0 + 2 * e + 1));
                hw[e] = *reinterpret_cast<const uint32_t*>(&h);
            }
            reinterpret_cast<uint4*>(H)[i] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        }
    } else {
        for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < T * d; i += stride)
            H[i] = __float2bfloat16_rn(__bfloat162float(Z[i]) * coef(i % d));
    }
}

}  // namespace qlora

// fp8.cuh -- FP8 (E4M3) activations: the per-tensor scale and the activation quantizer, the
// weight's scale, and the low-rank pre-pass that reads the E4M3 activation.
//
// "LoRA and QLoRA Fine-Tuning Under the Hood", section "1.3 Activation Memory Savings via
// FlashAttention-2 & Activation Checkpointing": activations held in the FP8 formats (E4M3,
// E5M2) that Blackwell's tensor cores take natively halve the activation bytes.  Here:
//   sigma = 2^(8 - ceil(log2 amax))       (1 for amax = 0; exponent kept in [-126, 126])
//   X8    = E4M3(fl32(x * sigma))         round to nearest even, saturating at 448
// so amax * sigma lies in (128, 256] and X ~ X8 / sigma.  A power-of-two scale makes every
// rescaling exact.  The weight's scale sigma_w comes from the largest second-level constant
// (every decoded weight is L * s_b with |L| <= 1 and s_b <= c2 of its group).  The upstream
// gradient of the backward takes E5M2 (range to 57344) with sigma = 2^(15 - ceil(log2 amax)).
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace qlora {

// 2^(top - ceil(log2 amax)); top = 8 (E4M3) or 15 (E5M2)
__device__ __forceinline__ float fp8_pow2_scale(float amax, int top = 8) {
    if (!(amax > 0.f)) return 1.f;
    const uint32_t b = __float_as_uint(amax);
    const int e = static_cast<int>((b >> 23) & 255u);
    const uint32_t m = b & 0x7FFFFFu;
    int c;                                        // ceil(log2 amax)
    if (e == 0) {                                 // subnormal: amax = m 2^-149
        const int hb = 31 - __clz(m);
        c = hb - 149 + ((m & (m - 1)) ? 1 : 0);
    } else {
        c = e - 127 + (m ? 1 : 0);
    }
    const int k = min(max(top - c, -126), 126);
    return __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
}

__device__ __forceinline__ float block_max_256(float m, float* s_red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s_red[warp] = m;
    __syncthreads();
    float r = s_red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) r = fmaxf(r, s_red[i]);
    return r;
}

// max |x| over n bf16 values into *amax_bits (fp32 bits, zero before the launch).  NaNs are
// ignored.  256 threads per block.
__global__ void __launch_bounds__(256) k_fp8_amax(const __nv_bfloat16* __restrict__ X, int64_t n,
                                                  unsigned* __restrict__ amax_bits) {
    griddep_enter();
    __shared__ float s_red[8];
    float m = 0.f;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t n8 = n / 8;
    for (int64_t i = i0; i < n8; i += stride) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(X) + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            m = fmaxf(m, fabsf(__uint_as_float(w[k] << 16)));
            m = fmaxf(m, fabsf(__uint_as_float(w[k] & 0xFFFF0000u)));
        }
    }
    for (int64_t i = n8 * 8 + i0; i < n; i += stride) m = fmaxf(m, fabsf(__bfloat162float(X[i])));
    m = block_max_256(m, s_red);
    if (threadIdx.x == 0 && m > 0.f) atomicMax(amax_bits, __float_as_uint(m));
}

// X8 = E4M3 (or E5M2) of fl32(x * sigma), sigma from the amax; block 0 stores sigma into *scale.
template <bool E5M2>
__global__ void __launch_bounds__(256) k_fp8_quant(const __nv_bfloat16* __restrict__ X, int64_t n,
                                                   const unsigned* __restrict__ amax_bits,
                                                   uint8_t* __restrict__ X8, float* __restrict__ scale) {
    griddep_enter();
    constexpr __nv_fp8_interpretation_t kFmt = E5M2 ? __NV_E5M2 : __NV_E4M3;
    const float sig = fp8_pow2_scale(__uint_as_float(*amax_bits), E5M2 ? 15 : 8);
    if (blockIdx.x == 0 && threadIdx.x == 0) *scale = sig;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t n8 = n / 8;
    for (int64_t i = i0; i < n8; i += stride) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(X) + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t b[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            b[k] = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(
                make_float2(__fmul_rn(__uint_as_float(w[k] << 16), sig),
                            __fmul_rn(__uint_as_float(w[k] & 0xFFFF0000u), sig)),
                __NV_SATFINITE, kFmt));
        reinterpret_cast<uint2*>(X8)[i] = make_uint2(b[0] | (b[1] << 16), b[2] | (b[3] << 16));
    }
    for (int64_t i = n8 * 8 + i0; i < n; i += stride)
        X8[i] = static_cast<uint8_t>(
            __nv_cvt_float_to_fp8(__fmul_rn(__bfloat162float(X[i]), sig), __NV_SATFINITE, kFmt));
}

// dst = bf16(value(src) / sigma) for n FP8 bytes: exact (every E4M3 / E5M2 value times a power
// of two is a bf16 value), the stored activation or gradient back in its own units.
template <bool E5M2>
__global__ void __launch_bounds__(256) k_fp8_dequant(const uint8_t* __restrict__ src, int64_t n,
                                                     const float* __restrict__ scale,
                                                     __nv_bfloat16* __restrict__ dst) {
    griddep_enter();
    constexpr __nv_fp8_interpretation_t kFmt = E5M2 ? __NV_E5M2 : __NV_E4M3;
    const float inv = __frcp_rn(__ldg(scale));
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t n8 = n / 8;
    for (int64_t i = i0; i < n8; i += stride) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(src) + i);
        const uint32_t w[2] = {v.x, v.y};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
                    static_cast<__nv_fp8x2_storage_t>((w[k] >> (16 * h)) & 0xFFFFu), kFmt);
                const float2 f = __half22float2(__half2(hr));
                o[2 * k + h] = pack_bf16x2(__fmul_rn(f.x, inv), __fmul_rn(f.y, inv));
            }
        }
        reinterpret_cast<uint4*>(dst)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    for (int64_t i = n8 * 8 + i0; i < n; i += stride) {
        const __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(src[i]), kFmt);
        dst[i] = __float2bfloat16_rn(__fmul_rn(__half2float(__half(hr)), inv));
    }
}

// dst = bf16(src * a * b) for n bf16 values, a and b device scalars (powers of two: exact).
__global__ void __launch_bounds__(256) k_scale2_bf16(const __nv_bfloat16* __restrict__ src, int64_t n,
                                                     const float* __restrict__ a, const float* __restrict__ b,
                                                     __nv_bfloat16* __restrict__ dst) {
    griddep_enter();
    const float f = __fmul_rn(__ldg(a), __ldg(b));
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        dst[i] = __float2bfloat16_rn(__fmul_rn(__bfloat162float(src[i]), f));
}

// sigma_w of a stored weight from its n second-level constants; one block of 256 threads.
__global__ void __launch_bounds__(256) k_fp8_wscale(const float* __restrict__ c2, int64_t n,
                                                    float* __restrict__ w_scale) {
    griddep_enter();
    __shared__ float s_red[8];
    float m = 0.f;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, c2[i]);
    m = block_max_256(m, s_red);
    if (threadIdx.x == 0) *w_scale = fp8_pow2_scale(m);
}

// Two E4M3 bytes (low byte first) to a bf16x2 word; exact (E4M3 values are bf16 values).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t v) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(v & 0xFFFFu), __NV_E4M3);
    const float2 f = __half22float2(__half2(h));
    return pack_bf16x2(f.x, f.y);
}

// The low-rank pre-pass on the E4M3 activation, 16 tokens per CTA:
//   U'[t, j] = bf16(fl32(s * sigma_w) * sum_k X8v[t, k] A[j, k])   (j < r; zero for r <= j < ldu)
// X8v the E4M3 values of X8 (X times sigma_x), so U' = sigma_x sigma_w bf16(s X A^T) up to the
// activation's rounding: the adapter term in the units of the FP8 accumulator.  fp32
// accumulation with mma.sync m16n8k16; the WARPS warps split K in 64-wide chunks (each warp
// issuing the loads of UNR chunks before their MMAs, to keep many loads in flight) and their
// partials are summed in a fixed order.  Within a chunk, thread quad t owns the 16 consecutive
// columns 16t..16t+15 of both operands (the same permutation of K for A and B leaves every dot
// product unchanged), so each operand fragment is one contiguous load.
template <int NT, int WARPS, int UNR>
__global__ void __launch_bounds__(32 * WARPS) k_fp8_u(const uint8_t* __restrict__ X8, int64_t T, int d_in,
                                                      const __nv_bfloat16* __restrict__ A, int r, float s,
                                                      const float* __restrict__ w_scale,
                                                      __nv_bfloat16* __restrict__ U, int ldu) {
    griddep_enter();
    __shared__ float s_part[WARPS][16][NT * 8 + 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * 16;
    const int64_t ra = t0 + g, rb = t0 + g + 8;
    const uint8_t* xa = X8 + (ra < T ? ra : 0) * d_in + 16 * t;
    const uint8_t* xb = X8 + (rb < T ? rb : 0) * d_in + 16 * t;
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
    const uint4 z4 = make_uint4(0, 0, 0, 0);
    constexpr int kStride = 64 * WARPS;
    for (int kb = 64 * warp; kb < d_in; kb += kStride * UNR) {
        uint4 qa[UNR], qb[UNR], b0[UNR][NT], b1[UNR][NT];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int k0 = kb + u * kStride;
            const bool kin = k0 < d_in;
            qa[u] = kin && ra < T ? __ldg(reinterpret_cast<const uint4*>(xa + k0)) : z4;
            qb[u] = kin && rb < T ? __ldg(reinterpret_cast<const uint4*>(xb + k0)) : z4;
#pragma unroll
            for (int nn = 0; nn < NT; ++nn) {
                const int n = 8 * nn + g;
                b0[u][nn] = z4;
                b1[u][nn] = z4;
                if (kin && n < r) {
                    const uint4* ap = reinterpret_cast<const uint4*>(A + static_cast<int64_t>(n) * d_in + k0 + 16 * t);
                    b0[u][nn] = __ldg(ap);
                    b1[u][nn] = __ldg(ap + 1);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            uint32_t fa[8], fb[8];
            const uint32_t wa[4] = {qa[u].x, qa[u].y, qa[u].z, qa[u].w};
            const uint32_t wb[4] = {qb[u].x, qb[u].y, qb[u].z, qb[u].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                fa[2 * k] = e4m3x2_to_bf16x2(wa[k]);
                fa[2 * k + 1] = e4m3x2_to_bf16x2(wa[k] >> 16);
                fb[2 * k] = e4m3x2_to_bf16x2(wb[k]);
                fb[2 * k + 1] = e4m3x2_to_bf16x2(wb[k] >> 16);
            }
#pragma unroll
            for (int nn = 0; nn < NT; ++nn) {
                const uint32_t bw[8] = {b0[u][nn].x, b0[u][nn].y, b0[u][nn].z, b0[u][nn].w,
                                        b1[u][nn].x, b1[u][nn].y, b1[u][nn].z, b1[u][nn].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t a4[4] = {fa[2 * j], fb[2 * j], fa[2 * j + 1], fb[2 * j + 1]};
                    mma_bf16_16816(acc[nn], a4, bw[2 * j], bw[2 * j + 1], true);
                }
            }
        }
    }
#pragma unroll
    for (int nn = 0; nn < NT; ++nn) {
        s_part[warp][g][8 * nn + 2 * t] = acc[nn][0];
        s_part[warp][g][8 * nn + 2 * t + 1] = acc[nn][1];
        s_part[warp][g + 8][8 * nn + 2 * t] = acc[nn][2];
        s_part[warp][g + 8][8 * nn + 2 * t + 1] = acc[nn][3];
    }
    __syncthreads();
    const float fac = __fmul_rn(s, __ldg(w_scale));
    for (int e = threadIdx.x; e < 16 * ldu; e += blockDim.x) {
        const int row = e / ldu, col = e - row * ldu;
        const int64_t tok = t0 + row;
        if (tok >= T) continue;
        float v = 0.f;
        if (col < r) {
            v = s_part[0][row][col];
#pragma unroll
            for (int w = 1; w < WARPS; ++w) v += s_part[w][row][col];
            v = __fmul_rn(fac, v);
        }
        U[tok * ldu + col] = __float2bfloat16_rn(v);
    }
}

}  // namespace qlora

// nf4.cuh -- NF4 + double-quantization: block quantizer, exact decoder, and the
// byte-permute decode used inside the tensor-core GEMMs.
//
// Format ("Low-Rank Adaptation (LoRA) and QLoRA: Mathematical Foundations...", section
// "QLoRA: 4-Bit NormalFloat and Memory Optimization", subsections "1. 4-bit NormalFloat (NF4)
// Quantization" and "2. Double Quantization (DQ)"; block 64 / group 256 from "Large Language
// Model Fine-tuning and LoRA", section "Quantizing the frozen weights: NF4 and double
// quantization"):
//   per 64-block:   c1 = max|w|, x = fl32(w / c1), code = nearest level (ties upward)
//   per 256 blocks: c2 = max c1, q8 = rint(fl32(fl32(c1/c2) * 127)) in [0, 127]
//   decode:         s = fl32(fl32(q8 * c2) / 127), w = fl32(L[code] * s), bf16 = RN(w)
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"
#include "nf4_table.cuh"

namespace qlora {

constexpr int kBlock = 64;
constexpr int kGroup = 256;

__constant__ float c_nf4_levels[16] = QLORA_NF4_LEVELS;
__constant__ float c_nf4_thresholds[15] = QLORA_NF4_THRESHOLDS;

__device__ __forceinline__ float nf4_block_scale(uint32_t q8, float c2) {
    return __fdiv_rn(__fmul_rn(static_cast<float>(q8), c2), 127.0f);
}

// Per-block decode table for the byte-permute decoder.  The level table is symmetric
// (L[15-i] = -L[i] exactly), so only the 8 positive magnitudes P[j] = RN_bf16(fl32(L[8+j]*s))
// are formed; a negative code c < 8 decodes to -P[7-c].  The bf16 magnitudes are held as
// two byte planes (low bytes, high bytes) of 8 entries each, two registers per plane.
struct Nf4Planes {
    uint32_t lo0, lo1, hi0, hi1;
};

__device__ __forceinline__ Nf4Planes nf4_make_planes(float s) {
    const uint32_t w01 = pack_bf16x2(__fmul_rn(c_nf4_levels[8], s), __fmul_rn(c_nf4_levels[9], s));
    const uint32_t w23 = pack_bf16x2(__fmul_rn(c_nf4_levels[10], s), __fmul_rn(c_nf4_levels[11], s));
    const uint32_t w45 = pack_bf16x2(__fmul_rn(c_nf4_levels[12], s), __fmul_rn(c_nf4_levels[13], s));
    const uint32_t w67 = pack_bf16x2(__fmul_rn(c_nf4_levels[14], s), __fmul_rn(c_nf4_levels[15], s));
    Nf4Planes p;
    p.lo0 = prmt(w01, w23, 0x6420);
    p.hi0 = prmt(w01, w23, 0x7531);
    p.lo1 = prmt(w45, w67, 0x6420);
    p.hi1 = prmt(w45, w67, 0x7531);
    return p;
}

// Decode 8 packed codes (element e in nibble e) into 8 bf16 values in element order
// (returned as 4 words, low half = even element).
__device__ __forceinline__ uint4 nf4_decode8(uint32_t q, const Nf4Planes& p) {
    const uint32_t t = ~q & 0x88888888u;          // 8 in each nibble whose code is < 8
    const uint32_t f = t - (t >> 3);              // -> 7 there, 0 elsewhere
    const uint32_t m = (q ^ f) & 0x77777777u;     // magnitude index: c-8, or 7-c
    const uint32_t mh = m >> 16;
    const uint32_t lo_a = prmt(p.lo0, p.lo1, m);
    const uint32_t lo_b = prmt(p.lo0, p.lo1, mh);
    uint32_t hi_a = prmt(p.hi0, p.hi1, m);
    uint32_t hi_b = prmt(p.hi0, p.hi1, mh);
    // 0xFF in each byte whose code has bit 3 set (the positive half), from the sign bits of
    // the code bytes: element 2j's bit 3 is the msb of byte j of (q << 4), element 2j+1's
    // bit 3 is the msb of byte j of q.
    const uint32_t q4 = q << 4;
    const uint32_t pos_a = prmt(q4, q, 0xD9C8);
    const uint32_t pos_b = prmt(q4, q, 0xFBEA);
    hi_a |= ~pos_a & 0x80808080u;
    hi_b |= ~pos_b & 0x80808080u;
    uint4 out;
    out.x = prmt(lo_a, hi_a, 0x5140);
    out.y = prmt(lo_a, hi_a, 0x7362);
    out.z = prmt(lo_b, hi_b, 0x5140);
    out.w = prmt(lo_b, hi_b, 0x7362);
    return out;
}

// E4M3 decode for the FP8 GEMM.  The 8 positive magnitudes P[j] = E4M3(fl32(L[8+j] * s))
// (round to nearest even, saturating at 448; s already carries the weight's power-of-two
// scale) are bytes 0..7 of two registers; a code c < 8 decodes to P[7-c] with the sign bit set.
struct Nf4Fp8Planes {
    uint32_t lo, hi;
};

// Two fp32 values to two E4M3 bytes (a in the low byte).
__device__ __forceinline__ uint32_t e4m3x2_bits(float a, float b) {
    return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ Nf4Fp8Planes nf4_make_planes_e4m3(float s) {
    const uint32_t p01 = e4m3x2_bits(__fmul_rn(c_nf4_levels[8], s), __fmul_rn(c_nf4_levels[9], s));
    const uint32_t p23 = e4m3x2_bits(__fmul_rn(c_nf4_levels[10], s), __fmul_rn(c_nf4_levels[11], s));
    const uint32_t p45 = e4m3x2_bits(__fmul_rn(c_nf4_levels[12], s), __fmul_rn(c_nf4_levels[13], s));
    const uint32_t p67 = e4m3x2_bits(__fmul_rn(c_nf4_levels[14], s), __fmul_rn(c_nf4_levels[15], s));
    return Nf4Fp8Planes{p01 | (p23 << 16), p45 | (p67 << 16)};
}

// Decode 8 packed codes (element e in nibble e) into 8 E4M3 bytes in element order.
__device__ __forceinline__ uint2 nf4_decode8_e4m3(uint32_t q, const Nf4Fp8Planes& p) {
    const uint32_t t = ~q & 0x88888888u;          // 8 in each nibble whose code is < 8
    const uint32_t f = t - (t >> 3);              // -> 7 there, 0 elsewhere
    const uint32_t m = (q ^ f) & 0x77777777u;     // magnitude index: c-8, or 7-c
    uint32_t a = prmt(p.lo, p.hi, m);
    uint32_t b = prmt(p.lo, p.hi, m >> 16);
    // sign bytes (as in nf4_decode8): 0xFF where the element's code has bit 3 set
    const uint32_t q4 = q << 4;
    a |= ~prmt(q4, q, 0xD9C8) & 0x80808080u;
    b |= ~prmt(q4, q, 0xFBEA) & 0x80808080u;
    return make_uint2(a, b);
}

// ------------------------------------------------------------------ quantize

// One CTA (256 threads) per group of 256 blocks.  Each warp quantizes 32 blocks, one block
// at a time: lane l handles elements 2l and 2l+1 and writes code byte l.
template <typename TW>
__global__ void __launch_bounds__(256) k_nf4_quantize(const TW* __restrict__ W, int64_t nblocks,
                                                      uint8_t* __restrict__ codes,
                                                      uint8_t* __restrict__ absmax_q,
                                                      float* __restrict__ c2_out) {
    __shared__ float s_c1[kGroup];
    __shared__ float s_red[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t g = blockIdx.x;
    for (int b = warp; b < kGroup; b += 8) {
        const int64_t blk = g * kGroup + b;
        float c1 = 0.0f;
        if (blk < nblocks) {
            const int64_t e = blk * kBlock + 2 * lane;
            float w0, w1;
            if constexpr (sizeof(TW) == 4) {
                const float2 v = *reinterpret_cast<const float2*>(W + e);
                w0 = v.x;
                w1 = v.y;
            } else {
                const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(W + e);
                w0 = __bfloat162float(v.x);
                w1 = __bfloat162float(v.y);
            }
            float a = fmaxf(fabsf(w0), fabsf(w1));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
            c1 = a;
            float x0 = 0.0f, x1 = 0.0f;
            if (c1 > 0.0f) {
                x0 = __fdiv_rn(w0, c1);
                x1 = __fdiv_rn(w1, c1);
            }
            uint32_t k0 = 0, k1 = 0;
#pragma unroll
            for (int i = 0; i < 15; ++i) {
                k0 += (x0 >= c_nf4_thresholds[i]) ? 1u : 0u;
                k1 += (x1 >= c_nf4_thresholds[i]) ? 1u : 0u;
            }
            codes[blk * (kBlock / 2) + lane] = static_cast<uint8_t>(k0 | (k1 << 4));
        }
        if (lane == 0) s_c1[b] = c1;
    }
    __syncthreads();
    // c2 = max over the group's constants
    float m = s_c1[threadIdx.x];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s_red[warp] = m;
    __syncthreads();
    float c2 = s_red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) c2 = fmaxf(c2, s_red[i]);
    if (threadIdx.x == 0) c2_out[g] = c2;
    const int64_t blk = g * kGroup + threadIdx.x;
    if (blk < nblocks) {
        uint32_t q8 = 0;
        if (c2 > 0.0f) {
            const float v = __fmul_rn(__fdiv_rn(s_c1[threadIdx.x], c2), 127.0f);
            q8 = static_cast<uint32_t>(fminf(fmaxf(rintf(v), 0.0f), 127.0f));
        }
        absmax_q[blk] = static_cast<uint8_t>(q8);
    }
}

// ------------------------------------------------------------------ decode (stand-alone)

// bf16 output: one thread per 64-block through the same byte-permute decoder as the GEMMs.
__global__ void __launch_bounds__(256) k_nf4_dequant_bf16(const uint8_t* __restrict__ codes,
                                                          const uint8_t* __restrict__ absmax_q,
                                                          const float* __restrict__ c2,
                                                          int64_t nblocks,
                                                          __nv_bfloat16* __restrict__ out) {
    const int64_t blk = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (blk >= nblocks) return;
    const float s = nf4_block_scale(absmax_q[blk], c2[blk / kGroup]);
    const Nf4Planes p = nf4_make_planes(s);
    const uint4* src = reinterpret_cast<const uint4*>(codes + blk * (kBlock / 2));
    uint4* dst = reinterpret_cast<uint4*>(out + blk * kBlock);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint4 q = src[h];
        dst[4 * h + 0] = nf4_decode8(q.x, p);
        dst[4 * h + 1] = nf4_decode8(q.y, p);
        dst[4 * h + 2] = nf4_decode8(q.z, p);
        dst[4 * h + 3] = nf4_decode8(q.w, p);
    }
}

// fp32 output: one thread per code byte (two weights).
__global__ void __launch_bounds__(256) k_nf4_dequant_f32(const uint8_t* __restrict__ codes,
                                                         const uint8_t* __restrict__ absmax_q,
                                                         const float* __restrict__ c2,
                                                         int64_t nbytes, float* __restrict__ out) {
    const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (j >= nbytes) return;
    const int64_t blk = (2 * j) / kBlock;
    const float s = nf4_block_scale(absmax_q[blk], c2[blk / kGroup]);
    const uint32_t b = codes[j];
    float2 v;
    v.x = __fmul_rn(c_nf4_levels[b & 15u], s);
    v.y = __fmul_rn(c_nf4_levels[b >> 4], s);
    reinterpret_cast<float2*>(out)[j] = v;
}

}  // namespace qlora

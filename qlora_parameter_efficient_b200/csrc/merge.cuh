// merge.cuh -- dense merge W_final = W^ + s B A on the tensor cores (bf16 adapters).
//
// "Low-Rank Adaptation (LoRA) and QLoRA: Mathematical Foundations...", section "Static Weight
// Merging": after training, the adapter product is folded into the base weight once,
// W_final = W0 + (alpha / r) B A; with an NF4 base W0 is the decoded weight W^.  The result is
// dense (bf16 or fp32) and is not re-quantized; W^ is the decode in the output dtype.
//
// One CTA makes a 128 x 64 tile of W_final (one NF4 block column, so every tile is whole:
// d_in is a multiple of 64) with 8 warps; warp w owns rows 32 (w / 2) .. +31 and columns
// 32 (w % 2) .. +31 as 2 x 4 m16n8 fragments.  B A is formed with mma.sync
// m16n8k16 (bf16 x bf16 products are exact in fp32, fp32 accumulation), operands staged in
// shared memory and read with ldmatrix (A's rows are K x N with N contiguous: .trans).  The
// epilogue decodes, for each accumulator pair (row, columns 2t, 2t+1), the one code byte that
// holds those two weights, scales by the row's block scale (q8 c2 / 127, fp32), rounds to the
// output dtype, adds s * (B A) in fp32 and writes the value into a staged copy of the tile in
// shared memory, which is then stored with 16-byte vectors along whole rows.  The tile reads
// 4 KB of codes and writes 16 KB (bf16) or 32 KB (fp32): the kernel is bound by the output
// stream.
#pragma once

#include "common.cuh"
#include "nf4.cuh"

namespace qlora {

constexpr int kMergeThreads = 256;

// Row strides (elements) of the staged A rows and of the output tile: 72 keeps the ldmatrix
// rows and the fragment writes of a warp (bf16 words) or half-warp (fp32 pairs) on distinct
// banks.
constexpr int kMergeLda = 72;
constexpr int kMergeLdo = 72;

struct MergeSmem {
    // sB [128][rp + 8] bf16, sA [rp][72] bf16, sC [128][32] u8, sS [128] f32, levels [16],
    // sO [128][72] output elements
    static int bytes(int rp, int out_bytes) {
        return 128 * (rp + 8) * 2 + rp * kMergeLda * 2 + 128 * 32 + 128 * 4 + 64 + 128 * kMergeLdo * out_bytes;
    }
};

// NORM = true (DoRA): the tile's values are not stored; instead out_norm[row * (d_in / 64) +
// tile column] receives the sum of squares of the row's 64 values in the tile (fp32, summed
// in a fixed order), TOut giving the decode's rounding (bf16).
template <typename TOut, bool NORM = false>
__global__ void __launch_bounds__(kMergeThreads, 4) k_merge_tc(const uint8_t* __restrict__ codes,
                                                            const uint8_t* __restrict__ absmax_q,
                                                            const float* __restrict__ c2,
                                                            int64_t d_out, int64_t d_in,
                                                            const __nv_bfloat16* __restrict__ A,
                                                            const __nv_bfloat16* __restrict__ B,
                                                            int r, float s, TOut* __restrict__ out,
                                                            float* __restrict__ out_norm = nullptr) {
    extern __shared__ __align__(16) uint8_t mtc_smem[];
    const int rp = (r + 15) & ~15;
    const int ldb = rp + 8;                      // bf16 elements per staged B row
    __nv_bfloat16* sB = reinterpret_cast<__nv_bfloat16*>(mtc_smem);
    __nv_bfloat16* sA = sB + 128 * ldb;          // [rp][kMergeLda]
    uint8_t* sC = reinterpret_cast<uint8_t*>(sA + rp * kMergeLda);   // [128][32]
    float* sS = reinterpret_cast<float*>(sC + 128 * 32);             // [128]
    float* sL = sS + 128;                                            // [16]
    TOut* sO = reinterpret_cast<TOut*>(sL + 16);                     // [128][kMergeLdo]

    const int64_t row0 = static_cast<int64_t>(blockIdx.y) * 128;
    const int64_t col0 = static_cast<int64_t>(blockIdx.x) * 64;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t bpr = d_in / 64;               // 64-blocks per weight row

    griddep_enter();
    if (tid < 16) sL[tid] = c_nf4_levels[tid];
    // B rows (rank-padded with zeros); 16-byte vectors when every row is whole 16-byte units
    if (r % 8 == 0) {
        const int vpr = rp / 8;
        for (int i = tid; i < 128 * vpr; i += kMergeThreads) {
            const int rr = i / vpr, v = i % vpr;
            const int64_t gr = row0 + rr;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (8 * v < r && gr < d_out) val = *reinterpret_cast<const uint4*>(B + gr * r + 8 * v);
            *reinterpret_cast<uint4*>(sB + rr * ldb + 8 * v) = val;
        }
    } else {
        for (int i = tid; i < 128 * rp; i += kMergeThreads) {
            const int rr = i / rp, j = i % rp;
            const int64_t gr = row0 + rr;
            sB[rr * ldb + j] = (j < r && gr < d_out) ? B[gr * r + j] : __float2bfloat16_rn(0.f);
        }
    }
    // A rows: 16-byte vectors (d_in is a multiple of 64, the tile's columns of 8 are aligned)
    for (int i = tid; i < rp * 8; i += kMergeThreads) {
        const int j = i >> 3, v = i & 7;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (j < r) val = *reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j) * d_in + col0 + 8 * v);
        *reinterpret_cast<uint4*>(sA + j * kMergeLda + 8 * v) = val;
    }
    // code bytes of the tile (one block per row): 128 rows x 32 bytes
    {
        const int rr = tid >> 1, v = tid & 1;
        const int64_t gr = row0 + rr;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (gr < d_out) val = *reinterpret_cast<const uint4*>(codes + gr * (d_in / 2) + col0 / 2 + 16 * v);
        *reinterpret_cast<uint4*>(sC + rr * 32 + 16 * v) = val;
    }
    // block scales: one 64-block per row of the tile
    if (tid < 128) {
        const int64_t gr = row0 + tid;
        float sc = 0.f;
        if (gr < d_out) {
            const int64_t blk = gr * bpr + col0 / 64;
            sc = nf4_block_scale(absmax_q[blk], c2[blk / kGroup]);
        }
        sS[tid] = sc;
    }
    __syncthreads();

    const int wr = (warp >> 1) * 32, wc = (warp & 1) * 32;
    float acc[2][4][4];
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mi][ni][e] = 0.f;
    const uint32_t sB_u = smem_u32(sB), sA_u = smem_u32(sA);
    for (int k0 = 0; k0 < rp; k0 += 16) {
        uint32_t af[2][4];
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
            const int arow = wr + 16 * mi + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int acol = k0 + (lane >> 4) * 8;
            ldsm_x4(af[mi], sB_u + static_cast<uint32_t>((arow * ldb + acol) * 2));
        }
#pragma unroll
        for (int nj = 0; nj < 2; ++nj) {
            // two n8 tiles per x4.trans: lanes 0-15 give K rows 0..15 at column n, lanes 16-31
            // the same rows at column n + 8
            uint32_t bf[4];
            const int brow = k0 + (lane & 15);
            const int bcol = wc + 16 * nj + (lane >> 4) * 8;
            ldsm_x4_trans(bf, sA_u + static_cast<uint32_t>((brow * kMergeLda + bcol) * 2));
#pragma unroll
            for (int mi = 0; mi < 2; ++mi) {
                mma_bf16_16816(acc[mi][2 * nj], af[mi], bf[0], bf[1], true);
                mma_bf16_16816(acc[mi][2 * nj + 1], af[mi], bf[2], bf[3], true);
            }
        }
    }

    // epilogue: accumulator (row g [+8], columns 2t, 2t+1) of each fragment
    const int g = lane >> 2, t = lane & 3;
    float sq[2][2] = {{0.f, 0.f}, {0.f, 0.f}};      // NORM: per (mi, h) row of the thread
#pragma unroll
    for (int mi = 0; mi < 2; ++mi) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int rr = wr + 16 * mi + g + 8 * h;
            const float sc = sS[rr];
#pragma unroll
            for (int ni = 0; ni < 4; ++ni) {
                const int cc = wc + 8 * ni + 2 * t;
                const uint32_t byte = sC[rr * 32 + (cc >> 1)];
                float w0 = __fmul_rn(sL[byte & 15u], sc), w1 = __fmul_rn(sL[byte >> 4], sc);
                if constexpr (sizeof(TOut) == 2) {
                    w0 = __bfloat162float(__float2bfloat16_rn(w0));
                    w1 = __bfloat162float(__float2bfloat16_rn(w1));
                }
                const float v0 = w0 + s * acc[mi][ni][2 * h], v1 = w1 + s * acc[mi][ni][2 * h + 1];
                if constexpr (NORM) {
                    sq[mi][h] = fmaf(v0, v0, sq[mi][h]);
                    sq[mi][h] = fmaf(v1, v1, sq[mi][h]);
                    continue;
                }
                if constexpr (sizeof(TOut) == 2) {
                    *reinterpret_cast<__nv_bfloat162*>(sO + rr * kMergeLdo + cc) = __floats2bfloat162_rn(v0, v1);
                } else {
                    *reinterpret_cast<float2*>(sO + rr * kMergeLdo + cc) = make_float2(v0, v1);
                }
            }
        }
    }
    if constexpr (NORM) {
        // the 4 threads of a row (t = 0..3), then the 2 warps of a row group (32 columns each)
        float* s_sq = reinterpret_cast<float*>(sO);                   // [128][2]
#pragma unroll
        for (int mi = 0; mi < 2; ++mi)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float x = sq[mi][h];
                x += __shfl_xor_sync(0xffffffffu, x, 1);
                x += __shfl_xor_sync(0xffffffffu, x, 2);
                if (t == 0) s_sq[(wr + 16 * mi + g + 8 * h) * 2 + (warp & 1)] = x;
            }
        __syncthreads();
        if (tid < 128 && row0 + tid < d_out)
            out_norm[(row0 + tid) * (d_in / 64) + blockIdx.x] = s_sq[tid * 2] + s_sq[tid * 2 + 1];
        return;
    }
    __syncthreads();
    // whole rows of the tile, 16 bytes per thread per store
    constexpr int kVec = 16 / static_cast<int>(sizeof(TOut));     // elements per 16 bytes
    constexpr int kVpr = 64 / kVec;                                // vectors per tile row
    for (int i = tid; i < 128 * kVpr; i += kMergeThreads) {
        const int rr = i / kVpr, v = i % kVpr;
        const int64_t gr = row0 + rr, gc = col0 + v * kVec;
        if (gr < d_out)
            *reinterpret_cast<uint4*>(out + gr * d_in + gc) =
                *reinterpret_cast<const uint4*>(sO + rr * kMergeLdo + v * kVec);
    }
}

// DoRA column scale of the layer output: scale[j] = magnitude[j] / sqrt(sum_c partial[j][c])
// (partials from k_merge_tc<., true>, summed in column order); magnitude == nullptr writes the
// norms themselves.  A row of norm 0 has no direction: its scale is 0.
__global__ void k_dora_scale(const float* __restrict__ partial, int64_t d_out, int n_cb,
                             const float* __restrict__ magnitude, float* __restrict__ out) {
    griddep_enter();
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < d_out;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float acc = 0.f;
        for (int c = 0; c < n_cb; ++c) acc += partial[j * n_cb + c];
        const float nrm = sqrtf(acc);
        out[j] = magnitude ? (nrm > 0.f ? magnitude[j] / nrm : 0.f) : nrm;
    }
}

}  // namespace qlora

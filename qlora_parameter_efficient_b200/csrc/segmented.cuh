// segmented.cuh -- multi-adapter forward for many adapters: token sort + segmented shrink/expand.
//
// "Large Language Model Fine-tuning and LoRA", section "Serving many adapters at once: the
// multi-tenant problem": one resident (quantized) base, every tenant's A_i, B_i kept as small
// separate objects, the shared x W term computed once per batch and each request's correction
// x (B_i A_i) added by grouped kernels that handle adapters of different ranks in one batch;
// "LoRA and QLoRA Fine-Tuning Under the Hood", section "6.2 Multi-Adapter Serving at Scale
// (S-LoRA & Punica)": thousands of adapters applied on the fly over one base.
//
//   H[t] = X[t] W^T + s_i (X[t] A_i^T) B_i^T,   i = id[t],  s_i = alpha_i / r_i
//
// The base term is the fused NF4 GEMM without adapter steps.  The adapter term:
//   1. k_seg_count:   per-adapter token counts (an id outside [0, n) is a device error and the
//                     token gets no adapter term).
//   2. k_seg_plan:    one CTA: exclusive scans of the counts (segment starts) and of the
//                     per-adapter tile counts (16 tokens per tile), the tile list (adapter,
//                     first sorted slot) and the scatter cursors.
//   3. k_seg_scatter: perm[slot] = t, tokens grouped by adapter (the order inside a segment is
//                     whatever the atomics give; every token's result depends on its own row
//                     only, so the output does not depend on it).
//   4. k_seg_shrink:  one CTA per tile: U[slot, 0..r_i) = bf16(s_i X[perm[slot]] A_i^T), fp32
//                     accumulation (mma.sync m16n8k16, K split over 4 warps, summed in order).
//   5. k_seg_expand:  per tile, all columns: H[perm[slot]] = bf16(H + U[slot] B_i^T).
// Kernels 4 and 5 run persistent grids over the planned tiles.
#pragma once

#include "common.cuh"

namespace qlora {

constexpr int kSegTile = 16;          // tokens per tile
constexpr int kSegMaxAdapters = 65536;

struct SegArgs {
    int64_t T;
    int n;                            // adapters
    int d_in, d_out;
    int ldu;                          // row stride of U (max rank rounded up to 16)
    const __nv_bfloat16* X;           // [T, d_in]
    __nv_bfloat16* H;                 // [T, d_out], holds X W^T on entry to k_seg_expand
    const int32_t* ids;               // [T]
    const __nv_bfloat16* const* A;    // [n] -> A_i [r_i, d_in]
    const __nv_bfloat16* const* B;    // [n] -> B_i [d_out, r_i]
    const int32_t* ranks;             // [n]
    const float* alphas;              // [n] alpha_i; s_i = alpha_i / r_i is formed here
    int32_t* cnt;                     // [n] zero at launch of k_seg_count
    int32_t* seg_start;               // [n]
    int32_t* cursor;                  // [n]
    int32_t* n_tiles;                 // [1]
    int4* tiles;                      // [max_tiles] (adapter, first slot, rows, rank)
    int32_t* perm;                    // [T] slot -> token
    __nv_bfloat16* U;                 // [T, ldu] by slot
    int* err;
};

__global__ void k_seg_count(SegArgs a) {
    griddep_enter();
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < a.T;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int id = a.ids[t];
        if (id < 0 || id >= a.n) set_error(a.err, kErrDevice);
        else atomicAdd(a.cnt + id, 1);
    }
}

// Block-wide exclusive scan of one value per thread (1024 threads); returns the block total.
__device__ __forceinline__ int seg_block_scan(int v, int* s_warp, int& excl) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;            // inclusive prefix over warps
    }
    __syncthreads();
    const int warp_base = warp > 0 ? s_warp[warp - 1] : 0;
    excl = warp_base + x - v;
    const int total = s_warp[31];
    __syncthreads();
    return total;
}

__global__ void __launch_bounds__(1024) k_seg_plan(SegArgs a) {
    griddep_enter();
    __shared__ int s_warp[32];
    int slot_base = 0, tile_base = 0;
    for (int c0 = 0; c0 < a.n; c0 += 1024) {
        const int i = c0 + static_cast<int>(threadIdx.x);
        const int c = i < a.n ? a.cnt[i] : 0;
        const int nt = (c + kSegTile - 1) / kSegTile;
        int ex_c, ex_t;
        const int tot_c = seg_block_scan(c, s_warp, ex_c);
        const int tot_t = seg_block_scan(nt, s_warp, ex_t);
        if (i < a.n) {
            const int start = slot_base + ex_c;
            a.seg_start[i] = start;
            a.cursor[i] = start;
            const int r = a.ranks[i];
            for (int j = 0; j < nt; ++j)
                a.tiles[tile_base + ex_t + j] = make_int4(i, start + j * kSegTile, min(kSegTile, c - j * kSegTile), r);
        }
        slot_base += tot_c;
        tile_base += tot_t;
    }
    if (threadIdx.x == 0) *a.n_tiles = tile_base;
}

__global__ void k_seg_scatter(SegArgs a) {
    griddep_enter();
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < a.T;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int id = a.ids[t];
        if (id < 0 || id >= a.n) continue;
        const int slot = atomicAdd(a.cursor + id, 1);
        if (dcheck(slot >= 0 && slot < a.T, a.err)) a.perm[slot] = static_cast<int32_t>(t);
    }
}

// Persistent grids: CTA b takes tiles b, b + gridDim.x, ... below the planned count.  A tile
// entry is one 16-byte load: (adapter, first slot, rows, rank).

// An adapter the kernels can serve: rank within [1, ldu] (U rows hold ldu columns) and A_i on a
// 16-byte boundary (its rows are read as 16-byte vectors).  Others get no adapter term; the
// shrink reports them as QLORA_ERR_DEVICE.
__device__ __forceinline__ bool seg_adapter_ok(const SegArgs& a, int r, const __nv_bfloat16* Ai) {
    return r >= 1 && r <= a.ldu && (reinterpret_cast<uintptr_t>(Ai) & 15u) == 0;
}

// 32-bit pair of bf16 at p (p even-aligned) or zero.
__device__ __forceinline__ uint32_t ld_pair(const __nv_bfloat16* p, bool ok) {
    return ok ? __ldg(reinterpret_cast<const uint32_t*>(p)) : 0u;
}

// K order inside the MMA.  A dot product over K may take its terms in any order as long as both
// operands use the same one, so inside each chunk of 64 (shrink) or 16 (expand) elements the
// m16n8k16 K slots are mapped to elements so that a thread's fragments are contiguous in memory:
// in k16 step s of a 64-chunk, thread-column t's slots {2t, 2t+1} and {2t+8, 2t+9} hold elements
// 16t + 4s + {0, 1} and 16t + 4s + {2, 3}; so the thread loads elements 16t .. 16t+15 of each of
// its rows as two 16-byte vectors and uses words 2s and 2s+1 in step s.

// One CTA (4 warps) per tile.  Warp w takes the 64-element K chunks w, w + 4, ...; the four
// warps' sums are added in warp order.  NT: n8 tiles of the largest rank (ranks up to 8 NT);
// fewer accumulators let more K chunks' loads be in flight (UNR chunks per iteration).
#ifndef QLORA_SEG_SHRINK_MINB
#define QLORA_SEG_SHRINK_MINB 3
#endif
template <int NT, int UNR>
__global__ void __launch_bounds__(128, QLORA_SEG_SHRINK_MINB) k_seg_shrink(SegArgs a) {
    griddep_enter();
    __shared__ float s_part[4][kSegTile][129];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int n_tiles = *a.n_tiles;
    for (int b = blockIdx.x; b < n_tiles; b += gridDim.x) {
    const int4 tl = a.tiles[b];
    const int i = tl.x, start = tl.y, rows = tl.z, r = tl.w;
    if (!dcheck(i >= 0 && i < a.n && start >= 0 && rows >= 1 && rows <= kSegTile && start + rows <= a.T, a.err))
        continue;                     // (uniform over the CTA: every thread reads the same entry)
    const __nv_bfloat16* Ai = a.A[i];
    if (!seg_adapter_ok(a, r, Ai)) {
        if (threadIdx.x == 0) set_error(a.err, kErrDevice);
        continue;
    }
    const int nt8 = (r + 7) / 8;      // n8 tiles of the rank (<= 16)
    const int tok_a = g < rows ? a.perm[start + g] : -1;
    const int tok_b = g + 8 < rows ? a.perm[start + g + 8] : -1;
    const __nv_bfloat16* xa = a.X + static_cast<int64_t>(tok_a < 0 ? 0 : tok_a) * a.d_in + 16 * t;
    const __nv_bfloat16* xb = a.X + static_cast<int64_t>(tok_b < 0 ? 0 : tok_b) * a.d_in + 16 * t;
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
    const uint4 z4 = make_uint4(0, 0, 0, 0);
    // UNR chunks of 64 columns per pass: every load of the pass is issued before its MMAs
    for (int kb = 64 * warp; kb < a.d_in; kb += 256 * UNR) {
        uint4 x[UNR][4], y[UNR][NT][2];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int k0 = kb + 256 * u;
            const bool kin = k0 < a.d_in;
            x[u][0] = kin && tok_a >= 0 ? __ldg(reinterpret_cast<const uint4*>(xa + k0)) : z4;
            x[u][1] = kin && tok_a >= 0 ? __ldg(reinterpret_cast<const uint4*>(xa + k0 + 8)) : z4;
            x[u][2] = kin && tok_b >= 0 ? __ldg(reinterpret_cast<const uint4*>(xb + k0)) : z4;
            x[u][3] = kin && tok_b >= 0 ? __ldg(reinterpret_cast<const uint4*>(xb + k0 + 8)) : z4;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int j = 8 * n + g;                      // adapter row = output column
                const bool ok = kin && n < nt8 && j < r;
                const __nv_bfloat16* arow = Ai + static_cast<int64_t>(ok ? j : 0) * a.d_in + (kin ? k0 : 0) + 16 * t;
                y[u][n][0] = ok ? __ldg(reinterpret_cast<const uint4*>(arow)) : z4;
                y[u][n][1] = ok ? __ldg(reinterpret_cast<const uint4*>(arow + 8)) : z4;
            }
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const uint32_t* wa = reinterpret_cast<const uint32_t*>(&x[u][0]);   // row g: 8 words
            const uint32_t* wb = reinterpret_cast<const uint32_t*>(&x[u][2]);   // row g + 8
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                if (n < nt8) {
                    const uint32_t* wy = reinterpret_cast<const uint32_t*>(&y[u][n][0]);
#pragma unroll
                    for (int st = 0; st < 4; ++st) {
                        const uint32_t af[4] = {wa[2 * st], wb[2 * st], wa[2 * st + 1], wb[2 * st + 1]};
                        mma_bf16_16816(acc[n], af, wy[2 * st], wy[2 * st + 1], true);
                    }
                }
            }
        }
    }
    // accumulator (row g [+8], columns 8n + 2t, +1) -> shared, then summed over the warps
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        if (n < nt8) {
            s_part[warp][g][8 * n + 2 * t] = acc[n][0];
            s_part[warp][g][8 * n + 2 * t + 1] = acc[n][1];
            s_part[warp][g + 8][8 * n + 2 * t] = acc[n][2];
            s_part[warp][g + 8][8 * n + 2 * t + 1] = acc[n][3];
        }
    }
    __syncthreads();
    const float s = __fdiv_rn(a.alphas[i], static_cast<float>(r));   // alpha_i / r_i
    const int rp = (r + 15) & ~15;
    for (int e = threadIdx.x; e < kSegTile * rp; e += blockDim.x) {
        const int row = e / rp, j = e % rp;
        if (row >= rows) continue;
        float v = 0.f;
        if (j < r) v = s * (((s_part[0][row][j] + s_part[1][row][j]) + s_part[2][row][j]) + s_part[3][row][j]);
        a.U[static_cast<int64_t>(start + row) * a.ldu + j] = __float2bfloat16_rn(v);
    }
    __syncthreads();                  // s_part is rewritten by the next tile
    }
}

// 4 bf16 of a row at element j (j a multiple of 4) as two words, zero beyond `valid`; aligned
// 8-byte load when the whole quad is valid and the row start allows it.
__device__ __forceinline__ uint2 ld_quad(const __nv_bfloat16* row, int j, int valid, bool aligned8) {
    if (aligned8 && j + 4 <= valid) return __ldg(reinterpret_cast<const uint2*>(row + j));
    uint16_t v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
        v[e] = j + e < valid ? __ldg(reinterpret_cast<const uint16_t*>(row + j + e)) : 0;
    return make_uint2(v[0] | (static_cast<uint32_t>(v[1]) << 16), v[2] | (static_cast<uint32_t>(v[3]) << 16));
}

// Persistent over tiles; for a tile, warp w takes the 64-column blocks w, w + 4, ... of H as
// eight n8 fragments each.  K = the adapter's rank rounded up to 16 (U is zero beyond r), the K
// slots of each 16-step mapped as in the shrink (thread-column t holds elements 4t .. 4t+3).
// The tile's U fragments stay in registers for all its column blocks; each warp loads the H
// values and first B quads of UNR blocks before multiplying and storing them.
// KS: K steps of 16 of the largest rank (ranks up to 16 KS).
#ifndef QLORA_SEG_EXPAND_UNR
#define QLORA_SEG_EXPAND_UNR 2
#endif
#ifndef QLORA_SEG_EXPAND_MINB
#define QLORA_SEG_EXPAND_MINB 4
#endif
// ODD: d_out is odd, so H's rows are not whole bf16 pairs and are read and written element by
// element (a separate instance keeps the common even case free of the per-element branches).
template <int KS, bool ODD>
__global__ void __launch_bounds__(128, QLORA_SEG_EXPAND_MINB) k_seg_expand(SegArgs a) {
    constexpr int UNR = QLORA_SEG_EXPAND_UNR;     // column blocks per pass of a warp
    griddep_enter();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int n_tiles = *a.n_tiles;
    const int n_blocks = (a.d_out + 63) / 64;
    for (int b = blockIdx.x; b < n_tiles; b += gridDim.x) {
        const int4 tl = a.tiles[b];
        const int i = tl.x, start = tl.y, rows = tl.z, r = tl.w;
        if (!dcheck(i >= 0 && i < a.n && start >= 0 && rows >= 1 && rows <= kSegTile && start + rows <= a.T,
                    a.err))
            continue;
        if (!seg_adapter_ok(a, r, a.A[i])) continue;     // reported by k_seg_shrink
        const int ksteps = (r + 15) / 16;
        const __nv_bfloat16* Bi = a.B[i];
        const bool ra = g < rows, rb = g + 8 < rows;
        const int tok_a = ra ? a.perm[start + g] : -1;
        const int tok_b = rb ? a.perm[start + g + 8] : -1;
        // U fragments of the tile, all K steps (<= KS)
        uint32_t uf[KS][4];
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            uint2 qa = make_uint2(0, 0), qb = make_uint2(0, 0);
            if (ks < ksteps) {
                if (ra) qa = __ldg(reinterpret_cast<const uint2*>(a.U + static_cast<int64_t>(start + g) * a.ldu + 16 * ks + 4 * t));
                if (rb) qb = __ldg(reinterpret_cast<const uint2*>(a.U + static_cast<int64_t>(start + g + 8) * a.ldu + 16 * ks + 4 * t));
            }
            uf[ks][0] = qa.x;
            uf[ks][1] = qb.x;
            uf[ks][2] = qa.y;
            uf[ks][3] = qb.y;
        }
        // B_i rows start on 8-byte boundaries
        const bool b_al8 = (r % 4) == 0 && (reinterpret_cast<uintptr_t>(Bi) & 7u) == 0;
        const __nv_bfloat16* ha = a.H + static_cast<int64_t>(tok_a < 0 ? 0 : tok_a) * a.d_out;
        const __nv_bfloat16* hb = a.H + static_cast<int64_t>(tok_b < 0 ? 0 : tok_b) * a.d_out;
        auto load_h = [&](int blk, uint32_t (&h)[8][2]) {
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                const int col = 64 * blk + 8 * n + 2 * t;
                const bool okc = col < a.d_out;
                // two adjacent bf16 of a row (read one by one when rows have an odd length)
                auto pair = [&](const __nv_bfloat16* row) -> uint32_t {
                    if constexpr (!ODD) return *reinterpret_cast<const uint32_t*>(row + col);
                    const uint32_t lo = *reinterpret_cast<const unsigned short*>(row + col);
                    const uint32_t hi = col + 1 < a.d_out ? *reinterpret_cast<const unsigned short*>(row + col + 1) : 0u;
                    return lo | (hi << 16);
                };
                h[n][0] = (okc && ra) ? pair(ha) : 0u;
                h[n][1] = (okc && rb) ? pair(hb) : 0u;
            }
        };
        // B_i quads of one K step of a 64-column block (rows = output columns)
        auto load_b = [&](int blk, int ks, uint2 (&bq)[8]) {
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                const int col = 64 * blk + 8 * n + g;
                bq[n] = col < a.d_out ? ld_quad(Bi + static_cast<int64_t>(col) * r, 16 * ks + 4 * t, r, b_al8)
                                      : make_uint2(0, 0);
            }
        };
        // warp w takes blocks w, w + 4, ...; UNR of them per pass, every H value and K step 0
        // B quad of the pass loaded before its MMAs
        for (int blk0 = warp; blk0 < n_blocks; blk0 += 4 * UNR) {
            uint32_t hv[UNR][8][2];
            uint2 bq0[UNR][8];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int blk = blk0 + 4 * u;
                if (blk < n_blocks) {
                    load_h(blk, hv[u]);
                    load_b(blk, 0, bq0[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int blk = blk0 + 4 * u;
                if (blk >= n_blocks) break;
                float acc[8][4];
#pragma unroll
                for (int n = 0; n < 8; ++n)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
#pragma unroll
                for (int n = 0; n < 8; ++n) mma_bf16_16816(acc[n], uf[0], bq0[u][n].x, bq0[u][n].y, true);
#pragma unroll
                for (int ks = 1; ks < KS; ++ks) {
                    if (ks < ksteps) {
                        uint2 bq[8];
                        load_b(blk, ks, bq);
#pragma unroll
                        for (int n = 0; n < 8; ++n) mma_bf16_16816(acc[n], uf[ks], bq[n].x, bq[n].y, true);
                    }
                }
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    const int col = 64 * blk + 8 * n + 2 * t;
                    if (col >= a.d_out) continue;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int tok = hh ? tok_b : tok_a;
                        if (tok < 0) continue;
                        __nv_bfloat162 base;
                        *reinterpret_cast<uint32_t*>(&base) = hv[u][n][hh];
                        const float2 bf = __bfloat1622float2(base);
                        __nv_bfloat16* dst = a.H + static_cast<int64_t>(tok) * a.d_out + col;
                        if constexpr (!ODD) {
                            *reinterpret_cast<__nv_bfloat162*>(dst) =
                                __floats2bfloat162_rn(bf.x + acc[n][2 * hh], bf.y + acc[n][2 * hh + 1]);
                        } else {
                            dst[0] = __float2bfloat16_rn(bf.x + acc[n][2 * hh]);
                            if (col + 1 < a.d_out) dst[1] = __float2bfloat16_rn(bf.y + acc[n][2 * hh + 1]);
                        }
                    }
                }
            }
        }
    }
}

}  // namespace qlora

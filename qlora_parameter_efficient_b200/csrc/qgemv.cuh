// qgemv.cuh -- decode-size forward (T <= 32 tokens): an HBM-bound stream over the NF4 codes.
//
//   H[t, n] = sum_b s_b(n) * sum_{k in b} L16(code(n, k)) x[t, k]  +  (s U[t, :]) . B[n, :]
//
// With a handful of tokens every weight is used T times, so the layer is a weight stream
// (0.516 B per weight) and the decode must keep up with HBM: about 44 weights per SM cycle.
// The exact per-block table of the large-T kernels (a bf16 product per level and block) costs
// ~2 integer ops per weight, too many here.  This kernel factors the block scale out of the
// block's dot product instead -- dequantize = LUT(code) x s_b ("Low-Rank Adaptation (LoRA) and
// QLoRA: Mathematical Foundations...", section "1. 4-bit NormalFloat (NF4) Quantization";
// the block scale is that of "2. Double Quantization (DQ)") evaluated as
// s_b * sum(LUT(code) x): a fixed 256-entry table maps a code byte to its two levels as a
// bf16 pair (one shared-memory load per two weights, replicated per lane so a warp's loads
// never conflict), the tensor cores form the block's partial dot products, and s_b multiplies
// the fp32 partial.  Identical in exact arithmetic; the levels are rounded to bf16 before the
// scale instead of after (relative 2^-9 per weight, averaging out in the sum).
//
// Work: units of (128 weight rows) x (256 K) = four NF4 blocks per row, i.e. 128 contiguous code
// bytes per row (whole cache lines; the code stream is read once, straight from HBM), with one
// accumulator per block so each block's scale applies to its own partial; a persistent grid splits
// the unit sequence (row tile major) into equal contiguous ranges.  Per CTA (448 threads):
//   warp 0       TMA: the unit's code tile (128 x 128 B, 128-byte swizzle) and X tiles
//                (4 x N x 64 bf16, rows past T zero-filled) into a 4-stage ring.
//   warp 1       issues tcgen05.mma (M = 128, N = 16/32, K = 16, A from tensor memory) into a
//                per-unit accumulator (a ring of four in tensor memory).
//   warps 2..9   decoders in two groups of four warps taking units in turn: one row per
//                thread; 32 table loads per block give the row's 64 bf16, written to tensor
//                memory with one tcgen05.st per block (A operand, 2 stages of 4 x 32 columns).
//   warps 10..13 accumulate: read the unit's partial from tensor memory, add s_b * partial in
//                fp32.  At the end of a row tile's range they write a partial row; the last CTA
//                to finish a tile (semaphore) sums the partials in CTA order, adds the adapter
//                term and writes H -- deterministic.
#pragma once

#include "common.cuh"
#include "nf4.cuh"

namespace qlora {

constexpr int kGvBlk = 4;       // NF4 blocks per row per unit: 128 contiguous code bytes
constexpr int kGvStagesC = 4;   // code + X tiles
constexpr int kGvStagesA = 2;   // decoded A tiles in tensor memory (4 x 32 columns each)
constexpr int kGvDecGroups = 2; // groups of 4 decoder warps taking units in turn
constexpr int kGvDBufs = 2;     // per-unit accumulators in tensor memory (4 x NT columns)
constexpr int kGvEpiWarp = 2 + 4 * kGvDecGroups;     // first accumulate warp
constexpr int kGvThreads = 32 * (kGvEpiWarp + 4);
// Decoder group g handles units g, g + groups, ...; with both ring depths multiples of the
// group count the previous phase of every barrier a group waits on is one it has seen.
static_assert(kGvStagesC % kGvDecGroups == 0 && kGvStagesA % kGvDecGroups == 0, "ring depths");
constexpr int kGvLut = 256 * 32 * 4;   // 256 entries x 32 lanes x 4 bytes
constexpr int kGvUsMax = 32 * 128;     // s*U staging: T <= 32 tokens x r <= 128

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
// D[tmem] (+)= A[tmem] * B[smem desc]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

struct GvArgs {
    int T;                  // tokens (1..NT)
    int d_out, d_in, kt;    // kt = d_in / 64 blocks per row
    int kt4;                // units per row tile: ceil(kt / kGvBlk)
    int rt;                 // row tiles of 128
    int units;              // rt * kt4
    int tiles_per_cta;      // partial slots per CTA
    const uint8_t* absmax_q;
    const float* c2;
    float* part;            // [grid][tiles_per_cta][128][NT]
    int* counters;          // [rt], zeroed by the pre-pass
    const float* us;        // [T][r]  s * U in fp32, from the pre-pass
    const __nv_bfloat16* B; // [d_out][r]
    int r;
    __nv_bfloat16* H;       // [T][d_out]
    int* err;
    uint64_t wait_ns;
};

__device__ __forceinline__ int gv_start(int c, int units, int grid) {
    return static_cast<int>((static_cast<int64_t>(c) * units) / grid);
}

template <int NT>
__global__ void __launch_bounds__(kGvThreads, 1)
    k_qgemv(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmX,
            const GvArgs args) {
    static_assert(NT == 16 || NT == 32, "token tile");
    constexpr int SC = kGvStagesC, SA = kGvStagesA, ND = kGvDBufs;
    constexpr int kCodes = 128 * 32 * kGvBlk;     // bytes per unit (128 rows x 128 B)
    constexpr int kXb = NT * 128;                 // bytes per block (NT rows x 64 bf16)
    constexpr int kX = kXb * kGvBlk;              // bytes per unit
    constexpr uint32_t kTmemCols = 512;
    constexpr uint32_t kACols = 32 * kGvBlk;      // tensor-memory columns per A stage
    constexpr uint32_t kDCols = NT * kGvBlk;      // tensor-memory columns per accumulator set
    constexpr uint32_t kDCol = kACols * kGvStagesA;   // accumulators after the A stages
    static_assert(kDCol + kDCols * kGvDBufs <= kTmemCols, "tensor memory budget");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem);          // [256][32]
    uint8_t* sX = smem + kGvLut;                                 // [SC][kX]
    uint8_t* sC = sX + SC * kX;                                  // [SC][kCodes]
    float* s_us = reinterpret_cast<float*>(sC + SC * kCodes);   // [T][r] s*U (reduction only)
    uint64_t* bars = reinterpret_cast<uint64_t*>(s_us + kGvUsMax);
    uint64_t* full = bars;                 // [SC] codes + X landed
    uint64_t* empty = full + SC;           // [SC] decoders (4) + MMA (1) done with the stage
    uint64_t* a_full = empty + SC;         // [SA] decoded rows in tensor memory (4 warps)
    uint64_t* a_free = a_full + SA;        // [SA] MMA done with the stage
    uint64_t* d_full = a_free + SA;        // [ND] unit accumulator ready
    uint64_t* d_free = d_full + ND;        // [ND] accumulator read (4 warps)
    uint64_t* seg_bar = d_free + ND;       // [2]  accumulate warps meet at a row-tile end
    uint64_t* us_bar = seg_bar + 2;        // [1]  s*U staged (used once)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(us_bar + 1);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* last_flag = abort + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u0 = gv_start(blockIdx.x, args.units, gridDim.x);
    const int u1 = gv_start(blockIdx.x + 1, args.units, gridDim.x);
    const int n_units = u1 - u0;

    // level-pair table: entry b = (bf16(L[b & 15]), bf16(L[b >> 4])), one copy per lane
    for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
        const int b = i >> 5;
        lut[i] = pack_bf16x2(c_nf4_levels[b & 15], c_nf4_levels[b >> 4]);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < SC; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 5);
        }
        for (int s = 0; s < SA; ++s) {
            mbar_init(&a_full[s], 4);
            mbar_init(&a_free[s], 1);
        }
        for (int b = 0; b < ND; ++b) {
            mbar_init(&d_full[b], 1);
            mbar_init(&d_free[b], 4);
        }
        for (int b = 0; b < 2; ++b) mbar_init(&seg_bar[b], 4);
        mbar_init(us_bar, 4);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmC);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto fail = [&]() {
        set_error(args.err, kErrTimeout);
        *abort = 1;
    };

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < n_units; ++i) {
                const int u = u0 + i;
                const int tile = u / args.kt4, ks = u % args.kt4;
                const int s = i % SC;
                if (!mbar_wait(&empty[s], ((i / SC) & 1) ^ 1, abort, args.wait_ns)) {
                    fail();
                    break;
                }
                mbar_arrive_expect_tx(&full[s], kCodes + kX);
                tma_load_2d(sC + s * kCodes, &tmC, &full[s], ks * 32 * kGvBlk, tile * 128);
#pragma unroll
                for (int b = 0; b < kGvBlk; ++b)
                    tma_load_2d(sX + s * kX + b * kXb, &tmX, &full[s], (ks * kGvBlk + b) * 64, 0);
                issued = i + 1;
            }
            if (*abort)
                for (int g = max(0, issued - SC); g < issued; ++g)
                    mbar_wait(&full[g % SC], (g / SC) & 1, nullptr, args.wait_ns);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = make_idesc_bf16(128, NT, false, false);
            for (int i = 0; i < n_units; ++i) {
                const int s = i % SC, sa = i % SA, db = i % ND;
                bool ok = mbar_wait(&full[s], (i / SC) & 1, abort, args.wait_ns);
                ok = ok && mbar_wait(&a_full[sa], (i / SA) & 1, abort, args.wait_ns);
                ok = ok && mbar_wait(&d_free[db], ((i / ND) & 1) ^ 1, abort, args.wait_ns);
                if (!ok) {
                    fail();
                    break;
                }
                tc_fence_after();
                const uint32_t xs = smem_u32(sX + s * kX);
                for (int b = 0; b < kGvBlk; ++b)
                    for (int k = 0; k < 4; ++k)
                        umma_bf16_ts(tmem + kDCol + db * kDCols + static_cast<uint32_t>(b * NT),
                                     tmem + sa * kACols + static_cast<uint32_t>(b * 32 + k * 8),
                                     make_sw128_desc(xs + b * kXb + k * 32, 16, 1024), idesc,
                                     k > 0 ? 1u : 0u);
                umma_commit(&empty[s]);
                umma_commit(&a_free[sa]);
                umma_commit(&d_full[db]);
            }
        }
    } else if (warp < kGvEpiWarp) {
        // ------------------------------------------------------------------ decoders
        const int q = warp & 3;
        const int grp = (warp - 2) >> 2;
        const int row = q * 32 + lane;
        const uint32_t tlane = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t* mylut = lut + lane;
        for (int i = grp; i < n_units; i += kGvDecGroups) {
            const int s = i % SC, sa = i % SA;
            if (!mbar_wait_warp(&full[s], (i / SC) & 1, abort, args.wait_ns)) {
                fail();
                break;
            }
            if (!mbar_wait_warp(&a_free[sa], ((i / SA) & 1) ^ 1, abort, args.wait_ns)) {
                fail();
                break;
            }
            // row's 128 code bytes (4 blocks): one 32-column tensor-memory store per block
            // (the code tile is stored with the 128-byte swizzle: chunk j of row r sits at
            //  chunk j ^ (r & 7), so a warp's reads spread over all banks)
            const uint8_t* crow = sC + s * kCodes + row * 32 * kGvBlk;
            const uint32_t sw = static_cast<uint32_t>(row & 7);
#pragma unroll
            for (int b = 0; b < kGvBlk; ++b) {
                const uint4 c0 = *reinterpret_cast<const uint4*>(crow + (((2 * b) ^ sw) << 4));
                const uint4 c1 = *reinterpret_cast<const uint4*>(crow + (((2 * b + 1) ^ sw) << 4));
                const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                uint32_t v[32];
#pragma unroll
                for (int w = 0; w < 8; ++w) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) v[4 * w + e] = mylut[((cw[w] >> (8 * e)) & 0xFFu) * 32];
                }
                tmem_st_32x32b_x32(tmem + tlane + sa * kACols + static_cast<uint32_t>(b * 32), v);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);         // codes consumed
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[sa]);
        }
    } else {
        // ------------------------------------------------------------------ accumulate
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const int et = threadIdx.x - 32 * kGvEpiWarp;     // 0..127 within the 4 warps
        const uint32_t tlane = static_cast<uint32_t>(q * 32) << 16;
        float acc[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = 0.f;
        bool waited_primary = false;
        bool us_staged = false;
        int tile_slot = 0;
        // bounded meeting point of the four accumulate warps (no hardware barrier that a warp
        // leaving on a timeout could strand the others at)
        auto epi_sync = [&](int which, int seg) -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(&seg_bar[which]);
            return mbar_wait_warp(&seg_bar[which], static_cast<uint32_t>(seg & 1), abort, args.wait_ns);
        };
        // Block-scale inputs of a unit (kGvBlk consecutive blocks of this row), loaded two
        // units ahead (an L2 round trip is longer than a unit) and rotated through registers.
        struct ScaleIn {
            uint32_t q8[kGvBlk];
            float c2[kGvBlk];
        };
        auto load_scale = [&](int i) -> ScaleIn {
            ScaleIn v;
#pragma unroll
            for (int b = 0; b < kGvBlk; ++b) {
                v.q8[b] = 0u;
                v.c2[b] = 0.f;
            }
            if (i < n_units) {
                const int u = u0 + i;
                const int64_t grow = static_cast<int64_t>(u / args.kt4) * 128 + row;
                const int kb0 = (u % args.kt4) * kGvBlk;
                if (grow < args.d_out) {
#pragma unroll
                    for (int b = 0; b < kGvBlk; ++b) {
                        if (kb0 + b < args.kt) {
                            const int64_t blk = grow * args.kt + kb0 + b;
                            v.q8[b] = __ldg(args.absmax_q + blk);
                            v.c2[b] = __ldg(args.c2 + (blk >> 8));
                        }
                    }
                }
            }
            return v;
        };
        ScaleIn p0 = load_scale(0), p1 = load_scale(1);
        for (int i = 0; i < n_units; ++i) {
            const int u = u0 + i;
            const int db = i % ND;
            float sc[kGvBlk];
#pragma unroll
            for (int b = 0; b < kGvBlk; ++b) sc[b] = nf4_block_scale(p0.q8[b], p0.c2[b]);
            p0 = p1;
            p1 = load_scale(i + 2);
            if (!mbar_wait_warp(&d_full[db], (i / ND) & 1, abort, args.wait_ns)) {
                fail();
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int b = 0; b < kGvBlk; ++b) {
                const uint32_t dcol = kDCol + db * kDCols + static_cast<uint32_t>(b * NT);
                uint32_t r0[16], r1[16];
                tmem_ld_32x32b_x16(tmem + tlane + dcol, r0);
                if constexpr (NT == 32) tmem_ld_32x32b_x16(tmem + tlane + dcol + 16, r1);
                tmem_ld_wait();
#pragma unroll
                for (int t = 0; t < 16; ++t) acc[t] = fmaf(sc[b], __uint_as_float(r0[t]), acc[t]);
                if constexpr (NT == 32) {
#pragma unroll
                    for (int t = 0; t < 16; ++t) acc[16 + t] = fmaf(sc[b], __uint_as_float(r1[t]), acc[16 + t]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_free[db]);
            // end of this CTA's range inside the row tile?
            const int tile = u / args.kt4;
            const bool seg_end = (u + 1 == u1) || ((u + 1) % args.kt4 == 0);
            if (!seg_end) continue;
            float* pp = args.part + ((static_cast<int64_t>(blockIdx.x) * args.tiles_per_cta + tile_slot) * 128 + row) * NT;
#pragma unroll
            for (int t = 0; t < NT; t += 4)
                *reinterpret_cast<float4*>(pp + t) = make_float4(acc[t], acc[t + 1], acc[t + 2], acc[t + 3]);
#pragma unroll
            for (int t = 0; t < NT; ++t) acc[t] = 0.f;
            const int seg = tile_slot++;
            __threadfence();
            if (!epi_sync(0, seg)) {
                fail();
                break;
            }
            if (et == 0) {
                if (!waited_primary) griddep_wait();     // counters / s*U from the pre-pass
                // CTAs whose ranges touch this tile
                const int first_u = tile * args.kt4, last_u = min(args.units, (tile + 1) * args.kt4) - 1;
                int c_first = static_cast<int>((static_cast<int64_t>(first_u) * gridDim.x) / args.units);
                while (c_first + 1 < static_cast<int>(gridDim.x) && gv_start(c_first + 1, args.units, gridDim.x) <= first_u) ++c_first;
                while (gv_start(c_first, args.units, gridDim.x) > first_u) --c_first;
                int c_last = static_cast<int>((static_cast<int64_t>(last_u) * gridDim.x) / args.units);
                while (c_last + 1 < static_cast<int>(gridDim.x) && gv_start(c_last + 1, args.units, gridDim.x) <= last_u) ++c_last;
                while (gv_start(c_last, args.units, gridDim.x) > last_u) --c_last;
                const int need = c_last - c_first + 1;
                const int done = atomicAdd(args.counters + tile, 1) + 1;
                *last_flag = (done == need) ? (c_first + 1) : 0;    // 0: not last
                if (done == need) *(last_flag + 1) = c_last;
            }
            waited_primary = true;
            if (!epi_sync(1, seg)) {
                fail();
                break;
            }
            const int lf = *last_flag;
            if (lf == 0) continue;
            __threadfence();
            griddep_wait();
            if (!us_staged) {      // s*U of all tokens into shared memory, once per CTA
                for (int e = et; e < args.T * args.r; e += 128) s_us[e] = args.us[e];
                us_staged = true;
                __syncwarp();
                if (lane == 0) mbar_arrive(us_bar);
                if (!mbar_wait_warp(us_bar, 0, abort, args.wait_ns)) {
                    fail();
                    break;
                }
            }
            const int c_first = lf - 1, c_last = *(last_flag + 1);
            const int64_t grow = static_cast<int64_t>(tile) * 128 + row;
            if (grow < args.d_out) {
                float out[NT];
#pragma unroll
                for (int t = 0; t < NT; ++t) out[t] = 0.f;
                for (int c = c_first; c <= c_last; ++c) {
                    const int slot = tile - gv_start(c, args.units, gridDim.x) / args.kt4;
                    const float* src = args.part + ((static_cast<int64_t>(c) * args.tiles_per_cta + slot) * 128 + row) * NT;
#pragma unroll
                    for (int t = 0; t < NT; t += 4) {
                        const float4 p4 = __ldcg(reinterpret_cast<const float4*>(src + t));
                        out[t] += p4.x;
                        out[t + 1] += p4.y;
                        out[t + 2] += p4.z;
                        out[t + 3] += p4.w;
                    }
                }
                // adapter term: (s U[t, :]) . B[row, :], the B row in chunks of 8 from registers
                const __nv_bfloat16* brow = args.B + grow * args.r;
                for (int j0 = 0; j0 < args.r; j0 += 8) {
                    float b8[8];
                    if (j0 + 8 <= args.r && (args.r & 7) == 0) {
                        const uint4 bv = __ldg(reinterpret_cast<const uint4*>(brow + j0));
                        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&bv);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(b2[e]);
                            b8[2 * e] = f.x;
                            b8[2 * e + 1] = f.y;
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) b8[e] = j0 + e < args.r ? __bfloat162float(brow[j0 + e]) : 0.f;
                    }
                    const int jn = min(8, args.r - j0);
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        if (t < args.T) {
                            const float* ust = s_us + t * args.r + j0;
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                if (e < jn) out[t] = fmaf(ust[e], b8[e], out[t]);
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    if (t < args.T)
                        args.H[static_cast<int64_t>(t) * args.d_out + grow] = __float2bfloat16_rn(out[t]);
            }
        }
        if (!waited_primary) griddep_wait();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Pre-pass for the decode-size forward: U = X A^T (fp32 accumulation), s U in fp32 for the
// adapter term, U in the call dtype for the backward, and zeroed tile counters.  Grid
// (r, ceil(T / 4)): each warp computes one (token, adapter row) dot product with all of its
// loads in flight at once.  Lets the dependent stream kernel start immediately.
__global__ void __launch_bounds__(128) k_small_u(const __nv_bfloat16* __restrict__ X, int T,
                                                 int d_in, const __nv_bfloat16* __restrict__ A,
                                                 int r, float s, float* __restrict__ us,
                                                 __nv_bfloat16* __restrict__ u_save,
                                                 int* __restrict__ counters, int n_counters) {
    griddep_launch_dependents();
    const int j = blockIdx.x;
    const int t = blockIdx.y * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (j == 0 && blockIdx.y == 0)
        for (int i = threadIdx.x; i < n_counters; i += blockDim.x) counters[i] = 0;
    if (t >= T) return;
    const __nv_bfloat16* a = A + static_cast<int64_t>(j) * d_in;
    const __nv_bfloat16* x = X + static_cast<int64_t>(t) * d_in;
    float acc = 0.f;
    for (int k0 = lane * 8; k0 < d_in; k0 += 32 * 8 * 4) {
        uint4 av[4], xv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int k = k0 + u * 256;
            av[u] = k < d_in ? __ldg(reinterpret_cast<const uint4*>(a + k)) : make_uint4(0, 0, 0, 0);
            xv[u] = k < d_in ? __ldg(reinterpret_cast<const uint4*>(x + k)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&av[u]);
            const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&xv[u]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 af = __bfloat1622float2(a2[e]);
                const float2 xf = __bfloat1622float2(x2[e]);
                acc = fmaf(af.x, xf.x, acc);
                acc = fmaf(af.y, xf.y, acc);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
        us[static_cast<int64_t>(t) * r + j] = s * acc;
        if (u_save) u_save[static_cast<int64_t>(t) * r + j] = __float2bfloat16_rn(acc);
    }
}

}  // namespace qlora

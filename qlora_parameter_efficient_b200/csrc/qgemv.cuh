// qgemv.cuh -- decode-size forward (T <= 16 tokens): an HBM-bound stream over the NF4 codes.
//
//   H[t, n] = (1/127) sum_b q8_b(n) c2_b(n) sum_{k in b} L16(code(n, k)) x[t, k]
//             + (s U[t, :]) . B[n, :]
//
// With a handful of tokens every weight is used T times, so the layer is a weight stream
// (0.516 B per weight) and the decode has to keep pace with HBM.  The block scale is factored
// out of the block's dot product -- dequantize = L(code) x s_b ("Low-Rank Adaptation (LoRA) and
// QLoRA: Mathematical Foundations...", section "1. 4-bit NormalFloat (NF4) Quantization";
// s_b = q8_b c2_b / 127 is the block constant of "2. Double Quantization (DQ)"): each weight
// decodes to its unscaled level rounded to bf16, the tensor cores form the block's partial dot
// product in fp32, q8_b c2_b multiplies the fp32 partial and the common 1/127 is applied once to
// the output.  Identical in exact arithmetic; the level is rounded to bf16 before the scale
// instead of after (relative 2^-9 per weight, averaging out in the sum).
//
// Why warp-level mma.sync and not tcgen05 here: one tcgen05.mma of M = 128, K = 16 occupies
// the SM's tensor core for ~130-190 cycles whatever N is (measured on B200 with N = 16..256),
// i.e. at most ~16 weights per cycle when the weights are the M x K operand -- well below the
// stream rate.  mma.sync m16n8k16 (~900 MAC per SM cycle measured) takes its operands from
// registers, so the codes decode (byte-permute arithmetic on the symmetric level table) straight
// into A fragments.
//
// K order inside a block.  The dot product over a block's 64 K is order-free, so K is permuted
// consistently in A and X: in k16 step j, mma K positions {2c, 2c+1, 2c+8, 2c+9} (thread c of
// a quad) are block elements 16c + 4j + {0, 1, 2, 3}.  A thread's 8 code bytes 8c..8c+7 of a row
// then supply its A registers of all four steps, and its X fragment is the 16 consecutive
// elements 16c..16c+15 of the token's row.
//
// Work split.  The rows are cut into tiles of M rows (a multiple of 16, chosen per shape so
// that the tiles fill the SMs); a cluster of C CTAs (C = 1, 2, 4 or 8) owns a contiguous range
// of tiles and CTA rank p owns K blocks [kb_lo, kb_hi) of every row.  Warp w owns the blocks
// kb_lo + w + 8j: their X fragments are loaded once into registers and stay there.  A stage is
// 16 consecutive rows x the rank's K range -- 16 contiguous runs, one 3-D TMA box (pieces of 128
// bytes, 128-byte swizzle, so the fragment reads are bank-conflict free); the warps take turns
// issuing the refills.  Across the M/16 stages of a tile each warp accumulates q8 c2 x partial
// in fp32 registers; the tile's absmax bytes and c2 values come in once per tile by cp.async.
// At the end of a tile warp w sums 16-row group w over the 8 warps in warp order, the ranks' sums
// meet in rank 0's shared memory over DSMEM, and rank 0 sums them in rank order, applies 1/127,
// adds the adapter term (a few mma steps) and writes H.  No global partials, atomics or
// semaphores: the sums are deterministic and the tail is on-chip.
#pragma once

#include "common.cuh"
#include "nf4.cuh"

namespace qlora {

constexpr int kGvWarps = 8;
constexpr int kGvThreads = 32 * kGvWarps;
constexpr int kGvUsMax = 16 * 128; // s*U staging (bf16): T <= 16 tokens x r <= 128
constexpr int kGvTabS = 6144;      // a tile's block scales: M x (kb_hi - kb_lo + 1) <= this
constexpr int kGvRawC2 = 320;      // a tile's c2 groups: M x kt / 256 + 2 <= this
constexpr int kGvBrowMax = 8192;  // a tile's adapter rows: M x (r + 8) bf16 <= this

template <int NT8>
struct GvCfg {
    static constexpr int NT = 8 * NT8;                 // token tile
    static constexpr int NBW = 8 / NT8;                // blocks per warp (X fragments in registers)
    static constexpr int kMaxBlk = 8 * NBW;            // blocks of a CTA's K range
    static constexpr int MW = NT8 == 1 ? 8 : 6;        // max 16-row groups per tile
    static constexpr int kStage = 16 * kMaxBlk * 32;   // 16 rows x the K range (<= 32 KB)
    static constexpr int S = NT8 == 1 ? 3 : 4;
    static constexpr int kMaxRanks = NT8 == 1 ? 4 : 8;  // cluster size limit
    static constexpr int kSlot = 32 * MW * NT8 * 16;   // one warp's partials of a tile
    static constexpr int kTree = 8 * kSlot;            // every warp's partials
    static constexpr int kRing = kMaxRanks * kSlot;    // rank 0: one CTA sum per rank
    static constexpr int kStageOff = 0;
    static constexpr int kTreeOff = kStageOff + S * kStage;
    static constexpr int kRingOff = kTreeOff + kTree;
    static constexpr int kUsOff = kRingOff + kRing;
    static constexpr int kTabOff = kUsOff + kGvUsMax * 2;   // the tile's scales [M][nbk + 1] fp32
    static constexpr int kBrowOff = kTabOff + kGvTabS * 4;  // the tile's B rows [M][r + 8] bf16
    static constexpr int kRawOff = kBrowOff + kGvBrowMax * 2;   // [2] absmax bytes, then c2
    static constexpr int kRawBuf = kGvTabS + kGvRawC2 * 4;
    static constexpr int kBarOff = kRawOff + 2 * kRawBuf;
    static constexpr int kSmem = kBarOff + 256 + 1024;   // barriers + alignment slack
    static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

// 4-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros without reading.
__device__ __forceinline__ void cp_async_4(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(src_bytes)
                 : "memory");
}
// 16-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros without reading.
__device__ __forceinline__ void cp_async_16(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x),
                 "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}


struct GvArgs {
    int T;                   // tokens (1..NT)
    int d_out, d_in, kt;     // kt = d_in / 64 blocks per row (a multiple of 4)
    int M;                   // rows per tile (multiple of 16, <= MMAX)
    int tiles;               // ceil(d_out / M)
    int C;                   // CTAs per cluster (K ranks)
    int clusters;            // grid / C
    int pieces;              // 128-byte pieces per row in a stage box: ceil(kt / 4 / C)
    const __nv_bfloat16* X;  // [T][d_in]
    const uint8_t* absmax_q;
    const float* c2;
    const float* us;         // [T][r]  s * U in fp32, from the pre-pass
    const __nv_bfloat16* B;  // [d_out][r]
    int r;
    int b_vec;               // r % 8 == 0 (B rows are 16-byte aligned)
    __nv_bfloat16* H;        // [T][d_out]
    int* err;
    uint64_t wait_ns;
};

template <int NT8>
__global__ void __launch_bounds__(kGvThreads, 1)
    k_qgemv(const __grid_constant__ CUtensorMap tmC, const GvArgs args) {
    using Cf = GvCfg<NT8>;
    constexpr int S = Cf::S, MW = Cf::MW, NT = Cf::NT, NBW = Cf::NBW;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* stages = smem + Cf::kStageOff;
    float4* part = reinterpret_cast<float4*>(smem + Cf::kTreeOff);           // [8 warps][MW][NT8][32]
    float4* ring = reinterpret_cast<float4*>(smem + Cf::kRingOff);           // [ranks][MW][NT8][32]
    __nv_bfloat16* s_us = reinterpret_cast<__nv_bfloat16*>(smem + Cf::kUsOff);   // [NT][rp]
    float* tab_s = reinterpret_cast<float*>(smem + Cf::kTabOff);             // [M][nbk + 1]
    __nv_bfloat16* s_b = reinterpret_cast<__nv_bfloat16*>(smem + Cf::kBrowOff);  // [M][r + 8]
    uint8_t* raw = smem + Cf::kRawOff;        // [2][absmax bytes [M][nbk] | c2 groups], by tile parity
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cf::kBarOff);
    uint64_t* full = bars;                     // [S] the stage's code box landed
    uint64_t* empty = full + S;                // [S] all warps done with the stage
    uint64_t* csync_bar = empty + S;           // the 8 warps meet
    uint64_t* ring_full = csync_bar + 1;       // rank 0: every rank's sum of the tile is in
    uint64_t* ring_free = ring_full + 1;       // every rank: rank 0 has consumed the ring
    volatile int* abort = reinterpret_cast<volatile int*>(ring_free + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;          // mma fragment coordinates
    const int C = args.C;
    const int rank = static_cast<int>(blockIdx.x) % C;      // cluster dims (C, 1, 1)
    const int cl = static_cast<int>(blockIdx.x) / C;
    const int t_lo = static_cast<int>((static_cast<int64_t>(cl) * args.tiles) / args.clusters);
    const int t_hi = static_cast<int>((static_cast<int64_t>(cl + 1) * args.tiles) / args.clusters);
    const int q4 = args.kt / 4;
    const int kb_lo = 4 * ((rank * q4) / C), kb_hi = 4 * (((rank + 1) * q4) / C);
    const int nbk = kb_hi - kb_lo;
    const int M = args.M, mw = M / 16;
    const int n_units = (t_hi - t_lo) * mw;          // (tile, 16-row group) sequence

    auto fail = [&]() {
        set_error(args.err, kErrTimeout);
        *abort = 1;
    };
    // ---- stage issue (one warp in turn, lane 0): 16 full rows of the rank's K range as one box
    auto issue = [&](int u) {
        if (lane != 0) return;
        const int s = u % S;
        const int row0 = (t_lo + u / mw) * M + (u % mw) * 16;
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(16 * 128 * args.pieces));
        tma_load_3d(stages + s * Cf::kStage, &tmC, &full[s], 0, row0, kb_lo / 4);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kGvWarps);
        }
        mbar_init(csync_bar, kGvWarps);
        mbar_init(ring_full, 32 * mw * C);
        mbar_init(ring_free, 1);
        *abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmC);
        for (int u = 0; u < S - 1 && u < n_units; ++u) issue(u);
    }
    const Nf4Planes planes = nf4_make_planes(1.0f);
    // X fragments of this warp's blocks, held for the whole kernel: token 8n + g, elements
    // 16c .. 16c + 15 of block kb_lo + warp + 8j
    uint32_t xw[NBW][NT8][8];
#pragma unroll
    for (int j = 0; j < NBW; ++j) {
        const int L = warp + 8 * j;
#pragma unroll
        for (int n = 0; n < NT8; ++n) {
            const int t = 8 * n + g;
            uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
            if (L < nbk && t < args.T) {
                const uint4* src = reinterpret_cast<const uint4*>(args.X + static_cast<int64_t>(t) * args.d_in + (kb_lo + L) * 64 + 16 * c);
                x0 = __ldg(src);
                x1 = __ldg(src + 1);
            }
            xw[j][n][0] = x0.x; xw[j][n][1] = x0.y; xw[j][n][2] = x0.z; xw[j][n][3] = x0.w;
            xw[j][n][4] = x1.x; xw[j][n][5] = x1.y; xw[j][n][6] = x1.z; xw[j][n][7] = x1.w;
        }
    }
    // barriers initialised (and visible cluster-wide) before any remote arrive or store
    if (C > 1) cluster_barrier();
    else __syncthreads();

    uint32_t phase = 0;
    // bounded meeting point of the 8 warps (no hardware barrier that a warp leaving on a timeout
    // could strand the others at)
    auto csync = [&]() -> bool {
        __syncwarp();
        if (lane == 0) mbar_arrive(csync_bar);
        const bool ok = mbar_spin(csync_bar, phase & 1, abort, args.wait_ns);
        ++phase;
        return ok;
    };

    // the raw tables of a tile: absmax bytes [M][nbk] and its c2 groups, by all threads, into the
    // buffer of the tile's parity
    auto prefetch_tables = [&](int tile) {
        const int row0 = tile * M;
        uint8_t* rabs = raw + ((tile - t_lo) & 1) * Cf::kRawBuf;
        float* rc2 = reinterpret_cast<float*>(rabs + kGvTabS);
        const int wpr = nbk / 4;
        for (int wi = threadIdx.x; wi < M * wpr; wi += kGvThreads) {
            const int rr = wi / wpr, q = wi % wpr;
            const bool ok = row0 + rr < args.d_out;
            cp_async_4(rabs + rr * nbk + 4 * q,
                       args.absmax_q + (ok ? static_cast<int64_t>(row0 + rr) * args.kt + kb_lo + 4 * q : 0),
                       ok ? 4u : 0u);
        }
        const int64_t rlast = min(row0 + M, args.d_out) - 1;
        const int64_t g_first = (static_cast<int64_t>(row0) * args.kt + kb_lo) >> 8;
        const int n_c2 = static_cast<int>(((rlast * args.kt + kb_hi - 1) >> 8) - g_first + 1);
        for (int e = threadIdx.x; e < n_c2; e += kGvThreads) cp_async_4(rc2 + e, args.c2 + g_first + e, 4u);
    };
    if (t_lo < t_hi) prefetch_tables(t_lo);
    int last_issued = -1;       // latest stage this warp issued (beyond the initial ones)
    bool ok_all = true;
    int tiles_done = 0;

    for (int tile = t_lo; tile < t_hi && ok_all; ++tile) {
        const int row0 = tile * M;
        // ---- the tile's block scales q8 * c2 [M][nbk + 1] from its raw tables (prefetched during
        // the previous tile), then the next tile's raw tables and (rank 0) this tile's adapter
        // rows go out; the previous tile's readers are past its end-of-tile meetings
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (!csync()) {
            fail();
            break;
        }
        const int sld = nbk + 1;                  // padded row: the 8 rows a warp reads hit 8 banks
        {
            const uint8_t* rabs = raw + ((tile - t_lo) & 1) * Cf::kRawBuf;
            const float* rc2 = reinterpret_cast<const float*>(rabs + kGvTabS);
            const int64_t g_first = (static_cast<int64_t>(row0) * args.kt + kb_lo) >> 8;
            for (int e = threadIdx.x; e < M * nbk; e += kGvThreads) {
                const int rr = e / nbk, L = e % nbk;
                const int64_t blk = static_cast<int64_t>(row0 + rr) * args.kt + kb_lo + L;
                tab_s[rr * sld + L] = row0 + rr < args.d_out
                    ? static_cast<float>(rabs[e]) * rc2[(blk >> 8) - g_first] : 0.f;
            }
        }
        if (!csync()) {
            fail();
            break;
        }
        if (rank == 0 && args.b_vec) {
            const int cpr = args.r / 8;           // 16-byte pieces per row
            for (int e = threadIdx.x; e < M * cpr; e += kGvThreads) {
                const int rr = e / cpr, q = e % cpr;
                const bool ok = row0 + rr < args.d_out;
                cp_async_16(s_b + rr * (args.r + 8) + 8 * q,
                            args.B + (ok ? static_cast<int64_t>(row0 + rr) * args.r + 8 * q : 0), ok ? 16u : 0u);
            }
        }
        if (tile + 1 < t_hi) prefetch_tables(tile + 1);
        // ---- the tile's 16-row groups, one stage each (a runtime loop: its body is emitted once)
#pragma unroll 1
        for (int m = 0; m < mw; ++m) {
            const int u = (tile - t_lo) * mw + m;
            const int s = u % S;
            if (warp == u % kGvWarps && u + S - 1 < n_units) {
                // refill the slot of stage u - 1 with stage u + S - 1 once every warp has left it
                // (the warps take this duty in turn)
                const int nxt = u + S - 1;
                if (!mbar_wait_warp(&empty[nxt % S], ((nxt / S) & 1) ^ 1, abort, args.wait_ns)) {
                    ok_all = false;
                    break;
                }
                issue(nxt);
                last_issued = nxt;
            }
            if (!mbar_wait_warp(&full[s], (u / S) & 1, abort, args.wait_ns)) {
                ok_all = false;
                break;
            }
            const uint8_t* st = stages + s * Cf::kStage;
            const int ra_ = 16 * m + g, rb_ = ra_ + 8;          // rows within the tile
            float acc[NT8][4];
#pragma unroll
            for (int n = 0; n < NT8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
#pragma unroll
            for (int j = 0; j < NBW; ++j) {
                const int L = warp + 8 * j;
                // (no early exit: past the rank's K range the X fragments are zero and the scale
                // is 0, and every read stays inside the stage buffer and the scale table)
                // stage layout [piece L/4][16 rows][128 B], 128-byte swizzle: block L of a row is
                // 16-byte chunks 2(L%4), 2(L%4)+1, stored at chunk ^ (row & 7)
                const uint8_t* piece = st + (L >> 2) * 2048;
                const int chunk = ((((L & 3) * 2 + (c >> 1)) ^ g) << 4) + (c & 1) * 8;
                const uint2 ca = *reinterpret_cast<const uint2*>(piece + g * 128 + chunk);
                const uint2 cb = *reinterpret_cast<const uint2*>(piece + (g + 8) * 128 + chunk);
                const uint4 a0 = nf4_decode8(ca.x, planes), a1 = nf4_decode8(ca.y, planes);
                const uint4 b0 = nf4_decode8(cb.x, planes), b1 = nf4_decode8(cb.y, planes);
                // A registers per k16 step: {row g: byte 2k, row g+8: byte 2k, row g: byte 2k+1,
                // row g+8: byte 2k+1} of the thread's 8 bytes
                const uint32_t A[4][4] = {{a0.x, b0.x, a0.y, b0.y}, {a0.z, b0.z, a0.w, b0.w},
                                          {a1.x, b1.x, a1.y, b1.y}, {a1.z, b1.z, a1.w, b1.w}};
                float tmp[NT8][4];
#pragma unroll
                for (int k = 0; k < 4; ++k)
#pragma unroll
                    for (int n = 0; n < NT8; ++n)
                        mma_bf16_16816(tmp[n], A[k], xw[j][n][2 * k], xw[j][n][2 * k + 1], k > 0);
                // q8 * c2 of rows ra_, rb_ from the tile's scale table
                const bool in_tab = L < nbk && dcheck(rb_ * sld + L < kGvTabS, args.err);
                const float sa = in_tab ? tab_s[ra_ * sld + L] : 0.f;
                const float sb = in_tab ? tab_s[rb_ * sld + L] : 0.f;
#pragma unroll
                for (int n = 0; n < NT8; ++n) {
                    acc[n][0] = fmaf(sa, tmp[n][0], acc[n][0]);
                    acc[n][1] = fmaf(sa, tmp[n][1], acc[n][1]);
                    acc[n][2] = fmaf(sb, tmp[n][2], acc[n][2]);
                    acc[n][3] = fmaf(sb, tmp[n][3], acc[n][3]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            // the warp's partial of this 16-row group
#pragma unroll
            for (int n = 0; n < NT8; ++n)
                part[((warp * MW + m) * NT8 + n) * 32 + lane] = make_float4(acc[n][0], acc[n][1], acc[n][2], acc[n][3]);
        }
        if (!ok_all) {
            fail();
            break;
        }

        asm volatile("cp.async.wait_all;" ::: "memory");   // this tile's adapter rows
        if (tiles_done == 0 && rank == 0) {
            // s*U from the pre-pass as bf16 [NT][rp] (zero beyond T and r), once per CTA; the
            // pre-pass has long finished by the end of the first tile
            const int rp = (args.r + 15) & ~15;
            griddep_wait();
            for (int e = threadIdx.x; e < NT * rp; e += kGvThreads) {
                const int t = e / rp, jj = e % rp;
                s_us[e] = __float2bfloat16_rn(t < args.T && jj < args.r ? args.us[t * args.r + jj] : 0.f);
            }
        }
        // ---- end of the tile: warp w sums group w over the 8 warps in warp order and sends it to
        // rank 0 (its own ring when C == 1)
        if (!csync()) {
            fail();
            break;
        }
        if (warp < mw) {
            float4 sum[NT8];
#pragma unroll
            for (int n = 0; n < NT8; ++n) {
                sum[n] = part[(warp * NT8 + n) * 32 + lane];
#pragma unroll
                for (int w = 1; w < kGvWarps; ++w) {
                    const float4 v = part[((w * MW + warp) * NT8 + n) * 32 + lane];
                    sum[n].x += v.x;
                    sum[n].y += v.y;
                    sum[n].z += v.z;
                    sum[n].w += v.w;
                }
            }
            if (tiles_done > 0 && !mbar_wait_warp(ring_free, (tiles_done - 1) & 1, abort, args.wait_ns)) {
                fail();
                break;
            }
            const uint32_t dst = mapa_shared(smem_u32(ring + rank * (Cf::kSlot / 16) + (warp * NT8) * 32 + lane), 0);
#pragma unroll
            for (int n = 0; n < NT8; ++n) st_cluster_v4(dst + n * 32 * 16, sum[n]);
            mbar_arrive_remote(mapa_shared(smem_u32(ring_full), 0));   // release.cluster
        }
        ++tiles_done;
        if (rank != 0) continue;

        // ---- rank 0: finalize the tile -- ranks in order, 1/127, adapter term, H.  Warp w
        // takes m16 tiles w, w + 8, ...
        if (!mbar_wait_cluster(ring_full, (tiles_done - 1) & 1, abort, args.wait_ns)) {
            fail();
            break;
        }
        const int rp = (args.r + 15) & ~15;          // adapter rank padded to the mma K
        for (int m = warp; m < mw; m += kGvWarps) {
            float4 tot[NT8];
#pragma unroll
            for (int n = 0; n < NT8; ++n) tot[n] = ring[(m * NT8 + n) * 32 + lane];
            for (int rr = 1; rr < C; ++rr) {
#pragma unroll
                for (int n = 0; n < NT8; ++n) {
                    const float4 v = ring[rr * (Cf::kSlot / 16) + (m * NT8 + n) * 32 + lane];
                    tot[n].x += v.x;
                    tot[n].y += v.y;
                    tot[n].z += v.z;
                    tot[n].w += v.w;
                }
            }
            const int rbase = row0 + 16 * m;
            // this thread's outputs: rows rbase + g, rbase + g + 8; tokens 8n + 2c, 8n + 2c + 1
            float out[2][NT8][2];
#pragma unroll
            for (int n = 0; n < NT8; ++n) {
                out[0][n][0] = __fdiv_rn(tot[n].x, 127.0f);
                out[0][n][1] = __fdiv_rn(tot[n].y, 127.0f);
                out[1][n][0] = __fdiv_rn(tot[n].z, 127.0f);
                out[1][n][1] = __fdiv_rn(tot[n].w, 127.0f);
            }
            if (args.b_vec) {
                // adapter term on the tensor cores: [16 rows x rp] B rows times [rp x NT]
                // (s U)^T, fp32 accumulation
                float adp[NT8][4];
                for (int k0 = 0; k0 < rp; k0 += 16) {
                    uint32_t a[4];
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2) {
                        const int rr = 16 * m + g + 8 * (q2 & 1);     // row within the tile
                        const int col = k0 + 2 * c + 8 * (q2 >> 1);
                        a[q2] = col < args.r ? *reinterpret_cast<const uint32_t*>(s_b + rr * (args.r + 8) + col) : 0u;
                    }
#pragma unroll
                    for (int n = 0; n < NT8; ++n) {
                        const __nv_bfloat16* ub = s_us + (8 * n + g) * rp + k0 + 2 * c;
                        mma_bf16_16816(adp[n], a, *reinterpret_cast<const uint32_t*>(ub),
                                       *reinterpret_cast<const uint32_t*>(ub + 8), k0 > 0);
                    }
                }
#pragma unroll
                for (int n = 0; n < NT8; ++n) {
                    out[0][n][0] += adp[n][0];
                    out[0][n][1] += adp[n][1];
                    out[1][n][0] += adp[n][2];
                    out[1][n][1] += adp[n][3];
                }
            } else {
                // r % 8 != 0: scalar adapter term
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int64_t grow = rbase + g + 8 * h;
                    if (grow >= args.d_out) continue;
                    const __nv_bfloat16* brow = args.B + grow * args.r;
                    for (int j = 0; j < args.r; ++j) {
                        const float bj = __bfloat162float(brow[j]);
#pragma unroll
                        for (int n = 0; n < NT8; ++n)
#pragma unroll
                            for (int e2 = 0; e2 < 2; ++e2)
                                out[h][n][e2] = fmaf(__bfloat162float(s_us[(8 * n + 2 * c + e2) * rp + j]), bj, out[h][n][e2]);
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t grow = rbase + g + 8 * h;
                if (grow >= args.d_out) continue;
#pragma unroll
                for (int n = 0; n < NT8; ++n)
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        const int t = 8 * n + 2 * c + e2;
                        if (t < args.T) args.H[static_cast<int64_t>(t) * args.d_out + grow] = __float2bfloat16_rn(out[h][n][e2]);
                    }
            }
        }
        // everyone is done with the ring: release it to every rank (the last tile needs none)
        if (!csync()) {
            fail();
            break;
        }
        if (warp == 0 && lane < C && tile + 1 < t_hi)
            mbar_arrive_remote(mapa_shared(smem_u32(ring_free), static_cast<uint32_t>(lane)));
    }
    if (lane == 0 && *abort) {
        // leave no copy in flight into shared memory of an exiting CTA: the stages this warp
        // issued (thread 0 also the initial ones) are waited for, each bounded
        if (warp == 0)
            for (int i = 0; i < min(S - 1, n_units); ++i)
                mbar_wait(&full[i % S], (i / S) & 1, nullptr, args.wait_ns);
        if (last_issued >= 0)
            mbar_wait(&full[last_issued % S], (last_issued / S) & 1, nullptr, args.wait_ns);
    }
}

// Pre-pass for the decode-size forward: U = X A^T (fp32 accumulation), s U in fp32 for the
// adapter term and U in the call dtype for the backward.  Few CTAs (ceil(r / 8), 8 warps each)
// so that they fit beside the stream kernel, which it overlaps through programmatic dependent
// launch: warp w of CTA b computes adapter row j = 8b + w for the tokens two at a time, each
// pass over a 4096-element chunk of K with all of its loads in flight at once.
// u_spad (nullable): bf16(s U) [T, ldp] for a tensor-core K-extension (columns >= r are left
// as they are: the caller zeroes them).
__global__ void __launch_bounds__(256) k_small_u(const __nv_bfloat16* __restrict__ X, int T,
                                                 int d_in, const __nv_bfloat16* __restrict__ A,
                                                 int r, float s, float* __restrict__ us,
                                                 __nv_bfloat16* __restrict__ u_save,
                                                 __nv_bfloat16* __restrict__ u_spad = nullptr,
                                                 int ldp = 0) {
    griddep_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = blockIdx.x * 8 + warp;
    if (j >= r) return;
    const __nv_bfloat16* a = A + static_cast<int64_t>(j) * d_in;
    auto dot8 = [](const uint4& p, const uint4& q, float acc) {
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&p);
        const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 pf = __bfloat1622float2(p2[e]);
            const float2 qf = __bfloat1622float2(q2[e]);
            acc = fmaf(pf.x, qf.x, acc);
            acc = fmaf(pf.y, qf.y, acc);
        }
        return acc;
    };
    for (int t0 = 0; t0 < T; t0 += 2) {
        const bool two = t0 + 1 < T;
        const __nv_bfloat16* x0p = X + static_cast<int64_t>(t0) * d_in;
        const __nv_bfloat16* x1p = X + static_cast<int64_t>(two ? t0 + 1 : t0) * d_in;
        float acc0 = 0.f, acc1 = 0.f;
        for (int kc = 0; kc < d_in; kc += 4096) {
            uint4 av[16], xv0[16], xv1[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int k = kc + 256 * i + 8 * lane;
                const bool ok = k < d_in;
                av[i] = ok ? __ldg(reinterpret_cast<const uint4*>(a + k)) : make_uint4(0, 0, 0, 0);
                xv0[i] = ok ? __ldg(reinterpret_cast<const uint4*>(x0p + k)) : make_uint4(0, 0, 0, 0);
                xv1[i] = (ok && two) ? __ldg(reinterpret_cast<const uint4*>(x1p + k)) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                acc0 = dot8(av[i], xv0[i], acc0);
                acc1 = dot8(av[i], xv1[i], acc1);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            acc0 += __shfl_xor_sync(0xffffffffu, acc0, o);
            acc1 += __shfl_xor_sync(0xffffffffu, acc1, o);
        }
        if (lane == 0) {
            us[static_cast<int64_t>(t0) * r + j] = s * acc0;
            if (u_save) u_save[static_cast<int64_t>(t0) * r + j] = __float2bfloat16_rn(acc0);
            if (u_spad) u_spad[static_cast<int64_t>(t0) * ldp + j] = __float2bfloat16_rn(s * acc0);
            if (two) {
                us[static_cast<int64_t>(t0 + 1) * r + j] = s * acc1;
                if (u_save) u_save[static_cast<int64_t>(t0 + 1) * r + j] = __float2bfloat16_rn(acc1);
                if (u_spad) u_spad[static_cast<int64_t>(t0 + 1) * ldp + j] = __float2bfloat16_rn(s * acc1);
            }
        }
    }
}

}  // namespace qlora

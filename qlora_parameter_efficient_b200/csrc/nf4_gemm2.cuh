// nf4_gemm2.cuh -- persistent 2-SM (tcgen05 cta_group::2) fused NF4-decode GEMM.
//
//   forward (B_MN = false):  H[T, d_out]  = X[T, d_in]  W^T + sU[T, RP] B_pad[d_out, RP]^T
//   dX      (B_MN = true):   dX[T, d_in]  = dH[T, d_out] W  + sG[T, RP] A_pad[RP, d_in]
//   FP8 forward (FP8 = true): H = (X8 W8^T + U'[T, RP] B_pad^T) / (sigma_x sigma_w), X8 the
//     E4M3 activation, W8 the weight decoded to E4M3 in sigma_w units, U' the adapter term
//     already in those units; the main K steps are kind::f8f6f4 MMAs (K = 128 per step), the
//     adapter steps stay kind::f16 bf16 MMAs into the same fp32 accumulator.
//   FP8 dX (FP8 = B_MN = true): dX = (dH8 W8 + G'[T, RP] A_pad) / (sigma_g sigma_w), dH8 the
//     E5M2 gradient, W8 decoded MN-major (a K step is 128 weight rows x this CTA's 128 columns,
//     one 128-byte swizzled row per weight row).
//
// A cluster of two CTAs (a "pair") computes 256 x 256 output tiles with 256x256x16 UMMA
// instructions issued by the leader CTA.  Each CTA holds half of the A tile (128 token rows)
// and half of the B tile (128 of the 256 weight columns), so each SM decodes only its half of
// the weight tile and every decoded weight feeds 256 tokens; each CTA's tensor memory holds
// its 128 accumulator rows x 256 columns, double-buffered (512 columns) so the epilogue of one
// tile overlaps the main loop of the next.  The grid is persistent: pair p handles tiles
// p, p + npairs, ...  When the last wave would leave most pairs idle (its tile count is at most
// half the pairs), its tiles are each split in two along K and run on two pairs: the first half
// takes main K steps [0, k/2), the second the rest plus the adapter steps.  Each epilogue warp
// of a split tile writes its fp32 partial (32 rows x 256 columns) to a workspace slot and takes
// a ticket from a per-warp counter; the second finisher adds the other half's partial to its
// own and writes the bf16 output.  fp32 addition of two terms is commutative, so the result does
// not depend on which half finishes first, and no CTA ever waits for another.
//
// Warp roles per CTA (6 + 4 x decoder groups warps):
//   warp 0       TMA producer: this CTA's A half and NF4 code tile (or the K-extension
//                adapter tiles) into a 6-stage ring, completing on the local full[s]; the
//                decoded B halves live in a separate 6-slot ring (the adapter K
//                step's B tile is loaded straight into its slot).
//   warp 1       leader CTA only: issues the MMAs, commits stage release (empty[s]) and
//                accumulator-ready (accf[b]) to both CTAs.
//   warps 2..5   epilogue: TMEM -> bf16 -> global, then release the accumulator buffer to the
//                leader (acc_empty[b]).
//   warps 6..    NF4 decoders in groups of four warps that take K steps in turn: wait
//                for the stage's code tile, decode 128 blocks of 64 weights into the stage's
//                B half (one block per thread, written in the 128-byte-swizzled UMMA layout),
//                then arrive on a local barrier: the leader's ready[s] directly, the peer's
//                dec_done[s], which the peer's warp 1 forwards to the leader's ready[s] with
//                one remote arrive.  For the adapter K steps the group only reports
//                "landed".  ready[s] thus certifies, for both CTAs, that the A half has
//                landed and the B half is in place.
// The peer's remote arrives (ready, acc_empty) carry no generic-proxy payload: the decoded
// tile was handed to the async proxy by fence.proxy.async in every writing thread, and TMEM
// reads are retired by tcgen05.wait::ld before tcgen05.fence::before_thread_sync; so they use
// the default CTA-scope release (a cluster-scope release costs ~0.5 us per arrive and, made
// once per K step by one thread, set the step period).
// Every wait is bounded (QLORA_ERR_TIMEOUT on expiry); all TMA loads are plain local loads.
#pragma once

#include "common.cuh"
#include "nf4.cuh"

namespace qlora {

// ------------------------------------------------------------------ cluster / 2-SM PTX

__device__ __forceinline__ void tmem_alloc_2sm(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_2sm() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_2sm(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void umma_bf16_ss_2sm(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                 uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the barrier at this offset in both CTAs of the pair when all previously
// issued tcgen05 operations of this thread have completed.
__device__ __forceinline__ void umma_commit_2sm_both(uint64_t* bar) {
    const uint16_t mask = 0x3;
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"(mask)
        : "memory");
}

// ------------------------------------------------------------------ kernel

#ifndef QLORA_G2_DEC_GROUPS
#define QLORA_G2_DEC_GROUPS 3
#endif
constexpr int kG2DecGroups = QLORA_G2_DEC_GROUPS;   // groups of 4 decoder warps
#ifndef QLORA_G2_STAGES_A
#define QLORA_G2_STAGES_A 6
#endif
#ifndef QLORA_G2_STAGES_B
#define QLORA_G2_STAGES_B 6
#endif
constexpr int kG2StagesA = QLORA_G2_STAGES_A;   // A half + NF4 codes: covers the TMA latency
constexpr int kG2StagesB = QLORA_G2_STAGES_B;   // decoded B half: covers the signalling latency
static_assert(kG2StagesA >= kG2StagesB, "B-slot reuse is gated through the A ring");
// (bf16: 3 groups with 6 A stages and 6 B slots measured best against 4 groups with (8, 4) and
// 3 groups with (6, 5), (6, 4); a B slot freed SB - 1 MMA steps back gives the hand-off from
// the decoders that much slack.)
// Each decoder group waits on full[] of the steps it handles; with the ring depth a multiple
// of the group count, the previous phase of every such barrier belongs to a step the same
// group has already observed, so no parity wait can alias.
static_assert(kG2StagesA % kG2DecGroups == 0, "A-ring depth must be a multiple of the groups");
// FP8: a K step is 128 E4M3 columns (the same 128-byte rows), its codes tile twice as large,
// so shared memory holds fewer stages: 3 decoder groups with 6 A stages and 3 decoded-B slots
// (measured best of 1, 2, 3 or 4 groups with (8, 2), (6, 4), (6, 3), (6, 2), (4, 4) rings).
#ifndef QLORA_G2_FP8_DEC_GROUPS
#define QLORA_G2_FP8_DEC_GROUPS 3
#endif
#ifndef QLORA_G2_FP8_STAGES_A
#define QLORA_G2_FP8_STAGES_A 6
#endif
#ifndef QLORA_G2_FP8_STAGES_B
#define QLORA_G2_FP8_STAGES_B 3
#endif
static_assert(QLORA_G2_FP8_STAGES_A >= QLORA_G2_FP8_STAGES_B, "B-slot reuse is gated through the A ring");
static_assert(QLORA_G2_FP8_STAGES_A % QLORA_G2_FP8_DEC_GROUPS == 0,
              "A-ring depth must be a multiple of the groups");

template <bool FP8 = false>
struct G2Smem {
    static constexpr int kGroups = FP8 ? QLORA_G2_FP8_DEC_GROUPS : kG2DecGroups;
    static constexpr int kThreads = 32 * (6 + 4 * kGroups);
    static constexpr int SA = FP8 ? QLORA_G2_FP8_STAGES_A : kG2StagesA;
    static constexpr int SB = FP8 ? QLORA_G2_FP8_STAGES_B : kG2StagesB;
    static constexpr int kKStep = FP8 ? 128 : 64;  // K columns per step
    static constexpr int kA = 128 * 128;          // this CTA's A half, one K step (128-byte rows)
    static constexpr int kC = 128 * kKStep / 2;   // NF4 codes of the B half
    static constexpr int kB = 128 * 128;          // this CTA's decoded B half
    static constexpr int kStageA = kA + kC;
    static constexpr int kBars = 512;
    static constexpr int kTotal = 1024 + SA * kStageA + SB * kB + kBars;
    static_assert(kTotal <= 232448, "shared memory budget");
};

// Instruction descriptor for kind::f8f6f4, fp32 D, dense: A E4M3 (or E5M2), B E4M3 K-major
// (or MN-major).
__host__ __device__ constexpr uint32_t make_idesc_f8(int M, int N, bool a_e5m2, bool b_mn) {
    return (1u << 4)                                  // D format fp32
           | (static_cast<uint32_t>(a_e5m2) << 7)     // A format: 0 E4M3, 1 E5M2
           | (0u << 10)                               // B format E4M3
           | (static_cast<uint32_t>(b_mn) << 16)      // B major (0 = K)
           | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

__device__ __forceinline__ void umma_e4m3_ss_2sm(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                 uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

struct Gemm2Args {
    int M, N;              // output rows (tokens) and columns
    int k_steps;           // main K steps of 64
    int ext_steps;         // adapter K-extension steps of 64
    int ext_k16_last;      // K=16 MMAs in the last extension step
    int m_tiles, n_tiles;  // 256 x 256 tiles
    const uint8_t* absmax_q;
    const float* c2;
    int nf4_rows;          // d_out of the stored weight
    int nf4_bpr;           // d_in / 64
    __nv_bfloat16* out;
    int64_t ld_out;
    const float* col_scale;  // [N] factor applied to output column n before rounding, or NULL
    int split_tiles;       // trailing tiles split in two along K (0 = none)
    float* part;           // [split_tiles][2 ranks][4 warps][2 halves][2048 float4] fp32 partials
    int* cnt;              // [split_tiles][2 ranks][4 warps] tickets, zero at launch
    const float* x_scale;  // FP8: sigma_x (device scalar)
    const float* w_scale;  // FP8: sigma_w (device scalar)
    int* err;
    uint64_t wait_ns;
};

// Float4 index of (row = lane, columns 32c + 4g .. +3) in a warp's 32 x 256 partial slot:
// consecutive lanes of one store are consecutive 16-byte words.
__device__ __forceinline__ int g2_part_idx(int c, int g, int lane) { return (c * 8 + g) * 32 + lane; }

template <bool B_MN, bool FP8 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(G2Smem<FP8>::kThreads, 1)
    k_nf4_gemm2(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmC,
                const __grid_constant__ CUtensorMap tmAx, const __grid_constant__ CUtensorMap tmBx,
                const Gemm2Args args) {
    using L = G2Smem<FP8>;
    constexpr int SA = L::SA;
    constexpr int SB = L::SB;
    constexpr int NG = L::kGroups;          // decoder groups of 4 warps
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;                          // [SA][kA]
    uint8_t* sB = smem + SA * L::kA;             // [SB][kB]
    uint8_t* sC = sB + SB * L::kB;               // [SA][kC]
    uint64_t* bars = reinterpret_cast<uint64_t*>(sC + SA * L::kC);
    uint64_t* full = bars;                  // [SA] local: A half + codes (or ext tiles) landed
    uint64_t* empty = full + SA;            // [SA] both: A stage consumed by the MMAs
    uint64_t* ready = empty + SA;           // [SA] leader: both halves ready for this K step
    uint64_t* dec_done = ready + SA;        // [SA] peer: its decoder warps finished the step
    uint64_t* accf = dec_done + SA;         // [2]  both: accumulator buffer complete
    uint64_t* acc_empty = accf + 2;         // [2]  leader: buffer drained (8 warp arrivals)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();          // 0 = leader, 1 = peer
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int n_tiles_total = args.m_tiles * args.n_tiles;
    const int iters_per_tile = args.k_steps + args.ext_steps;
    // Schedule of this pair: n_full whole tiles pair, pair + npairs, ..., then (split only)
    // one half tile, K steps [hb, he) of tile half_tile.
    const int split_base = n_tiles_total - args.split_tiles;   // a multiple of npairs when split
    int n_full, half = -1, half_tile = 0, hb = 0, he = 0;
    if (args.split_tiles > 0) {
        n_full = split_base / npairs;
        if (pair < 2 * args.split_tiles) {
            half = pair & 1;
            half_tile = split_base + (pair >> 1);
            const int h0 = args.k_steps / 2;
            hb = half ? h0 : 0;
            he = half ? iters_per_tile : h0;
        }
    } else {
        n_full = max(0, (n_tiles_total - pair + npairs - 1) / npairs);
    }
    const int n_units = n_full + (half >= 0 ? 1 : 0);
    const int full_iters = n_full * iters_per_tile;
    const int total_iters = full_iters + (half >= 0 ? he - hb : 0);
    // (tile, K step within the tile) of this pair's git-th step
    auto step_of = [&](int git, int& tile, int& ks) {
        if (git < full_iters) {
            tile = pair + (git / iters_per_tile) * npairs;
            ks = git % iters_per_tile;
        } else {
            tile = half_tile;
            ks = hb + (git - full_iters);
        }
    };

    // Decoder cursor: (tile, K step) of the steps git = grp, grp + NG, ... of one decoder group,
    // advanced incrementally (no integer division per step).
    struct Cur {
        int git, tile, it;
    };
    auto cur_at = [&](int git) {
        Cur c;
        c.git = git;
        c.tile = 0;
        c.it = 0;
        if (git < total_iters) step_of(git, c.tile, c.it);
        return c;
    };
    auto cur_next = [&](Cur& c) {
        c.git += NG;
        if (c.git >= full_iters) {
            c.tile = half_tile;
            c.it = hb + (c.git - full_iters);
            return;
        }
        c.it += NG;
        while (c.it >= iters_per_tile) {
            c.it -= iters_per_tile;
            c.tile += npairs;
        }
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < SA; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&ready[s], 5);      // 4 leader decoder warps + the peer's forwarder
            mbar_init(&dec_done[s], 4);   // 4 peer decoder warps
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&acc_empty[b], 8);
        }
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmC);
        if (args.ext_steps > 0) {
            tma_prefetch_desc(&tmAx);
            tma_prefetch_desc(&tmBx);
        }
    }
    if (warp == 1) {
        tmem_alloc_2sm(tmem_slot, 512);
        tmem_relinquish_2sm();
    }
    tc_fence_before();
    cluster_barrier();          // barriers of both CTAs initialised; TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    griddep_enter();

    auto fail = [&]() {
        set_error(args.err, kErrTimeout);
        *abort = 1;
    };
    // Decoded-B slot git % SB is free once the MMAs of step git - SB (its previous user) have
    // completed, i.e. once empty[] of that step's A stage has fired.  Every waiter here is
    // already past full[] of step git, so the MMAs of step git - SA are done and this barrier
    // is at most one phase behind the awaited one: the parity test cannot alias.
    auto wait_slot_free = [&](int git) -> bool {
        if (git < SB) return true;
        const int g = git - SB;
        return mbar_wait(&empty[g % SA], (g / SA) & 1, abort, args.wait_ns);
    };
    auto wait_slot_free_warp = [&](int git) -> bool {
        if (git < SB) return true;
        const int g = git - SB;
        return mbar_wait_warp(&empty[g % SA], (g / SA) & 1, abort, args.wait_ns);
    };

    if (warp == 0) {
        // -------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int git = 0; git < total_iters; ++git) {
                int tile, it;
                step_of(git, tile, it);
                const int m0 = (tile % args.m_tiles) * 256 + static_cast<int>(rank) * 128;
                const int n0 = (tile / args.m_tiles) * 256 + static_cast<int>(rank) * 128;
                const int s = git % SA;
                const uint32_t ph = (git / SA) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, abort, args.wait_ns)) {
                    fail();
                    break;
                }
                uint8_t* a = sA + s * L::kA;
                uint8_t* c = sC + s * L::kC;
                if (it < args.k_steps) {
                    const int kx = it * L::kKStep;
                    mbar_arrive_expect_tx(&full[s], L::kA + L::kC);
                    tma_load_2d(a, &tmA, &full[s], kx, m0);
                    if (B_MN) tma_load_2d(c, &tmC, &full[s], n0 / 2, kx);
                    else tma_load_2d(c, &tmC, &full[s], kx / 2, n0);
                } else {
                    // adapter K step: the B tile goes straight into its decoded-B slot, once
                    // the slot's previous user (step git - SB) has been consumed
                    if (!wait_slot_free(git)) {
                        fail();
                        break;
                    }
                    uint8_t* b = sB + (git % SB) * L::kB;
                    const int kx = (it - args.k_steps) * 64;
                    mbar_arrive_expect_tx(&full[s], L::kA + L::kB);
                    tma_load_2d(a, &tmAx, &full[s], kx, m0);
                    if (B_MN) {
                        tma_load_2d(b, &tmBx, &full[s], n0, kx);
                        tma_load_2d(b + 8192, &tmBx, &full[s], n0 + 64, kx);
                    } else {
                        tma_load_2d(b, &tmBx, &full[s], kx, n0);
                    }
                }
                issued = git + 1;
            }
            if (*abort) {
                for (int g = max(0, issued - SA); g < issued; ++g)
                    mbar_wait(&full[g % SA], (g / SA) & 1, nullptr, args.wait_ns);
            }
        }
    } else if (warp == 1) {
        if (rank == 0 && lane == 0) {
            // ---------------------------------------------------------- MMA issuer (leader)
            const uint32_t idesc = make_idesc_bf16(256, 256, false, B_MN);
            const uint32_t idesc8 = make_idesc_f8(256, 256, B_MN, B_MN);
            int git = 0;
            bool ok = true;
            for (int tc = 0; ok && tc < n_units; ++tc) {
                const int buf = tc & 1;
                const uint32_t aph = (tc >> 1) & 1;
                const int it0 = tc < n_full ? 0 : hb;
                const int it1 = tc < n_full ? iters_per_tile : he;
                if (!mbar_wait_cluster(&acc_empty[buf], aph ^ 1, abort, args.wait_ns)) {
                    fail();
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * 256);
                for (int it = it0; it < it1; ++it, ++git) {
                    const int s = git % SA;
                    const int sb = git % SB;
                    if (!mbar_wait_cluster(&ready[s], (git / SA) & 1, abort, args.wait_ns)) {
                        fail();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a = smem_u32(sA + s * L::kA);
                    const uint32_t b = smem_u32(sB + sb * L::kB);
                    const int nk = (it == iters_per_tile - 1 && it >= args.k_steps) ? args.ext_k16_last : 4;
                    if (FP8 && it < args.k_steps) {
                        // 4 x K = 32 FP8 columns: 32 bytes of each 128-byte A row per MMA; B
                        // K-major the same, B MN-major 32 rows of 128 bytes
                        for (int k = 0; k < 4; ++k)
                            umma_e4m3_ss_2sm(d_tmem, make_sw128_desc(a + k * 32, 16, 1024),
                                             B_MN ? make_sw128_desc(b + k * 4096, 8192, 1024)
                                                  : make_sw128_desc(b + k * 32, 16, 1024),
                                             idesc8, (it > it0 || k > 0) ? 1u : 0u);
                    } else {
                        for (int k = 0; k < nk; ++k) {
                            const uint64_t ad = make_sw128_desc(a + k * 32, 16, 1024);
                            const uint64_t bd = B_MN ? make_sw128_desc(b + k * 2048, 8192, 1024)
                                                     : make_sw128_desc(b + k * 32, 16, 1024);
                            umma_bf16_ss_2sm(d_tmem, ad, bd, idesc, (it > it0 || k > 0) ? 1u : 0u);
                        }
                    }
                    umma_commit_2sm_both(&empty[s]);
                }
                umma_commit_2sm_both(&accf[buf]);
            }
        }
        if (rank == 1 && lane == 0) {
            // ---------------------------------------------------------- peer forwarder
            // One remote arrive per K step on the leader's ready[s].
            const uint32_t ready_leader = mapa_shared(smem_u32(&ready[0]), 0);
            for (int git = 0; git < total_iters; ++git) {
                const int s = git % SA;
                if (!mbar_wait(&dec_done[s], (git / SA) & 1, abort, args.wait_ns)) {
                    fail();
                    break;
                }
                mbar_arrive_remote_async_payload(ready_leader + static_cast<uint32_t>(s * 8));
            }
        }
    } else if (warp < 6) {
        // -------------------------------------------------------------- epilogue
        const int q = warp & 3;                    // TMEM lane quarter of this warp
        const uint32_t acc_empty_leader = mapa_shared(smem_u32(&acc_empty[0]), 0);
        // FP8: the accumulator holds sigma_x sigma_w H; both scales are powers of two
        float out_scale = 1.f;
        if constexpr (FP8) out_scale = __frcp_rn(__fmul_rn(__ldg(args.x_scale), __ldg(args.w_scale)));
        for (int tc = 0; tc < n_units; ++tc) {
            const bool is_half = tc >= n_full;
            const int tile = is_half ? half_tile : pair + tc * npairs;
            const int buf = tc & 1;
            const uint32_t aph = (tc >> 1) & 1;
            if (!mbar_wait_warp(&accf[buf], aph, abort, args.wait_ns)) {
                fail();
                break;
            }
            tc_fence_after();
            const int mt = tile % args.m_tiles, nt = tile / args.m_tiles;
            const int64_t grow = static_cast<int64_t>(mt) * 256 + rank * 128 + q * 32 + lane;
            const int gc0 = nt * 256;
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(buf * 256);
            const float4* other = nullptr;
            if (is_half) {
                // publish this half's partial, then take a ticket: the second finisher adds
                const int64_t slot = (static_cast<int64_t>(half_tile - split_base) * 2 + rank) * 4 + q;
                float4* mine = reinterpret_cast<float4*>(args.part) + ((slot * 2 + half) << 11);
#pragma unroll 1
                for (int c = 0; c < 8; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int g = 0; g < 8; ++g)
                        mine[g2_part_idx(c, g, lane)] =
                            make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]),
                                        __uint_as_float(r[4 * g + 2]), __uint_as_float(r[4 * g + 3]));
                }
                __threadfence();
                __syncwarp();
                int ticket = 0;
                if (lane == 0) ticket = atomicAdd(args.cnt + slot, 1);
                ticket = __shfl_sync(0xffffffffu, ticket, 0);
                if (ticket == 1) {
                    __threadfence();
                    other = reinterpret_cast<const float4*>(args.part) + ((slot * 2 + (half ^ 1)) << 11);
                }
            }
#pragma unroll 1
            for (int c0 = 0; c0 < 256 && (!is_half || other != nullptr); c0 += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tbase + c0, r);
                tmem_ld_wait();
                if (other != nullptr) {
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        const float4 o = __ldcg(other + g2_part_idx(c0 >> 5, g, lane));
                        r[4 * g + 0] = __float_as_uint(__uint_as_float(r[4 * g + 0]) + o.x);
                        r[4 * g + 1] = __float_as_uint(__uint_as_float(r[4 * g + 1]) + o.y);
                        r[4 * g + 2] = __float_as_uint(__uint_as_float(r[4 * g + 2]) + o.z);
                        r[4 * g + 3] = __float_as_uint(__uint_as_float(r[4 * g + 3]) + o.w);
                    }
                }
                if (grow < args.M) {
                    const int gc = gc0 + c0;
                    __nv_bfloat16* o = args.out + grow * args.ld_out + gc;
                    const bool vec_rows = (args.ld_out & 7) == 0;      // every row 16-byte aligned
                    if constexpr (FP8) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * out_scale);
                    }
                    if (args.col_scale != nullptr) {
                        // per-output-column factor (DoRA's m / ||W + sBA|| row norms)
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (gc + e < args.N)
                                r[e] = __float_as_uint(__uint_as_float(r[e]) * __ldg(args.col_scale + gc + e));
                    }
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        if (gc + 8 * g + 8 <= args.N && vec_rows) {
                            uint4 v;
                            v.x = pack_bf16x2(__uint_as_float(r[8 * g + 0]), __uint_as_float(r[8 * g + 1]));
                            v.y = pack_bf16x2(__uint_as_float(r[8 * g + 2]), __uint_as_float(r[8 * g + 3]));
                            v.z = pack_bf16x2(__uint_as_float(r[8 * g + 4]), __uint_as_float(r[8 * g + 5]));
                            v.w = pack_bf16x2(__uint_as_float(r[8 * g + 6]), __uint_as_float(r[8 * g + 7]));
                            *reinterpret_cast<uint4*>(o + 8 * g) = v;
                        } else {
                            // a ragged last column block, or rows that are not whole 16-byte units
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                if (gc + 8 * g + e < args.N) o[8 * g + e] = __float2bfloat16_rn(__uint_as_float(r[8 * g + e]));
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote_async_payload(acc_empty_leader + static_cast<uint32_t>(buf * 8));
        }
    } else if constexpr (FP8) {
        // -------------------------------------------------------------- NF4 -> E4M3 decoders
        // Forward: thread j owns weight row j of this CTA's 128 and, per K step, that row's two
        // consecutive 64-blocks: 128 E4M3 bytes, one whole 128-byte row of the swizzled tile.
        // dX: thread j owns weight row j of the K step and this CTA's 128 columns of it (two
        // 64-blocks): again one whole 128-byte row, now of the MN-major tile.
        const int grp = (warp - 6) >> 2;
        const int j = ((warp - 6) & 3) * 32 + lane;
        const float wsc = __ldg(args.w_scale);
        struct Pre {
            int nv;              // valid blocks of the step (0, 1 or 2)
            uint32_t q8[2];
            float c2[2];
        };
        int row_tile = -1;
        int64_t col0 = 0;                     // first of this CTA's 128 columns of the tile
        Cur fc = cur_at(grp);                 // the next step to fetch scales for
        auto fetch = [&](Pre& pr) {
            pr.nv = 0;
            const Cur c = fc;
            cur_next(fc);
            if (c.git >= total_iters || c.it >= args.k_steps) return;
            if (c.tile != row_tile) {
                row_tile = c.tile;
                col0 = static_cast<int64_t>(c.tile / args.m_tiles) * 256 + rank * 128;
            }
            const int64_t wrow = B_MN ? static_cast<int64_t>(c.it) * 128 + j : col0 + j;
            const int64_t wblk = B_MN ? col0 / 64 : 2 * static_cast<int64_t>(c.it);
            if (wrow >= args.nf4_rows || wblk >= args.nf4_bpr) return;
            pr.nv = wblk + 1 < args.nf4_bpr ? 2 : 1;
            const int64_t b0 = wrow * args.nf4_bpr + wblk;
            if (!dcheck(b0 + pr.nv <= static_cast<int64_t>(args.nf4_rows) * args.nf4_bpr, args.err)) {
                pr.nv = 0;
                return;
            }
            for (int h = 0; h < pr.nv; ++h) {
                pr.q8[h] = __ldg(args.absmax_q + b0 + h);
                pr.c2[h] = __ldg(args.c2 + ((b0 + h) >> 8));
            }
        };
        uint4 dec[8];
        auto decode_into_regs = [&](int git, const Pre& pr) {
            const uint8_t* src = sC + (git % SA) * L::kC + j * 64;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (h < pr.nv) {
                    const Nf4Fp8Planes p = nf4_make_planes_e4m3(__fmul_rn(nf4_block_scale(pr.q8[h], pr.c2[h]), wsc));
                    const uint4 qa = *reinterpret_cast<const uint4*>(src + 32 * h);
                    const uint4 qb = *reinterpret_cast<const uint4*>(src + 32 * h + 16);
                    const uint2 e0 = nf4_decode8_e4m3(qa.x, p), e1 = nf4_decode8_e4m3(qa.y, p);
                    const uint2 e2 = nf4_decode8_e4m3(qa.z, p), e3 = nf4_decode8_e4m3(qa.w, p);
                    const uint2 e4 = nf4_decode8_e4m3(qb.x, p), e5 = nf4_decode8_e4m3(qb.y, p);
                    const uint2 e6 = nf4_decode8_e4m3(qb.z, p), e7 = nf4_decode8_e4m3(qb.w, p);
                    dec[4 * h + 0] = make_uint4(e0.x, e0.y, e1.x, e1.y);
                    dec[4 * h + 1] = make_uint4(e2.x, e2.y, e3.x, e3.y);
                    dec[4 * h + 2] = make_uint4(e4.x, e4.y, e5.x, e5.y);
                    dec[4 * h + 3] = make_uint4(e6.x, e6.y, e7.x, e7.y);
                } else {
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) dec[4 * h + ch] = make_uint4(0, 0, 0, 0);
                }
            }
        };
        uint64_t* arrive_bar = rank == 0 ? ready : dec_done;
        Pre nxt;
        fetch(nxt);
        bool have = false;          // dec[] holds step `git` (decoded ahead)
        Cur mc = cur_at(grp);
        for (int git = grp; git < total_iters; git += NG) {
            const int s = git % SA;
            const bool main_step = mc.it < args.k_steps;
            Cur nc = mc;
            cur_next(nc);
            if (!have) {
                const Pre cur = nxt;
                fetch(nxt);
                if (!mbar_wait_warp(&full[s], (git / SA) & 1, abort, args.wait_ns)) {
                    fail();
                    break;
                }
                if (main_step) decode_into_regs(git, cur);
            }
            if (main_step) {
                if (!wait_slot_free_warp(git)) {
                    fail();
                    break;
                }
                uint8_t* dst_row = sB + (git % SB) * L::kB + j * 128;
                const uint32_t sw = j & 7;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4*>(dst_row + ((ch ^ sw) << 4)) = dec[ch];
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&arrive_bar[s]);
            have = false;
            const int gn = git + NG;
            if (gn < total_iters && nc.it < args.k_steps) {
                const Pre cur = nxt;
                fetch(nxt);
                if (!mbar_wait_warp(&full[gn % SA], (gn / SA) & 1, abort, args.wait_ns)) {
                    fail();
                    break;
                }
                decode_into_regs(gn, cur);
                have = true;
            }
            mc = nc;
        }
    } else {
        // -------------------------------------------------------------- NF4 decoders
        const int grp = (warp - 6) >> 2;
        const int j = ((warp - 6) & 3) * 32 + lane;      // 0..127: block of this thread
        int row_in_tile, blk_col_off;
        if (B_MN) {
            row_in_tile = j >> 1;           // weight row (K) within the step
            blk_col_off = j & 1;            // which 64-wide chunk of this CTA's 128 columns
        } else {
            row_in_tile = j;                // weight row within this CTA's 128
            blk_col_off = 0;
        }
        // block of the step at the fetch cursor (then advanced); -1 outside the weight
        Cur fc = cur_at(grp);
        int row_tile = -1, n0 = 0;
        auto next_block = [&]() -> int64_t {
            const Cur c = fc;
            cur_next(fc);
            if (c.git >= total_iters || c.it >= args.k_steps) return -1;
            if (c.tile != row_tile) {
                row_tile = c.tile;
                n0 = (c.tile / args.m_tiles) * 256 + static_cast<int>(rank) * 128;
            }
            const int it = c.it;
            int64_t wrow, wblk;
            if (B_MN) {
                wrow = static_cast<int64_t>(it) * 64 + row_in_tile;
                wblk = n0 / 64 + blk_col_off;
            } else {
                wrow = n0 + row_in_tile;
                wblk = it;
            }
            if (wrow >= args.nf4_rows || wblk >= args.nf4_bpr) return -1;
            const int64_t blk = wrow * args.nf4_bpr + wblk;
            return dcheck(blk < static_cast<int64_t>(args.nf4_rows) * args.nf4_bpr, args.err) ? blk : -1;
        };
        uint64_t* arrive_bar = rank == 0 ? ready : dec_done;   // local arrive either way
        // Software pipeline per handled step: the step's 64 weights are decoded into registers
        // as soon as its code tile has landed -- before its decoded-B slot is free -- so the
        // slot is held only for the stores; the next block's tables are built after that.
        uint4 dec[8];
        auto decode_into_regs = [&](int git, int64_t blk, const Nf4Planes& p) {
            const int s = git % SA;
            const uint8_t* c = sC + s * L::kC;
            const uint8_t* src = B_MN ? c + row_in_tile * 64 + blk_col_off * 32 : c + row_in_tile * 32;
            if (blk >= 0) {
                const uint4 q0 = *reinterpret_cast<const uint4*>(src);
                const uint4 q1 = *reinterpret_cast<const uint4*>(src + 16);
                dec[0] = nf4_decode8(q0.x, p);
                dec[1] = nf4_decode8(q0.y, p);
                dec[2] = nf4_decode8(q0.z, p);
                dec[3] = nf4_decode8(q0.w, p);
                dec[4] = nf4_decode8(q1.x, p);
                dec[5] = nf4_decode8(q1.y, p);
                dec[6] = nf4_decode8(q1.z, p);
                dec[7] = nf4_decode8(q1.w, p);
            } else {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) dec[ch] = make_uint4(0, 0, 0, 0);
            }
        };
        int64_t blk_nxt = next_block();
        uint32_t q8_nxt = 0;
        float c2_nxt = 0.f;
        if (blk_nxt >= 0) {
            q8_nxt = __ldg(args.absmax_q + blk_nxt);
            c2_nxt = __ldg(args.c2 + (blk_nxt >> 8));
        }
        bool have = false;          // dec[] holds step `git` (decoded ahead)
        Cur mc = cur_at(grp);
        for (int git = grp; git < total_iters; git += NG) {
            const int s = git % SA;
            const bool main_step = mc.it < args.k_steps;
            Cur nc = mc;
            cur_next(nc);
            if (!have) {
                // (first step, or after an adapter step) decode now
                const int64_t blk = blk_nxt;
                Nf4Planes p{};
                if (blk >= 0) p = nf4_make_planes(nf4_block_scale(q8_nxt, c2_nxt));
                blk_nxt = next_block();
                if (blk_nxt >= 0) {
                    q8_nxt = __ldg(args.absmax_q + blk_nxt);
                    c2_nxt = __ldg(args.c2 + (blk_nxt >> 8));
                }
                if (!mbar_wait_warp(&full[s], (git / SA) & 1, abort, args.wait_ns)) {
                    fail();
                    break;
                }
                if (main_step) decode_into_regs(git, blk, p);
            }
            if (main_step) {
                if (!wait_slot_free_warp(git)) {
                    fail();
                    break;
                }
                uint8_t* dst_row = sB + (git % SB) * L::kB +
                                   (B_MN ? blk_col_off * 8192 + row_in_tile * 128 : row_in_tile * 128);
                const uint32_t sw = row_in_tile & 7;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4*>(dst_row + ((ch ^ sw) << 4)) = dec[ch];
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&arrive_bar[s]);
            // decode the next handled step ahead, as soon as its codes have landed
            have = false;
            const int gn = git + NG;
            if (gn < total_iters && nc.it < args.k_steps) {
                const int64_t blk = blk_nxt;
                Nf4Planes p{};
                if (blk >= 0) p = nf4_make_planes(nf4_block_scale(q8_nxt, c2_nxt));
                blk_nxt = next_block();
                if (blk_nxt >= 0) {
                    q8_nxt = __ldg(args.absmax_q + blk_nxt);
                    c2_nxt = __ldg(args.c2 + (blk_nxt >> 8));
                }
                if (!mbar_wait_warp(&full[gn % SA], (gn / SA) & 1, abort, args.wait_ns)) {
                    fail();
                    break;
                }
                decode_into_regs(gn, blk, p);
                have = true;
            }
            mc = nc;
        }
    }

    // ---------------------------------------------------------------- teardown
    if (*abort) {
        // give in-flight copies of the pair time to land before shared memory is released
        __nanosleep(100000);
    }
    tc_fence_before();
    cluster_barrier();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_2sm(tmem_base, 512);
    }
}

}  // namespace qlora

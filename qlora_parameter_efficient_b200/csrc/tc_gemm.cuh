// tc_gemm.cuh -- the tcgen05/TMEM/TMA GEMM engine of libqlora (sm_100a).
//
//   D[M, N] = sum_K A[M, K] * B[N, K]        (fp32 accumulator in tensor memory)
//
// One CTA computes a 128 x BN tile.  Warp roles (320 threads):
//   warp 0      TMA producer: A tiles, and either B tiles or the packed NF4 code tiles.
//   warp 1      allocates TMEM and issues tcgen05.mma from one thread, 4 x (K = 16) per stage.
//   warps 2..9  NF4 decoders during the main loop (one thread per 64-weight block per stage:
//               the block's 64 bf16 weights become one 128-byte row of the swizzled operand
//               tile), then the epilogue (TMEM -> registers -> global).
// The weight operand is therefore dequantized on the fly into shared memory and consumed by
// the tensor cores without ever existing as a bf16 matrix in HBM ("Low-Rank Adaptation (LoRA)
// and QLoRA: Mathematical Foundations...", section "1. 4-bit NormalFloat (NF4) Quantization":
// dequantized on the fly into BF16 before the matrix multiplication; "LoRA and QLoRA
// Fine-Tuning Under the Hood", section "3.4 CUDA Block Dequantization and SRAM Paging
// Mechanics").
//
// The LoRA branch enters as extra K steps ("K-extension") after the main loop:
//   forward:  H  = [X  | sU] [W^ | B ]^T       (sU = s X A^T, zero-padded to 64 columns)
//   dX:       dX = [dH | sG] [W^ ; A ]         (sG = s dH B)
// so h is accumulated in one TMEM tile and written once.
//
// Operand layouts in shared memory are the UMMA canonical 128-byte-swizzle layouts:
//   K-major  (rows of 64 K elements = 128 B, 8-row atoms of 1024 B)
//   MN-major (64 M/N elements = 128 B per K row, 8-K-row atoms of 1024 B, 64-element chunks
//             8 KB apart).
// Every mbarrier wait is bounded; on a timeout the CTA records QLORA_ERR_TIMEOUT, drains its
// in-flight copies and MMAs, frees TMEM and returns.
#pragma once

#include "common.cuh"
#include "nf4.cuh"

namespace qlora {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kGemmThreads = 320;

enum : int { kBTma = 0, kBNf4 = 1 };

struct GemmArgs {
    int M, N;                 // valid rows / columns of the whole output
    int k_steps;              // main-loop K steps of 64
    int ext_steps;            // K-extension steps of 64 (0: none)
    int ext_k16_last;         // K=16 MMAs issued in the last extension step (1..4)
    int split;                // split-K over the main steps (grid.z); the extension steps are
                              // taken by the last split only
    const uint8_t* absmax_q;  // NF4 operand
    const float* c2;
    int nf4_rows;             // d_out of the stored weight
    int nf4_bpr;              // 64-blocks per stored row (d_in / 64)
    void* out;                // bf16 [M, ld_out] or fp32 partials [split][M][ld_out]
    int64_t ld_out;
    int64_t split_stride;     // elements between fp32 partials
    // 1: the kernel reads nothing the previous kernel on the stream writes, so it lets the next
    // kernel launch, starts at once, and waits for the previous one only before it exits (so a
    // kernel after it still sees both finished).  0: it waits before its first global access.
    int late_wait;
    int* err;
    uint64_t wait_ns;
};

template <int BN, int BMODE, int STAGES>
struct GemmSmem {
    static constexpr int kABytes = kBM * kBK * 2;
    static constexpr int kBBytes = BN * kBK * 2;
    static constexpr int kCBytes = (BMODE == kBNf4) ? BN * kBK / 2 : 0;
    static constexpr int kStage = kABytes + kBBytes + kCBytes;
    static constexpr int kBar = 256;
    static constexpr int kTotal = 1024 + STAGES * kStage + kBar;
    static_assert(kTotal <= 232448, "shared memory budget");
};

template <int BN>
struct TmemCols {
    static constexpr uint32_t value = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
};

// A_MN / B_MN: operand majorness.  BMODE kBNf4 decodes B from NF4 codes (B_MN = false: the
// forward orientation, B rows = weight rows; B_MN = true: the dX orientation, B = W^T).
// OUT_F32: fp32 split-K partials instead of bf16 output.
template <bool A_MN, bool B_MN, int BMODE, int BN, int STAGES, bool OUT_F32>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_tc_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmAx, const __grid_constant__ CUtensorMap tmBx,
              const GemmArgs args) {
    using L = GemmSmem<BN, BMODE, STAGES>;
    constexpr uint32_t kTmemCols = TmemCols<BN>::value;
    static_assert(BMODE == kBTma || BN == 256, "NF4 operand tiles are 256 wide");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * L::kABytes;
    uint8_t* sC = sB + STAGES * L::kBBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * L::kStage);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* decoded = bars + 2 * STAGES;
    uint64_t* accf = bars + 3 * STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * STAGES + 1);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BN;
    const int m0 = blockIdx.y * kBM;
    const int z = blockIdx.z;
    // main K steps owned by this CTA
    const int per = (args.k_steps + args.split - 1) / args.split;
    const int k_begin = z * per;
    const int k_end = min(args.k_steps, k_begin + per);
    const int n_main = max(0, k_end - k_begin);
    const int n_iters = n_main + (z == args.split - 1 ? args.ext_steps : 0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&decoded[s], 8);
        }
        mbar_init(accf, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (args.ext_steps > 0) {
            tma_prefetch_desc(&tmAx);
            tma_prefetch_desc(&tmBx);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_acc = *tmem_slot;
    if (args.late_wait) griddep_launch_dependents();
    else griddep_enter();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int it = 0; it < n_iters; ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, abort, args.wait_ns)) {
                    set_error(args.err, kErrTimeout);
                    *abort = 1;
                    break;
                }
                uint8_t* a = sA + s * L::kABytes;
                uint8_t* b = sB + s * L::kBBytes;
                const bool main_step = it < n_main;
                // late-wait launches: the extension operands come from the previous kernel
                if (args.late_wait && it == n_main) griddep_wait();
                const CUtensorMap* ma = main_step ? &tmA : &tmAx;
                const int kx = main_step ? (k_begin + it) * kBK : (it - n_main) * kBK;
                uint32_t bytes = L::kABytes;
                if (main_step && BMODE == kBNf4) bytes += L::kCBytes;
                else bytes += L::kBBytes;
                mbar_arrive_expect_tx(&full[s], bytes);
                if (A_MN) {
                    tma_load_2d(a, ma, &full[s], m0, kx);
                    tma_load_2d(a + 8192, ma, &full[s], m0 + 64, kx);
                } else {
                    tma_load_2d(a, ma, &full[s], kx, m0);
                }
                if (main_step && BMODE == kBNf4) {
                    uint8_t* c = sC + s * L::kCBytes;
                    if (B_MN) tma_load_2d(c, &tmB, &full[s], n0 / 2, kx);
                    else tma_load_2d(c, &tmB, &full[s], kx / 2, n0);
                } else {
                    const CUtensorMap* mb = main_step ? &tmB : &tmBx;
                    if (B_MN) {
#pragma unroll
                        for (int cch = 0; cch < BN / 64; ++cch)
                            tma_load_2d(b + cch * 8192, mb, &full[s], n0 + cch * 64, kx);
                    } else {
                        tma_load_2d(b, mb, &full[s], kx, n0);
                    }
                }
                issued = it + 1;
            }
            if (*abort) {
                // drain copies still in flight before the CTA's shared memory goes away
                for (int it = max(0, issued - STAGES); it < issued; ++it) {
                    const int s = it % STAGES;
                    mbar_wait(&full[s], (it / STAGES) & 1, nullptr, args.wait_ns);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = make_idesc_bf16(kBM, BN, A_MN, B_MN);
            for (int it = 0; it < n_iters; ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                bool ok = mbar_wait(&full[s], ph, abort, args.wait_ns);
                if (ok && BMODE == kBNf4 && it < n_main)
                    ok = mbar_wait(&decoded[s], ph, abort, args.wait_ns);
                if (!ok) {
                    set_error(args.err, kErrTimeout);
                    *abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t a = smem_u32(sA + s * L::kABytes);
                const uint32_t b = smem_u32(sB + s * L::kBBytes);
                const int nk = (it == n_iters - 1 && it >= n_main) ? args.ext_k16_last : 4;
                for (int k = 0; k < nk; ++k) {
                    const uint64_t ad = A_MN ? make_sw128_desc(a + k * 2048, 8192, 1024)
                                             : make_sw128_desc(a + k * 32, 16, 1024);
                    const uint64_t bd = B_MN ? make_sw128_desc(b + k * 2048, 8192, 1024)
                                             : make_sw128_desc(b + k * 32, 16, 1024);
                    umma_bf16_ss(tmem_acc, ad, bd, idesc, (it > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit(&empty[s]);
            }
            umma_commit(accf);
        }
    } else {
        const int td = threadIdx.x - 64;   // 0..255
        if (BMODE == kBNf4) {
            // -------------------------------------------------------- NF4 decoders
            // Each thread owns one 64-weight block per stage.
            int row_in_tile, blk_col_off;
            if (B_MN) {
                row_in_tile = td >> 2;      // K row (weight row) within the stage
                blk_col_off = td & 3;       // 64-element chunk of the N range
            } else {
                row_in_tile = td;           // weight row within the N tile
                blk_col_off = 0;
            }
            auto block_of = [&](int kt) -> int64_t {
                int64_t wrow, wblk;
                if (B_MN) {
                    wrow = static_cast<int64_t>(kt) * kBK + row_in_tile;
                    wblk = n0 / 64 + blk_col_off;
                } else {
                    wrow = n0 + row_in_tile;
                    wblk = kt;
                }
                if (wrow >= args.nf4_rows || wblk >= args.nf4_bpr) return -1;
                return wrow * args.nf4_bpr + wblk;
            };
            int64_t blk = n_main > 0 ? block_of(k_begin) : -1;
            uint32_t q8 = 0;
            float c2v = 0.0f;
            if (blk >= 0) {
                q8 = __ldg(args.absmax_q + blk);
                c2v = __ldg(args.c2 + (blk >> 8));
            }
            for (int it = 0; it < n_main; ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                const int64_t cur = blk;
                const uint32_t cq8 = q8;
                const float cc2 = c2v;
                if (it + 1 < n_main) {   // prefetch the next stage's scale inputs
                    blk = block_of(k_begin + it + 1);
                    if (blk >= 0) {
                        q8 = __ldg(args.absmax_q + blk);
                        c2v = __ldg(args.c2 + (blk >> 8));
                    }
                }
                if (!mbar_wait(&full[s], ph, abort, args.wait_ns)) {
                    set_error(args.err, kErrTimeout);
                    *abort = 1;
                    break;
                }
                uint8_t* b = sB + s * L::kBBytes;
                const uint8_t* c = sC + s * L::kCBytes;
                uint8_t* dst_row;
                const uint8_t* src;
                if (B_MN) {
                    dst_row = b + blk_col_off * 8192 + row_in_tile * 128;
                    src = c + row_in_tile * 128 + blk_col_off * 32;
                } else {
                    dst_row = b + row_in_tile * 128;
                    src = c + row_in_tile * 32;
                }
                const uint32_t sw = row_in_tile & 7;
                if (cur >= 0) {
                    const Nf4Planes p = nf4_make_planes(nf4_block_scale(cq8, cc2));
                    const uint4 q0 = *reinterpret_cast<const uint4*>(src);
                    const uint4 q1 = *reinterpret_cast<const uint4*>(src + 16);
                    const uint32_t qs[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        *reinterpret_cast<uint4*>(dst_row + ((ch ^ sw) << 4)) =
                            nf4_decode8(qs[ch], p);
                } else {
                    const uint4 zero = make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        *reinterpret_cast<uint4*>(dst_row + ((ch ^ sw) << 4)) = zero;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&decoded[s]);
            }
        }
        // ------------------------------------------------------------ epilogue
        if (!mbar_wait(accf, 0, nullptr, args.wait_ns)) {
            set_error(args.err, kErrTimeout);
            *abort = 1;
        }
        tc_fence_after();
        if (!*abort) {
            const int q = warp & 3;                 // TMEM lane quarter of this warp
            const int half = (warp - 2) >> 2;       // which half of the columns
            const int row = q * 32 + lane;
            const int64_t grow = m0 + row;
            constexpr int kHalf = BN / 2;
#pragma unroll 1
            for (int c0 = half * kHalf; c0 < (half + 1) * kHalf; c0 += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_acc + (static_cast<uint32_t>(q * 32) << 16) + c0, r);
                tmem_ld_wait();
                if (grow < args.M) {
                    const int gc = n0 + c0;
                    if (OUT_F32) {
                        float* o = reinterpret_cast<float*>(args.out) + z * args.split_stride +
                                   grow * args.ld_out + gc;
                        // 16-byte stores where the row and the block are whole, else one by one
                        const bool vec = (args.ld_out & 3) == 0 && (args.split_stride & 3) == 0;
#pragma unroll
                        for (int g = 0; g < 8; ++g) {
                            if (vec && gc + 4 * g + 4 <= args.N) {
                                *reinterpret_cast<uint4*>(o + 4 * g) =
                                    make_uint4(r[4 * g], r[4 * g + 1], r[4 * g + 2], r[4 * g + 3]);
                            } else {
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    if (gc + 4 * g + e < args.N) o[4 * g + e] = __uint_as_float(r[4 * g + e]);
                            }
                        }
                    } else {
                        __nv_bfloat16* o =
                            reinterpret_cast<__nv_bfloat16*>(args.out) + grow * args.ld_out + gc;
                        const bool vec = (args.ld_out & 7) == 0;
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            if (vec && gc + 8 * g + 8 <= args.N) {
                                uint4 v;
                                v.x = pack_bf16x2(__uint_as_float(r[8 * g + 0]), __uint_as_float(r[8 * g + 1]));
                                v.y = pack_bf16x2(__uint_as_float(r[8 * g + 2]), __uint_as_float(r[8 * g + 3]));
                                v.z = pack_bf16x2(__uint_as_float(r[8 * g + 4]), __uint_as_float(r[8 * g + 5]));
                                v.w = pack_bf16x2(__uint_as_float(r[8 * g + 6]), __uint_as_float(r[8 * g + 7]));
                                *reinterpret_cast<uint4*>(o + 8 * g) = v;
                            } else {
#pragma unroll
                                for (int e = 0; e < 8; ++e)
                                    if (gc + 8 * g + e < args.N) o[8 * g + e] = __float2bfloat16_rn(__uint_as_float(r[8 * g + e]));
                            }
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_acc, kTmemCols);
    }
    if (args.late_wait) griddep_wait();
}

// Bounded-wait self-test: waits on a barrier that nothing arrives on.
__global__ void k_wait_timeout_selftest(int* err, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (!mbar_wait(&bar, 0, nullptr, limit_ns)) set_error(err, kErrTimeout);
    }
}

}  // namespace qlora

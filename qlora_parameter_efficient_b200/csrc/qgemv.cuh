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
// Decode by table look-up.  A code byte holds two consecutive weights, and with the scale
// factored out the pair's two bf16 levels depend on the byte alone: a 256-entry table of bf16x2
// words turns a byte into an mma A register with one shared-memory load.  The table is
// replicated per lane (entry e, lane l at byte e * 256 + 4 l), so the 32 loads of a warp hit 32
// different banks whatever the bytes are, and the table starts on a 64 KB boundary of the
// shared window: the load address of byte i of a code word is then a single byte permute of the
// word and a per-lane constant (table address | 4 lane).  Two instructions per two weights, one of them on
// the memory pipe, against ~4.5 integer instructions per two weights for arithmetic decoding.
//
// Work split.  Rows come in tiles of 16; a cluster of C CTAs (C = 1, 2, 4 or 8) owns a
// contiguous range of tiles and its 16 warps x C ranks split K: warp w of rank p owns the KB
// consecutive 64-blocks starting at (16 p + w) KB (KB = 4 for up to 8 tokens, 2 for up to 16).
// The warp's X fragments stay in registers for the whole kernel; the codes of its 16 rows x KB
// blocks of a tile (a "slice") come through its own ring of S slices in shared memory, filled by
// 16-byte cp.async S - 1 tiles ahead of use (XOR-swizzled 16-byte chunks, so that the fragment
// reads of 8 rows fall in different banks).  A thread reads 8 bytes of a row per block, the k
// order inside a block permuted consistently in the codes and X so that those 8 bytes are the
// thread's A registers of the block's four k16 steps.  Up to 8 tokens the slice's block scales
// (16 absmax words and 16 c2 values) ride in the same copy group, one 4-byte cp.async per lane,
// and are read from shared memory; for 9..16 tokens (half the weights per warp and tile, more
// registers in use) each warp loads them into registers a tile ahead, which measured faster
// there (21.9 against 20.9 us at 16 tokens; 12.4 against 13.3 us at 1 token the other way).  Each warp writes its tile partial to one
// of NBUF shared buffers; a dedicated finaliser warp per buffer sums the 16 partials in warp
// order, the ranks' sums meet in rank 0 over DSMEM (rank order), and rank 0 applies 1/127, adds
// the adapter term with a few mma steps over bf16 s U (from the pre-pass) and the tile's B rows,
// and writes H, while the compute warps run on into the next tiles.  No global partials,
// atomics or semaphores: the sums are deterministic and the tail is on-chip.
//
// Why warp-level mma.sync and not tcgen05 here: one tcgen05.mma of M = 128, K = 16 occupies the
// SM's tensor core for ~130-190 cycles whatever N is (measured on B200 with N = 16..256), i.e. at
// most ~16 weights per cycle when the weights are the M x K operand, well below the stream rate;
// mma.sync takes its A operand from registers, where the table look-up leaves it.
#pragma once

#include "common.cuh"
#include "nf4.cuh"

namespace qlora {

constexpr int kLvWarps = 16;                 // compute warps
constexpr int kLvTableBytes = 0x10000;       // 256 entries x 256 bytes (lanes' words in the low half)
constexpr int kLvMaxRanks = 8;
constexpr int kLvRpMax = 128;                // adapter rank padded to 16
constexpr int kLvSuLd = kLvRpMax + 8;        // row stride (bf16) of s U and of staged B rows

template <int NT8>
struct LvCfg {
    static constexpr int KB = NT8 == 1 ? 4 : 2;                      // 64-blocks per warp
    static constexpr int NBUF = 3;                                   // tile partial buffers
    static constexpr int S = 3;                                      // code slices in flight per warp
    static constexpr int kThreads = 32 * (kLvWarps + NBUF);          // + one finaliser per buffer
    static constexpr int kMaxRanks = NT8 == 1 ? 8 : 4;
    static constexpr int kRowBytes = KB * 32;                         // a warp's bytes of a row
    static constexpr int kSlice = 16 * kRowBytes;                     // a warp's bytes of a tile
    static constexpr int kCodes = kLvWarps * S * kSlice;              // [warp][stage] slices
    static constexpr int kPart = NBUF * kLvWarps * NT8 * 512;         // [buf][warp][n][lane] float4
    static constexpr int kRing = NBUF * kMaxRanks * NT8 * 512;        // [buf][rank][n][lane] float4
    static constexpr int kSu = 16 * kLvSuLd * 2;                      // bf16 s U [16][kLvSuLd]
    static constexpr int kSb = NBUF * 16 * kLvSuLd * 2;               // bf16 B rows [NBUF][16][kLvSuLd]
    static constexpr bool kSmemScales = NT8 == 1;                    // scales through the copy ring
    static constexpr int kScl = kSmemScales ? kLvWarps * S * 32 * 4 : 0;   // [warp][stage] absmax words, c2
    // The table sits on the first 64 KB boundary of the shared window above the buffers placed
    // below it (at most 62 KB of them: the window starts within the first KB); the others follow
    // it.  Up to 8 tokens the tile partials live in the unused upper halves of the table entries
    // (128-byte pieces, a quarter warp's float4 each) and the code slices follow the table; for
    // 9..16 tokens the code slices go below the table and the partials after it.
    static constexpr bool kPartInTable = NT8 == 1;
    static_assert(!kPartInTable || NBUF * kLvWarps * NT8 * 4 <= 256, "partials must fit in the table");
    static constexpr int kBelow = kPartInTable ? kRing + kSu + kSb + kScl + 256 : kCodes + kSu + kScl + 256;
    static constexpr int kAbove = kPartInTable ? kCodes : kPart + kRing + kSb;
    static_assert(kBelow <= 62 * 1024, "buffers below the table");
    static constexpr int kSmem = 64 * 1024 + kLvTableBytes + kAbove;    // window start .. end
    static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

struct LvArgs {
    int T;                   // tokens (1..8 NT8)
    int d_out, d_in, kt;     // kt = d_in / 64 (a multiple of 4)
    int tiles;               // ceil(d_out / 16)
    int C;                   // CTAs per cluster (K ranks)
    int clusters;            // grid / C
    int r, rp;               // adapter rank and its padding to 16
    const uint8_t* codes;
    const uint8_t* absmax_q;
    const float* c2;
    const __nv_bfloat16* X;       // [T][d_in]
    const __nv_bfloat16* us_pad;  // [16][kLvSuLd] bf16(s U), zero beyond T and r (pre-pass)
    const __nv_bfloat16* B;       // [d_out][r]
    __nv_bfloat16* H;             // [T][d_out]
    int* err;
    uint64_t wait_ns;
    uint32_t lv16[8];        // the 16 levels rounded to bf16, two per word (level 2i low)
};

// A load from the byte table or from a warp's own code slice: both are read-only while read (the
// table after a barrier, a slice between its cp.async wait and the warp's next refill), so the
// load is a pure function of its address and the compiler may batch and hoist it.
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint2 lds_v2(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(src_bytes)
                 : "memory");
}
// 4-byte copy (src_bytes 0: zero fill), through L1
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x),
                 "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

// Bounded wait for a finaliser: polls the barrier with a short sleep between tries, so that a
// finaliser waiting for its next tile takes few issue slots from the compute warps of its
// scheduler.  Gives up (false) on *abort or after limit_ns, like mbar_wait_warp.
__device__ __forceinline__ bool mbar_wait_idle(uint64_t* bar, uint32_t parity, volatile int* abort,
                                               uint64_t limit_ns) {
    const uint32_t addr = smem_u32(bar);
    uint32_t ok = mbar_test_wait(addr, parity) ? 1u : 0u;
    if (!__shfl_sync(0xffffffffu, ok, 0)) {
        const uint64_t t0 = globaltimer_ns();
        while (true) {
            __nanosleep(128);
            if (mbar_test_wait(addr, parity)) {
                ok = 1u;
                break;
            }
            if (*abort || globaltimer_ns() - t0 > limit_ns) break;
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    return ok != 0u;
}

template <int NT8>
__global__ void __maxnreg__(96) k_qgemv_lut(const __grid_constant__ LvArgs a) {
    using Cf = LvCfg<NT8>;
    constexpr int KB = Cf::KB, NBUF = Cf::NBUF, MR = Cf::kMaxRanks, S = Cf::S;
    extern __shared__ __align__(1024) uint8_t smem[];
    // the table on the first 64 KB boundary above the buffers placed below it: the table address
    // of a code byte is then a single byte permute (table address bits 16+, byte, 4 lane)
    const uint32_t sbase = smem_u32(smem);
    const uint32_t tab_addr = (sbase + Cf::kBelow + 0xFFFFu) & ~0xFFFFu;
    if (tab_addr + kLvTableBytes + Cf::kAbove > sbase + Cf::kSmem) {
        if (threadIdx.x == 0) set_error(a.err, kErrDevice);
        // still meet the other ranks at both cluster barriers (theirs time out on the missing
        // partials and reach the last one)
        if (a.C > 1) {
            cluster_barrier();
            cluster_barrier();
        }
        return;
    }
    uint8_t* const below = smem;
    uint8_t* const above = smem + (tab_addr - sbase) + kLvTableBytes;
    uint32_t* table = reinterpret_cast<uint32_t*>(smem + (tab_addr - sbase));
    uint8_t* const codes_sm = Cf::kPartInTable ? above : below;
    float4* const part_lin = reinterpret_cast<float4*>(above);             // (9..16 tokens)
    float4* const ring = reinterpret_cast<float4*>(Cf::kPartInTable ? below : above + Cf::kPart);
    __nv_bfloat16* s_us = reinterpret_cast<__nv_bfloat16*>(Cf::kPartInTable ? below + Cf::kRing : below + Cf::kCodes);
    __nv_bfloat16* s_b = reinterpret_cast<__nv_bfloat16*>(Cf::kPartInTable ? below + Cf::kRing + Cf::kSu
                                                                            : above + Cf::kPart + Cf::kRing);
    uint32_t* scl = reinterpret_cast<uint32_t*>(Cf::kPartInTable ? below + Cf::kRing + Cf::kSu + Cf::kSb
                                                                  : below + Cf::kCodes + Cf::kSu);
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(scl) + Cf::kScl);
    // the float4 of lane ln for (buffer, warp, n) of the tile partials
    auto part_at = [&](int buf, int w, int n, int ln) -> float4* {
        const int idx = (buf * kLvWarps + w) * NT8 + n;
        if constexpr (Cf::kPartInTable)
            return reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(table) + (idx * 4 + (ln >> 3)) * 256 + 128) + (ln & 7);
        else
            return part_lin + idx * 32 + ln;
    };
    uint64_t* full = bars;                  // [NBUF] the 16 warps' partials of a tile are in
    uint64_t* freeb = bars + NBUF;          // [NBUF] the finaliser has read them
    uint64_t* ring_full = bars + 2 * NBUF;  // [NBUF] rank 0: the other ranks' sums are in
    uint64_t* ring_free = bars + 3 * NBUF;  // [NBUF] rank p: rank 0 has read this rank's sum
    uint64_t* us_bar = bars + 4 * NBUF;     // rank 0: s U is staged
    volatile int* abort = reinterpret_cast<volatile int*>(bars + 4 * NBUF + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int C = a.C;
    const int rank = static_cast<int>(blockIdx.x) % C;
    const int cl = static_cast<int>(blockIdx.x) / C;
    const int t_lo = static_cast<int>((static_cast<int64_t>(cl) * a.tiles) / a.clusters);
    const int t_hi = static_cast<int>((static_cast<int64_t>(cl + 1) * a.tiles) / a.clusters);
    const int ntl = t_hi - t_lo;
    const int64_t row_bytes = a.d_in / 2;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NBUF; ++i) {
            mbar_init(&full[i], kLvWarps);
            mbar_init(&freeb[i], 1);
            mbar_init(&ring_full[i], C > 1 ? C - 1 : 1);
            mbar_init(&ring_free[i], 1);
        }
        mbar_init(us_bar, 1);
        *abort = 0;
        if (C > 1) fence_mbar_init();       // other CTAs of the cluster arrive on these
    }

    const bool compute = warp < kLvWarps;
    const int kb0 = (rank * kLvWarps + warp) * KB;          // this warp's first 64-block
    const bool k_ok = compute && kb0 < a.kt;                // kt % 4 == 0: all KB blocks or none
    // ---- compute warps: the warp's slice of tile li (16 rows x KB blocks) into its ring stage
    // li % S, a row's 16-byte chunk c at chunk c ^ swz(row) (so that the fragment reads of 8 rows
    // fall in different banks); rows past d_out are zero-filled
    const uint32_t slices = smem_u32(codes_sm) + warp * S * Cf::kSlice;
    auto swz = [](int row) { return KB == 4 ? (row & 7) : ((row >> 1) & 3); };
    const uint8_t* const w0 = a.codes + static_cast<int64_t>(t_lo) * 16 * row_bytes + kb0 * 32;
    // the slice's block scales: lane l < 16 copies the absmax word of row l (the aligned 4 bytes
    // holding its KB bytes), lane 16 + l the second-level constant of row l (KB blocks never
    // straddle a group of 256 blocks: kt and kb0 are multiples of KB)
    const uint32_t scl_w = smem_u32(scl) + warp * S * 128;
    const int rr = lane & 15;
    const int64_t i_row = static_cast<int64_t>(t_lo * 16 + rr) * a.kt + kb0;   // absmax index, tile 0
    const uint8_t* const q_src0 = a.absmax_q + (i_row & ~static_cast<int64_t>(3));
    const int64_t tile_q = 16 * static_cast<int64_t>(a.kt);                 // absmax bytes per tile
    auto issue_slice = [&](int li) {
        if (k_ok && li < ntl) {
            if constexpr (Cf::kSmemScales) {
                const bool ok = (t_lo + li) * 16 + rr < a.d_out;
                const int64_t iq = static_cast<int64_t>(li) * tile_q;
                const void* src = lane < 16 ? static_cast<const void*>(q_src0 + iq)
                                            : static_cast<const void*>(a.c2 + ((i_row + iq) >> 8));
                cp_async4(scl_w + ((li % S) * 32 + lane) * 4, ok ? src : static_cast<const void*>(a.c2),
                          ok ? 4u : 0u);
            }
            const uint32_t dst = slices + (li % S) * Cf::kSlice;
            constexpr int kChunks = 16 * 2 * KB;            // 16-byte chunks of a slice
#pragma unroll
            for (int i = 0; i < kChunks / 32; ++i) {
                const int idx = lane + 32 * i, row = idx / (2 * KB), c = idx % (2 * KB);
                const bool ok = (t_lo + li) * 16 + row < a.d_out && dcheck(kb0 + KB <= a.kt, a.err);
                cp_async16(dst + row * Cf::kRowBytes + ((c ^ swz(row)) << 4),
                           ok ? static_cast<const void*>(w0 + (static_cast<int64_t>(li) * 16 + row) * row_bytes + 16 * c)
                              : static_cast<const void*>(a.codes),
                           ok ? 16u : 0u);
            }
        }
        cp_async_commit();
    };
    // the absmax word of a row holds its KB bytes at this shift (KB = 2: kb0 may be 2 mod 4)
    const int q_shift = (kb0 & 3) * 8;
    // (9..16 tokens) the tile's absmax bytes of rows g, g + 8 and each row's second-level constant (a warp's
    // KB blocks never straddle a group of 256 blocks: kt and kb0 are multiples of KB)
    struct Scales {
        uint32_t qa, qb;
        float c2a, c2b;
    };
    const int64_t ia0 = static_cast<int64_t>(t_lo * 16 + g) * a.kt + kb0;
    auto load_scales = [&](int li, Scales& R) {
        const int ra = (t_lo + li) * 16 + g, rb = ra + 8;
        const bool va = k_ok && li < ntl && ra < a.d_out, vb = k_ok && li < ntl && rb < a.d_out;
        const int64_t ia = ia0 + static_cast<int64_t>(li) * 16 * a.kt, ib = ia + 8 * static_cast<int64_t>(a.kt);
        if constexpr (KB == 4) {
            R.qa = va ? __ldg(reinterpret_cast<const uint32_t*>(a.absmax_q + ia)) : 0u;
            R.qb = vb ? __ldg(reinterpret_cast<const uint32_t*>(a.absmax_q + ib)) : 0u;
        } else {
            R.qa = va ? static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short*>(a.absmax_q + ia))) : 0u;
            R.qb = vb ? static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short*>(a.absmax_q + ib))) : 0u;
        }
        R.c2a = va ? __ldg(a.c2 + (ia >> 8)) : 0.f;
        R.c2b = vb ? __ldg(a.c2 + (ib >> 8)) : 0.f;
    };


    Scales sc_cur;
    if constexpr (Cf::kSmemScales) sc_cur = Scales{};
    uint32_t xw[KB][NT8][8];
    if (compute) {
        for (int st = 0; st < S - 1; ++st) issue_slice(st);
        // the byte table: entry e = (high code << 4) | low code -> bf16x2 (L[low], L[high]), the
        // same word in every lane's slot; warp w writes the entries of low code w
        {
            const uint32_t lo = (a.lv16[warp >> 1] >> (16 * (warp & 1))) & 0xFFFFu;
#pragma unroll
            for (int j = 0; j < 16; ++j)
                table[(16 * j + warp) * 64 + lane] = lo | (a.lv16[j >> 1] >> (16 * (j & 1)) << 16);
        }
        if constexpr (!Cf::kSmemScales) load_scales(0, sc_cur);
        // X fragments of this warp's blocks, held for the whole kernel: token 8n + g, elements
        // 16q .. 16q + 15 of block kb0 + b
#pragma unroll
        for (int b = 0; b < KB; ++b) {
#pragma unroll
            for (int n = 0; n < NT8; ++n) {
                const int t = 8 * n + g;
                uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
                if (k_ok && t < a.T) {
                    const uint4* src = reinterpret_cast<const uint4*>(a.X + static_cast<int64_t>(t) * a.d_in + (kb0 + b) * 64 + 16 * q);
                    x0 = __ldg(src);
                    x1 = __ldg(src + 1);
                }
                xw[b][n][0] = x0.x; xw[b][n][1] = x0.y; xw[b][n][2] = x0.z; xw[b][n][3] = x0.w;
                xw[b][n][4] = x1.x; xw[b][n][5] = x1.y; xw[b][n][6] = x1.z; xw[b][n][7] = x1.w;
            }
        }
    }
    // barriers initialised (and visible cluster-wide) and the table written before use
    if (C > 1) cluster_barrier();
    else __syncthreads();

    if (compute) {
        // ================================================================ compute warps
        const uint32_t lb = tab_addr | (static_cast<uint32_t>(lane) << 2);
        // table address of byte i of a code word: bits 16+ and the lane's word from lb, the byte as
        // bits 8..15 (entry stride 256 bytes)
        auto tab = [&](uint32_t w, uint32_t i) -> uint32_t { return prmt(w, lb, 0x7604u | (i << 4)); };
        // the warp's part of tile li (its slice in stage li % S; its scales there too, or in R);
        // false on a failed wait
        auto process = [&](int li, const Scales& R) -> bool {
            const int buf = li % NBUF;
            const int st = li % S;
            const uint32_t slc = slices + st * Cf::kSlice;
            uint32_t qa_w = R.qa, qb_w = R.qb;
            float c2a = R.c2a, c2b = R.c2b;
            if constexpr (Cf::kSmemScales) {
                // (a warp past its rank's K range copies no scales: it contributes zeros)
                qa_w = k_ok ? lds_u32(scl_w + (st * 32 + g) * 4) >> q_shift : 0u;
                qb_w = k_ok ? lds_u32(scl_w + (st * 32 + g + 8) * 4) >> q_shift : 0u;
                c2a = k_ok ? __uint_as_float(lds_u32(scl_w + (st * 32 + 16 + g) * 4)) : 0.f;
                c2b = k_ok ? __uint_as_float(lds_u32(scl_w + (st * 32 + 24 + g) * 4)) : 0.f;
            }
            float acc[NT8][4];
#pragma unroll
            for (int n = 0; n < NT8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
            // the thread's 8 code bytes of each block in rows g and g + 8 (logical chunk 2b + q / 2,
            // half q % 2), all loaded before the look-ups
            uint2 ca[KB], cb[KB];
#pragma unroll
            for (int b = 0; b < KB; ++b) {
                const int c = 2 * b + (q >> 1);
                ca[b] = lds_v2(slc + g * Cf::kRowBytes + ((c ^ swz(g)) << 4) + ((q & 1) << 3));
                cb[b] = lds_v2(slc + (g + 8) * Cf::kRowBytes + ((c ^ swz(g + 8)) << 4) + ((q & 1) << 3));
            }
#pragma unroll
            for (int b = 0; b < KB; ++b) {
                float tmp[NT8][4];
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    // A registers of k16 step s: bytes 2s (slots 2q, 2q+1) and 2s + 1 (slots
                    // 2q+8, 2q+9) of the thread's 8 code bytes, rows g and g + 8
                    const uint32_t wa = (s < 2) ? ca[b].x : ca[b].y;
                    const uint32_t wb = (s < 2) ? cb[b].x : cb[b].y;
                    const uint32_t i0 = 2 * (s & 1), i1 = i0 + 1;
                    const uint32_t A[4] = {lds_u32(tab(wa, i0)), lds_u32(tab(wb, i0)), lds_u32(tab(wa, i1)),
                                           lds_u32(tab(wb, i1))};
#pragma unroll
                    for (int n = 0; n < NT8; ++n)
                        mma_bf16_16816(tmp[n], A, xw[b][n][2 * s], xw[b][n][2 * s + 1], s > 0);
                }
                // the unscaled block partial times the block's absmax byte; c2 multiplies the sum
                const float qa = static_cast<float>((qa_w >> (8 * b)) & 0xFFu);
                const float qb = static_cast<float>((qb_w >> (8 * b)) & 0xFFu);
#pragma unroll
                for (int n = 0; n < NT8; ++n) {
                    acc[n][0] = fmaf(qa, tmp[n][0], acc[n][0]);
                    acc[n][1] = fmaf(qa, tmp[n][1], acc[n][1]);
                    acc[n][2] = fmaf(qb, tmp[n][2], acc[n][2]);
                    acc[n][3] = fmaf(qb, tmp[n][3], acc[n][3]);
                }
            }
            // the warp's partial into this tile's buffer, free once the finaliser has read the
            // tile NBUF back (1/127 is applied to the output)
            if (li >= NBUF && !mbar_wait_warp(&freeb[buf], ((li / NBUF) - 1) & 1, abort, a.wait_ns)) {
                set_error(a.err, kErrTimeout);
                *abort = 1;
                return false;
            }
#pragma unroll
            for (int n = 0; n < NT8; ++n)
                *part_at(buf, warp, n, lane) =
                    make_float4(c2a * acc[n][0], c2a * acc[n][1], c2b * acc[n][2], c2b * acc[n][3]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[buf]);
            return !*abort;
        };
        // per tile: refill the stage of the previous tile with the slice S - 1 ahead, wait for this
        // tile's slice (and scales: the warp's own copies), then compute
        if constexpr (Cf::kSmemScales) {
            for (int li = 0; li < ntl; ++li) {
                __syncwarp();
                issue_slice(li + S - 1);
                cp_async_wait<S - 1>();
                __syncwarp();
                if (!process(li, sc_cur)) break;
            }
        } else {
            // scales ping-pong one tile ahead in registers
            Scales sc_nxt;
            for (int li = 0; li < ntl; li += 2) {
                __syncwarp();
                issue_slice(li + S - 1);
                load_scales(li + 1, sc_nxt);
                cp_async_wait<S - 1>();
                __syncwarp();
                if (!process(li, sc_cur) || li + 1 >= ntl) break;
                __syncwarp();
                issue_slice(li + S);
                load_scales(li + 2, sc_cur);
                cp_async_wait<S - 1>();
                __syncwarp();
                if (!process(li + 1, sc_nxt)) break;
            }
        }
        cp_async_wait<0>();     // no copy in flight into the shared memory of an exiting CTA
    } else {
        // ================================================================ finaliser warps
        // Finaliser f takes the tiles of buffer f (tile li -> warp 16 + li % NBUF): it sums the 16
        // partials in warp order, sends the sum to rank 0 or (rank 0) adds the other ranks' sums in
        // rank order, applies 1/127, adds the adapter term and writes H.  Each keeps the adapter
        // rows of its next tile in flight (cp.async into its own s_b buffer).
        const int f = warp - kLvWarps;
        // the adapter rows of tile li into this finaliser's s_b buffer (one cp.async group; rows
        // whose r bf16 are not whole 16-byte units are read at use instead)
        const bool b_vec = (a.r % 8) == 0;
        const int cpr = a.r / 8;                            // 16-byte pieces of a B row
        __nv_bfloat16* const sbf = s_b + f * 16 * kLvSuLd;
        auto stage_b = [&](int li) {
            if (rank == 0 && b_vec && li < ntl) {
                const int row0 = (t_lo + li) * 16;
                for (int rr = 0; rr < 16; ++rr) {
                    if (lane < cpr && row0 + rr < a.d_out)
                        cp_async16(smem_u32(sbf + rr * kLvSuLd + 8 * lane),
                                   a.B + static_cast<int64_t>(row0 + rr) * a.r + 8 * lane, 16u);
                }
            }
            cp_async_commit();
        };
        // B fragment e of k16 step kk for tile li: rows g (+8 for odd e), columns 16 kk + 2q (+8)
        auto b_frag = [&](int li, int kk, int e) -> uint32_t {
            const int rr = g + 8 * (e & 1), col = 16 * kk + 2 * q + 8 * (e >> 1);
            const int row = (t_lo + li) * 16 + rr;
            if (row >= a.d_out || col >= a.r) return 0u;
            if (b_vec) return *reinterpret_cast<const uint32_t*>(sbf + rr * kLvSuLd + col);
            const __nv_bfloat16* p = a.B + static_cast<int64_t>(row) * a.r + col;
            const uint32_t lo = __ldg(reinterpret_cast<const unsigned short*>(p));
            const uint32_t hi = col + 1 < a.r ? __ldg(reinterpret_cast<const unsigned short*>(p + 1)) : 0u;
            return lo | (hi << 16);
        };
        stage_b(f);
        bool us_ready = false;
        for (int li = f; li < ntl; li += NBUF) {
            const int buf = f;                              // li % NBUF
            // ---- the 16 partials of the tile in warp order
            if (!mbar_wait_idle(&full[buf], (li / NBUF) & 1, abort, a.wait_ns)) {
                set_error(a.err, kErrTimeout);
                *abort = 1;
                break;
            }
            float4 tot[NT8];
#pragma unroll
            for (int n = 0; n < NT8; ++n) {
                tot[n] = *part_at(buf, 0, n, lane);
#pragma unroll
                for (int w = 1; w < kLvWarps; ++w) {
                    const float4 v = *part_at(buf, w, n, lane);
                    tot[n].x += v.x;
                    tot[n].y += v.y;
                    tot[n].z += v.z;
                    tot[n].w += v.w;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&freeb[buf]);
            if (C > 1) {
                if (rank != 0) {
                    // this rank's sum to rank 0 (its ring slot is free once rank 0 has read the
                    // sum of the tile NBUF back)
                    if (li >= NBUF && !mbar_wait_warp(&ring_free[buf], ((li / NBUF) - 1) & 1, abort, a.wait_ns)) {
                        set_error(a.err, kErrTimeout);
                        *abort = 1;
                        break;
                    }
                    if (!dcheck(rank < MR, a.err)) break;
#pragma unroll
                    for (int n = 0; n < NT8; ++n)
                        st_cluster_v4(mapa_shared(smem_u32(ring + ((buf * MR + rank) * NT8 + n) * 32 + lane), 0), tot[n]);
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&ring_full[buf]), 0));
                    continue;
                }
                bool got = mbar_try_wait_acq_cluster(smem_u32(&ring_full[buf]), (li / NBUF) & 1);
                if (!got) got = mbar_wait_cluster(&ring_full[buf], (li / NBUF) & 1, abort, a.wait_ns);
                if (__shfl_sync(0xffffffffu, got ? 1u : 0u, 0) == 0u) {
                    set_error(a.err, kErrTimeout);
                    *abort = 1;
                    break;
                }
                for (int p = 1; p < C; ++p) {
#pragma unroll
                    for (int n = 0; n < NT8; ++n) {
                        const float4 v = ring[((buf * MR + p) * NT8 + n) * 32 + lane];
                        tot[n].x += v.x;
                        tot[n].y += v.y;
                        tot[n].z += v.z;
                        tot[n].w += v.w;
                    }
                }
                __syncwarp();
                // every rank's slot of this buffer is free again (its last use needs none)
                if (lane >= 1 && lane < C && li + NBUF < ntl)
                    mbar_arrive_remote(mapa_shared(smem_u32(&ring_free[buf]), static_cast<uint32_t>(lane)));
            }
            // ---- rank 0: 1/127, the adapter term (B rows times bf16 s U on the tensor cores,
            // fp32 accumulation), H
            // s U from the pre-pass, staged by finaliser 0 once its first tile is summed (the
            // sums never wait for the pre-pass)
            if (!us_ready) {
                if (f == 0) {
                    griddep_wait();
                    cp_async_wait<0>();                     // this tile's B rows (group order)
                    const uint32_t dst = smem_u32(s_us);
                    for (int i = lane; i < 16 * kLvSuLd / 8; i += 32) cp_async16(dst + 16 * i, a.us_pad + 8 * i, 16u);
                    cp_async_commit();
                    cp_async_wait<0>();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(us_bar);
                } else if (!mbar_wait_warp(us_bar, 0, abort, a.wait_ns)) {
                    set_error(a.err, kErrTimeout);
                    *abort = 1;
                    break;
                }
                us_ready = true;
            }
            float out[2][NT8][2];
#pragma unroll
            for (int n = 0; n < NT8; ++n) {
                out[0][n][0] = __fdiv_rn(tot[n].x, 127.0f);
                out[0][n][1] = __fdiv_rn(tot[n].y, 127.0f);
                out[1][n][0] = __fdiv_rn(tot[n].z, 127.0f);
                out[1][n][1] = __fdiv_rn(tot[n].w, 127.0f);
            }
            float adp[NT8][4];
#pragma unroll
            for (int n = 0; n < NT8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) adp[n][e] = 0.f;
            cp_async_wait<0>();                             // this tile's B rows
            __syncwarp();
#pragma unroll
            for (int kk = 0; kk < kLvRpMax / 16; ++kk) {
                if (16 * kk >= a.rp) break;
                const uint32_t af[4] = {b_frag(li, kk, 0), b_frag(li, kk, 1), b_frag(li, kk, 2), b_frag(li, kk, 3)};
#pragma unroll
                for (int n = 0; n < NT8; ++n) {
                    const __nv_bfloat16* ub = s_us + (8 * n + g) * kLvSuLd + 16 * kk + 2 * q;
                    mma_bf16_16816(adp[n], af, *reinterpret_cast<const uint32_t*>(ub),
                                   *reinterpret_cast<const uint32_t*>(ub + 8), true);
                }
            }
            __syncwarp();
            stage_b(li + NBUF);                             // this finaliser's next tile
            const int ra = (t_lo + li) * 16 + g, rb = ra + 8;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = h ? rb : ra;
                if (row >= a.d_out) continue;
#pragma unroll
                for (int n = 0; n < NT8; ++n)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int t = 8 * n + 2 * q + e;
                        if (t < a.T)
                            a.H[static_cast<int64_t>(t) * a.d_out + row] =
                                __float2bfloat16_rn(out[h][n][e] + adp[n][2 * h + e]);
                    }
            }
        }
        cp_async_wait<0>();
    }
    // a rank's shared memory is the target of the others' remote stores and arrives: no CTA of a
    // cluster leaves before all are done (every wait above is bounded, so all arrive here)
    if (C > 1) cluster_barrier();
}

// Pre-pass of the decode-size forward: U = X A^T on the tensor cores.  A cluster of KS CTAs owns
// 16 adapter rows and splits K; warp w of rank p takes every 8th 64-block of the rank's share (the
// same in-block k order as the stream kernel, at most 4 blocks per warp so that its loads are in
// flight together); the warps' and then the ranks' partials are summed in order in rank 0, which
// writes bf16(s U) into the padded [16][kLvSuLd] layout the stream kernel stages (zero beyond T
// and r) and U (the call dtype, unscaled) for the backward.  It takes a few SMs of its own (the
// stream kernel's grid leaves them free) and is launched with programmatic dependent launch: it
// waits for the previous kernel, then lets the stream kernel start, whose finaliser reads its
// output once it has finished.
constexpr int kLuWarps = 8;
struct LuArgs {
    const __nv_bfloat16* X;
    int T, d_in, kt;
    const __nv_bfloat16* A;
    int r;
    float s;
    int KS;                         // CTAs per cluster
    __nv_bfloat16* us_pad;          // [16][kLvSuLd]
    __nv_bfloat16* u_save;          // nullable [T][r]
};

__global__ void __launch_bounds__(32 * kLuWarps) k_lora_u_tc(const LuArgs a) {
    griddep_wait();
    griddep_launch_dependents();
    __shared__ float4 red[kLuWarps][2][32];       // the warps' partials
    __shared__ float4 rsum[kLvMaxRanks][2][32];   // rank 0: the ranks' sums
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int KS = a.KS;
    const int rank = static_cast<int>(blockIdx.x) % KS;
    const int j0 = (static_cast<int>(blockIdx.x) / KS) * 16;
    const int lo = (rank * a.kt) / KS, hi = ((rank + 1) * a.kt) / KS;
    const int ja = j0 + g, jb = ja + 8;
    float acc[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
    const int nt8 = a.T > 8 ? 2 : 1;
    // at most 4 blocks per warp (the launch sizes KS for it): all of their loads in flight at once
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int blk = lo + warp + i * kLuWarps;
        if (blk >= hi) break;
        uint32_t ra[8], rb[8], xf[2][8];
        auto ld8 = [&](uint32_t (&dst)[8], const __nv_bfloat16* src, bool ok) {
            uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
            if (ok) {
                v0 = __ldg(reinterpret_cast<const uint4*>(src));
                v1 = __ldg(reinterpret_cast<const uint4*>(src) + 1);
            }
            dst[0] = v0.x; dst[1] = v0.y; dst[2] = v0.z; dst[3] = v0.w;
            dst[4] = v1.x; dst[5] = v1.y; dst[6] = v1.z; dst[7] = v1.w;
        };
        const int64_t col = static_cast<int64_t>(blk) * 64 + 16 * q;
        ld8(ra, a.A + static_cast<int64_t>(ja) * a.d_in + col, ja < a.r);
        ld8(rb, a.A + static_cast<int64_t>(jb) * a.d_in + col, jb < a.r);
        ld8(xf[0], a.X + static_cast<int64_t>(g) * a.d_in + col, g < a.T);
        ld8(xf[1], a.X + static_cast<int64_t>(8 + g) * a.d_in + col, nt8 > 1 && 8 + g < a.T);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const uint32_t af[4] = {ra[2 * s], rb[2 * s], ra[2 * s + 1], rb[2 * s + 1]};
            mma_bf16_16816(acc[0], af, xf[0][2 * s], xf[0][2 * s + 1], true);
            if (nt8 > 1) mma_bf16_16816(acc[1], af, xf[1][2 * s], xf[1][2 * s + 1], true);
        }
    }
#pragma unroll
    for (int n = 0; n < 2; ++n) red[warp][n][lane] = make_float4(acc[n][0], acc[n][1], acc[n][2], acc[n][3]);
    __syncthreads();
    if (warp == 0) {
        float4 tot[2];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            tot[n] = red[0][n][lane];
            for (int w = 1; w < kLuWarps; ++w) {
                tot[n].x += red[w][n][lane].x;
                tot[n].y += red[w][n][lane].y;
                tot[n].z += red[w][n][lane].z;
                tot[n].w += red[w][n][lane].w;
            }
        }
        if (KS > 1) {
            const uint32_t dst = mapa_shared(smem_u32(&rsum[rank][0][lane]), 0);
#pragma unroll
            for (int n = 0; n < 2; ++n) st_cluster_v4(dst + n * 32 * 16, tot[n]);
        } else {
#pragma unroll
            for (int n = 0; n < 2; ++n) rsum[0][n][lane] = tot[n];
        }
    }
    if (KS > 1) cluster_barrier();
    else __syncthreads();
    if (rank != 0 || warp != 0) return;
    float4 tot[2];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
        tot[n] = rsum[0][n][lane];
        for (int p = 1; p < KS; ++p) {
            tot[n].x += rsum[p][n][lane].x;
            tot[n].y += rsum[p][n][lane].y;
            tot[n].z += rsum[p][n][lane].z;
            tot[n].w += rsum[p][n][lane].w;
        }
    }
    // thread (g, q) holds U[t][j] for j = ja, jb and t = 8n + 2q + e
#pragma unroll
    for (int n = 0; n < 2; ++n) {
        const float v[2][2] = {{tot[n].x, tot[n].y}, {tot[n].z, tot[n].w}};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int j = h ? jb : ja;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int t = 8 * n + 2 * q + e;
                const bool valid = t < a.T && j < a.r;
                a.us_pad[t * kLvSuLd + j] = __float2bfloat16_rn(valid ? a.s * v[h][e] : 0.f);
                if (valid && a.u_save) a.u_save[static_cast<int64_t>(t) * a.r + j] = __float2bfloat16_rn(v[h][e]);
            }
        }
    }
    // the padding columns past the last group (one group writes them)
    if (j0 == 0) {
        const int rp = (a.r + 15) & ~15;
        for (int i = lane; i < 16 * (kLvSuLd - rp); i += 32) {
            const int t = i / (kLvSuLd - rp), j = rp + i % (kLvSuLd - rp);
            a.us_pad[t * kLvSuLd + j] = __float2bfloat16_rn(0.f);
        }
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

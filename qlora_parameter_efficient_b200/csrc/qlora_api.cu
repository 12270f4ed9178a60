// qlora_api.cu -- the C ABI of libqlora (see include/qlora.h): argument validation, workspace
// planning, TMA descriptor construction and the launch sequence of each entry point.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/qlora.h"
#include "common.cuh"
#include "nf4.cuh"
#include "simt.cuh"
#include "tc_gemm.cuh"
#include "nf4_gemm2.cuh"
#include "merge.cuh"
#include "segmented.cuh"
#include "optim.cuh"
#include "fp8.cuh"
#include "qgemv.cuh"
#include "dora.cuh"

using namespace qlora;

// ======================================================================= globals

__device__ int g_qlora_error;   // the device error word (one per device context)

namespace {

constexpr int kMaxDevices = 64;
constexpr int kSmsForSplit = 148;         // split-K is sized for a B200's 148 SMs
constexpr uint64_t kWaitNs = 4000000000ull;
constexpr int kTmaStages = 4;
constexpr int kNf4Stages = 4;          // the mid-size NF4 GEMM: 4 x 56 KB stages

std::atomic<uint64_t> g_launches{0};
int* g_err_ptr[kMaxDevices] = {};
std::mutex g_mu;
cudaEvent_t g_ev_start = nullptr, g_ev_stop = nullptr;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

inline void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }


#define QL_TRY(expr)                         \
    do {                                     \
        qlora_status _s = (expr);            \
        if (_s != QLORA_OK) return _s;       \
    } while (0)

#define QL_LAUNCH_CHECK()                                              \
    do {                                                               \
        count_launch();                                                \
        if (cudaPeekAtLastError() != cudaSuccess) return QLORA_ERR_CUDA; \
    } while (0)

// Launch a kernel that begins with griddep_enter() with programmatic stream serialization, so
// that its launch and prologue overlap the end of the previous kernel on the stream.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// The device address of a __device__ variable on the current device.  Looked up again on
// every call made outside stream capture (a context torn down by cudaDeviceReset and re-created
// may place the module's variables elsewhere), and taken from the per-device cache while the
// stream is being captured, where the lookup may not be allowed; the first call on a device must
// therefore come before any capture.
qlora_status symbol_address(const void* symbol, void** cache, cudaStream_t stream, void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ERR_CUDA;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    const bool capturing = cudaStreamIsCapturing(stream, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone;
    if (capturing) cudaGetLastError();   // a refused query leaves no sticky error behind
    std::lock_guard<std::mutex> lk(g_mu);
    if (!capturing || !cache[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess || !p) return QLORA_ERR_CUDA;
        cache[dev] = p;
    }
    *out = cache[dev];
    return QLORA_OK;
}

qlora_status err_word(int** out, cudaStream_t stream) {
    void* p = nullptr;
    QL_TRY(symbol_address(reinterpret_cast<const void*>(&g_qlora_error), reinterpret_cast<void**>(g_err_ptr),
                          stream, &p));
    *out = static_cast<int*>(p);
    return QLORA_OK;
}

qlora_status get_encoder() {
    if (g_encode) return QLORA_OK;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode) return QLORA_OK;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return QLORA_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return QLORA_OK;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned16_or_null(const void* p) { return !p || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// bf16 bits of a finite fp32 value, round to nearest even (the NF4 levels, on the host)
inline uint32_t bf16_bits(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    return (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
}
inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// ======================================================================= TMA descriptors

qlora_status tmap_bf16(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld,
                       uint32_t box_rows) {
    QL_TRY(get_encoder());
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                          strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? QLORA_OK : QLORA_ERR_CUDA;
}

// byte matrix [rows, cols_bytes], no swizzle, box = box_x bytes x box_y rows.
qlora_status tmap_u8(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld,
                     uint32_t box_x, uint32_t box_y) {
    QL_TRY(get_encoder());
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld)};
    cuuint32_t box[2] = {box_x, box_y};
    cuuint32_t es[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                          strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? QLORA_OK : QLORA_ERR_CUDA;
}

// byte matrix [rows, cols] (row stride ld bytes), 128-byte swizzle, box = 128 bytes x box_rows:
// an E4M3 operand tile in the UMMA K-major layout.
qlora_status tmap_u8_sw128(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld,
                           uint32_t box_rows) {
    QL_TRY(get_encoder());
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld)};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                          strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? QLORA_OK : QLORA_ERR_CUDA;
}

// ======================================================================= planning

int choose_split(int64_t tiles, int64_t k_steps) {
    // the skinny kernel fits two CTAs per SM: fill one wave of 2 x 148 slots, never more
    int64_t s = std::max<int64_t>(1, (2 * kSmsForSplit) / std::max<int64_t>(tiles, 1));
    s = std::min<int64_t>(s, std::max<int64_t>(1, k_steps / 4));
    s = std::max<int64_t>(1, std::min<int64_t>(s, 32));
    const int64_t per = cdiv(k_steps, s);
    return static_cast<int>(cdiv(k_steps, per));   // no empty splits
}

int pad_rank(int r) { return r <= 64 ? 64 : 128; }

// Decode-size forward (bf16, T <= 16, d_in a multiple of 256): clusters of C CTAs own tiles of
// M rows, the C ranks split K.  (C, M) is picked at launch by balanced cost.
constexpr int kSmallT = 16;   // above this the large-T path is faster (measured)
// Mid-size forward (bf16, 8 < T <= kMidT, or T <= 8 when the decode-size kernel does not
// apply): split-K NF4 GEMM over all SMs with fp32 partials, then one finalize with the adapter.
constexpr int64_t kMidT = 64;
struct MidPlan {
    bool ok = false;
    int split = 1, n_tiles = 1;
};
MidPlan make_mid_plan(int64_t T, int64_t d_out, int64_t d_in) {
    MidPlan mp;
    if (T < 1 || T > kMidT) return mp;
    mp.n_tiles = static_cast<int>(cdiv(d_out, 256));
    const int64_t k_steps = d_in / 64;
    int64_t s = std::max<int64_t>(1, kSmsForSplit / mp.n_tiles);   // one CTA per SM, one wave
    s = std::min<int64_t>(s, std::max<int64_t>(1, k_steps / 2));
    const int64_t per = cdiv(k_steps, s);
    mp.split = static_cast<int>(cdiv(k_steps, per));                // no empty splits
    mp.ok = true;
    return mp;
}

struct SmallPlan {
    bool ok = false;
    int nt8 = 1, kt = 0, C = 1, ks = 1;
};
// Decode-size forward: 16 warps x C ranks split K in slices of KB 64-blocks (4 for up to 8
// tokens, 2 for up to 16); d_in a multiple of 256 and at most 8 ranks.
SmallPlan make_small_plan(int64_t T, int64_t d_out, int64_t d_in) {
    SmallPlan sp;
    (void)d_out;
    if (T < 1 || T > kSmallT) return sp;
    sp.nt8 = T <= 8 ? 1 : 2;
    sp.kt = static_cast<int>(d_in / 64);
    const int kb = sp.nt8 == 1 ? 4 : 2;
    sp.C = static_cast<int>(cdiv(sp.kt, kLvWarps * kb));
    // U pre-pass: K ranks per cluster, at most 4 blocks for each of a CTA's warps
    sp.ks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(kLvMaxRanks, cdiv(sp.kt, 4 * kLuWarps))));
    sp.ok = sp.kt % 4 == 0 && sp.C <= (sp.nt8 == 1 ? LvCfg<1>::kMaxRanks : LvCfg<2>::kMaxRanks);
    return sp;
}

// Persistent schedule of the fused NF4 GEMM: pairs of SMs, and how many trailing tiles are
// split in two along K (only when the last wave has at most half the pairs' worth of tiles).
struct G2Sched {
    int pairs = 1, split_tiles = 0;
    size_t part_bytes = 0, cnt_bytes = 0;
    size_t bytes() const { return part_bytes + cnt_bytes; }
};
G2Sched g2_schedule(int64_t T, int64_t N, int64_t K, int64_t k_step = 64) {
    G2Sched g;
    const int64_t tiles = cdiv(T, 256) * cdiv(N, 256);
    g.pairs = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(tiles, kSmsForSplit / 2)));
    const int64_t rem = tiles % g.pairs;
    if (tiles > g.pairs && rem > 0 && 2 * rem <= g.pairs && cdiv(K, k_step) >= 2) {
        g.split_tiles = static_cast<int>(rem);
        g.part_bytes = align256(static_cast<size_t>(rem) * 2 * 4 * 2 * 2048 * 16);
        g.cnt_bytes = align256(static_cast<size_t>(rem) * 2 * 4 * sizeof(int));
    }
    return g;
}

struct Plan {
    int RP = 0;
    bool small = false;
    size_t s_us = 0;
    bool mid = false;
    size_t mid_part = 0;
    int mid_split = 1;
    int split_u = 1, split_g = 1, split_da = 1, split_db = 1;
    size_t a_pad = 0, b_pad = 0, u_spad = 0, u_pad = 0, g_spad = 0, part = 0;
    size_t w32 = 0, uf = 0, gf = 0;
    size_t g2 = 0;         // fused-GEMM split-tail partials and tickets
    // segmented multi-adapter forward
    size_t seg_cnt = 0, seg_start = 0, seg_cursor = 0, seg_ntiles = 0, seg_tiles = 0, seg_perm = 0,
           seg_u = 0;
    int seg_ldu = 0, seg_max_tiles = 0;
    size_t dora_part = 0, dora_scale = 0;   // DoRA row-norm partials and column scale
    size_t f8_x = 0, f8_dh = 0, f8_g = 0;    // FP8 backward: bf16 X~, dH~ and sigma sigma_w s G
    size_t dh_pad = 0;     // bf16 backward, d_out not a multiple of 8: dH with 16-byte rows
    size_t total = 0;
};

Plan make_plan(int op, qlora_dtype dtype, int64_t T, int64_t d_out, int64_t d_in, int r) {
    // (QLORA_OP_DORA_FWD: the forward's workspace plus the DoRA row norms)
    Plan p;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    if (op == QLORA_OP_MERGE) return p;
    if (op == QLORA_OP_FP8_QUANT) {
        p.total = 256;      // the amax word
        return p;
    }
    if (op == QLORA_OP_BWD_FP8) {
        p = make_plan(QLORA_OP_BWD, QLORA_BF16, T, d_out, d_in, r);
        off = p.total;
        p.f8_x = take(static_cast<size_t>(T) * d_in * 2);
        p.f8_dh = take(static_cast<size_t>(T) * d_out * 2);
        p.f8_g = take(static_cast<size_t>(T) * p.RP * 2);
        p.total = off;
        return p;
    }
    if (op == QLORA_OP_FWD_FP8) {
        p.RP = pad_rank(r);
        if (r % 8 != 0) p.b_pad = take(static_cast<size_t>(d_out) * p.RP * 2);
        p.u_spad = take(static_cast<size_t>(T) * p.RP * 2);
        p.g2 = take(g2_schedule(T, d_out, d_in, 128).bytes());
        p.total = off;
        return p;
    }
    if (op == QLORA_OP_FWD_MULTI) {
        // base GEMM split tail, then the segmented adapter term (r = the largest rank)
        p.g2 = take(g2_schedule(T, d_out, d_in).bytes());
        p.seg_ldu = (r + 15) & ~15;
        p.seg_cnt = take(static_cast<size_t>(kSegMaxAdapters) * 4);
        p.seg_start = take(static_cast<size_t>(kSegMaxAdapters) * 4);
        p.seg_cursor = take(static_cast<size_t>(kSegMaxAdapters) * 4);
        p.seg_ntiles = take(4);
        p.seg_max_tiles = static_cast<int>(cdiv(T, kSegTile) + std::min<int64_t>(T, kSegMaxAdapters));
        p.seg_tiles = take(static_cast<size_t>(p.seg_max_tiles) * 16);
        p.seg_perm = take(static_cast<size_t>(T) * 4);
        p.seg_u = take(static_cast<size_t>(T) * p.seg_ldu * 2);
        p.total = off;
        return p;
    }
    const bool dora = op == QLORA_OP_DORA_FWD;
    if (dora) op = QLORA_OP_FWD;          // the forward's plan, never the decode-size path
    if (!dora && op == QLORA_OP_FWD && dtype == QLORA_BF16 && make_small_plan(T, d_out, d_in).ok) {
        p.small = true;
        p.s_us = take(static_cast<size_t>(16) * kLvSuLd * 2);   // bf16 s U, padded
        p.total = off;
        return p;
    }
    if (!dora && op == QLORA_OP_FWD && dtype == QLORA_BF16) {
        const MidPlan mp = make_mid_plan(T, d_out, d_in);
        if (mp.ok) {
            p.mid = true;
            p.mid_split = mp.split;
            p.RP = pad_rank(r);
            p.s_us = take(static_cast<size_t>(T) * r * 4);
            p.u_spad = take(static_cast<size_t>(T) * p.RP * 2);
            p.b_pad = take(static_cast<size_t>(d_out) * p.RP * 2);
            p.mid_part = take(static_cast<size_t>(mp.split) * T * d_out * 4);
            p.total = off;
            return p;
        }
    }
    if (dtype == QLORA_BF16) {
        p.RP = pad_rank(r);
        const int64_t RP = p.RP;
        const int64_t mt = cdiv(T, kBM);
        p.a_pad = take(RP * d_in * 2);
        p.b_pad = take(d_out * RP * 2);
        p.split_u = choose_split(mt, cdiv(d_in, kBK));
        size_t part = static_cast<size_t>(p.split_u) * T * RP * 4;
        if (op == QLORA_OP_FWD || op == QLORA_OP_FWD_BATCHED) {
            p.u_spad = take(T * RP * 2);
        } else {
            p.u_pad = take(T * RP * 2);
            p.g_spad = take(T * RP * 2);
            p.split_g = choose_split(mt, cdiv(d_out, kBK));
            p.split_da = choose_split(cdiv(d_in, kBM), cdiv(T, kBK));
            p.split_db = choose_split(cdiv(d_out, kBM), cdiv(T, kBK));
            if (d_out % 8 != 0) p.dh_pad = take(static_cast<size_t>(T) * (d_out + 7) / 8 * 8 * 2);
            part = std::max(part, static_cast<size_t>(p.split_g) * T * RP * 4);
            part = std::max(part, static_cast<size_t>(p.split_da) * d_in * RP * 4);
            part = std::max(part, static_cast<size_t>(p.split_db) * d_out * RP * 4);
        }
        p.part = take(part);
        const size_t g2 = op == QLORA_OP_BWD ? g2_schedule(T, d_in, d_out).bytes()
                                             : g2_schedule(T, d_out, d_in).bytes();
        p.g2 = take(g2);
    } else {
        p.w32 = take(static_cast<size_t>(d_out) * d_in * 4);
        if (op == QLORA_OP_FWD_BATCHED) {
            p.a_pad = take(static_cast<size_t>(r) * d_in * 4);
            p.b_pad = take(static_cast<size_t>(d_out) * r * 4);
            p.uf = take(static_cast<size_t>(T) * r * 4);
        } else {
            p.uf = take(static_cast<size_t>(T) * r * 4);
            if (op == QLORA_OP_BWD) p.gf = take(static_cast<size_t>(T) * r * 4);
        }
    }
    if (dora) {
        p.dora_part = take(static_cast<size_t>(d_out) * (d_in / 64) * 4);
        p.dora_scale = take(static_cast<size_t>(d_out) * 4);
    }
    p.total = off;
    return p;
}

// DoRA backward workspace: one region shared in turn by the large-T forward (the pre-scale
// output Z), the LoRA backward of dZ and the two weight passes with the adapter rows as tokens,
// then the DoRA buffers.
struct DoraBwdLayout {
    size_t shared = 0, merge_part = 0, norms = 0, e = 0, colpart = 0, z = 0, u = 0, dz = 0, ge = 0,
           pm = 0, qm = 0, aat = 0, beb = 0, total = 0;
};
DoraBwdLayout dora_bwd_layout(int64_t T, int64_t d, int64_t k, int r) {
    DoraBwdLayout L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    const size_t shared = std::max({make_plan(QLORA_OP_DORA_FWD, QLORA_BF16, T, d, k, r).total,
                                    make_plan(QLORA_OP_BWD, QLORA_BF16, T, d, k, r).total,
                                    g2_schedule(r, d, k).bytes(), g2_schedule(r, k, d).bytes()});
    L.shared = take(shared);
    L.merge_part = take(static_cast<size_t>(d) * (k / 64) * 4);
    L.norms = take(static_cast<size_t>(d) * 4);
    L.e = take(static_cast<size_t>(d) * 4);
    L.colpart = take(static_cast<size_t>(kDoraChunks) * d * 4);
    L.z = take(static_cast<size_t>(T) * d * 2);
    L.u = take(static_cast<size_t>(T) * r * 2);
    L.dz = take(static_cast<size_t>(T) * d * 2);
    L.ge = take(static_cast<size_t>(r) * ((d + 7) / 8 * 8) * 2);
    L.pm = take(static_cast<size_t>(r) * d * 2);
    L.qm = take(static_cast<size_t>(r) * k * 2);
    L.aat = take(static_cast<size_t>(r) * r * 4);
    L.beb = take(static_cast<size_t>(r) * r * 4);
    L.total = off;
    return L;
}

template <typename P>
P* at(void* ws, size_t off) {
    return reinterpret_cast<P*>(static_cast<uint8_t*>(ws) + off);
}

dim3 grid1d(int64_t n) {
    return dim3(static_cast<unsigned>(std::min<int64_t>(std::max<int64_t>(cdiv(n, 256), 1), 148 * 16)));
}

// ======================================================================= validation

qlora_status check_nf4(const qlora_nf4* w) {
    if (!w || !aligned16(w->codes) || !aligned16(w->absmax_q) || !aligned16(w->c2))
        return QLORA_ERR_INVALID_ARG;
    if (w->d_out < 1 || w->d_in < 64 || w->d_in % 64) return QLORA_ERR_UNSUPPORTED;
    if (w->d_out > (1 << 30) || w->d_in > (1 << 30)) return QLORA_ERR_UNSUPPORTED;
    return QLORA_OK;
}

qlora_status check_layer(const qlora_nf4* w, int64_t T, int r, qlora_dtype dtype) {
    QL_TRY(check_nf4(w));
    if (dtype != QLORA_BF16 && dtype != QLORA_F32) return QLORA_ERR_INVALID_ARG;
    if (T < 1 || T > (1LL << 30) || r < 1 || r > 128) return QLORA_ERR_UNSUPPORTED;
    return QLORA_OK;
}

qlora_status check_ws(const void* ws, size_t ws_bytes, size_t need) {
    if (need == 0) return QLORA_OK;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < need) return QLORA_ERR_INVALID_ARG;
    return QLORA_OK;
}

// ======================================================================= GEMM launchers

template <bool A_MN, bool B_MN, int BMODE, int BN, int STAGES, bool OUT_F32>
qlora_status launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& ax,
                         const CUtensorMap& bx, const GemmArgs& args, dim3 grid,
                         cudaStream_t st, bool timed) {
    auto kern = k_tc_gemm<A_MN, B_MN, BMODE, BN, STAGES, OUT_F32>;
    constexpr int smem = GemmSmem<BN, BMODE, STAGES>::kTotal;
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
            return QLORA_ERR_CUDA;
        configured.fetch_or(bit);
    }
    const bool ev = timed && g_ev_start && g_ev_stop;
    if (ev) cudaEventRecord(g_ev_start, st);
    if (launch_pdl(kern, grid, dim3(kGemmThreads), smem, st, a, b, ax, bx, args) != cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    if (ev) cudaEventRecord(g_ev_stop, st);
    return QLORA_OK;
}

GemmArgs base_args(int M, int N, int k_steps, int* err) {
    GemmArgs g{};
    g.M = M;
    g.N = N;
    g.k_steps = k_steps;
    g.ext_steps = 0;
    g.ext_k16_last = 4;
    g.split = 1;
    g.err = err;
    g.wait_ns = kWaitNs;
    return g;
}

// Skinny tensor-core contraction D[M, RP] = sum_K A[M,K] B[RP,K] written as fp32 split-K
// partials.  a_mn / b_mn give the operand majorness of the two TMA maps.
qlora_status skinny_gemm(bool a_mn, bool b_mn, int RP, int n_valid, const CUtensorMap& ta,
                         const CUtensorMap& tb, int64_t M, int64_t k_steps, int split,
                         float* part, int* err, cudaStream_t st) {
    // partial columns >= n_valid are never read: only the first n_valid are stored
    GemmArgs g = base_args(static_cast<int>(M), n_valid, static_cast<int>(k_steps), err);
    g.split = split;
    g.out = part;
    g.ld_out = RP;
    g.split_stride = M * RP;
    dim3 grid(1, static_cast<unsigned>(cdiv(M, kBM)), static_cast<unsigned>(split));
    if (RP == 64) {
        if (!a_mn && !b_mn) return launch_gemm<false, false, kBTma, 64, kTmaStages, true>(ta, tb, ta, tb, g, grid, st, false);
        if (!a_mn && b_mn) return launch_gemm<false, true, kBTma, 64, kTmaStages, true>(ta, tb, ta, tb, g, grid, st, false);
        if (a_mn && b_mn) return launch_gemm<true, true, kBTma, 64, kTmaStages, true>(ta, tb, ta, tb, g, grid, st, false);
    } else {
        if (!a_mn && !b_mn) return launch_gemm<false, false, kBTma, 128, kTmaStages, true>(ta, tb, ta, tb, g, grid, st, false);
        if (!a_mn && b_mn) return launch_gemm<false, true, kBTma, 128, kTmaStages, true>(ta, tb, ta, tb, g, grid, st, false);
        if (a_mn && b_mn) return launch_gemm<true, true, kBTma, 128, kTmaStages, true>(ta, tb, ta, tb, g, grid, st, false);
    }
    return QLORA_ERR_UNSUPPORTED;
}

// Fused NF4-decode GEMM with the adapter K-extension (persistent 2-SM kernel).
//   forward (dx = false): out[T, d_out]  = act[T, d_in]  W^T + ext_a[T, RP] ext_b[d_out, RP]^T
//   dX      (dx = true):  out[T, d_in]   = act[T, d_out] W   + ext_a[T, RP] ext_b[RP, d_in]
// ext_b_rank: the rank extent stored in ext_b (RP for a zero-padded copy, or the caller's r
// when the TMA zero-fills the rank padding out of bounds).
qlora_status nf4_gemm(bool dx, const qlora_nf4* w, const void* act, int64_t T, const void* ext_a,
                      const void* ext_b, int RP, int r_used, int ext_b_rank, void* out,
                      void* g2ws, int* err, cudaStream_t st, const float* col_scale = nullptr,
                      const float* x_scale = nullptr, const float* w_scale = nullptr,
                      int64_t act_ld = 0) {
    // x_scale != NULL: the FP8 variant (act is the E4M3 activation or, for dX, the E5M2
    // gradient; ext_a the adapter term in sigma sigma_w units; x_scale that tensor's sigma)
    const bool fp8 = x_scale != nullptr;
    const int64_t d_out = w->d_out, d_in = w->d_in;
    CUtensorMap ta, tc, tax, tbx;
    const int64_t K = dx ? d_out : d_in;
    const int64_t N = dx ? d_in : d_out;
    const int64_t k_step = fp8 ? 128 : 64;
    if (fp8) {
        QL_TRY(tmap_u8_sw128(&ta, act, T, K, K, 128));
        QL_TRY(tmap_u8(&tc, w->codes, d_out, d_in / 2, d_in / 2, 64, 128));
    } else {
        QL_TRY(tmap_bf16(&ta, act, T, K, act_ld > 0 ? act_ld : K, 128));
        if (dx) QL_TRY(tmap_u8(&tc, w->codes, d_out, d_in / 2, d_in / 2, 64, 64));
        else QL_TRY(tmap_u8(&tc, w->codes, d_out, d_in / 2, d_in / 2, 32, 128));
    }
    if (RP > 0) {
        QL_TRY(tmap_bf16(&tax, ext_a, T, RP, RP, 128));
        if (dx) QL_TRY(tmap_bf16(&tbx, ext_b, ext_b_rank, d_in, d_in, 64));
        else QL_TRY(tmap_bf16(&tbx, ext_b, d_out, ext_b_rank, ext_b_rank, 128));
    } else {                 // no adapter steps: the maps are never read
        tax = ta;
        tbx = ta;
    }
    Gemm2Args g{};
    g.col_scale = col_scale;
    g.x_scale = x_scale;
    g.w_scale = w_scale;
    g.M = static_cast<int>(T);
    g.N = static_cast<int>(N);
    g.k_steps = static_cast<int>(cdiv(K, k_step));
    g.ext_steps = RP / 64;
    g.ext_k16_last = RP > 0 ? static_cast<int>(std::min<int64_t>(4, cdiv(r_used - 64 * (g.ext_steps - 1), 16))) : 4;
    g.m_tiles = static_cast<int>(cdiv(T, 256));
    g.n_tiles = static_cast<int>(cdiv(N, 256));
    g.absmax_q = w->absmax_q;
    g.c2 = w->c2;
    g.nf4_rows = static_cast<int>(d_out);
    g.nf4_bpr = static_cast<int>(d_in / 64);
    g.out = static_cast<__nv_bfloat16*>(out);
    g.ld_out = N;
    g.err = err;
    g.wait_ns = kWaitNs;
    const G2Sched sch = g2_schedule(T, N, K, k_step);
    const int pairs = sch.pairs;
    g.split_tiles = sch.split_tiles;
    if (sch.split_tiles > 0) {
        if (!g2ws || (reinterpret_cast<uintptr_t>(g2ws) & 255u)) return QLORA_ERR_INVALID_ARG;
        g.part = static_cast<float*>(g2ws);
        g.cnt = reinterpret_cast<int*>(static_cast<uint8_t*>(g2ws) + sch.part_bytes);
    }
    auto kern = fp8 ? (dx ? k_nf4_gemm2<true, true> : k_nf4_gemm2<false, true>)
                    : (dx ? k_nf4_gemm2<true> : k_nf4_gemm2<false>);
    const int smem = fp8 ? G2Smem<true>::kTotal : G2Smem<false>::kTotal;
    const int variant = (fp8 ? 2 : 0) + (dx ? 1 : 0);
    static std::atomic<uint64_t> configured[4] = {0, 0, 0, 0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured[variant].load() & bit)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return QLORA_ERR_CUDA;
        configured[variant].fetch_or(bit);
    }
    if (sch.split_tiles > 0 && cudaMemsetAsync(g.cnt, 0, sch.cnt_bytes, st) != cudaSuccess)
        return QLORA_ERR_CUDA;
    const bool ev = g_ev_start && g_ev_stop;
    if (ev) cudaEventRecord(g_ev_start, st);
    const int threads = fp8 ? G2Smem<true>::kThreads : G2Smem<false>::kThreads;
    if (launch_pdl(kern, dim3(2 * pairs), dim3(threads), smem, st, ta, tc, tax, tbx, g) !=
        cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    if (ev) cudaEventRecord(g_ev_stop, st);
    return QLORA_OK;
}

// Decode-size forward: the tensor-core U pre-pass (a few clusters of 128-thread CTAs that fit
// beside the stream kernel's CTAs) and the stream kernel, both launched with programmatic
// dependent launch so that the stream starts while U is computed.
template <int NT8>
qlora_status launch_qgemv(LvArgs g, int ks, const LuArgs& u, cudaStream_t st) {
    int dev = 0;
    cudaGetDevice(&dev);
    static std::atomic<uint64_t> configured{0};
    static std::atomic<int> fit[64][kLvMaxRanks + 1];   // clusters of C CTAs that fit at once
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        if (cudaFuncSetAttribute(k_qgemv_lut<NT8>, cudaFuncAttributeMaxDynamicSharedMemorySize, LvCfg<NT8>::kSmem) !=
            cudaSuccess)
            return QLORA_ERR_CUDA;
        configured.fetch_or(bit);
    }
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.attrs = attr;
    cfg.stream = st;
    // the U pre-pass
    attr[1].val.clusterDim.x = static_cast<unsigned>(ks);
    const int pre_ctas = static_cast<int>(cdiv(u.r, 16) * ks);
    cfg.gridDim = dim3(static_cast<unsigned>(pre_ctas));
    cfg.blockDim = dim3(32 * kLuWarps);
    cfg.dynamicSmemBytes = 0;
    cfg.numAttrs = ks > 1 ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, k_lora_u_tc, u) != cudaSuccess) return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    // the stream kernel
    const int C = g.C;
    int n = fit[dev & 63][C].load();
    cfg.blockDim = dim3(LvCfg<NT8>::kThreads);
    cfg.dynamicSmemBytes = LvCfg<NT8>::kSmem;
    attr[1].val.clusterDim.x = static_cast<unsigned>(C);
    cfg.numAttrs = C > 1 ? 2 : 1;
    // the stream kernel's CTAs take the SMs the pre-pass leaves (so that none waits for it)
    const int sms = std::max(C, kSmsForSplit - pre_ctas);
    if (n == 0) {
        n = kSmsForSplit / C;
        if (C > 1) {
            cfg.gridDim = dim3(static_cast<unsigned>(C * (kSmsForSplit / C)));
            int m = 0;
            if (cudaOccupancyMaxActiveClusters(&m, k_qgemv_lut<NT8>, &cfg) != cudaSuccess) {
                cudaGetLastError();
                m = 0;
            }
            n = std::min(n, std::max(m, 1));
        }
        fit[dev & 63][C].store(n);
    }
    g.clusters = static_cast<int>(std::min<int64_t>(std::min(n, sms / C), g.tiles));
    cfg.gridDim = dim3(static_cast<unsigned>(C * g.clusters));
    const bool ev = g_ev_start && g_ev_stop;
    if (ev) cudaEventRecord(g_ev_start, st);
    if (cudaLaunchKernelEx(&cfg, k_qgemv_lut<NT8>, g) != cudaSuccess) return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    if (ev) cudaEventRecord(g_ev_stop, st);
    return QLORA_OK;
}

qlora_status small_fwd(const qlora_nf4* w, const void* X, int64_t T, const void* A, const void* B,
                       int r, float s, void* H, void* U_save, const Plan& p, void* ws, int* err,
                       cudaStream_t st) {
    const int64_t d_out = w->d_out, d_in = w->d_in;
    const SmallPlan sp = make_small_plan(T, d_out, d_in);
    if (!sp.ok) return QLORA_ERR_UNSUPPORTED;
    auto* us_pad = at<__nv_bfloat16>(ws, p.s_us);
    LuArgs u{};
    u.X = static_cast<const __nv_bfloat16*>(X);
    u.T = static_cast<int>(T);
    u.d_in = static_cast<int>(d_in);
    u.kt = sp.kt;
    u.A = static_cast<const __nv_bfloat16*>(A);
    u.r = r;
    u.s = s;
    u.KS = sp.ks;
    u.us_pad = us_pad;
    u.u_save = static_cast<__nv_bfloat16*>(U_save);
    LvArgs g{};
    g.T = static_cast<int>(T);
    g.d_out = static_cast<int>(d_out);
    g.d_in = static_cast<int>(d_in);
    g.kt = sp.kt;
    g.tiles = static_cast<int>(cdiv(d_out, 16));
    g.C = sp.C;
    g.r = r;
    g.rp = (r + 15) & ~15;
    g.codes = w->codes;
    g.absmax_q = w->absmax_q;
    g.c2 = w->c2;
    g.X = static_cast<const __nv_bfloat16*>(X);
    g.us_pad = us_pad;
    g.B = static_cast<const __nv_bfloat16*>(B);
    g.H = static_cast<__nv_bfloat16*>(H);
    g.err = err;
    g.wait_ns = kWaitNs;
    {
        static const float lv[16] = QLORA_NF4_LEVELS;
        for (int i = 0; i < 8; ++i) g.lv16[i] = bf16_bits(lv[2 * i]) | (bf16_bits(lv[2 * i + 1]) << 16);
    }
    if (sp.nt8 == 1) return launch_qgemv<1>(g, sp.ks, u, st);
    return launch_qgemv<2>(g, sp.ks, u, st);
}

qlora_status sgemm(cudaStream_t st, int64_t M, int64_t N, int64_t K, float alpha, const float* A,
                   int64_t lda, bool ta, const float* B, int64_t ldb, bool tb, float beta,
                   float* C, int64_t ldc) {
    dim3 grid(static_cast<unsigned>(cdiv(N, 64)), static_cast<unsigned>(cdiv(M, 64)));
    k_sgemm<<<grid, 256, 0, st>>>(static_cast<int>(M), static_cast<int>(N), static_cast<int>(K),
                                  alpha, A, lda, ta ? 1 : 0, B, ldb, tb ? 1 : 0, beta, C, ldc);
    QL_LAUNCH_CHECK();
    return QLORA_OK;
}

qlora_status dequant_f32(const qlora_nf4* w, float* out, cudaStream_t st) {
    const int64_t nbytes = w->d_out * w->d_in / 2;
    k_nf4_dequant_f32<<<static_cast<unsigned>(cdiv(nbytes, 256)), 256, 0, st>>>(
        w->codes, w->absmax_q, w->c2, nbytes, out);
    QL_LAUNCH_CHECK();
    return QLORA_OK;
}

template <typename T>
qlora_status pad_bf16(const T* src, int64_t rows, int64_t cols, int64_t ld, __nv_bfloat16* dst,
                      int64_t rows_pad, int64_t ld_dst, int64_t col_off, int64_t col_span,
                      cudaStream_t st) {
    if (launch_pdl(k_pad_copy_bf16<T>, grid1d(rows_pad * col_span), dim3(256), 0, st, src, rows,
                   cols, ld, dst, rows_pad, ld_dst, col_off, col_span) != cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    return QLORA_OK;
}

// U = X A^T on the tensor cores (split-K), finalized into the requested outputs.
// a_src holds a_rows rows of d_in (a_rows = RP for a padded copy, r for the caller's A).
qlora_status compute_u_bf16(const void* X, int64_t T, int64_t d_in, const void* a_src, int a_rows,
                            int RP, int r, float s, int split, float* part, __nv_bfloat16* u_save,
                            __nv_bfloat16* u_pad, __nv_bfloat16* u_spad, int* err,
                            cudaStream_t st) {
    CUtensorMap tx, tap;
    QL_TRY(tmap_bf16(&tx, X, T, d_in, d_in, kBM));
    QL_TRY(tmap_bf16(&tap, a_src, a_rows, d_in, d_in, RP));
    QL_TRY(skinny_gemm(false, false, RP, r, tx, tap, T, cdiv(d_in, kBK), split, part, err, st));
    if (launch_pdl(k_finalize_rows<__nv_bfloat16>, grid1d(T * RP), dim3(256), 0, st, part, split,
                   T * RP, T, r, RP, s, u_save, u_pad, u_spad) != cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    return QLORA_OK;
}

// Mid-size forward: the U pre-pass (few CTAs) runs beside the split-K NF4 GEMM, which waits
// for it only before exiting; the finalize then sums the partials and adds s U B^T.
qlora_status mid_fwd(const qlora_nf4* w, const void* X, int64_t T, const void* A, const void* B,
                     int r, float s, void* H, void* U_save, const Plan& p, void* ws, int* err,
                     cudaStream_t st) {
    const int64_t d_out = w->d_out, d_in = w->d_in;
    const MidPlan mp = make_mid_plan(T, d_out, d_in);
    const int RP = p.RP;
    float* us = at<float>(ws, p.s_us);
    float* part = at<float>(ws, p.mid_part);
    auto* u_spad = at<__nv_bfloat16>(ws, p.u_spad);
    // the adapter's B as the extension's B operand: the caller's B when its rows are whole
    // 16-byte units (the map zero-fills the rank padding), else a zero-padded copy
    const void* b_src = B;
    int b_ld = r;
    if (r % 8 != 0) {
        auto* b_pad = at<__nv_bfloat16>(ws, p.b_pad);
        QL_TRY(pad_bf16(static_cast<const __nv_bfloat16*>(B), d_out, r, r, b_pad, d_out, RP, 0, RP, st));
        b_src = b_pad;
        b_ld = RP;
    }
    if (cudaMemsetAsync(u_spad, 0, static_cast<size_t>(T) * RP * 2, st) != cudaSuccess) return QLORA_ERR_CUDA;
    k_small_u<<<static_cast<unsigned>(cdiv(r, 8)), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(X), static_cast<int>(T), static_cast<int>(d_in),
        static_cast<const __nv_bfloat16*>(A), r, s, us, static_cast<__nv_bfloat16*>(U_save), u_spad, RP);
    QL_LAUNCH_CHECK();
    CUtensorMap ta, tc, tax, tbx;
    QL_TRY(tmap_bf16(&ta, X, T, d_in, d_in, kBM));
    QL_TRY(tmap_u8(&tc, w->codes, d_out, d_in / 2, d_in / 2, 32, 256));
    QL_TRY(tmap_bf16(&tax, u_spad, T, RP, RP, kBM));
    QL_TRY(tmap_bf16(&tbx, b_src, d_out, b_ld, b_ld, 256));
    GemmArgs g = base_args(static_cast<int>(T), static_cast<int>(d_out), static_cast<int>(d_in / 64), err);
    g.ext_steps = RP / 64;              // s U B^T as extra K steps of the last split
    g.ext_k16_last = static_cast<int>(std::min<int64_t>(4, cdiv(r - 64 * (g.ext_steps - 1), 16)));
    g.split = mp.split;
    g.absmax_q = w->absmax_q;
    g.c2 = w->c2;
    g.nf4_rows = static_cast<int>(d_out);
    g.nf4_bpr = static_cast<int>(d_in / 64);
    g.out = part;
    g.ld_out = d_out;
    g.split_stride = T * d_out;
    g.late_wait = 1;    // the main steps read only X and W; the extension waits for k_small_u
    dim3 grid(static_cast<unsigned>(mp.n_tiles), 1, static_cast<unsigned>(mp.split));
    QL_TRY((launch_gemm<false, false, kBNf4, 256, kNf4Stages, true>(ta, tc, tax, tbx, g, grid, st, true)));
    if (launch_pdl(k_finalize_mid, grid1d(T * d_out), dim3(256), 0, st, part, mp.split, T * d_out,
                   static_cast<__nv_bfloat16*>(H)) != cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    return QLORA_OK;
}


// The large-T bf16 forward: U pre-pass, then the fused NF4 GEMM with the adapter K-extension;
// col_scale (nullable) multiplies output column n before rounding (DoRA).
qlora_status fwd_bf16_large(const qlora_nf4* w, const void* X, int64_t T, const void* A,
                            const void* B, int32_t r, float s, void* H, void* U_save,
                            const Plan& p, void* ws, int* err, cudaStream_t stream,
                            const float* col_scale) {
    const int64_t d_out = w->d_out, d_in = w->d_in;
    {
        const int RP = p.RP;
        auto* a_pad = at<__nv_bfloat16>(ws, p.a_pad);
        auto* b_pad = at<__nv_bfloat16>(ws, p.b_pad);
        auto* u_spad = at<__nv_bfloat16>(ws, p.u_spad);
        auto* part = at<float>(ws, p.part);
        // With r a multiple of 8 every row of A, B is a whole number of 16-byte units, so the
        // tensor maps address the caller's tensors and zero-fill the rank padding out of
        // bounds; otherwise zero-padded copies are made.
        const bool direct = r % 8 == 0;
        const void* a_src = A;
        const void* b_src = B;
        int a_rows = r, b_ld = r;
        if (!direct) {
            QL_TRY(pad_bf16(static_cast<const __nv_bfloat16*>(A), r, d_in, d_in, a_pad, RP, d_in, 0, d_in, stream));
            QL_TRY(pad_bf16(static_cast<const __nv_bfloat16*>(B), d_out, r, r, b_pad, d_out, RP, 0, RP, stream));
            a_src = a_pad;
            b_src = b_pad;
            a_rows = b_ld = RP;
        }
        QL_TRY(compute_u_bf16(X, T, d_in, a_src, a_rows, RP, r, s, p.split_u, part,
                              static_cast<__nv_bfloat16*>(U_save), nullptr, u_spad, err, stream));
        return nf4_gemm(false, w, X, T, u_spad, b_src, RP, r, b_ld, H, at<void>(ws, p.g2), err, stream,
                        col_scale);
    }
}

// DoRA: scale[j] = magnitude[j] / ||(W^ + s B A)[j, :]|| (or the norms when magnitude is NULL),
// from the tensor-core merge tile in its row-norm mode and one reduction over the 64-column
// tiles.
qlora_status dora_scale(const qlora_nf4* w, const void* A, const void* B, int32_t r, float s,
                        const float* magnitude, float* partial, float* out, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    auto kern = k_merge_tc<bf, true>;
    const int rp = (r + 15) & ~15;
    const int tsmem = MergeSmem::bytes(rp, 2);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, tsmem) != cudaSuccess)
        return QLORA_ERR_CUDA;
    dim3 tgrid(static_cast<unsigned>(w->d_in / 64), static_cast<unsigned>(cdiv(w->d_out, 128)));
    kern<<<tgrid, kMergeThreads, tsmem, stream>>>(w->codes, w->absmax_q, w->c2, w->d_out, w->d_in,
                                                   static_cast<const bf*>(A), static_cast<const bf*>(B),
                                                   r, s, nullptr, partial);
    QL_LAUNCH_CHECK();
    if (launch_pdl(k_dora_scale, grid1d(w->d_out), dim3(256), 0, stream, partial, w->d_out,
                   static_cast<int>(w->d_in / 64), magnitude, out) != cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    return QLORA_OK;
}

// FP8 operands of the dX GEMM: the E5M2 gradient and its scale, the weight's scale, and the
// workspace for sigma_g sigma_w bf16(s G).
struct Fp8Dx {
    const uint8_t* dH8;
    const float* g_scale;
    const float* w_scale;
    __nv_bfloat16* g8;
};

// The bf16 backward: U (or U_saved), G = dH B, dX (bf16 GEMM, or the FP8 GEMM when f8 is set),
// dA, dB by split-K tensor-core products and their finalizes.
// phase: kBwdAll (G, dX, dA, dB), kBwdGrads (G, dA, dB; bf16(sG) stays in the workspace) or
// kBwdDx (dX only, from the bf16(sG) a kBwdGrads call left in the same workspace).
enum BwdPhase { kBwdAll = 0, kBwdGrads = 1, kBwdDx = 2 };
qlora_status bwd_bf16(const qlora_nf4* w, const void* X, const void* dH, int64_t T, const void* A,
                      const void* B, int32_t r, float s, const void* U_saved, void* dX, float* dA,
                      float* dB, const Plan& p, void* ws, int* err, int acc_grads, cudaStream_t stream,
                      const Fp8Dx* f8, BwdPhase phase = kBwdAll) {
    const int64_t d_out = w->d_out, d_in = w->d_in;
    const int RP = p.RP;
    auto* a_pad = at<__nv_bfloat16>(ws, p.a_pad);
    auto* b_pad = at<__nv_bfloat16>(ws, p.b_pad);
    auto* u_pad = at<__nv_bfloat16>(ws, p.u_pad);
    auto* g_spad = at<__nv_bfloat16>(ws, p.g_spad);
    auto* part = at<float>(ws, p.part);
    // pad-free operands when r is a multiple of 8 (see the forward)
    const bool direct = r % 8 == 0;
    const void* a_src = A;
    const void* b_src = B;
    const void* u_src = u_pad;
    int a_rows = r, b_ld = r, u_ld = RP;
    if (!direct) {
        QL_TRY(pad_bf16(static_cast<const __nv_bfloat16*>(A), r, d_in, d_in, a_pad, RP, d_in, 0, d_in, stream));
        QL_TRY(pad_bf16(static_cast<const __nv_bfloat16*>(B), d_out, r, r, b_pad, d_out, RP, 0, RP, stream));
        a_src = a_pad;
        b_src = b_pad;
        a_rows = b_ld = RP;
    }
    if (phase == kBwdDx) {
        // U is not needed for dX
    } else if (U_saved && direct) {
        u_src = U_saved;
        u_ld = r;
    } else if (U_saved) {
        QL_TRY(pad_bf16(static_cast<const __nv_bfloat16*>(U_saved), T, r, r, u_pad, T, RP, 0, RP, stream));
    } else {
        QL_TRY(compute_u_bf16(X, T, d_in, a_src, a_rows, RP, r, s, p.split_u, part, nullptr,
                              u_pad, nullptr, err, stream));
    }
    // Rows of d_out bf16 that are not whole 16-byte units cannot be read by a tensor map: such a
    // dH is copied into rows of d_out rounded up to 8 (the maps still stop at column d_out).
    int64_t dh_ld = d_out;
    if (d_out % 8 != 0 && !f8) {
        dh_ld = (d_out + 7) / 8 * 8;
        auto* dh_pad = at<__nv_bfloat16>(ws, p.dh_pad);
        QL_TRY(pad_bf16(static_cast<const __nv_bfloat16*>(dH), T, d_out, d_out, dh_pad, T, dh_ld, 0, dh_ld, stream));
        dH = dh_pad;
    }
    // G = dH B  ->  g_spad = bf16(s G)
    if (phase != kBwdDx) {
        CUtensorMap tdh, tbp;
        QL_TRY(tmap_bf16(&tdh, dH, T, d_out, dh_ld, kBM));
        QL_TRY(tmap_bf16(&tbp, b_src, d_out, b_ld, b_ld, 64));
        QL_TRY(skinny_gemm(false, true, RP, r, tdh, tbp, T, cdiv(d_out, kBK), p.split_g, part, err, stream));
        if (launch_pdl(k_finalize_rows<__nv_bfloat16>, grid1d(T * RP), dim3(256), 0, stream,
                       part, p.split_g, T * RP, T, r, RP, s, nullptr, nullptr, g_spad) !=
            cudaSuccess)
            return QLORA_ERR_CUDA;
        QL_LAUNCH_CHECK();
    }
    // dX = dH W^ + (sG) A
    if (phase == kBwdGrads) dX = nullptr;
    if (dX && !f8)
        QL_TRY(nf4_gemm(true, w, dH, T, g_spad, a_src, RP, r, a_rows, dX, at<void>(ws, p.g2), err, stream,
                        nullptr, nullptr, nullptr, dh_ld));
    if (dX && f8) {
        // FP8: the adapter operand in the accumulator's units (sigma_g sigma_w, powers of two),
        // then the E5M2 x E4M3 GEMM with the epilogue factor 1 / (sigma_g sigma_w)
        if (launch_pdl(k_scale2_bf16, grid1d(T * RP), dim3(256), 0, stream,
                       static_cast<const __nv_bfloat16*>(g_spad), T * RP, f8->g_scale, f8->w_scale,
                       f8->g8) != cudaSuccess)
            return QLORA_ERR_CUDA;
        QL_LAUNCH_CHECK();
        QL_TRY(nf4_gemm(true, w, f8->dH8, T, f8->g8, a_src, RP, r, a_rows, dX, at<void>(ws, p.g2), err, stream,
                        nullptr, f8->g_scale, f8->w_scale));
    }
    if (phase == kBwdDx) return QLORA_OK;
    // dA^T[d_in, RP] = X^T (sG)
    {
        CUtensorMap txm, tgm;
        QL_TRY(tmap_bf16(&txm, X, T, d_in, d_in, 64));
        QL_TRY(tmap_bf16(&tgm, g_spad, T, RP, RP, 64));
        QL_TRY(skinny_gemm(true, true, RP, r, txm, tgm, d_in, cdiv(T, kBK), p.split_da, part, err, stream));
        if (launch_pdl(k_finalize_dA, grid1d(static_cast<int64_t>(r) * d_in), dim3(256), 0,
                       stream, part, p.split_da, d_in * RP, d_in, r, RP, dA, acc_grads) != cudaSuccess)
            return QLORA_ERR_CUDA;
        QL_LAUNCH_CHECK();
    }
    // dB[d_out, RP] = s dH^T U
    {
        CUtensorMap thm, tum;
        QL_TRY(tmap_bf16(&thm, dH, T, d_out, dh_ld, 64));
        QL_TRY(tmap_bf16(&tum, u_src, T, u_ld, u_ld, 64));
        QL_TRY(skinny_gemm(true, true, RP, r, thm, tum, d_out, cdiv(T, kBK), p.split_db, part, err, stream));
        if (launch_pdl(k_finalize_dB, grid1d(d_out * r), dim3(256), 0, stream, part, p.split_db,
                       d_out * RP, d_out, r, RP, s, dB, acc_grads) != cudaSuccess)
            return QLORA_ERR_CUDA;
        QL_LAUNCH_CHECK();
    }
    return QLORA_OK;
}

}  // namespace

// ======================================================================= C ABI

extern "C" {

const char* qlora_status_string(qlora_status s) {
    switch (s) {
        case QLORA_OK: return "QLORA_OK";
        case QLORA_ERR_INVALID_ARG: return "QLORA_ERR_INVALID_ARG";
        case QLORA_ERR_UNSUPPORTED: return "QLORA_ERR_UNSUPPORTED";
        case QLORA_ERR_CUDA: return "QLORA_ERR_CUDA";
        case QLORA_ERR_TIMEOUT: return "QLORA_ERR_TIMEOUT";
        case QLORA_ERR_DEVICE: return "QLORA_ERR_DEVICE";
    }
    return "QLORA_ERR_UNKNOWN";
}

uint64_t qlora_launch_count(void) { return g_launches.load(); }

qlora_status qlora_nf4_sizes(int64_t d_out, int64_t d_in, size_t* codes_bytes,
                             size_t* absmax_bytes, size_t* c2_bytes) {
    if (!codes_bytes || !absmax_bytes || !c2_bytes) return QLORA_ERR_INVALID_ARG;
    if (d_out < 1 || d_in < 64 || d_in % 64) return QLORA_ERR_UNSUPPORTED;
    const int64_t n = d_out * d_in;
    *codes_bytes = static_cast<size_t>(n / 2);
    *absmax_bytes = static_cast<size_t>(n / 64);
    *c2_bytes = static_cast<size_t>(4 * cdiv(n / 64, 256));
    return QLORA_OK;
}

qlora_status qlora_nf4_levels(float* out) {
    if (!out) return QLORA_ERR_INVALID_ARG;
    static const float levels[16] = QLORA_NF4_LEVELS;
    std::memcpy(out, levels, sizeof(levels));
    return QLORA_OK;
}

size_t qlora_workspace_bytes(int op, qlora_dtype dtype, int64_t T, int64_t d_out, int64_t d_in,
                             int32_t r_total) {
    if (op < QLORA_OP_FWD || op > QLORA_OP_DORA_BWD) return 0;
    if ((op == QLORA_OP_FWD_MULTI || op == QLORA_OP_DORA_FWD || op == QLORA_OP_FWD_FP8 ||
         op == QLORA_OP_FP8_QUANT || op == QLORA_OP_BWD_FP8 || op == QLORA_OP_DORA_BWD) &&
        dtype != QLORA_BF16)
        return 0;
    if ((dtype != QLORA_BF16 && dtype != QLORA_F32) || T < 1 || d_out < 1 || d_in < 64 ||
        r_total < 1 || r_total > 128)
        return 0;
    if (op == QLORA_OP_DORA_BWD) return dora_bwd_layout(T, d_out, d_in, r_total).total;
    return make_plan(op, dtype, T, d_out, d_in, r_total).total;
}

qlora_status nf4_quantize(const void* W, qlora_dtype w_dtype, int64_t d_out, int64_t d_in,
                          uint8_t* codes, uint8_t* absmax_q, float* c2, cudaStream_t stream) {
    if (!aligned16(W) || !aligned16(codes) || !aligned16(absmax_q) || !aligned16(c2))
        return QLORA_ERR_INVALID_ARG;
    if (d_out < 1 || d_in < 64 || d_in % 64) return QLORA_ERR_UNSUPPORTED;
    const int64_t nblocks = d_out * d_in / 64;
    const unsigned groups = static_cast<unsigned>(cdiv(nblocks, 256));
    if (w_dtype == QLORA_F32) {
        k_nf4_quantize<float><<<groups, 256, 0, stream>>>(static_cast<const float*>(W), nblocks,
                                                          codes, absmax_q, c2);
    } else if (w_dtype == QLORA_BF16) {
        k_nf4_quantize<__nv_bfloat16><<<groups, 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(W), nblocks, codes, absmax_q, c2);
    } else {
        return QLORA_ERR_INVALID_ARG;
    }
    QL_LAUNCH_CHECK();
    return QLORA_OK;
}

qlora_status nf4_dequantize(const qlora_nf4* w, void* W_out, qlora_dtype out_dtype,
                            cudaStream_t stream) {
    if (!w || !aligned16(w->codes) || !aligned16(w->absmax_q) || !aligned16(w->c2) ||
        !aligned16(W_out))
        return QLORA_ERR_INVALID_ARG;
    if (w->d_out < 1 || w->d_in < 64 || w->d_in % 64) return QLORA_ERR_UNSUPPORTED;
    const int64_t nblocks = w->d_out * w->d_in / 64;
    if (out_dtype == QLORA_BF16) {
        k_nf4_dequant_bf16<<<static_cast<unsigned>(cdiv(nblocks, 256)), 256, 0, stream>>>(
            w->codes, w->absmax_q, w->c2, nblocks, static_cast<__nv_bfloat16*>(W_out));
        QL_LAUNCH_CHECK();
        return QLORA_OK;
    }
    if (out_dtype == QLORA_F32) return dequant_f32(w, static_cast<float*>(W_out), stream);
    return QLORA_ERR_INVALID_ARG;
}

// Argument checks of qlora_linear_fwd (everything but the workspace), shared with
// qlora_linear_fwd_noalloc so that both return the same status for the same arguments.
__attribute__((visibility("hidden"))) qlora_status qlora_fwd_check_args(
    const qlora_nf4* w, const void* X, int64_t T, const void* A, const void* B, int32_t r,
    qlora_dtype dtype, const void* H, const void* U_save) {
    QL_TRY(check_layer(w, T, r, dtype));
    if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(H) ||
        !aligned16_or_null(U_save))
        return QLORA_ERR_INVALID_ARG;
    return QLORA_OK;
}

qlora_status qlora_linear_fwd(const qlora_nf4* w, const void* X, int64_t T, const void* A,
                              const void* B, int32_t r, float alpha, qlora_dtype dtype, void* H,
                              void* U_save, void* ws, size_t ws_bytes, cudaStream_t stream) {
    QL_TRY(qlora_fwd_check_args(w, X, T, A, B, r, dtype, H, U_save));
    const Plan p = make_plan(QLORA_OP_FWD, dtype, T, w->d_out, w->d_in, r);
    QL_TRY(check_ws(ws, ws_bytes, p.total));
    int* err = nullptr;
    QL_TRY(err_word(&err, stream));
    const int64_t d_out = w->d_out, d_in = w->d_in;
    const float s = alpha / static_cast<float>(r);
    if (p.small)
        return small_fwd(w, X, T, A, B, r, s, H, U_save, p, ws, err, stream);
    if (p.mid)
        return mid_fwd(w, X, T, A, B, r, s, H, U_save, p, ws, err, stream);
    if (dtype == QLORA_BF16) return fwd_bf16_large(w, X, T, A, B, r, s, H, U_save, p, ws, err, stream, nullptr);
    // exact fp32 path
    float* w32 = at<float>(ws, p.w32);
    float* U = U_save ? static_cast<float*>(U_save) : at<float>(ws, p.uf);
    const float* Xf = static_cast<const float*>(X);
    QL_TRY(dequant_f32(w, w32, stream));
    QL_TRY(sgemm(stream, T, r, d_in, 1.f, Xf, d_in, false, static_cast<const float*>(A), d_in, true, 0.f, U, r));
    QL_TRY(sgemm(stream, T, d_out, d_in, 1.f, Xf, d_in, false, w32, d_in, true, 0.f, static_cast<float*>(H), d_out));
    return sgemm(stream, T, d_out, r, s, U, r, false, static_cast<const float*>(B), r, true, 1.f,
                 static_cast<float*>(H), d_out);
}

qlora_status qlora_dora_row_norms(const qlora_nf4* w, const void* A, const void* B, int32_t r,
                                  float alpha, float* norms, void* ws, size_t ws_bytes,
                                  cudaStream_t stream) {
    QL_TRY(check_layer(w, 1, r, QLORA_BF16));
    if (!aligned16(A) || !aligned16(B) || !norms) return QLORA_ERR_INVALID_ARG;
    const size_t need = static_cast<size_t>(w->d_out) * (w->d_in / 64) * 4;
    QL_TRY(check_ws(ws, ws_bytes, need));
    return dora_scale(w, A, B, r, alpha / static_cast<float>(r), nullptr, static_cast<float*>(ws), norms,
                      stream);
}

qlora_status qlora_dora_fwd(const qlora_nf4* w, const void* X, int64_t T, const void* A,
                            const void* B, int32_t r, float alpha, const float* magnitude,
                            void* H, void* U_save, void* ws, size_t ws_bytes, cudaStream_t stream) {
    QL_TRY(check_layer(w, T, r, QLORA_BF16));
    if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(H) || !magnitude ||
        !aligned16_or_null(U_save))
        return QLORA_ERR_INVALID_ARG;
    const Plan p = make_plan(QLORA_OP_DORA_FWD, QLORA_BF16, T, w->d_out, w->d_in, r);
    QL_TRY(check_ws(ws, ws_bytes, p.total));
    int* err = nullptr;
    QL_TRY(err_word(&err, stream));
    const float s = alpha / static_cast<float>(r);
    float* scale = at<float>(ws, p.dora_scale);
    QL_TRY(dora_scale(w, A, B, r, s, magnitude, at<float>(ws, p.dora_part), scale, stream));
    return fwd_bf16_large(w, X, T, A, B, r, s, H, U_save, p, ws, err, stream, scale);
}

qlora_status qlora_dora_fwd_save(const qlora_nf4* w, const void* X, int64_t T, const void* A,
                                 const void* B, int32_t r, float alpha, const float* magnitude,
                                 void* H, void* Z_save, void* U_save, float* norms_save, void* ws,
                                 size_t ws_bytes, cudaStream_t stream) {
    QL_TRY(check_layer(w, T, r, QLORA_BF16));
    if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(H) || !magnitude ||
        !aligned16(Z_save) || !aligned16(U_save) || !norms_save)
        return QLORA_ERR_INVALID_ARG;
    const Plan p = make_plan(QLORA_OP_DORA_FWD, QLORA_BF16, T, w->d_out, w->d_in, r);
    QL_TRY(check_ws(ws, ws_bytes, p.total));
    int* err = nullptr;
    QL_TRY(err_word(&err, stream));
    const float s = alpha / static_cast<float>(r);
    // n (the merge tile's row-norm mode), Z and U (the plain large-T forward), then H = Z c
    QL_TRY(dora_scale(w, A, B, r, s, nullptr, at<float>(ws, p.dora_part), norms_save, stream));
    QL_TRY(fwd_bf16_large(w, X, T, A, B, r, s, Z_save, U_save, p, ws, err, stream, nullptr));
    const int64_t n = (w->d_out % 8 == 0) ? T * w->d_out / 8 : T * w->d_out;
    if (launch_pdl(k_dora_apply, grid1d(n), dim3(256), 0, stream, static_cast<const __nv_bfloat16*>(Z_save),
                   magnitude, static_cast<const float*>(norms_save), T, w->d_out,
                   static_cast<__nv_bfloat16*>(H)) != cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    return QLORA_OK;
}

// The DoRA backward; Zs, Us, ns: the pre-scale output, U and the row norms saved by the forward,
// or all null (recomputed here).
qlora_status dora_bwd_impl(const qlora_nf4* w, const void* X, const void* dH, int64_t T,
                           const void* A, const void* B, int32_t r, float alpha,
                           const float* magnitude, const void* Zs, const void* Us, const float* ns,
                           void* dX, float* dA, float* dB, float* dm, void* ws, size_t ws_bytes,
                           cudaStream_t stream) {
    QL_TRY(check_layer(w, T, r, QLORA_BF16));
    if (!aligned16(X) || !aligned16(dH) || !aligned16(A) || !aligned16(B) || !magnitude ||
        !aligned16(dA) || !aligned16(dB) || !dm || !aligned16_or_null(dX))
        return QLORA_ERR_INVALID_ARG;
    const bool saved = Zs != nullptr;
    if (saved ? (!aligned16(Zs) || !aligned16(Us) || !ns) : (Us != nullptr || ns != nullptr))
        return QLORA_ERR_INVALID_ARG;
    const int64_t d = w->d_out, k = w->d_in;
    const DoraBwdLayout L = dora_bwd_layout(T, d, k, r);
    QL_TRY(check_ws(ws, ws_bytes, L.total));
    int* err = nullptr;
    QL_TRY(err_word(&err, stream));
    using bf = __nv_bfloat16;
    const float s = alpha / static_cast<float>(r);
    void* shared = at<void>(ws, L.shared);
    const float* norms = saved ? ns : at<float>(ws, L.norms);
    float* e = at<float>(ws, L.e);
    float* colpart = at<float>(ws, L.colpart);
    const bf* Z = saved ? static_cast<const bf*>(Zs) : at<bf>(ws, L.z);
    const bf* U = saved ? static_cast<const bf*>(Us) : at<bf>(ws, L.u);
    bf* dZ = at<bf>(ws, L.dz);
    bf* ge = at<bf>(ws, L.ge);
    bf* pm = at<bf>(ws, L.pm);
    bf* qm = at<bf>(ws, L.qm);
    float* aat = at<float>(ws, L.aat);
    float* beb = at<float>(ws, L.beb);
    // n_j = ||(W^ + s B A)[j, :]|| and the pre-scale output Z = X V^T (with U for the backward),
    // unless the forward saved them
    if (!saved) {
        QL_TRY(dora_scale(w, A, B, r, s, nullptr, at<float>(ws, L.merge_part), at<float>(ws, L.norms), stream));
        const Plan pf = make_plan(QLORA_OP_DORA_FWD, QLORA_BF16, T, d, k, r);
        QL_TRY(fwd_bf16_large(w, X, T, A, B, r, s, at<bf>(ws, L.z), at<bf>(ws, L.u), pf, shared, err, stream,
                              nullptr));
    }
    // dZ = dH diag(m / n), dc_j = sum_t dH[t, j] Z[t, j], dm = dc / n, e = -dc m / n^3
    const dim3 cgrid(static_cast<unsigned>(cdiv(d / 2, 256)), static_cast<unsigned>(kDoraChunks));
    if (launch_pdl(k_dora_colred, cgrid, dim3(256), 0, stream, static_cast<const bf*>(dH),
                   static_cast<const bf*>(Z), magnitude, static_cast<const float*>(norms), T, d, dZ,
                   colpart) != cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    if (launch_pdl(k_dora_coef, grid1d(d), dim3(256), 0, stream, static_cast<const float*>(colpart),
                   kDoraChunks, d, magnitude, static_cast<const float*>(norms), dm, e) != cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    // the LoRA backward of dZ: dX = dZ V, dA and dB without the norm's term
    const Plan pb = make_plan(QLORA_OP_BWD, QLORA_BF16, T, d, k, r);
    QL_TRY(bwd_bf16(w, X, dZ, T, A, B, r, s, U, dX, dA, dB, pb, shared, err, 0, stream, nullptr));
    // the norm's term: P = A W^T and Q = (B^T diag(e)) W^ by the fused NF4 GEMM with the r
    // adapter rows as tokens, then the r x r Gram products and the two updates
    const int64_t ge_ld = (d + 7) / 8 * 8;
    if (launch_pdl(k_dora_ge, grid1d(r * ge_ld), dim3(256), 0, stream, static_cast<const bf*>(B),
                   static_cast<const float*>(e), static_cast<int>(r), d, ge_ld, ge) != cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    QL_TRY(nf4_gemm(false, w, A, r, nullptr, nullptr, 0, 0, 0, pm, shared, err, stream));
    QL_TRY(nf4_gemm(true, w, ge, r, nullptr, nullptr, 0, 0, 0, qm, shared, err, stream, nullptr, nullptr,
                    nullptr, ge_ld));
    if (launch_pdl(k_dora_gram, dim3(static_cast<unsigned>(r * r), 2), dim3(256), 0, stream,
                   static_cast<const bf*>(A), static_cast<const bf*>(B), static_cast<const float*>(e),
                   static_cast<int>(r), d, k, aat, beb) != cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    if (launch_pdl(k_dora_add_db, grid1d(d * r), dim3(256), 0, stream, static_cast<const bf*>(pm),
                   static_cast<const bf*>(B), static_cast<const float*>(aat), static_cast<const float*>(e),
                   static_cast<int>(r), d, s, dB) != cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    if (launch_pdl(k_dora_add_da, grid1d(r * k), dim3(256), 0, stream, static_cast<const bf*>(qm),
                   static_cast<const bf*>(A), static_cast<const float*>(beb), static_cast<int>(r), k, s,
                   dA) != cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    return QLORA_OK;
}

qlora_status qlora_dora_bwd(const qlora_nf4* w, const void* X, const void* dH, int64_t T,
                            const void* A, const void* B, int32_t r, float alpha,
                            const float* magnitude, void* dX, float* dA, float* dB, float* dm,
                            void* ws, size_t ws_bytes, cudaStream_t stream) {
    return dora_bwd_impl(w, X, dH, T, A, B, r, alpha, magnitude, nullptr, nullptr, nullptr, dX, dA, dB,
                         dm, ws, ws_bytes, stream);
}

qlora_status qlora_dora_bwd_saved(const qlora_nf4* w, const void* X, const void* dH, int64_t T,
                                  const void* A, const void* B, int32_t r, float alpha,
                                  const float* magnitude, const void* Z_saved, const void* U_saved,
                                  const float* norms_saved, void* dX, float* dA, float* dB, float* dm,
                                  void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (!Z_saved || !U_saved || !norms_saved) return QLORA_ERR_INVALID_ARG;
    return dora_bwd_impl(w, X, dH, T, A, B, r, alpha, magnitude, Z_saved, U_saved, norms_saved, dX, dA,
                         dB, dm, ws, ws_bytes, stream);
}

qlora_status qlora_fp8_quantize(const void* X, int64_t n, uint8_t* X8, float* scale, void* ws,
                                size_t ws_bytes, cudaStream_t stream) {
    if (!aligned16(X) || !aligned16(X8) || !scale) return QLORA_ERR_INVALID_ARG;
    if (n < 1) return QLORA_ERR_UNSUPPORTED;
    QL_TRY(check_ws(ws, ws_bytes, 256));
    auto* amax = static_cast<unsigned*>(ws);
    if (cudaMemsetAsync(amax, 0, 4, stream) != cudaSuccess) return QLORA_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>(std::min<int64_t>(std::max<int64_t>(cdiv(n, 8 * 256), 1), 148 * 8)));
    if (launch_pdl(k_fp8_amax, grid, dim3(256), 0, stream, static_cast<const __nv_bfloat16*>(X), n, amax) !=
        cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    if (launch_pdl(k_fp8_quant<false>, grid, dim3(256), 0, stream, static_cast<const __nv_bfloat16*>(X), n,
                   static_cast<const unsigned*>(amax), X8, scale) != cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    return QLORA_OK;
}

qlora_status qlora_fp8_quantize_grad(const void* dH, int64_t n, uint8_t* dH8, float* scale, void* ws,
                                     size_t ws_bytes, cudaStream_t stream) {
    if (!aligned16(dH) || !aligned16(dH8) || !scale) return QLORA_ERR_INVALID_ARG;
    if (n < 1) return QLORA_ERR_UNSUPPORTED;
    QL_TRY(check_ws(ws, ws_bytes, 256));
    auto* amax = static_cast<unsigned*>(ws);
    if (cudaMemsetAsync(amax, 0, 4, stream) != cudaSuccess) return QLORA_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>(std::min<int64_t>(std::max<int64_t>(cdiv(n, 8 * 256), 1), 148 * 8)));
    if (launch_pdl(k_fp8_amax, grid, dim3(256), 0, stream, static_cast<const __nv_bfloat16*>(dH), n, amax) !=
        cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    if (launch_pdl(k_fp8_quant<true>, grid, dim3(256), 0, stream, static_cast<const __nv_bfloat16*>(dH), n,
                   static_cast<const unsigned*>(amax), dH8, scale) != cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    return QLORA_OK;
}

qlora_status qlora_linear_bwd_fp8(const qlora_nf4* w, const uint8_t* X8, const float* x_scale,
                                  const uint8_t* dH8, const float* g_scale, const float* w_scale,
                                  int64_t T, const void* A, const void* B, int32_t r, float alpha,
                                  void* dX, float* dA, float* dB, void* ws, size_t ws_bytes,
                                  uint32_t flags, cudaStream_t stream) {
    if (flags & ~static_cast<uint32_t>(QLORA_BWD_ACCUMULATE)) return QLORA_ERR_INVALID_ARG;
    const int acc_grads = (flags & QLORA_BWD_ACCUMULATE) ? 1 : 0;
    QL_TRY(check_layer(w, T, r, QLORA_BF16));
    if (!aligned16(X8) || !aligned16(dH8) || !aligned16(A) || !aligned16(B) || !aligned16(dA) ||
        !aligned16(dB) || !aligned16_or_null(dX) || !x_scale || !g_scale || !w_scale)
        return QLORA_ERR_INVALID_ARG;
    // the E5M2 gradient's rows are d_out bytes: a TMA row stride must be a multiple of 16
    if (w->d_out % 16 != 0) return QLORA_ERR_UNSUPPORTED;
    const Plan p = make_plan(QLORA_OP_BWD_FP8, QLORA_BF16, T, w->d_out, w->d_in, r);
    QL_TRY(check_ws(ws, ws_bytes, p.total));
    int* err = nullptr;
    QL_TRY(err_word(&err, stream));
    const int64_t d_out = w->d_out, d_in = w->d_in;
    // the stored FP8 tensors back in their own units (exact in bf16) for the skinny products
    auto* xb = at<__nv_bfloat16>(ws, p.f8_x);
    auto* hb = at<__nv_bfloat16>(ws, p.f8_dh);
    if (launch_pdl(k_fp8_dequant<false>, grid1d(T * d_in / 8), dim3(256), 0, stream, X8, T * d_in, x_scale, xb) !=
        cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    if (launch_pdl(k_fp8_dequant<true>, grid1d(T * d_out / 8), dim3(256), 0, stream, dH8, T * d_out, g_scale, hb) !=
        cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    const Fp8Dx f8{dH8, g_scale, w_scale, at<__nv_bfloat16>(ws, p.f8_g)};
    return bwd_bf16(w, xb, hb, T, A, B, r, alpha / static_cast<float>(r), nullptr, dX, dA, dB, p, ws, err,
                    acc_grads, stream, &f8);
}

qlora_status qlora_fp8_weight_scale(const qlora_nf4* w, float* w_scale, cudaStream_t stream) {
    QL_TRY(check_nf4(w));
    if (!w_scale) return QLORA_ERR_INVALID_ARG;
    const int64_t groups = cdiv(w->d_out * w->d_in / 64, 256);
    if (launch_pdl(k_fp8_wscale, dim3(1), dim3(256), 0, stream, w->c2, groups, w_scale) != cudaSuccess)
        return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    return QLORA_OK;
}

qlora_status qlora_linear_fwd_fp8(const qlora_nf4* w, const uint8_t* X8, int64_t T,
                                  const float* x_scale, const float* w_scale, const void* A,
                                  const void* B, int32_t r, float alpha, void* H, void* ws,
                                  size_t ws_bytes, cudaStream_t stream) {
    QL_TRY(check_layer(w, T, r, QLORA_BF16));
    if (!aligned16(X8) || !aligned16(A) || !aligned16(B) || !aligned16(H) || !x_scale || !w_scale)
        return QLORA_ERR_INVALID_ARG;
    const Plan p = make_plan(QLORA_OP_FWD_FP8, QLORA_BF16, T, w->d_out, w->d_in, r);
    QL_TRY(check_ws(ws, ws_bytes, p.total));
    int* err = nullptr;
    QL_TRY(err_word(&err, stream));
    const int64_t d_out = w->d_out, d_in = w->d_in;
    const float s = alpha / static_cast<float>(r);
    const int RP = p.RP;
    // B as the extension's B operand: the caller's B when its rows are whole 16-byte units
    // (the map zero-fills the rank padding), else a zero-padded copy
    const void* b_src = B;
    int b_ld = r;
    if (r % 8 != 0) {
        auto* b_pad = at<__nv_bfloat16>(ws, p.b_pad);
        QL_TRY(pad_bf16(static_cast<const __nv_bfloat16*>(B), d_out, r, r, b_pad, d_out, RP, 0, RP, stream));
        b_src = b_pad;
        b_ld = RP;
    }
    auto* u = at<__nv_bfloat16>(ws, p.u_spad);
    const auto* Ab = static_cast<const __nv_bfloat16*>(A);
    const dim3 ug(static_cast<unsigned>(cdiv(T, 16)));
    const int di = static_cast<int>(d_in);
    cudaError_t e;
    if (r <= 16) e = launch_pdl(k_fp8_u<2, 8, 4>, ug, dim3(256), 0, stream, X8, T, di, Ab, r, s, w_scale, u, RP);
    else if (r <= 32) e = launch_pdl(k_fp8_u<4, 8, 2>, ug, dim3(256), 0, stream, X8, T, di, Ab, r, s, w_scale, u, RP);
    else if (r <= 64) e = launch_pdl(k_fp8_u<8, 8, 1>, ug, dim3(256), 0, stream, X8, T, di, Ab, r, s, w_scale, u, RP);
    else e = launch_pdl(k_fp8_u<16, 4, 1>, ug, dim3(128), 0, stream, X8, T, di, Ab, r, s, w_scale, u, RP);
    if (e != cudaSuccess) return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    return nf4_gemm(false, w, X8, T, u, b_src, RP, r, b_ld, H, at<void>(ws, p.g2), err, stream, nullptr,
                    x_scale, w_scale);
}

qlora_status qlora_linear_bwd_ex(const qlora_nf4* w, const void* X, const void* dH, int64_t T,
                                 const void* A, const void* B, int32_t r, float alpha,
                                 const void* U_saved, qlora_dtype dtype, void* dX, float* dA,
                                 float* dB, void* ws, size_t ws_bytes, uint32_t flags,
                                 cudaStream_t stream) {
    constexpr uint32_t kKnown = QLORA_BWD_ACCUMULATE | QLORA_BWD_GRADS_ONLY | QLORA_BWD_DX_FROM_WS;
    if (flags & ~kKnown) return QLORA_ERR_INVALID_ARG;
    const bool grads_only = (flags & QLORA_BWD_GRADS_ONLY) != 0;
    const bool dx_only = (flags & QLORA_BWD_DX_FROM_WS) != 0;
    if (grads_only && dx_only) return QLORA_ERR_INVALID_ARG;
    const int acc_grads = (flags & QLORA_BWD_ACCUMULATE) ? 1 : 0;
    QL_TRY(check_layer(w, T, r, dtype));
    if (!aligned16(X) || !aligned16(dH) || !aligned16(A) || !aligned16(B) || !aligned16_or_null(dX) ||
        !aligned16_or_null(U_saved))
        return QLORA_ERR_INVALID_ARG;
    if (dx_only ? dX == nullptr : (!aligned16(dA) || !aligned16(dB))) return QLORA_ERR_INVALID_ARG;
    if (grads_only) dX = nullptr;
    const BwdPhase phase = grads_only ? kBwdGrads : dx_only ? kBwdDx : kBwdAll;
    const Plan p = make_plan(QLORA_OP_BWD, dtype, T, w->d_out, w->d_in, r);
    QL_TRY(check_ws(ws, ws_bytes, p.total));
    int* err = nullptr;
    QL_TRY(err_word(&err, stream));
    const int64_t d_out = w->d_out, d_in = w->d_in;
    const float s = alpha / static_cast<float>(r);
    if (dtype == QLORA_BF16)
        return bwd_bf16(w, X, dH, T, A, B, r, s, U_saved, dX, dA, dB, p, ws, err, acc_grads, stream, nullptr,
                        phase);
    // exact fp32 path
    const float* Xf = static_cast<const float*>(X);
    const float* dHf = static_cast<const float*>(dH);
    const float* Af = static_cast<const float*>(A);
    const float* Bf = static_cast<const float*>(B);
    float* w32 = at<float>(ws, p.w32);
    float* U = at<float>(ws, p.uf);
    float* G = at<float>(ws, p.gf);
    if (phase != kBwdGrads) QL_TRY(dequant_f32(w, w32, stream));
    const float* Uc = static_cast<const float*>(U_saved);
    if (!Uc && phase != kBwdDx) {
        QL_TRY(sgemm(stream, T, r, d_in, 1.f, Xf, d_in, false, Af, d_in, true, 0.f, U, r));
        Uc = U;
    }
    if (phase != kBwdDx) QL_TRY(sgemm(stream, T, r, d_out, 1.f, dHf, d_out, false, Bf, r, false, 0.f, G, r));
    if (dX) {
        float* dXf = static_cast<float*>(dX);
        QL_TRY(sgemm(stream, T, d_in, d_out, 1.f, dHf, d_out, false, w32, d_in, false, 0.f, dXf, d_in));
        QL_TRY(sgemm(stream, T, d_in, r, s, G, r, false, Af, d_in, false, 1.f, dXf, d_in));
    }
    if (phase == kBwdDx) return QLORA_OK;
    const float beta = acc_grads ? 1.f : 0.f;
    QL_TRY(sgemm(stream, r, d_in, T, s, G, r, true, Xf, d_in, false, beta, dA, d_in));
    return sgemm(stream, d_out, r, T, s, dHf, d_out, true, Uc, r, false, beta, dB, r);
}

qlora_status qlora_linear_bwd(const qlora_nf4* w, const void* X, const void* dH, int64_t T,
                              const void* A, const void* B, int32_t r, float alpha,
                              const void* U_saved, qlora_dtype dtype, void* dX, float* dA,
                              float* dB, void* ws, size_t ws_bytes, cudaStream_t stream) {
    return qlora_linear_bwd_ex(w, X, dH, T, A, B, r, alpha, U_saved, dtype, dX, dA, dB, ws,
                               ws_bytes, 0u, stream);
}

qlora_status qlora_adamw_step(void* param, qlora_dtype param_dtype, float* master,
                              const float* grad, float* m, float* v, int64_t n, int32_t step,
                              float lr, float beta1, float beta2, float eps, float weight_decay,
                              float grad_scale, cudaStream_t stream) {
    if (!param || !grad || !m || !v || n < 1 || step < 1) return QLORA_ERR_INVALID_ARG;
    if (param_dtype == QLORA_BF16 && (!master || master == param)) return QLORA_ERR_INVALID_ARG;
    if (param_dtype == QLORA_F32 && master && master != param) return QLORA_ERR_INVALID_ARG;
    if (param_dtype != QLORA_BF16 && param_dtype != QLORA_F32) return QLORA_ERR_INVALID_ARG;
    if (!(beta1 >= 0.f && beta1 < 1.f && beta2 >= 0.f && beta2 < 1.f)) return QLORA_ERR_INVALID_ARG;
    AdamArgs a{};
    a.n = n;
    a.lr = lr;
    a.beta1 = beta1;
    a.beta2 = beta2;
    a.eps = eps;
    a.wd = weight_decay;
    a.grad_scale = grad_scale;
    a.bc1 = static_cast<float>(1.0 - std::pow(static_cast<double>(beta1), step));
    a.bc2 = static_cast<float>(1.0 - std::pow(static_cast<double>(beta2), step));
    const bool vec = n % 4 == 0 && aligned16(param) && aligned16(grad) && aligned16(m) &&
                     aligned16(v) && (param_dtype == QLORA_F32 || aligned16(master)) &&
                     (param_dtype == QLORA_F32 || (reinterpret_cast<uintptr_t>(param) & 7u) == 0);
    const dim3 grid = grid1d(vec ? n / 4 : n);
    cudaError_t e;
    if (param_dtype == QLORA_BF16) {
        auto* pb = static_cast<__nv_bfloat16*>(param);
        e = vec ? launch_pdl(k_adamw<__nv_bfloat16, true>, grid, dim3(256), 0, stream, pb, master, grad, m, v, a)
                : launch_pdl(k_adamw<__nv_bfloat16, false>, grid, dim3(256), 0, stream, pb, master, grad, m, v, a);
    } else {
        auto* pf = static_cast<float*>(param);
        e = vec ? launch_pdl(k_adamw<float, true>, grid, dim3(256), 0, stream, pf, pf, grad, m, v, a)
                : launch_pdl(k_adamw<float, false>, grid, dim3(256), 0, stream, pf, pf, grad, m, v, a);
    }
    if (e != cudaSuccess) return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    return QLORA_OK;
}

qlora_status qlora_prefetch(const void* ptr, size_t bytes, int32_t to_device, cudaStream_t stream) {
    if (!ptr || bytes == 0) return QLORA_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
    cudaMemLocation loc{};
    loc.type = to_device ? cudaMemLocationTypeDevice : cudaMemLocationTypeHost;
    loc.id = to_device ? dev : 0;
    return cudaMemPrefetchAsync(ptr, bytes, loc, 0, stream) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status lora_merge(const qlora_nf4* w, const void* A, const void* B, int32_t r, float alpha,
                        qlora_dtype adapter_dtype, qlora_dtype out_dtype, void* W_final,
                        cudaStream_t stream) {
    QL_TRY(check_nf4(w));
    if (!aligned16(A) || !aligned16(B) || !aligned16(W_final)) return QLORA_ERR_INVALID_ARG;
    if (r < 1 || r > 128) return QLORA_ERR_UNSUPPORTED;
    const float s = alpha / static_cast<float>(r);
    dim3 grid(static_cast<unsigned>(cdiv(w->d_in, 128)), static_cast<unsigned>(cdiv(w->d_out, 64)));
    const size_t rp = static_cast<size_t>((r + 15) & ~15);
    const size_t smem = rp * 128 * 4 + 64 * rp * 4;
    auto run = [&](auto kern, auto a, auto b, auto o) -> qlora_status {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return QLORA_ERR_CUDA;
        kern<<<grid, 256, smem, stream>>>(w->codes, w->absmax_q, w->c2, w->d_out, w->d_in, a, b, r, s, o);
        QL_LAUNCH_CHECK();
        return QLORA_OK;
    };
    using bf = __nv_bfloat16;
    // bf16 adapters: B A on the tensor cores (exact products, fp32 accumulation)
    auto run_tc = [&](auto kern, auto o) -> qlora_status {
        const int tsmem = MergeSmem::bytes(static_cast<int>(rp), static_cast<int>(sizeof(*o)));
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, tsmem) != cudaSuccess)
            return QLORA_ERR_CUDA;
        dim3 tgrid(static_cast<unsigned>(w->d_in / 64), static_cast<unsigned>(cdiv(w->d_out, 128)));
        kern<<<tgrid, kMergeThreads, tsmem, stream>>>(w->codes, w->absmax_q, w->c2, w->d_out, w->d_in,
                                                       static_cast<const bf*>(A), static_cast<const bf*>(B),
                                                       r, s, o, nullptr);
        QL_LAUNCH_CHECK();
        return QLORA_OK;
    };
    if (adapter_dtype == QLORA_BF16 && out_dtype == QLORA_BF16)
        return run_tc(k_merge_tc<bf>, static_cast<bf*>(W_final));
    if (adapter_dtype == QLORA_BF16 && out_dtype == QLORA_F32)
        return run_tc(k_merge_tc<float>, static_cast<float*>(W_final));
    if (adapter_dtype == QLORA_F32 && out_dtype == QLORA_BF16)
        return run(k_merge<float, bf>, static_cast<const float*>(A), static_cast<const float*>(B), static_cast<bf*>(W_final));
    if (adapter_dtype == QLORA_F32 && out_dtype == QLORA_F32)
        return run(k_merge<float, float>, static_cast<const float*>(A), static_cast<const float*>(B), static_cast<float*>(W_final));
    return QLORA_ERR_INVALID_ARG;
}

qlora_status qlora_linear_fwd_multi(const qlora_nf4* w, const void* X, int64_t T,
                                    const int32_t* adapter_id, int32_t n_adapters,
                                    const void* const* A_ptrs, const void* const* B_ptrs,
                                    const int32_t* ranks, const float* alphas, int32_t r_max,
                                    void* H, void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (!A_ptrs || !B_ptrs || !ranks || !alphas || !adapter_id) return QLORA_ERR_INVALID_ARG;
    if (n_adapters < 1 || n_adapters > kSegMaxAdapters) return QLORA_ERR_UNSUPPORTED;
    QL_TRY(check_layer(w, T, r_max, QLORA_BF16));
    if (!aligned16(X) || !aligned16(H) || (reinterpret_cast<uintptr_t>(adapter_id) & 3u) ||
        (reinterpret_cast<uintptr_t>(A_ptrs) & 7u) || (reinterpret_cast<uintptr_t>(B_ptrs) & 7u) ||
        (reinterpret_cast<uintptr_t>(ranks) & 3u) || (reinterpret_cast<uintptr_t>(alphas) & 3u))
        return QLORA_ERR_INVALID_ARG;
    if (T > (1LL << 31) - 1) return QLORA_ERR_UNSUPPORTED;
    const Plan p = make_plan(QLORA_OP_FWD_MULTI, QLORA_BF16, T, w->d_out, w->d_in, r_max);
    QL_TRY(check_ws(ws, ws_bytes, p.total));
    int* err = nullptr;
    QL_TRY(err_word(&err, stream));
    SegArgs a{};
    a.T = T;
    a.n = n_adapters;
    a.d_in = static_cast<int>(w->d_in);
    a.d_out = static_cast<int>(w->d_out);
    a.ldu = p.seg_ldu;
    a.X = static_cast<const __nv_bfloat16*>(X);
    a.H = static_cast<__nv_bfloat16*>(H);
    a.ids = adapter_id;
    a.A = reinterpret_cast<const __nv_bfloat16* const*>(A_ptrs);
    a.B = reinterpret_cast<const __nv_bfloat16* const*>(B_ptrs);
    a.ranks = ranks;
    a.alphas = alphas;
    a.cnt = at<int32_t>(ws, p.seg_cnt);
    a.seg_start = at<int32_t>(ws, p.seg_start);
    a.cursor = at<int32_t>(ws, p.seg_cursor);
    a.n_tiles = at<int32_t>(ws, p.seg_ntiles);
    a.tiles = at<int4>(ws, p.seg_tiles);
    a.perm = at<int32_t>(ws, p.seg_perm);
    a.U = at<__nv_bfloat16>(ws, p.seg_u);
    a.err = err;
    // sort and shrink, then the shared base term (H = bf16(X W^T)), then the corrections
    if (cudaMemsetAsync(a.cnt, 0, static_cast<size_t>(n_adapters) * 4, stream) != cudaSuccess)
        return QLORA_ERR_CUDA;
    if (launch_pdl(k_seg_count, grid1d(T), dim3(256), 0, stream, a) != cudaSuccess) return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    if (launch_pdl(k_seg_plan, dim3(1), dim3(1024), 0, stream, a) != cudaSuccess) return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    if (launch_pdl(k_seg_scatter, grid1d(T), dim3(256), 0, stream, a) != cudaSuccess) return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    // persistent grids over the planned tiles: four resident CTAs of 128 threads per SM
    const unsigned seg_grid = static_cast<unsigned>(std::min<int64_t>(p.seg_max_tiles, 4 * kSmsForSplit));
    // accumulators for the largest rank's n8 tiles (a rank above r_max is rejected on the device)
    cudaError_t se;
    if (r_max <= 16) se = launch_pdl(k_seg_shrink<2, 4>, dim3(seg_grid), dim3(128), 0, stream, a);
    else if (r_max <= 32) se = launch_pdl(k_seg_shrink<4, 2>, dim3(seg_grid), dim3(128), 0, stream, a);
    else if (r_max <= 64) se = launch_pdl(k_seg_shrink<8, 2>, dim3(seg_grid), dim3(128), 0, stream, a);
    else se = launch_pdl(k_seg_shrink<16, 1>, dim3(seg_grid), dim3(128), 0, stream, a);
    if (se != cudaSuccess) return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    QL_TRY(nf4_gemm(false, w, X, T, nullptr, nullptr, 0, 0, 0, H, at<void>(ws, p.g2), err, stream));
    cudaError_t ee;
    const bool odd = (w->d_out & 1) != 0;
    if (r_max <= 16)
        ee = launch_pdl(odd ? k_seg_expand<1, true> : k_seg_expand<1, false>, dim3(seg_grid), dim3(128), 0, stream, a);
    else if (r_max <= 32)
        ee = launch_pdl(odd ? k_seg_expand<2, true> : k_seg_expand<2, false>, dim3(seg_grid), dim3(128), 0, stream, a);
    else if (r_max <= 64)
        ee = launch_pdl(odd ? k_seg_expand<4, true> : k_seg_expand<4, false>, dim3(seg_grid), dim3(128), 0, stream, a);
    else
        ee = launch_pdl(odd ? k_seg_expand<8, true> : k_seg_expand<8, false>, dim3(seg_grid), dim3(128), 0, stream, a);
    if (ee != cudaSuccess) return QLORA_ERR_CUDA;
    QL_LAUNCH_CHECK();
    return QLORA_OK;
}

qlora_status qlora_linear_fwd_batched(const qlora_nf4* w, const void* X, int64_t T,
                                      const int32_t* adapter_id, int32_t n_adapters,
                                      const void* const* A, const void* const* B,
                                      const int32_t* r, const float* alpha, qlora_dtype dtype,
                                      void* H, void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (!A || !B || !r || !alpha || n_adapters < 1 || n_adapters > 32) return QLORA_ERR_INVALID_ARG;
    int R = 0;
    for (int i = 0; i < n_adapters; ++i) {
        if (r[i] < 1 || r[i] > 128) return QLORA_ERR_UNSUPPORTED;
        if (!aligned16(A[i]) || !aligned16(B[i])) return QLORA_ERR_INVALID_ARG;
        R += r[i];
    }
    if (R > 128) return QLORA_ERR_UNSUPPORTED;
    QL_TRY(check_layer(w, T, R, dtype));
    if (!aligned16(X) || !aligned16(H) || !aligned16(adapter_id)) return QLORA_ERR_INVALID_ARG;
    const Plan p = make_plan(QLORA_OP_FWD_BATCHED, dtype, T, w->d_out, w->d_in, R);
    QL_TRY(check_ws(ws, ws_bytes, p.total));
    int* err = nullptr;
    QL_TRY(err_word(&err, stream));
    const int64_t d_out = w->d_out, d_in = w->d_in;
    SegTable seg;
    for (int j = 0; j < 128; ++j) seg.seg_of[j] = -1;
    for (int i = 0; i < 32; ++i) seg.scale[i] = 0.f;
    {
        int off = 0;
        for (int i = 0; i < n_adapters; ++i) {
            for (int j = 0; j < r[i]; ++j) seg.seg_of[off + j] = i;
            seg.scale[i] = alpha[i] / static_cast<float>(r[i]);
            off += r[i];
        }
    }
    if (dtype == QLORA_BF16) {
        const int RP = p.RP;
        auto* a_cat = at<__nv_bfloat16>(ws, p.a_pad);
        auto* b_cat = at<__nv_bfloat16>(ws, p.b_pad);
        auto* u_all = at<__nv_bfloat16>(ws, p.u_spad);
        auto* part = at<float>(ws, p.part);
        // all adapters concatenated (and zero-padded to RP) in one launch
        CatTable cat;
        for (int j = 0; j < 128; ++j) cat.seg_of[j] = static_cast<int8_t>(seg.seg_of[j]);
        for (int i = 0, off = 0; i < 32; ++i) {
            const bool used = i < n_adapters;
            cat.A[i] = used ? static_cast<const __nv_bfloat16*>(A[i]) : nullptr;
            cat.B[i] = used ? static_cast<const __nv_bfloat16*>(B[i]) : nullptr;
            cat.r[i] = used ? r[i] : 0;
            cat.off[i] = off;
            if (used) off += r[i];
        }
        if (launch_pdl(k_concat_adapters, grid1d(static_cast<int64_t>(RP) * (d_in / 8) + d_out * RP),
                       dim3(256), 0, stream, cat, d_out, d_in, RP, a_cat, b_cat) != cudaSuccess)
            return QLORA_ERR_CUDA;
        QL_LAUNCH_CHECK();
        CUtensorMap tx, tap;
        QL_TRY(tmap_bf16(&tx, X, T, d_in, d_in, kBM));
        QL_TRY(tmap_bf16(&tap, a_cat, RP, d_in, d_in, RP));
        QL_TRY(skinny_gemm(false, false, RP, R, tx, tap, T, cdiv(d_in, kBK), p.split_u, part, err, stream));
        if (launch_pdl(k_finalize_multi, grid1d(T * RP), dim3(256), 0, stream, part, p.split_u,
                       T * RP, T, RP, n_adapters, adapter_id, seg, u_all,
                       static_cast<float*>(nullptr), err) != cudaSuccess)
            return QLORA_ERR_CUDA;
        QL_LAUNCH_CHECK();
        return nf4_gemm(false, w, X, T, u_all, b_cat, RP, R, RP, H, at<void>(ws, p.g2), err, stream);
    }
    // exact fp32 path
    float* w32 = at<float>(ws, p.w32);
    float* a_cat = at<float>(ws, p.a_pad);
    float* b_cat = at<float>(ws, p.b_pad);
    float* U = at<float>(ws, p.uf);
    int off = 0;
    for (int i = 0; i < n_adapters; ++i) {
        k_pad_copy_f32<<<grid1d(static_cast<int64_t>(r[i]) * d_in), 256, 0, stream>>>(
            static_cast<const float*>(A[i]), r[i], d_in, d_in, a_cat + static_cast<int64_t>(off) * d_in,
            r[i], d_in, 0, d_in);
        QL_LAUNCH_CHECK();
        k_pad_copy_f32<<<grid1d(d_out * r[i]), 256, 0, stream>>>(
            static_cast<const float*>(B[i]), d_out, r[i], r[i], b_cat, d_out, R, off, r[i]);
        QL_LAUNCH_CHECK();
        off += r[i];
    }
    const float* Xf = static_cast<const float*>(X);
    QL_TRY(dequant_f32(w, w32, stream));
    QL_TRY(sgemm(stream, T, R, d_in, 1.f, Xf, d_in, false, a_cat, d_in, true, 0.f, U, R));
    k_mask_multi_f32<<<grid1d(T * R), 256, 0, stream>>>(U, T, R, n_adapters, adapter_id, seg, err);
    QL_LAUNCH_CHECK();
    QL_TRY(sgemm(stream, T, d_out, d_in, 1.f, Xf, d_in, false, w32, d_in, true, 0.f, static_cast<float*>(H), d_out));
    return sgemm(stream, T, d_out, R, 1.f, U, R, false, b_cat, R, true, 1.f, static_cast<float*>(H), d_out);
}

qlora_status qlora_get_device_error(cudaStream_t stream) {
    int* err = nullptr;
    QL_TRY(err_word(&err, stream));
    if (cudaStreamSynchronize(stream) != cudaSuccess) return QLORA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return QLORA_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
            return QLORA_ERR_CUDA;
    }
    return static_cast<qlora_status>(v);
}

qlora_status qlora_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream) {
    int* err = nullptr;
    QL_TRY(err_word(&err, stream));
    k_wait_timeout_selftest<<<1, 32, 0, stream>>>(err, limit_ns);
    QL_LAUNCH_CHECK();
    return QLORA_OK;
}

qlora_status qlora_set_gemm_events(cudaEvent_t start, cudaEvent_t stop) {
    g_ev_start = start;
    g_ev_stop = stop;
    return QLORA_OK;
}

}  // extern "C"

// simt.cuh -- CUDA-core kernels of libqlora: the exact-fp32 GEMM used by the fp32 dtype,
// adapter padding/packing, split-K finalizers for the skinny adapter contractions, and the
// merge kernel.
#pragma once

#include "common.cuh"
#include "nf4.cuh"

namespace qlora {

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

// ------------------------------------------------------------------ fp32 GEMM

// C[M,N] = alpha * op(A)[M,K] op(B)[K,N] + beta * C, fp32 FFMA (no TF32), 64x64 tiles,
// 256 threads with 4x4 outputs each.  op(A)(m,k) = ta ? A[k*lda+m] : A[m*lda+k];
// op(B)(k,n) = tb ? B[n*ldb+k] : B[k*ldb+n].
__global__ void __launch_bounds__(256) k_sgemm(int M, int N, int K, float alpha,
                                               const float* __restrict__ A, int64_t lda, int ta,
                                               const float* __restrict__ B, int64_t ldb, int tb,
                                               float beta, float* __restrict__ C, int64_t ldc) {
    __shared__ float sa[16][64 + 4];
    __shared__ float sb[16][64 + 4];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += 16) {
        for (int i = threadIdx.x; i < 16 * 64; i += 256) {
            const int kk = i >> 6, mm = i & 63;
            const int gm = m0 + mm, gk = k0 + kk;
            float va = 0.f, vb = 0.f;
            if (gm < M && gk < K) va = ta ? A[static_cast<int64_t>(gk) * lda + gm] : A[static_cast<int64_t>(gm) * lda + gk];
            const int gn = n0 + mm;
            if (gn < N && gk < K) vb = tb ? B[static_cast<int64_t>(gn) * ldb + gk] : B[static_cast<int64_t>(gk) * ldb + gn];
            sa[kk][mm] = va;
            sb[kk][mm] = vb;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = sa[kk][ty * 4 + i];
                b[i] = sb[kk][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int gm = m0 + ty * 4 + i;
        if (gm >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int gn = n0 + tx * 4 + j;
            if (gn >= N) continue;
            float* c = C + static_cast<int64_t>(gm) * ldc + gn;
            *c = (beta == 0.f) ? alpha * acc[i][j] : fmaf(beta, *c, alpha * acc[i][j]);
        }
    }
}

// ------------------------------------------------------------------ adapter packing

// dst[rows_pad, cols_pad] (bf16) <- src[rows, cols] (dtype T, row stride ld) with zero padding;
// column block [col_off, col_off + cols) of dst when packing several adapters side by side.
template <typename T>
__global__ void k_pad_copy_bf16(const T* __restrict__ src, int64_t rows, int64_t cols, int64_t ld,
                                __nv_bfloat16* __restrict__ dst, int64_t rows_pad, int64_t ld_dst,
                                int64_t col_off, int64_t col_span) {
    griddep_enter();
    const int64_t n = rows_pad * col_span;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t rr = i / col_span, cc = i % col_span;
        float v = 0.f;
        if (rr < rows && cc < cols) v = to_f(src[rr * ld + cc]);
        dst[rr * ld_dst + col_off + cc] = __float2bfloat16_rn(v);
    }
}

// fp32 version (used by the fp32 batched path)
__global__ void k_pad_copy_f32(const float* __restrict__ src, int64_t rows, int64_t cols,
                               int64_t ld, float* __restrict__ dst, int64_t rows_pad,
                               int64_t ld_dst, int64_t col_off, int64_t col_span) {
    const int64_t n = rows_pad * col_span;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t rr = i / col_span, cc = i % col_span;
        dst[rr * ld_dst + col_off + cc] = (rr < rows && cc < cols) ? src[rr * ld + cc] : 0.f;
    }
}

// ------------------------------------------------------------------ split-K finalizers

// Sum the fp32 partials P[z][t][j] (z < split, j < RP) in fixed order z = 0, 1, ...
// and emit, for j < r (zero for r <= j < RP):
//   out_raw   [t, r]  (dtype To, nullable): the unscaled sum      (U = X A^T for the save)
//   out_pad   [t, RP] (bf16, nullable):     the unscaled sum      (U for the dB contraction)
//   out_spad  [t, RP] (bf16, nullable):     scale * sum           (sU / sG for K-extension)
template <typename To>
__global__ void k_finalize_rows(const float* __restrict__ P, int split, int64_t split_stride,
                                int64_t T, int r, int RP, float scale, To* __restrict__ out_raw,
                                __nv_bfloat16* __restrict__ out_pad,
                                __nv_bfloat16* __restrict__ out_spad) {
    griddep_enter();
    const int64_t n = T * RP;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t t = i / RP;
        const int j = static_cast<int>(i % RP);
        float acc = 0.f;
        if (j < r)
            for (int zz = 0; zz < split; ++zz) acc += P[zz * split_stride + i];
        if (out_raw && j < r) {
            if constexpr (sizeof(To) == 4) out_raw[t * r + j] = acc;
            else out_raw[t * r + j] = __float2bfloat16_rn(acc);
        }
        if (out_pad) out_pad[i] = __float2bfloat16_rn(acc);
        if (out_spad) out_spad[i] = __float2bfloat16_rn(scale * acc);
    }
}

// Multi-adapter U: P[z][t][j] summed; column j belongs to adapter seg_of[j]; the value is
// kept (times that adapter's scale) only when it is token t's adapter, else 0.
struct SegTable {
    int32_t seg_of[128];
    float scale[32];
};

__global__ void k_finalize_multi(const float* __restrict__ P, int split, int64_t split_stride,
                                 int64_t T, int RP, int n_adapters, const int32_t* __restrict__ ids,
                                 SegTable seg, __nv_bfloat16* __restrict__ out_bf,
                                 float* __restrict__ out_f32, int* err) {
    griddep_enter();
    const int64_t n = T * RP;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t t = i / RP;
        const int j = static_cast<int>(i % RP);
        const int id = ids[t];
        if (j == 0 && (id < 0 || id >= n_adapters)) set_error(err, kErrDevice);
        const int a = seg.seg_of[j];
        float v = 0.f;
        if (a >= 0 && a == id) {
            float acc = 0.f;
            for (int zz = 0; zz < split; ++zz) acc += P[zz * split_stride + i];
            v = seg.scale[a] * acc;
        }
        if (out_bf) out_bf[i] = __float2bfloat16_rn(v);
        if (out_f32) out_f32[i] = v;
    }
}

// dA[j, n] = sum_z P[z][n][j]  (the dA GEMM computes dA^T tiles), j < r.
__global__ void k_finalize_dA(const float* __restrict__ P, int split, int64_t split_stride,
                              int64_t d_in, int r, int RP, float* __restrict__ dA, int accumulate) {
    griddep_enter();
    const int64_t n = static_cast<int64_t>(r) * d_in;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t j = i / d_in, col = i % d_in;
        float acc = 0.f;
        for (int zz = 0; zz < split; ++zz) acc += P[zz * split_stride + col * RP + j];
        dA[i] = accumulate ? dA[i] + acc : acc;
    }
}

// dB[i, j] = scale * sum_z P[z][i][j], j < r.
__global__ void k_finalize_dB(const float* __restrict__ P, int split, int64_t split_stride,
                              int64_t d_out, int r, int RP, float scale, float* __restrict__ dB,
                              int accumulate) {
    griddep_enter();
    const int64_t n = d_out * r;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = i / r;
        const int j = static_cast<int>(i % r);
        float acc = 0.f;
        for (int zz = 0; zz < split; ++zz) acc += P[zz * split_stride + row * RP + j];
        dB[i] = accumulate ? dB[i] + scale * acc : scale * acc;
    }
}

// Mid-size forward finalize: H = bf16(sum_z P[z]) over the split-K partials in z order (the
// adapter term is already in the last split's partial).
__global__ void k_finalize_mid(const float* __restrict__ P, int split, int64_t n_el,
                               __nv_bfloat16* __restrict__ H) {
    griddep_enter();
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_el;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float acc = 0.f;
        for (int z = 0; z < split; ++z) acc += P[z * n_el + i];
        H[i] = __float2bfloat16_rn(acc);
    }
}

// Concatenated adapters of the multi-adapter forward, built in one pass:
//   a_cat [RP, d_in]:  row j = row (j - off_i) of A_i for the adapter i holding column j, 0 for j >= R
//   b_cat [d_out, RP]: column j = column (j - off_i) of B_i, 0 for j >= R
struct CatTable {
    const __nv_bfloat16* A[32];
    const __nv_bfloat16* B[32];
    int32_t r[32];
    int32_t off[32];
    int8_t seg_of[128];      // adapter of concatenated column j, -1 beyond R
};

__global__ void k_concat_adapters(CatTable tab, int64_t d_out, int64_t d_in, int RP,
                                  __nv_bfloat16* __restrict__ a_cat,
                                  __nv_bfloat16* __restrict__ b_cat) {
    griddep_enter();
    const int64_t na = static_cast<int64_t>(RP) * (d_in / 8);      // 16-byte vectors of a_cat
    const int64_t nb = d_out * RP;                                  // elements of b_cat
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < na + nb;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        if (i < na) {
            const int j = static_cast<int>(i / (d_in / 8));
            const int64_t c = (i % (d_in / 8)) * 8;
            const int a = tab.seg_of[j];
            uint4 v = make_uint4(0, 0, 0, 0);
            if (a >= 0)
                v = *reinterpret_cast<const uint4*>(tab.A[a] + static_cast<int64_t>(j - tab.off[a]) * d_in + c);
            *reinterpret_cast<uint4*>(a_cat + static_cast<int64_t>(j) * d_in + c) = v;
        } else {
            const int64_t e = i - na;
            const int64_t n = e / RP;
            const int j = static_cast<int>(e % RP);
            const int a = tab.seg_of[j];
            b_cat[e] = a >= 0 ? tab.B[a][n * tab.r[a] + (j - tab.off[a])] : __float2bfloat16_rn(0.f);
        }
    }
}

// Zero columns of U_all[t, :] that do not belong to token t's adapter and scale the rest
// (fp32 batched path).
__global__ void k_mask_multi_f32(float* __restrict__ U, int64_t T, int R, int n_adapters,
                                 const int32_t* __restrict__ ids, SegTable seg, int* err) {
    const int64_t n = T * R;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t t = i / R;
        const int j = static_cast<int>(i % R);
        const int id = ids[t];
        if (j == 0 && (id < 0 || id >= n_adapters)) set_error(err, kErrDevice);
        const int a = seg.seg_of[j];
        U[i] = (a >= 0 && a == id) ? seg.scale[a] * U[i] : 0.f;
    }
}

// ------------------------------------------------------------------ merge

// W_final[n, kk] = W^[n, kk] + s * sum_j B[n, j] A[j, kk]; W^ is the decoded weight in the
// output dtype's decode (bf16 decode for bf16 output).  Tile: 64 rows x 128 columns, 256
// threads; thread (tx, ty) owns columns 2tx, 2tx+1 (one code byte per row) of rows
// 16ty .. 16ty+15.  The A tile is staged in shared memory in fp32 and read 16 adapter rows
// at a time into registers, the B rows are read as 4-wide broadcasts, so the products run at
// FMA rate; each element's sum over j is formed in j order (fp32 FMA), as before.  The level
// table sits in shared memory (a lookup by code would serialise in the constant cache).
template <typename TA, typename TOut>
__global__ void __launch_bounds__(256) k_merge(const uint8_t* __restrict__ codes,
                                               const uint8_t* __restrict__ absmax_q,
                                               const float* __restrict__ c2, int64_t d_out,
                                               int64_t d_in, const TA* __restrict__ A,
                                               const TA* __restrict__ B, int r, float s,
                                               TOut* __restrict__ out) {
    extern __shared__ float msm[];
    const int rp = (r + 15) & ~15;   // adapter rank padded to 16
    float* sA = msm;                 // [rp][128]
    float* sB = msm + rp * 128;      // [64][rp]
    __shared__ float sscale[64][2];
    __shared__ float s_lv[16];
    const int64_t row0 = static_cast<int64_t>(blockIdx.y) * 64;
    const int64_t col0 = static_cast<int64_t>(blockIdx.x) * 128;
    const int tid = threadIdx.x;
    if (tid < 16) s_lv[tid] = c_nf4_levels[tid];
    for (int i = tid; i < rp * 128; i += 256) {
        const int jj = i / 128, c = i % 128;
        const int64_t gc = col0 + c;
        sA[i] = (jj < r && gc < d_in) ? to_f(A[jj * d_in + gc]) : 0.f;
    }
    for (int i = tid; i < 64 * rp; i += 256) {
        const int rr = i / rp, jj = i % rp;
        const int64_t gr = row0 + rr;
        sB[i] = (jj < r && gr < d_out) ? to_f(B[gr * r + jj]) : 0.f;
    }
    if (tid < 128) {
        const int rr = tid >> 1, cb = tid & 1;
        const int64_t gr = row0 + rr, gcb = col0 / 64 + cb;
        float sc = 0.f;
        if (gr < d_out && gcb < d_in / 64) {
            const int64_t blk = gr * (d_in / 64) + gcb;
            sc = nf4_block_scale(absmax_q[blk], c2[blk / kGroup]);
        }
        sscale[rr][cb] = sc;
    }
    __syncthreads();
    const int tx = tid & 63, ty = tid >> 6;
    const int64_t gc = col0 + 2 * tx;
    if (gc >= d_in) return;
    float acc[16][2];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = 0.f;
    for (int j0 = 0; j0 < rp; j0 += 16) {
        float2 a[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) a[jj] = *reinterpret_cast<const float2*>(sA + (j0 + jj) * 128 + 2 * tx);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float* brow = sB + (16 * ty + i) * rp + j0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 b4 = *reinterpret_cast<const float4*>(brow + 4 * q);
                const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc[i][0] = fmaf(bv[e], a[4 * q + e].x, acc[i][0]);
                    acc[i][1] = fmaf(bv[e], a[4 * q + e].y, acc[i][1]);
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int rr = 16 * ty + i;
        const int64_t gr = row0 + rr;
        if (gr >= d_out) continue;
        const int64_t e = gr * d_in + gc;
        const uint32_t byte = codes[e >> 1];
        const float sc = sscale[rr][tx >> 5];
        float w0 = __fmul_rn(s_lv[byte & 15u], sc), w1 = __fmul_rn(s_lv[byte >> 4], sc);
        if constexpr (sizeof(TOut) == 2) {
            w0 = __bfloat162float(__float2bfloat16_rn(w0));
            w1 = __bfloat162float(__float2bfloat16_rn(w1));
        }
        const float v0 = w0 + s * acc[i][0], v1 = w1 + s * acc[i][1];
        if constexpr (sizeof(TOut) == 2) {
            *reinterpret_cast<__nv_bfloat162*>(out + e) = __floats2bfloat162_rn(v0, v1);
        } else {
            *reinterpret_cast<float2*>(out + e) = make_float2(v0, v1);
        }
    }
}

}  // namespace qlora

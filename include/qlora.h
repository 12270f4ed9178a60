/*
 * qlora.h -- C ABI of libqlora: the QLoRA-adapted linear layer on NVIDIA B200 (sm_100a).
 *
 * The frozen base weight W0[d_out, d_in] is stored as 4-bit NormalFloat codes in blocks of
 * 64 weights, each block's absmax double-quantized to uint8 in groups of 256 blocks with one
 * fp32 second-level constant per group.  The layer computes
 *     h = W0 x + (alpha/r) B (A x)
 * with W0 dequantized on the fly to bf16 inside the tensor-core GEMM, its backward pass, the
 * adapter merge, multi-adapter forwards over one shared base (a few adapters, or thousands of
 * mixed-rank adapters), DoRA's forward and backward, the adapter optimizer step (AdamW, gradient
 * accumulation, paged state), and the forward and backward with FP8 (E4M3 / E5M2) activations
 * and gradients on FP8 tensor cores.
 *
 * Sources of each definition (page title, then section):
 *  [MF]  "Low-Rank Adaptation (LoRA) and QLoRA: Mathematical Foundations, Intrinsic Rank
 *        Dynamics, NF4 Quantization, and Parameter-Efficient Fine-Tuning" (llms.blog)
 *  [CH]  "Large Language Model Fine-tuning and LoRA" (aicomputerinstitute.com)
 *  [UH]  "LoRA and QLoRA Fine-Tuning Under the Hood" (codingpancake.com)
 *  [L26] "Lesson 26: LoRA/QLoRA Theory" (teology.holyping.network)
 *
 * Conventions for every entry point
 *  - Layout: row-major, contiguous.  X[T, d_in], H[T, d_out], dH[T, d_out], dX[T, d_in],
 *    A[r, d_in], B[d_out, r], dA[r, d_in], dB[d_out, r].
 *  - Memory: every tensor argument is caller-allocated DEVICE memory unless marked "host";
 *    the library never allocates or frees device memory and never synchronises the host,
 *    except qlora_get_device_error().  All work is enqueued on the given stream.
 *  - Alignment: device pointers must be 16-byte aligned, else QLORA_ERR_INVALID_ARG.
 *  - Shapes: d_in % 64 == 0 (a block never straddles rows), d_out >= 1 (any value: ragged last
 *    rows are masked, and a backward whose dH rows are not whole 16-byte units copies dH into
 *    padded rows first), T >= 1, 1 <= r <= 128; otherwise QLORA_ERR_UNSUPPORTED.  The FP8
 *    backward alone needs d_out % 16 == 0 (its E5M2 gradient rows are read by a tensor map).
 *  - dtype: QLORA_BF16 or QLORA_F32 sets X, H, dH, dX, A and B.  dA and dB are always fp32 and
 *    are overwritten (not accumulated).  The fp32 path is exact fp32 arithmetic (no TF32).
 *  - Errors found on the host return at once and nothing is launched.  Errors found on the
 *    device (an adapter id out of range, a pipeline wait that ran past its time limit) set a
 *    device error word that the next qlora_get_device_error() returns and clears.
 *  - Workspace: calls that take (ws, ws_bytes) need at least qlora_workspace_bytes(...) bytes
 *    of device scratch, 256-byte aligned; contents need not be initialised and are clobbered.
 *  - The device error word's address is looked up again on every call made outside stream
 *    capture (so a context re-created after cudaDeviceReset is followed) and cached per device
 *    for calls made while the stream is captured: the first call on a device must precede any
 *    capture.
 */
#ifndef QLORA_H_
#define QLORA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QLORA_OK = 0,
    QLORA_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad dtype, short workspace */
    QLORA_ERR_UNSUPPORTED = 2,   /* shape outside the supported set (see conventions)    */
    QLORA_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed                    */
    QLORA_ERR_TIMEOUT = 4,       /* a device pipeline wait exceeded its time limit       */
    QLORA_ERR_DEVICE = 5         /* device-detected bad input (adapter id out of range)  */
} qlora_status;

typedef enum { QLORA_F32 = 0, QLORA_BF16 = 1 } qlora_dtype;

typedef enum {
    QLORA_OP_FWD = 0, QLORA_OP_BWD = 1, QLORA_OP_FWD_BATCHED = 2, QLORA_OP_MERGE = 3,
    QLORA_OP_FWD_MULTI = 4, QLORA_OP_DORA_FWD = 5, QLORA_OP_FWD_FP8 = 6, QLORA_OP_FP8_QUANT = 7,
    QLORA_OP_BWD_FP8 = 8, QLORA_OP_DORA_BWD = 9
} qlora_op;

/* Stored NF4 weight.  Block size 64 and group size 256 are fixed.
 *   codes    [d_out, d_in/2] bytes: element 2j in the low nibble of byte j, 2j+1 in the high.
 *   absmax_q [d_out*d_in/64] uint8: q8 = rint(fl32(fl32(c1/c2)*127)), c1 = block absmax.
 *   c2       [ceil(d_out*d_in/64/256)] fp32: max of each group of 256 consecutive c1.
 * Blocks are 64 consecutive row-major elements; groups are 256 consecutive blocks.
 * [MF] "QLoRA: 4-Bit NormalFloat and Memory Optimization", "1. 4-bit NormalFloat (NF4)
 * Quantization" and "2. Double Quantization (DQ)"; [CH] "Quantizing the frozen weights: NF4
 * and double quantization" (block 64, 256 constants per second-level block).                */
typedef struct {
    const uint8_t* codes;
    const uint8_t* absmax_q;
    const float*   c2;
    int64_t        d_out;
    int64_t        d_in;
} qlora_nf4;

/* Byte sizes of the three NF4 buffers for a [d_out, d_in] weight (host-only, no GPU call).
 * d_out*d_in/2, d_out*d_in/64 and 4*ceil(d_out*d_in/16384): 4.127 bits per weight as in
 * [CH] "Quantizing the frozen weights".  UNSUPPORTED if d_in % 64 != 0.                       */
qlora_status qlora_nf4_sizes(int64_t d_out, int64_t d_in,
                             size_t* codes_bytes, size_t* absmax_bytes, size_t* c2_bytes);

/* The 16 NF4 levels L[0..15] the kernels decode with (host copy, no GPU call): quantile
 * midpoints of 16 equal-probability bins of N(0,1), normalised to [-1, 1]
 * ([MF] "1. 4-bit NormalFloat (NF4) Quantization", q_i equation).  out: host float[16].   */
qlora_status qlora_nf4_levels(float* out);

/* Quantize W[d_out, d_in] (fp32 or bf16, device) into the NF4 + double-quant format.
 * Per block: c1 = max|w|, x = fl32(w/c1), code = nearest level (ties to the upper level);
 * per group: c2 = max c1, q8 as above.  Bit-exact, deterministic.
 * [MF] "1. 4-bit NormalFloat (NF4) Quantization" steps 1-3 and "2. Double Quantization (DQ)".
 * Outputs are device buffers of the sizes from qlora_nf4_sizes().                            */
qlora_status nf4_quantize(const void* W, qlora_dtype w_dtype, int64_t d_out, int64_t d_in,
                          uint8_t* codes, uint8_t* absmax_q, float* c2, cudaStream_t stream);

/* Decode the stored weight to W_out[d_out, d_in] (device): fp32 w = fl32(L[code] * s_b) with
 * s_b = fl32(fl32(q8*c2)/127); bf16 output is the round-to-nearest-even of that fp32 value.
 * Bit-exact.  [MF] "1. 4-bit NormalFloat (NF4) Quantization" (dequantized to BF16 before the
 * matrix multiplication); [CH] "Quantizing the frozen weights" (compute in bf16).           */
qlora_status nf4_dequantize(const qlora_nf4* w, void* W_out, qlora_dtype out_dtype,
                            cudaStream_t stream);

/* Scratch bytes needed by an operation (host-only).  op is a qlora_op, dtype the call's dtype;
 * r_total is r for the single-adapter calls, the sum of ranks for QLORA_OP_FWD_BATCHED and
 * the largest rank for QLORA_OP_FWD_MULTI.
 * Returns 0 for an unsupported combination.                                                  */
size_t qlora_workspace_bytes(int op, qlora_dtype dtype, int64_t T, int64_t d_out, int64_t d_in,
                             int32_t r_total);

/* Forward: H = X W^T + (alpha/r) (X A^T) B^T, with W = the decoded weight (bf16 when dtype is
 * QLORA_BF16, fp32 when QLORA_F32).  [MF] "Intrinsic Dimensionality and Low-Rank Parameter
 * Dynamics" (h = W0 x + (alpha/r) B A x); [L26] "2. LoRA", "The Decomposition".
 *   X [T, d_in], A [r, d_in], B [d_out, r] in dtype; H [T, d_out] out in dtype.
 *   U_save (nullable) [T, r] in dtype receives U = X A^T (unscaled) for the backward call.   */
qlora_status qlora_linear_fwd(const qlora_nf4* w, const void* X, int64_t T,
                              const void* A, const void* B, int32_t r, float alpha,
                              qlora_dtype dtype, void* H, void* U_save,
                              void* ws, size_t ws_bytes, cudaStream_t stream);

/* Backward for upstream dH[T, d_out]:
 *   dX = dH W + s (dH B) A,   dA = s (dH B)^T X,   dB = s dH^T (X A^T),   s = alpha/r.
 * [MF] "Gradient Dynamics and Backpropagation Mechanics" (all three equations, alpha/r kept);
 * W0 is read only by the dX GEMM and no dW0 is formed ([MF], same section; [CH] "Correcting a
 * common misconception").  U_saved (nullable) is the U from the forward call, else it is
 * recomputed.  dX (nullable: skipped) in dtype; dA [r, d_in], dB [d_out, r] fp32.            */
qlora_status qlora_linear_bwd(const qlora_nf4* w, const void* X, const void* dH, int64_t T,
                              const void* A, const void* B, int32_t r, float alpha,
                              const void* U_saved, qlora_dtype dtype, void* dX,
                              float* dA, float* dB, void* ws, size_t ws_bytes,
                              cudaStream_t stream);

/* qlora_linear_bwd with flags.  QLORA_BWD_ACCUMULATE adds the call's dA, dB into the caller's
 * buffers (dA += ..., dB += ...) instead of overwriting them: gradient accumulation over
 * micro-batches before one optimizer update ([UH], the gradient-accumulation paragraph next to
 * FlashAttention-2).  dX is always overwritten.  Unknown flag bits: QLORA_ERR_INVALID_ARG.    */
#define QLORA_BWD_ACCUMULATE 1u
/* The backward in two calls, so that a data-parallel caller can reduce dA and dB over ranks
 * while dX is computed ([MF] "Gradient Dynamics and Backpropagation Mechanics": dA and dB are
 * sums over tokens, dX is per token).  QLORA_BWD_GRADS_ONLY computes G, dA and dB (dX is
 * ignored and may be NULL) and leaves bf16(s G) in the workspace; QLORA_BWD_DX_FROM_WS then
 * computes dX only (dA, dB ignored, may be NULL; dX required), reading that bf16(s G) from the
 * same workspace, which the caller must not have reused in between, with the same w, dH, T, A,
 * B, r, alpha and dtype.  The pair gives results identical to one call.  Both bits together:
 * QLORA_ERR_INVALID_ARG. */
#define QLORA_BWD_GRADS_ONLY 2u
#define QLORA_BWD_DX_FROM_WS 4u
qlora_status qlora_linear_bwd_ex(const qlora_nf4* w, const void* X, const void* dH, int64_t T,
                                 const void* A, const void* B, int32_t r, float alpha,
                                 const void* U_saved, qlora_dtype dtype, void* dX,
                                 float* dA, float* dB, void* ws, size_t ws_bytes,
                                 uint32_t flags, cudaStream_t stream);

/* One AdamW step of an adapter tensor of n elements (decoupled weight decay):
 *   g' = grad_scale g;  m = beta1 m + (1 - beta1) g';  v = beta2 v + (1 - beta2) g'^2;
 *   w  = w (1 - lr weight_decay) - lr (m / (1 - beta1^step)) / (sqrt(v / (1 - beta2^step)) + eps)
 * in fp32, step counted from 1; grad_scale = 1 / micro-batches for accumulated gradients.
 * [MF] "The Memory Bottleneck of Full Parameter Fine-Tuning" (AdamW state: fp32 master, m, v);
 * the pages print no update rule, this is the published AdamW (reading R23).
 *   param   bf16 (then master, fp32 [n], is the weight and param gets its RN-even copy) or
 *           fp32 (updated in place; master must be NULL or equal to param)
 *   grad, m, v  fp32 [n]; m, v updated in place.  Any of the fp32 arrays may be unified
 *           memory (the "paged optimizer" state; see qlora_prefetch).
 * 16-byte aligned arrays with n % 4 == 0 take the vector path.  No allocation; asynchronous.  */
qlora_status qlora_adamw_step(void* param, qlora_dtype param_dtype, float* master,
                              const float* grad, float* m, float* v, int64_t n, int32_t step,
                              float lr, float beta1, float beta2, float eps, float weight_decay,
                              float grad_scale, cudaStream_t stream);

/* Page a caller-allocated unified-memory range (cudaMallocManaged) of optimizer state to the
 * current device (to_device != 0) before a step, or back to host memory after it, so that the
 * state occupies HBM only while it is used: [CH] "Paged optimizers", [MF] "3. Paged
 * Optimizers", [L26] "Paged Optimizers" (optimizer state in unified memory, paged between GPU
 * and CPU).  Asynchronous on `stream`; the library allocates nothing.                         */
qlora_status qlora_prefetch(const void* ptr, size_t bytes, int32_t to_device, cudaStream_t stream);

/* Merge: W_final = W + (alpha/r) B A, dense (not re-quantized), out_dtype fp32 or bf16;
 * W is the decoded weight in out_dtype's decode.  A, B are given in adapter_dtype.
 * [MF] "Production Serving and Multi-Tenant Routing", "1. Static Weight Merging";
 * [CH] "Merging adapters vs keeping them separate".                                          */
qlora_status lora_merge(const qlora_nf4* w, const void* A, const void* B, int32_t r,
                        float alpha, qlora_dtype adapter_dtype, qlora_dtype out_dtype,
                        void* W_final, cudaStream_t stream);

/* Multi-adapter forward over one shared base:
 *   H[t] = X[t] W^T + s_i (X[t] A_i^T) B_i^T,  i = adapter_id[t],  s_i = alpha[i]/r[i].
 * The base GEMM is shared by all tokens.  [CH] "Serving many adapters at once: the
 * multi-tenant problem"; [MF] "2. Multi-Tenant Dynamic Multiplexing"; [UH] "6.2 Multi-Adapter
 * Serving at Scale".  adapter_id: device int32[T]; A, B: HOST arrays of n_adapters device
 * pointers (A_i [r_i, d_in], B_i [d_out, r_i]); r, alpha: HOST arrays.  sum(r) <= 128,
 * n_adapters <= 32.  An id outside [0, n_adapters) contributes no adapter term for that token
 * and sets QLORA_ERR_DEVICE in the device error word.                                         */
qlora_status qlora_linear_fwd_batched(const qlora_nf4* w, const void* X, int64_t T,
                                      const int32_t* adapter_id, int32_t n_adapters,
                                      const void* const* A, const void* const* B,
                                      const int32_t* r, const float* alpha, qlora_dtype dtype,
                                      void* H, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Multi-adapter forward for many adapters (bf16), the same result as qlora_linear_fwd_batched
 * without its limits on the number and total rank of the adapters:
 *   H[t] = X[t] W^T + s_i (X[t] A_i^T) B_i^T,  i = adapter_id[t].
 * [CH] "Serving many adapters at once: the multi-tenant problem" (the shared x W once per
 * batch, each request's correction by grouped kernels over adapters of different ranks);
 * [UH] "6.2 Multi-Adapter Serving at Scale (S-LoRA & Punica)" (thousands of adapters over one
 * base).  The base term is the fused NF4 GEMM without adapter steps, rounded to bf16 into H;
 * the tokens are sorted by adapter on the device and each adapter's segment gets
 * U = bf16(s_i X A_i^T) and H = bf16(H + U B_i^T), fp32 accumulation.
 *   adapter_id  device int32 [T]
 *   A_ptrs      DEVICE array of n_adapters device pointers, A_i bf16 [r_i, d_in], 16-byte
 *               aligned (its rows then are too: d_in % 64 == 0 is already required)
 *   B_ptrs      DEVICE array of n_adapters device pointers, B_i bf16 [d_out, r_i]
 *   ranks       DEVICE int32 [n_adapters], 1 <= r_i <= r_max
 *   alphas      DEVICE float [n_adapters], alpha_i; the library forms s_i = alpha_i / r_i
 *               (IEEE fp32 division on the device, the same value the single-adapter calls use)
 *   r_max       host: the largest rank, 1..128; ws >= qlora_workspace_bytes(QLORA_OP_FWD_MULTI,
 *               QLORA_BF16, T, d_out, d_in, r_max)
 * 1 <= n_adapters <= 65536.  An id outside [0, n_adapters), or an adapter whose rank is
 * outside [1, r_max] or whose A_i is not 16-byte aligned, contributes no adapter term and sets
 * QLORA_ERR_DEVICE in the device error word.                                                 */
qlora_status qlora_linear_fwd_multi(const qlora_nf4* w, const void* X, int64_t T,
                                    const int32_t* adapter_id, int32_t n_adapters,
                                    const void* const* A_ptrs, const void* const* B_ptrs,
                                    const int32_t* ranks, const float* alphas, int32_t r_max,
                                    void* H, void* ws, size_t ws_bytes, cudaStream_t stream);

/* DoRA (bf16): one magnitude per output row, each row of the adapted weight W + s B A divided
 * by its Euclidean norm ([CH] "Choosing what to adapt": a magnitude vector of size d_out trained
 * directly, the low-rank update on the direction; [MF] "Advanced Variants: DoRA and LoRA+",
 * W = m (V + dW) / ||V + dW||; reading R24).  With per-row norms n_j = ||(W^ + s B A)[j, :]||_2:
 *   H[t, j] = (m_j / n_j) (X[t] W^T + s U[t] B^T)[j]        (a row of norm 0 gives 0)
 * W^ is the bf16 decode.  magnitude: device fp32 [d_out].  The norms are recomputed every call
 * (they depend on A, B) by the tensor-core merge tile in a row-norm mode, then the large-T
 * fused forward applies m / n to each output column before rounding.  U_save as in
 * qlora_linear_fwd.  ws >= qlora_workspace_bytes(QLORA_OP_DORA_FWD, QLORA_BF16, T, d_out,
 * d_in, r).  The backward is qlora_dora_bwd.                                                  */
qlora_status qlora_dora_fwd(const qlora_nf4* w, const void* X, int64_t T, const void* A,
                            const void* B, int32_t r, float alpha, const float* magnitude,
                            void* H, void* U_save, void* ws, size_t ws_bytes, cudaStream_t stream);

/* DoRA backward (bf16): the gradients of the DoRA forward above for the upstream gradient dH,
 * by the chain rule through every factor of H = Z diag(c), Z = X V^T, V = W^ + s B A,
 * c_j = m_j / n_j, n_j = ||V[j, :]||_2 -- the norm included (the pages give the forward only;
 * the derivative of the Euclidean norm is V[j, :] / n_j):
 *   dZ = dH diag(c),  dc_j = sum_t dH[t, j] Z[t, j],  dm_j = dc_j / n_j,  e_j = -dc_j m_j / n_j^3
 *   dX = dZ V,  dA = s B^T (dZ^T X + diag(e) V),  dB = s (dZ^T X + diag(e) V) A^T
 * A row of norm 0 contributes nothing.  The library recomputes n and Z (a large-T forward;
 * qlora_dora_bwd_saved takes them from qlora_dora_fwd_save instead), runs
 * the LoRA backward on dZ and adds the norm's term through two passes over the weight with the
 * adapter rows as tokens (A W^T and B^T diag(e) W^ on the fused NF4 GEMM) and r x r products.
 * [CH] "Choosing what to adapt: targets and rank"; [MF] "Advanced Variants: DoRA and LoRA+";
 * [MF] "Gradient Dynamics and Backpropagation Mechanics" (the LoRA part).
 *   X [T, d_in], dH [T, d_out], A, B bf16; magnitude fp32 [d_out]; dX (nullable) bf16 [T, d_in];
 *   dA fp32 [r, d_in], dB fp32 [d_out, r], dm fp32 [d_out], all overwritten.
 *   ws >= qlora_workspace_bytes(QLORA_OP_DORA_BWD, QLORA_BF16, T, d_out, d_in, r).            */
qlora_status qlora_dora_bwd(const qlora_nf4* w, const void* X, const void* dH, int64_t T,
                            const void* A, const void* B, int32_t r, float alpha,
                            const float* magnitude, void* dX, float* dA, float* dB, float* dm,
                            void* ws, size_t ws_bytes, cudaStream_t stream);

/* DoRA forward for training: the layer of qlora_dora_fwd that also keeps what its backward needs,
 * so that qlora_dora_bwd_saved does not recompute it.  It writes the row norms n (norms_save,
 * device fp32 [d_out]), the pre-scale output Z = X W^T + s U B^T (Z_save, bf16 [T, d_out], from
 * the large-T kernels whatever T), U (U_save, bf16 [T, r], required) and
 * H[t, j] = bf16(Z[t, j] (m_j / n_j)) (0 where n_j = 0) -- Z rounded to bf16 before the scale,
 * where qlora_dora_fwd scales the fp32 accumulator (one bf16 rounding more: a relative 2^-9;
 * reading R28).
 * Same sources, readings and ws size as qlora_dora_fwd.                                        */
qlora_status qlora_dora_fwd_save(const qlora_nf4* w, const void* X, int64_t T, const void* A,
                                 const void* B, int32_t r, float alpha, const float* magnitude,
                                 void* H, void* Z_save, void* U_save, float* norms_save, void* ws,
                                 size_t ws_bytes, cudaStream_t stream);

/* qlora_dora_bwd from the Z, U and norms that qlora_dora_fwd_save wrote for the same w, X, A, B,
 * alpha (the caller keeps them unchanged in between): the same results as qlora_dora_bwd bit
 * for bit (which recomputes exactly these three), without the norm pass and the forward.
 * Z_saved bf16 [T, d_out], U_saved bf16 [T, r], norms_saved fp32 [d_out]; the rest as in
 * qlora_dora_bwd, the same ws size.                                                           */
qlora_status qlora_dora_bwd_saved(const qlora_nf4* w, const void* X, const void* dH, int64_t T,
                                  const void* A, const void* B, int32_t r, float alpha,
                                  const float* magnitude, const void* Z_saved, const void* U_saved,
                                  const float* norms_saved, void* dX, float* dA, float* dB, float* dm,
                                  void* ws, size_t ws_bytes, cudaStream_t stream);

/* The DoRA row norms n_j = ||(W^ + (alpha/r) B A)[j, :]||_2 (bf16 adapters, W^ the bf16 decode)
 * into norms (device fp32 [d_out]); DoRA initialises the magnitude to them.  ws holds at least
 * d_out * (d_in / 64) floats.                                                                 */
qlora_status qlora_dora_row_norms(const qlora_nf4* w, const void* A, const void* B, int32_t r,
                                  float alpha, float* norms, void* ws, size_t ws_bytes,
                                  cudaStream_t stream);

/* ---- FP8 activations ------------------------------------------------------------------------
 * [UH] "1.3 Activation Memory Savings via FlashAttention-2 & Activation Checkpointing": the
 * FP8 formats E4M3 / E5M2, native on Blackwell, halve the activation bytes.  E4M3 is the OCP
 * 8-bit float (sign, 4 exponent bits with bias 7, 3 mantissa bits; largest finite 448).  A
 * tensor is held as bytes X8 with one per-tensor scale sigma (device fp32 scalar) such that
 * X ~ E4M3value(X8) / sigma; sigma = 2^(8 - ceil(log2 max|X|)) (1 for an all-zero tensor).    */

/* X8[n] = E4M3(fl32(X[i] * sigma)) (round to nearest even, saturating) and *scale = sigma, for
 * a bf16 X of n >= 1 elements (device).  NaNs are ignored by the max.  Bit-exact.
 * ws >= qlora_workspace_bytes(QLORA_OP_FP8_QUANT, QLORA_BF16, 1, 1, 64, 1) (256 bytes).      */
qlora_status qlora_fp8_quantize(const void* X, int64_t n, uint8_t* X8, float* scale, void* ws,
                                size_t ws_bytes, cudaStream_t stream);

/* *w_scale (device fp32) = sigma_w = 2^(8 - ceil(log2 max c2)): every decoded weight
 * L[code] * s_b has |L| <= 1 and s_b <= c2 of its group, so sigma_w * |w| <= 256.            */
qlora_status qlora_fp8_weight_scale(const qlora_nf4* w, float* w_scale, cudaStream_t stream);

/* Forward with the E4M3 activation X8[T, d_in] (scale *x_scale) and the weight decoded to E4M3
 * inside the tensor-core GEMM (w8 = E4M3(fl32(L[code] * s_b) * sigma_w), sigma_w = *w_scale):
 *   H = bf16( (X8 W8^T) / (sigma_x sigma_w) + s (X~ A^T) B^T ),   X~ = X8 / sigma_x,  s = alpha/r,
 * the base product on kind::f8f6f4 tensor cores, the adapter term in bf16 (A, B bf16) added in
 * the same fp32 accumulator.  x_scale and w_scale are device scalars from qlora_fp8_quantize /
 * qlora_fp8_weight_scale (powers of two make every rescaling exact; other positive values are
 * accepted).  ws >= qlora_workspace_bytes(QLORA_OP_FWD_FP8, QLORA_BF16, T, d_out, d_in, r).
 * Forward only: no U is saved.                                                               */
qlora_status qlora_linear_fwd_fp8(const qlora_nf4* w, const uint8_t* X8, int64_t T,
                                  const float* x_scale, const float* w_scale, const void* A,
                                  const void* B, int32_t r, float alpha, void* H, void* ws,
                                  size_t ws_bytes, cudaStream_t stream);

/* dH8[n] = E5M2(fl32(dH[i] * sigma_g)) (round to nearest even, saturating at 57344) and
 * *scale = sigma_g = 2^(15 - ceil(log2 max|dH|)), for the bf16 upstream gradient of n >= 1
 * elements: the wider-range FP8 format of [UH] "1.3 ..." for gradients.  E5M2 is the OCP 8-bit
 * float with 5 exponent bits (bias 15) and 2 mantissa bits.  Bit-exact.  ws as for
 * qlora_fp8_quantize.                                                                          */
qlora_status qlora_fp8_quantize_grad(const void* dH, int64_t n, uint8_t* dH8, float* scale, void* ws,
                                     size_t ws_bytes, cudaStream_t stream);

/* Backward from the saved E4M3 activation X8 (scale *x_scale) and the E5M2 upstream gradient
 * dH8[T, d_out] (scale *g_scale), the three gradient equations of [MF] "Gradient Dynamics and
 * Backpropagation Mechanics" with X~ = X8 / sigma_x and dH~ = dH8 / sigma_g in place of X, dH:
 *   G = dH~ B,  dX = bf16( (dH8 W8) / (sigma_g sigma_w) + s G A ),  dA = s G^T X~,
 *   dB = s dH~^T (X~ A^T),
 * W8 the weight decoded to E4M3 as in qlora_linear_fwd_fp8.  dX's weight product runs on
 * kind::f8f6f4 tensor cores (E5M2 x E4M3); G, U, dA, dB on bf16 tensor cores from X~, dH~
 * (exact bf16 copies in the workspace).  dX bf16 (nullable: skipped), dA, dB fp32;
 * QLORA_BWD_ACCUMULATE adds into dA, dB.  Needs d_out % 16 == 0 (the E5M2 rows are d_out bytes
 * and are read by TMA), else QLORA_ERR_UNSUPPORTED with nothing launched.
 * ws >= qlora_workspace_bytes(QLORA_OP_BWD_FP8, QLORA_BF16, T, d_out, d_in, r).              */
qlora_status qlora_linear_bwd_fp8(const qlora_nf4* w, const uint8_t* X8, const float* x_scale,
                                  const uint8_t* dH8, const float* g_scale, const float* w_scale,
                                  int64_t T, const void* A, const void* B, int32_t r, float alpha,
                                  void* dX, float* dA, float* dB, void* ws, size_t ws_bytes,
                                  uint32_t flags, cudaStream_t stream);

/* Size of the device scratch array behind qlora_linear_fwd_noalloc (bytes per GPU). */
#define QLORA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/* qlora_linear_fwd without a workspace argument, for callers that cannot allocate device
 * memory (an engine that owns all device memory through its own pool, or a hot path that
 * must not take the allocator's locks) and have none to lend.  It allocates nothing: its
 * scratch is a fixed QLORA_NOALLOC_SCRATCH_BYTES device array inside the library, held by
 * every GPU that loads the library until the process exits.  The pages have no counterpart;
 * the computation and the other arguments are exactly those of qlora_linear_fwd.
 *   - QLORA_ERR_UNSUPPORTED, with nothing launched, when qlora_workspace_bytes(QLORA_OP_FWD,
 *     dtype, T, d_out, d_in, r) exceeds QLORA_NOALLOC_SCRATCH_BYTES.
 *   - Other errors are those of qlora_linear_fwd for the same arguments.
 *   - All calls share the array, which keeps the previous call's contents (the forward's
 *     kernels write every scratch byte before they read it); calls whose work overlaps on the
 *     GPU (two streams, two host threads) race on it.
 *   - The array's device address is looked up on every call made outside stream capture;
 *     during a capture the address from the last such call on the device is used, so the first
 *     call on a device must come before any stream capture.                                  */
qlora_status qlora_linear_fwd_noalloc(const qlora_nf4* w, const void* X, int64_t T,
                                      const void* A, const void* B, int32_t r, float alpha,
                                      qlora_dtype dtype, void* H, void* U_save,
                                      cudaStream_t stream);

/* Synchronise `stream`, then read and clear the device error word of the current device.
 * Returns QLORA_OK, QLORA_ERR_TIMEOUT, QLORA_ERR_DEVICE or QLORA_ERR_CUDA.                   */
qlora_status qlora_get_device_error(cudaStream_t stream);

/* Self-test of the bounded pipeline wait: launches one block that waits on a shared-memory
 * barrier nothing ever arrives on, for at most limit_ns nanoseconds, then gives up and sets
 * QLORA_ERR_TIMEOUT in the device error word.  The context stays usable.                     */
qlora_status qlora_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream);

/* Benchmark instrumentation: while both events are non-NULL, every launch of the fused NF4
 * GEMM kernel (forward or dX) records `start` right before and `stop` right after itself on
 * the call's stream.  Pass NULL, NULL to stop.  Not thread-safe.                             */
qlora_status qlora_set_gemm_events(cudaEvent_t start, cudaEvent_t stop);

/* Number of kernels this library has launched since it was loaded (all entry points). */
uint64_t qlora_launch_count(void);

/* Human-readable name of a status code (static string). */
const char* qlora_status_string(qlora_status s);

#ifdef __cplusplus
}
#endif
#endif /* QLORA_H_ */

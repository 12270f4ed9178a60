"""Plain, slow, obviously-correct CPU oracle for the QLoRA-adapted linear layer.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The product library never calls it and shares no code, table or
constant with it.

What it computes, and where each step is defined:

* NF4 level table -- "Low-Rank Adaptation (LoRA) and QLoRA: Mathematical
  Foundations, Intrinsic Rank Dynamics, NF4 Quantization, and
  Parameter-Efficient Fine-Tuning" (llms.blog), section "QLoRA: 4-Bit
  NormalFloat and Memory Optimization", subsection "1. 4-bit NormalFloat (NF4)
  Quantization", the q_i equation and the sentence on normalising to [-1, 1].
* Block-wise absmax quantization (block 64) -- same subsection, steps 1-3;
  block size from "Large Language Model Fine-tuning and LoRA"
  (aicomputerinstitute.com), section "Quantizing the frozen weights: NF4 and
  double quantization".
* Double quantization (8-bit absmax, groups of 256, fp32 second level) --
  Mathematical Foundations page, subsection "2. Double Quantization (DQ)",
  the c1^{8bit} = round(c1/c2 * 127) equation; same section of the
  Fine-tuning-and-LoRA page for the group size.
* Forward h = W0 x + (alpha/r) B A x -- Mathematical Foundations page,
  section "Intrinsic Dimensionality and Low-Rank Parameter Dynamics".
* Gradients dB, dA, dx -- Mathematical Foundations page, section "Gradient
  Dynamics and Backpropagation Mechanics" (all three equations, alpha/r kept).
* Merge W_final = W0 + (alpha/r) B A -- Mathematical Foundations page,
  section "Production Serving and Multi-Tenant Routing", "1. Static Weight
  Merging"; "Large Language Model Fine-tuning and LoRA", section "Merging
  adapters vs keeping them separate".
* Multi-adapter forward (shared x W0, per-request B_i A_i) -- "Large Language
  Model Fine-tuning and LoRA", section "Serving many adapters at once: the
  multi-tenant problem".
* DoRA forward -- "Large Language Model Fine-tuning and LoRA", section
  "Choosing what to adapt" (a magnitude vector of size d_out trained directly,
  the low-rank update applied to the direction); Mathematical Foundations
  page, section "Advanced Variants: DoRA and LoRA+" (W = m (V + dW) / ||V + dW||).
  Reading R24: one magnitude per output row, each row of W0 + s B A divided by
  its Euclidean norm.
* Adapter optimizer step: AdamW with an fp32 master copy, first moment m and
  second moment v per trainable parameter -- Mathematical Foundations page,
  section "The Memory Bottleneck of Full Parameter Fine-Tuning" (the AdamW
  state list); gradient accumulation over micro-batches before one update --
  "LoRA and QLoRA Fine-Tuning Under the Hood", section on gradient
  accumulation (next to the FlashAttention-2 paragraph).  The pages name AdamW
  but print no update rule; the oracle writes out the published decoupled
  weight-decay rule (reading R23).
* FP8 activations: E4M3 activations with a per-tensor scale, the decoded
  weight rounded to E4M3 for the one FP8 contraction -- "LoRA and QLoRA
  Fine-Tuning Under the Hood", section "1.3 Activation Memory Savings via
  FlashAttention-2 & Activation Checkpointing" (FP8 formats E4M3 and E5M2 for
  activations on Hopper and Blackwell).  The pages name the formats only; the
  byte layout is the OCP 8-bit floating-point definition and the scaling,
  rounding and operand choices are reading R25.
* FP8 backward: the E5M2 upstream gradient (same section's E5M2) and the
  saved E4M3 activation in the three gradient equations of the Mathematical
  Foundations page, section "Gradient Dynamics and Backpropagation Mechanics";
  reading R26.

Where the pages are silent or garbled the oracle takes a reading (numbered R1,
R2, ...); each is cited by its number, with the choice it makes, where it is
applied.

Parity unpinned: the absolute NF4 code values and the double-quantization
rounding order are conventions (R1, R5, R8, R10, R11) -- no page prints a
worked NF4 example, so the tests pin their properties, not their bits.

Row-major throughout: X[T, d_in], H[T, d_out], W0[d_out, d_in], A[r, d_in],
B[d_out, r].  Floating-point arithmetic is fp64 except where the storage format
fixes an fp32 decision (quantization codes, scale rebuild, decoded weight), in
which case the IEEE fp32 operations are written out with numpy float32.
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 64          # weights per absmax block
GROUP = 256         # absmax constants per second-level group
Q8_MAX = 127        # 8-bit code range of the first-level constants

# ----------------------------------------------------------------------------
# NF4 level table (reading R1)
# ----------------------------------------------------------------------------


def normal_cdf(x: float) -> float:
    """Standard normal CDF, Phi(x) = erfc(-x/sqrt 2)/2, from libm's erfc."""
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def normal_quantile(p: float) -> float:
    """Q(p) = Phi^{-1}(p) by Newton's method on Phi(x) - p (fp64).

    Newton from x = 0 converges monotonically on each side because Phi is
    convex left of 0 and concave right of it; 200 steps is far more than the
    handful needed for p in [1/18, 17/18].
    """
    if not 0.0 < p < 1.0:
        raise ValueError("p must lie in (0, 1)")
    x = 0.0
    for _ in range(200):
        pdf = math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)
        step = (normal_cdf(x) - p) / pdf
        x -= step
        if abs(step) < 1e-17 * max(1.0, abs(x)):
            break
    return x


def nf4_unnormalised_levels() -> np.ndarray:
    """The 16 quantile midpoints before normalisation (fp64), reading R1.

    The pages' q_i = (Q(i/2^k) + Q((i+1)/2^k)) / 2 is infinite for the two end
    bins.  Reading R1 keeps the same construction on interior plotting
    positions: edges p_j = j/18, j = 1..17, and q_i = (Q(p_{i+1}) + Q(p_{i+2}))/2
    for i = 0..15 -- 16 equal-probability bins' quantile midpoints.
    """
    edges = [normal_quantile(j / 18.0) for j in range(1, 18)]
    return np.array([0.5 * (edges[i] + edges[i + 1]) for i in range(16)],
                    dtype=np.float64)


def nf4_levels() -> np.ndarray:
    """NF4 levels L[0..15] (fp32), normalised by max |q| to span [-1, 1]."""
    q = nf4_unnormalised_levels()
    return (q / np.max(np.abs(q))).astype(np.float32)


def nf4_midpoints(levels: np.ndarray) -> np.ndarray:
    """Decision thresholds m_i = fl32((L_i + L_{i+1}) / 2), computed in fp64 (R5)."""
    L = levels.astype(np.float64)
    return ((L[:-1] + L[1:]) / 2.0).astype(np.float32)


# ----------------------------------------------------------------------------
# Sizes of the stored format
# ----------------------------------------------------------------------------


def nf4_sizes(d_out: int, d_in: int) -> tuple[int, int, int]:
    """Byte sizes (codes, absmax_q, c2) for a [d_out, d_in] weight.

    Two 4-bit codes per byte, one uint8 per 64-block, one fp32 per group of
    256 blocks (the last group may be partial, reading R2).
    """
    if d_in % BLOCK:
        raise ValueError("d_in must be a multiple of 64")
    n = d_out * d_in
    nblocks = n // BLOCK
    ngroups = -(-nblocks // GROUP)
    return n // 2, nblocks, 4 * ngroups


# ----------------------------------------------------------------------------
# Quantize / double-quantize / pack   (readings R2-R9)
# ----------------------------------------------------------------------------


def nf4_codes_of_normalised(xn: np.ndarray, mids: np.ndarray) -> np.ndarray:
    """Nearest-level code of normalised values: #{i : x >= m_i} (R5, ties up)."""
    return np.searchsorted(mids, xn, side="right").astype(np.uint8)


def nf4_quantize(W: np.ndarray, levels: np.ndarray | None = None):
    """Quantize fp32 W[d_out, d_in] -> (codes u8, absmax_q u8, c2 f32, c1 f32).

    Steps, in the pages' order:
      1. c1 = max |w| over each block of 64 consecutive row-major elements.
      2. x~ = fl32(w / c1) (IEEE fp32 division; x~ = 0 when c1 = 0, R4).
      3. code = nearest NF4 level (R5).
      4. c2 = max of each group of 256 consecutive c1 (R7).
      5. q8 = rint(fl32(fl32(c1 / c2) * 127)), clamped to [0, 127]; 0 if c2 = 0 (R6, R8).
      6. Pack: element 2j in the low nibble of byte j, 2j+1 in the high nibble (R3).
    c1 is returned too (it is not stored; tests use it for bounds).
    """
    W = np.ascontiguousarray(W, dtype=np.float32)
    d_out, d_in = W.shape
    if d_in % BLOCK:
        raise ValueError("d_in must be a multiple of 64")
    L = nf4_levels() if levels is None else levels
    mids = nf4_midpoints(L)

    blocks = W.reshape(-1, BLOCK)                                   # R2
    c1 = np.max(np.abs(blocks), axis=1).astype(np.float32)          # step 1
    safe = np.where(c1 > 0, c1, np.float32(1.0)).astype(np.float32)
    xn = (blocks / safe[:, None]).astype(np.float32)                # step 2 (fp32 /)
    xn = np.where(c1[:, None] > 0, xn, np.float32(0.0)).astype(np.float32)
    codes = nf4_codes_of_normalised(xn, mids).reshape(-1)          # step 3

    nblocks = c1.shape[0]
    ngroups = -(-nblocks // GROUP)
    pad = ngroups * GROUP - nblocks
    c1p = np.concatenate([c1, np.zeros(pad, np.float32)])
    c2 = np.max(c1p.reshape(ngroups, GROUP), axis=1).astype(np.float32)  # step 4
    c2_of_block = np.repeat(c2, GROUP)[:nblocks]
    c2safe = np.where(c2_of_block > 0, c2_of_block, np.float32(1.0)).astype(np.float32)
    ratio = (c1 / c2safe).astype(np.float32)                         # fl32(c1/c2)
    scaled = (ratio * np.float32(Q8_MAX)).astype(np.float32)          # fl32(. * 127)
    q8 = np.clip(np.rint(scaled), 0, Q8_MAX)                          # rint = half-even
    q8 = np.where(c2_of_block > 0, q8, 0).astype(np.uint8)            # step 5

    packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)     # step 6 (R3)
    return packed.reshape(d_out, d_in // 2), q8, c2, c1


def nf4_unpack(codes: np.ndarray) -> np.ndarray:
    """Inverse of the packing: flat array of 4-bit codes in element order."""
    c = np.ascontiguousarray(codes, dtype=np.uint8).reshape(-1)
    out = np.empty(c.size * 2, dtype=np.uint8)
    out[0::2] = c & 0x0F
    out[1::2] = c >> 4
    return out


def nf4_block_scales(absmax_q: np.ndarray, c2: np.ndarray) -> np.ndarray:
    """Rebuilt block scale s_b = fl32(fl32(q8 * c2) / 127) (R10)."""
    q8 = np.asarray(absmax_q, dtype=np.uint8).astype(np.float32)
    c2b = np.repeat(np.asarray(c2, np.float32), GROUP)[: q8.size]
    prod = (q8 * c2b).astype(np.float32)
    return (prod / np.float32(Q8_MAX)).astype(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round-to-nearest-even), returned as fp32.

    The plain definition on the bit pattern: add 0x7FFF plus the lowest kept
    bit, then truncate the low 16 bits.  (No NaN/Inf ever reaches it here.)
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32)


def nf4_dequantize(codes, absmax_q, c2, d_out: int, d_in: int,
                   out: str = "f32", levels: np.ndarray | None = None) -> np.ndarray:
    """Decoded weight W^[d_out, d_in] (R11).

    w32 = fl32(L[code] * s_b); out="bf16" returns RN-even bf16 of w32 (as fp32
    values), out="f32" returns w32.
    """
    L = nf4_levels() if levels is None else levels
    cf = nf4_unpack(codes)[: d_out * d_in]
    s = nf4_block_scales(absmax_q, c2)
    w32 = (L[cf].reshape(-1, BLOCK) * s[:, None]).astype(np.float32).reshape(d_out, d_in)
    if out == "f32":
        return w32
    if out == "bf16":
        return bf16_round(w32)
    raise ValueError(out)


# ----------------------------------------------------------------------------
# LoRA forward / backward / merge in fp64
# ----------------------------------------------------------------------------


def lora_scale(alpha: float, r: int) -> float:
    """s = alpha / r (fp64)."""
    return float(alpha) / float(r)


def lora_forward(W_hat, X, A, B, alpha, r):
    """H = X W^T + s (X A^T) B^T: the batched row form of h = W0 x + (alpha/r) B A x."""
    W_hat, X, A, B = (np.asarray(t, np.float64) for t in (W_hat, X, A, B))
    s = lora_scale(alpha, r)
    U = X @ A.T
    return X @ W_hat.T + s * (U @ B.T)


def lora_backward(W_hat, X, dH, A, B, alpha, r):
    """(dX, dA, dB) for upstream gradient dH[T, d_out].

    Row form of the page's three equations, summed over the T tokens:
      dB = s dH^T (X A^T),   dA = s B^T dH^T X = s (dH B)^T X,
      dX = dH (W0 + s B A)  = dH W^ + s (dH B) A            (R12, R13).
    """
    W_hat, X, dH, A, B = (np.asarray(t, np.float64) for t in (W_hat, X, dH, A, B))
    s = lora_scale(alpha, r)
    G = dH @ B
    dX = dH @ W_hat + s * (G @ A)
    dA, dB = lora_adapter_grads(X, dH, A, B, alpha, r)
    return dX, dA, dB


def lora_adapter_grads(X, dH, A, B, alpha, r):
    """(dA, dB) alone: dA = s (dH B)^T X, dB = s dH^T (X A^T) (same section as above)."""
    X, dH, A, B = (np.asarray(t, np.float64) for t in (X, dH, A, B))
    s = lora_scale(alpha, r)
    U = X @ A.T
    G = dH @ B
    return s * (G.T @ X), s * (dH.T @ U)


def lora_merge(W_hat, A, B, alpha, r):
    """W_final = W^ + s B A (dense; not re-quantized, R17)."""
    W_hat, A, B = (np.asarray(t, np.float64) for t in (W_hat, A, B))
    return W_hat + lora_scale(alpha, r) * (B @ A)


def lora_forward_batched(W_hat, X, adapter_id, As, Bs, alphas, ranks):
    """Multi-adapter forward over one shared base (R18).

    The shared base term X W^T is computed once for the whole batch; each token
    t then adds its own adapter's correction s_i (x_t A_i^T) B_i^T.  An id
    outside [0, n) is an error.
    """
    W_hat = np.asarray(W_hat, np.float64)
    X = np.asarray(X, np.float64)
    ids = np.asarray(adapter_id).reshape(-1)
    n = len(As)
    if ids.size and (ids.min() < 0 or ids.max() >= n):
        raise ValueError("adapter id out of range")
    H = X @ W_hat.T
    for t in range(X.shape[0]):
        i = int(ids[t])
        A = np.asarray(As[i], np.float64)
        B = np.asarray(Bs[i], np.float64)
        H[t] += lora_scale(alphas[i], ranks[i]) * ((X[t] @ A.T) @ B.T)
    return H


# ----------------------------------------------------------------------------
# DoRA (reading R24)
# ----------------------------------------------------------------------------


def dora_row_norms(W_hat, A, B, alpha, r):
    """||W[j, :]||_2 of W = W_hat + s B A for every output row j (fp64)."""
    W = np.asarray(W_hat, np.float64) + lora_scale(alpha, r) * (
        np.asarray(B, np.float64) @ np.asarray(A, np.float64))
    return np.sqrt(np.sum(W * W, axis=1))


def dora_forward(W_hat, X, A, B, alpha, r, magnitude):
    """H = X W'^T with W'[j, :] = m_j (W_hat + s B A)[j, :] / ||(W_hat + s B A)[j, :]||.

    The decomposition puts the norm of every output row of the adapted weight into the
    trained magnitude m (size d_out) and keeps only its direction; written as the plain
    product with the full adapted weight.
    """
    W = np.asarray(W_hat, np.float64) + lora_scale(alpha, r) * (
        np.asarray(B, np.float64) @ np.asarray(A, np.float64))
    norms = np.sqrt(np.sum(W * W, axis=1))
    Wd = (np.asarray(magnitude, np.float64) / norms)[:, None] * W
    return np.asarray(X, np.float64) @ Wd.T


def dora_backward(W_hat, X, dH, A, B, alpha, r, magnitude):
    """(dX, dA, dB, dm) of the DoRA forward above for the upstream gradient dH[T, d_out].

    With V = W_hat + s B A, n_j = ||V[j, :]||, c_j = m_j / n_j and Z = X V^T (so H = Z diag(c)),
    the chain rule through every factor, the norm included:
      dZ = dH diag(c)
      dc_j = sum_t dH[t, j] Z[t, j],   dm_j = dc_j / n_j,   dn_j = -dc_j m_j / n_j^2
      dX = dZ V;   dV = dZ^T X + diag(dn / n) V   (dn_j V[j, :] / n_j is the norm's gradient)
      dA = s B^T dV,   dB = s dV A^T             (V depends on A, B through s B A only)
    A row with n_j = 0 contributes nothing (its output is 0 and its direction undefined).
    """
    W_hat, X, dH, A, B = (np.asarray(t, np.float64) for t in (W_hat, X, dH, A, B))
    m = np.asarray(magnitude, np.float64)
    s = lora_scale(alpha, r)
    V = W_hat + s * (B @ A)
    n = np.sqrt(np.sum(V * V, axis=1))
    ok = n > 0
    safe = np.where(ok, n, 1.0)
    c = np.where(ok, m / safe, 0.0)
    Z = X @ V.T
    dZ = dH * c[None, :]
    dc = np.sum(dH * Z, axis=0)
    dm = np.where(ok, dc / safe, 0.0)
    dn = np.where(ok, -dc * m / (safe * safe), 0.0)
    dX = dZ @ V
    dV = dZ.T @ X + (np.where(ok, dn / safe, 0.0))[:, None] * V
    return dX, s * (B.T @ dV), s * (dV @ A.T), dm


# ----------------------------------------------------------------------------
# Adapter optimizer step (reading R23)
# ----------------------------------------------------------------------------


def adamw_step(w, g, m, v, step: int, lr: float, beta1: float, beta2: float,
               eps: float, weight_decay: float, grad_scale: float = 1.0):
    """One AdamW update of a trainable tensor (fp64), returning (w, m, v).

    Decoupled weight decay (Loshchilov & Hutter's AdamW, the rule behind the
    pages' "AdamW optimizer states"): the decay shrinks w directly, it is not
    added to the gradient.  With step t >= 1 counted from 1 and the gradient
    first multiplied by grad_scale (1 / micro-batches when accumulated):

        g' = grad_scale * g
        m  = beta1 m + (1 - beta1) g'
        v  = beta2 v + (1 - beta2) g'^2
        w  = w (1 - lr wd) - lr (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps)
    """
    w = np.asarray(w, np.float64)
    g = np.asarray(g, np.float64) * grad_scale
    m = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** step)
    v_hat = v / (1.0 - beta2 ** step)
    w = w * (1.0 - lr * weight_decay) - lr * m_hat / (np.sqrt(v_hat) + eps)
    return w, m, v


# ----------------------------------------------------------------------------
# FP8 activations (reading R25)
# ----------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(code) -> np.ndarray:
    """Value (fp64) of each E4M3 byte, the OCP 8-bit floating-point format the
    pages name for activations: bit 7 sign, bits 6..3 exponent with bias 7,
    bits 2..0 mantissa.  Exponent 0 holds the subnormals m/8 * 2^-6; the one
    pattern S.1111.111 is NaN; there is no infinity (largest finite 448)."""
    c = np.asarray(code, np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 15
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


def e4m3_encode(x) -> np.ndarray:
    """E4M3 byte of each finite fp32 value: the nearest representable value,
    ties to the even code (mantissa lsb 0), magnitudes at or beyond 448
    saturated to 448; the sign bit is the input's (so -0 and negatives that
    round to zero give 0x80)."""
    a = np.abs(np.asarray(x, np.float32).astype(np.float64))
    neg = np.signbit(np.asarray(x, np.float32))
    mags = e4m3_decode(np.arange(127, dtype=np.uint8))      # codes 0x00..0x7E, increasing
    hi = np.minimum(np.searchsorted(mags, a, side="left"), 126)
    lo = np.maximum(hi - 1, 0)
    dlo = a - mags[lo]
    dhi = mags[hi] - a
    pick = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(a >= E4M3_MAX, 126, pick)
    return (pick.astype(np.uint8) | np.where(neg, 0x80, 0).astype(np.uint8)).astype(np.uint8)


def fp8_pow2_scale(amax: float) -> float:
    """Per-tensor scale sigma = 2^(8 - ceil(log2 amax)), so that amax * sigma
    lies in (128, 256] below the E4M3 limit; 1 when amax is 0.  The exponent is
    kept in [-126, 126] (an fp32 normal power of two)."""
    if not amax > 0.0:
        return 1.0
    m, e = math.frexp(amax)                 # amax = m 2^e, 0.5 <= m < 1
    c = e - 1 if m == 0.5 else e            # ceil(log2 amax)
    return math.ldexp(1.0, min(max(8 - c, -126), 126))


def fp8_quantize_act(X):
    """(X8, sigma_x): X8 = E4M3(fl32(X * sigma_x)), sigma_x = fp8_pow2_scale(max|X|).
    X is read as fp32 values (a bf16 activation is exact in fp32); X8 / sigma_x
    stands for X."""
    X32 = np.asarray(X, np.float32)
    amax = float(np.max(np.abs(X32))) if X32.size else 0.0
    sig = fp8_pow2_scale(amax)
    return e4m3_encode((X32 * np.float32(sig)).astype(np.float32)), sig


def fp8_weight_scale(c2) -> float:
    """sigma_w of a double-quantized weight: every decoded weight is L * s_b with
    |L| <= 1 and s_b <= c2 of its group (up to one fp32 rounding), so the
    largest second-level constant bounds the tensor."""
    c2 = np.asarray(c2, np.float32)
    return fp8_pow2_scale(float(np.max(c2)) if c2.size else 0.0)


def nf4_dequantize_e4m3(codes, absmax_q, c2, d_out: int, d_in: int, w_scale: float,
                        levels: np.ndarray | None = None) -> np.ndarray:
    """E4M3 bytes [d_out, d_in] of the decoded weight in sigma_w units:
    E4M3(fl32(L[code] * s_b) * sigma_w) -- the fp32 decode of R11, scaled by an
    exact power of two, rounded once to E4M3."""
    w32 = nf4_dequantize(codes, absmax_q, c2, d_out, d_in, out="f32", levels=levels)
    return e4m3_encode((w32 * np.float32(w_scale)).astype(np.float32))


E5M2_MAX = 57344.0


def e5m2_decode(code) -> np.ndarray:
    """Value (fp64) of each E5M2 byte, the OCP 8-bit float with the wider range
    (the gradient format): bit 7 sign, bits 6..2 exponent with bias 15, bits
    1..0 mantissa.  Exponent 0 holds the subnormals m/4 * 2^-14; exponent 31
    is infinity (mantissa 0) or NaN.  Largest finite 57344."""
    c = np.asarray(code, np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 2) & 31
    m = (c & 3).astype(np.float64)
    mag = np.where(e == 0, m / 4.0 * 2.0 ** -14, (1.0 + m / 4.0) * np.exp2(e - 15.0))
    mag = np.where(e == 31, np.where(m == 0, np.inf, np.nan), mag)
    return sign * mag


def e5m2_encode(x) -> np.ndarray:
    """E5M2 byte of each finite fp32 value: nearest finite value, ties to the
    even code, magnitudes at or beyond 57344 saturated to 57344; sign bit the
    input's."""
    a = np.abs(np.asarray(x, np.float32).astype(np.float64))
    neg = np.signbit(np.asarray(x, np.float32))
    mags = e5m2_decode(np.arange(124, dtype=np.uint8))      # codes 0x00..0x7B, increasing
    hi = np.minimum(np.searchsorted(mags, a, side="left"), 123)
    lo = np.maximum(hi - 1, 0)
    dlo = a - mags[lo]
    dhi = mags[hi] - a
    pick = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(a >= E5M2_MAX, 123, pick)
    return (pick.astype(np.uint8) | np.where(neg, 0x80, 0).astype(np.uint8)).astype(np.uint8)


def fp8_pow2_scale_e5m2(amax: float) -> float:
    """The gradient's scale sigma = 2^(15 - ceil(log2 amax)): amax * sigma in
    (2^14, 2^15], below the E5M2 limit; 1 for amax = 0; exponent in [-126, 126]."""
    if not amax > 0.0:
        return 1.0
    m, e = math.frexp(amax)
    c = e - 1 if m == 0.5 else e
    return math.ldexp(1.0, min(max(15 - c, -126), 126))


def fp8_quantize_grad(dH):
    """(dH8, sigma_g): dH8 = E5M2(fl32(dH * sigma_g)), sigma_g = fp8_pow2_scale_e5m2(max|dH|)."""
    G32 = np.asarray(dH, np.float32)
    amax = float(np.max(np.abs(G32))) if G32.size else 0.0
    sig = fp8_pow2_scale_e5m2(amax)
    return e5m2_encode((G32 * np.float32(sig)).astype(np.float32)), sig


def lora_forward_fp8(X8, x_scale, W8, w_scale, A, B, alpha, r):
    """Forward of the adapted layer with E4M3 activations and weights (fp64):

        H = (X8 W8^T) / (sigma_x sigma_w) + s (X~ A^T) B^T,   X~ = X8 / sigma_x,

    X8, W8 the E4M3 bytes (decoded here), the adapters A, B in their own dtype.
    The base product is the one FP8 contraction; the low-rank branch reads the
    same FP8 activation."""
    Xv = e4m3_decode(X8)
    Wv = e4m3_decode(W8)
    Xt = Xv / float(x_scale)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    return (Xv @ Wv.T) / (float(x_scale) * float(w_scale)) + lora_scale(alpha, r) * ((Xt @ A.T) @ B.T)


def lora_backward_fp8(X8, x_scale, dH8, g_scale, W8, w_scale, A, B, alpha, r):
    """Backward of the adapted layer from the saved E4M3 activation and the E5M2
    upstream gradient (fp64), returning (dX, dA, dB):

        X~ = X8 / sigma_x,  dH~ = dH8 / sigma_g,  G = dH~ B,  U = X~ A^T
        dX = (dH8 W8) / (sigma_g sigma_w) + s G A      (the FP8 contraction)
        dA = s G^T X~,      dB = s dH~^T U

    the page's three gradient equations with the stored FP8 tensors in place of
    X and dH, and the E4M3 weight of the forward's FP8 contraction in dX."""
    Xt = e4m3_decode(X8) / float(x_scale)
    Gv = e5m2_decode(dH8)
    dHt = Gv / float(g_scale)
    Wv = e4m3_decode(W8)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    s = lora_scale(alpha, r)
    G = dHt @ B
    dX = (Gv @ Wv) / (float(g_scale) * float(w_scale)) + s * (G @ A)
    return dX, s * (G.T @ Xt), s * (dHt.T @ (Xt @ A.T))


# ----------------------------------------------------------------------------
# Counting formulas printed on the pages
# ----------------------------------------------------------------------------


def trainable_params(d_out: int, d_in: int, r: int) -> int:
    """r (d_in + d_out): r d_out for B plus r d_in for A ("Choosing what to adapt")."""
    return r * (d_in + d_out)


def merge_flops(d_out: int, d_in: int, r: int) -> int:
    """2 d_out r d_in: cost of B @ A ("Merging adapters vs keeping them separate")."""
    return 2 * d_out * r * d_in


def storage_bits_per_param(d_out: int, d_in: int) -> float:
    """Stored bits per weight of the double-quantized format."""
    a, b, c = nf4_sizes(d_out, d_in)
    return 8.0 * (a + b + c) / (d_out * d_in)


def fwd_flops(T, d_out, d_in, r):
    """Algorithmic forward FLOPs: 2 T d k + 2 T r (d + k)."""
    return 2 * T * d_out * d_in + 2 * T * r * (d_out + d_in)


def bwd_flops(T, d_out, d_in, r):
    """Algorithmic backward FLOPs: 2 T d k + 4 T r (d + k) (U reused)."""
    return 2 * T * d_out * d_in + 4 * T * r * (d_out + d_in)

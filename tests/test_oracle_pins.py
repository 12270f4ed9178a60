"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these calls the CUDA path.  Each pin is chosen so that a plausible
mistake in the oracle (a dropped alpha/r, a transposed operand, a wrong sign,
swapped nibbles, the wrong rounding rule, 255 for 127) fails at least one of
them; ``test_pins_catch_planted_mistakes`` plants such mistakes in copies of
the oracle functions and checks that the pins reject them.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special as sp

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_numbers.json")


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ---------------------------------------------------------------- NF4 table


def test_levels_shape_symmetry_range():
    L = O.nf4_levels()
    assert L.dtype == np.float32 and L.shape == (16,)
    assert np.all(np.diff(L) > 0)                      # strictly increasing
    assert L[0] == -1.0 and L[15] == 1.0               # normalised to [-1, 1]
    assert np.array_equal(L, -L[::-1])                 # symmetric quantiles


def test_levels_against_independent_quantile():
    # Re-derive every level with scipy's ndtri (an independent inverse CDF).
    edges = [sp.ndtri(j / 18.0) for j in range(1, 18)]
    q = np.array([0.5 * (edges[i] + edges[i + 1]) for i in range(16)])
    assert np.max(np.abs(O.nf4_unnormalised_levels() - q)) < 1e-12
    assert np.array_equal(O.nf4_levels(), (q / np.max(np.abs(q))).astype(np.float32))


def test_levels_equal_probability_bins():
    # The bins whose quantile midpoints give the levels each hold 1/18 of N(0,1).
    edges = [O.normal_quantile(j / 18.0) for j in range(1, 18)]
    for j, e in enumerate(edges, start=1):
        assert abs(sp.ndtr(e) - j / 18.0) < 1e-14
    probs = np.diff([sp.ndtr(e) for e in edges])
    assert np.allclose(probs, 1.0 / 18.0, atol=1e-14)


# ---------------------------------------------------------------- quantize


def brute_force_codes(xn, L):
    """Nearest level by exhaustive fp64 search; ties to the upper level."""
    d = np.abs(xn.astype(np.float64)[:, None] - L.astype(np.float64)[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = np.where(d == best, np.arange(16)[None, :], -1)
    return cand.max(axis=1), np.sort(d, axis=1)


def test_codes_are_nearest_level():
    rng = np.random.default_rng(1)
    W = (rng.standard_normal((32, 256)) * 0.141).astype(np.float32)
    codes, q8, c2, c1 = O.nf4_quantize(W)
    L = O.nf4_levels()
    xn = (W.reshape(-1, 64) / c1[:, None]).astype(np.float32).reshape(-1)
    bf, dsorted = brute_force_codes(xn, L)
    got = O.nf4_unpack(codes)
    # Only values within rounding of a midpoint may legitimately differ.
    clear = (dsorted[:, 1] - dsorted[:, 0]) > 1e-6
    assert clear.mean() > 0.999
    assert np.array_equal(got[clear], bf[clear])


def test_zero_ties_up_and_zero_block():
    W = np.zeros((1, 128), np.float32)
    W[0, 0] = 1.0                         # block 0: max 1, zeros elsewhere
    W[0, 1] = -0.0
    codes, q8, c2, c1 = O.nf4_quantize(W)
    c = O.nf4_unpack(codes)
    assert c[1] == 8 and c[2] == 8        # 0 and -0 tie between L7, L8 -> upper
    assert c[0] == 15
    assert np.all(c[64:] == 8)            # all-zero block (c1 = 0) -> x~ = 0
    assert c1[1] == 0 and q8[1] == 0


def check_round_trip(quantize):
    """Violations of the level round trip (0 = pinned).  A block holding c * L_j plus one +-c
    entry must quantize to codes j, element 2i in the low nibble of byte i, and with c a power
    of two (every product exact) decode to c * L_j.  quantize has nf4_quantize's signature."""
    L = O.nf4_levels()
    rng = np.random.default_rng(2)
    c = np.float32(0.25)
    j = rng.integers(0, 16, size=(8, 64))
    j[:, 0] = 15                          # guarantees max |w| = c
    W = (L[j] * c).astype(np.float32)
    codes, q8, c2, c1 = quantize(W.reshape(8, 64))
    bad = int(np.sum(O.nf4_unpack(codes).reshape(8, 64) != j))
    bad += int(np.sum((codes.reshape(-1) & 0xF) != j.reshape(-1)[0::2]))
    bad += int(np.sum(q8 != 127)) + int(np.sum(c2 != c))
    w = O.nf4_dequantize(codes, q8, c2, 8, 64)
    bad += int(np.sum(w != W))
    return bad


def check_double_quant(quantize):
    """Violations of the second-level code (0 = pinned): q8 in [0, 127], c2 the group maximum,
    the group's largest block coded 127, and the rebuilt scale within half a step (c2/254) of
    c1 plus fp32 rounding."""
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((64, 1024)) * 0.141).astype(np.float32)
    W[5] *= 40.0                          # a few large blocks
    codes, q8, c2, c1 = quantize(W)
    bad = int(q8.dtype != np.uint8) + int(np.sum(q8 > 127))
    nb = c1.size
    for g in range(c2.size):
        blk = c1[g * 256:(g + 1) * 256]
        bad += int(c2[g] != blk.max())
        bad += int(q8[g * 256 + int(np.argmax(blk))] != 127)
    s = O.nf4_block_scales(q8, c2).astype(np.float64)
    c2b = np.repeat(c2, 256)[:nb].astype(np.float64)
    bad += int(np.sum(np.abs(s - c1) > c2b / 254.0 * (1 + 1e-5) + 1e-12))
    return bad


def test_round_trip_of_levels_and_nibble_order():
    assert check_round_trip(O.nf4_quantize) == 0


def test_double_quant_range_and_scale_error():
    assert check_double_quant(O.nf4_quantize) == 0


def test_identity_levels_reduce_to_textbook_matmul():
    # With the levels replaced by the identity map (L[i] = i), the second-level code bypassed
    # (block scales that the rebuild gives exactly) and B = 0, the decode
    # and forward must be the plain matrix product of X with (code x block scale), built here
    # straight from the nibbles with numpy.matmul: this pins the unpacking order, which block
    # each scale multiplies, and the orientation of the forward product.
    rng = np.random.default_rng(9)
    d_out, d_in, T, r = 6, 256, 5, 3
    nib = rng.integers(0, 16, size=(d_out, d_in)).astype(np.uint8)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    nblocks = d_out * d_in // 64
    # c2 = 127 * 2^-7 makes every rebuilt scale exact: s_b = q8 * c2 / 127 = q8 * 2^-7, a
    # different known scale for every block
    q8 = rng.integers(1, 128, size=nblocks).astype(np.uint8)
    c2 = np.array([127.0 * 2.0 ** -7], np.float32)
    ident = np.arange(16, dtype=np.float32)
    W_hat = O.nf4_dequantize(codes, q8, c2, d_out, d_in, levels=ident)
    X = rng.standard_normal((T, d_in))
    A = rng.standard_normal((r, d_in))
    H = O.lora_forward(W_hat, X, A, np.zeros((d_out, r)), 2.0 * r, r)
    W_direct = nib.astype(np.float64) * np.repeat(q8.astype(np.float64) * 2.0 ** -7, 64).reshape(d_out, d_in)
    assert np.array_equal(W_hat.astype(np.float64), W_direct)
    assert np.allclose(H, np.matmul(X, W_direct.T), rtol=0, atol=1e-12 * np.abs(X).sum() * 15)


def test_elementwise_error_bound():
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((16, 512)) * 0.141).astype(np.float32)
    codes, q8, c2, c1 = O.nf4_quantize(W)
    w = O.nf4_dequantize(codes, q8, c2, 16, 512).astype(np.float64)
    L = O.nf4_levels().astype(np.float64)
    half_gap = np.max(np.diff(L)) / 2.0
    s = O.nf4_block_scales(q8, c2).astype(np.float64)
    c1b = np.repeat(c1.astype(np.float64), 64)
    sb = np.repeat(s, 64)
    bound = c1b * (half_gap + 2.0 ** -22) + np.abs(c1b - sb) + 2.0 ** -23 * np.abs(w.reshape(-1))
    assert np.all(np.abs(W.reshape(-1) - w.reshape(-1)) <= bound)


def test_bf16_rounding_definition():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -1.0 - 2 ** -8,
                  3.0e-3, 65504.0], np.float32)
    import torch
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(O.bf16_round(x), ref)
    # halfway cases go to even
    assert O.bf16_round(np.array([1.0 + 2 ** -8], np.float32))[0] == 1.0
    assert O.bf16_round(np.array([1.0 + 3 * 2 ** -8], np.float32))[0] == 1.0 + 2 ** -6


# ---------------------------------------------------------------- storage rate


def test_storage_rate_matches_pages():
    g = json.load(open(GOLDEN))["storage"]
    a, b, c = O.nf4_sizes(4096, 4096)
    assert (a, b, c) == (4096 * 4096 // 2, 4096 * 4096 // 64, 4 * 1024)
    bits = O.storage_bits_per_param(4096, 4096)
    assert abs(bits - 4.126953125) < 1e-12
    assert round(bits, 3) == g["double_quant_bits"]
    assert round(4 + 32 / 64, 3) == g["single_level_bits"]
    assert round(g["single_level_bits"] - bits, 3) == g["saving_bits"]
    assert round(bits / 8, 4) == g["bytes_per_param"]
    assert round(bits - 4, 3) == g["dq_overhead_bits"]
    assert round(7e9 * bits / 8 / 1e9, 2) == g["gb_7b_base"]
    # a partial last group still costs one fp32 constant
    assert O.nf4_sizes(3, 128)[2] == 4


# ---------------------------------------------------------------- counting


def test_parameter_counts_and_calculator():
    g = json.load(open(GOLDEN))
    for e in g["trainable_params"]:
        assert O.trainable_params(e["d_out"], e["d_in"], e["r"]) == e["value"]
    c = g["calculator_output"]
    base = sum(O.trainable_params(d, k, c["baseline_rank"]) for d, k in c["baseline_targets"]) * c["layers"]
    exp = sum(O.trainable_params(d, k, c["expanded_rank"]) for d, k in c["expanded_targets"]) * c["layers"]
    assert (base, exp, exp / base) == (c["baseline"], c["expanded"], c["ratio"])
    v = g["v_proj_only"]
    assert O.trainable_params(4096, 4096, v["r"]) * v["layers"] == v["value"]


def test_merge_flops():
    g = json.load(open(GOLDEN))["merge_flops"]
    assert O.merge_flops(4096, 4096, 8) == g[0]["value"]
    base = 2 * O.merge_flops(4096, 4096, 8) * 32
    exp = (3 * O.merge_flops(4096, 4096, 16) + O.merge_flops(4096, 11008, 16)) * 32
    assert round(base / 1e9, 2) == g[1]["total_gflop_baseline"]
    assert round(exp / 1e9, 2) == g[1]["total_gflop_expanded"]


# ---------------------------------------------------------------- LoRA algebra


def small_layer(d=8, k=8, r=2, T=3, seed=5):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((d, k))
    X = rng.standard_normal((T, k))
    A = rng.standard_normal((r, k))
    B = rng.standard_normal((d, r))
    dH = rng.standard_normal((T, d))
    return W, X, A, B, dH


def check_init_invariant(fwd):
    W, X, A, B, dH = small_layer(d=12, k=10, r=3, T=4)
    H0 = fwd(W, X, A, np.zeros_like(B), 6.0, 3)
    return np.array_equal(H0, X @ W.T)


def check_forward_brute(fwd):
    W, X, A, B, dH = small_layer(d=6, k=5, r=2, T=3)
    alpha, r = 3.0, 2
    H = fwd(W, X, A, B, alpha, r)
    ref = np.zeros((3, 6))
    for t in range(3):
        for i in range(6):
            acc = 0.0
            for j in range(5):
                acc += W[i, j] * X[t, j]
            for q in range(r):
                ax = 0.0
                for j in range(5):
                    ax += A[q, j] * X[t, j]
                acc += (alpha / r) * B[i, q] * ax
            ref[t, i] = acc
    return rel(H, ref)


def check_gradients_fd(fwd, bwd):
    """Central differences of L = <dH, H>; exact up to rounding (L is linear
    in each single entry of X, A and B)."""
    W, X, A, B, dH = small_layer()
    alpha, r = 5.0, 2
    dX, dA, dB = bwd(W, X, dH, A, B, alpha, r)
    worst = 0.0
    for name, P, G in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        num = np.zeros_like(P)
        for idx in np.ndindex(P.shape):
            h = 0.5
            orig = P[idx]
            P[idx] = orig + h
            lp = np.sum(dH * fwd(W, X, A, B, alpha, r))
            P[idx] = orig - h
            lm = np.sum(dH * fwd(W, X, A, B, alpha, r))
            P[idx] = orig
            num[idx] = (lp - lm) / (2 * h)
        worst = max(worst, rel(G, num))
    return worst


def check_merge(fwd, merge):
    W, X, A, B, dH = small_layer(d=9, k=7, r=3, T=5)
    Wf = merge(W, A, B, 6.0, 3)
    return rel(X @ Wf.T, fwd(W, X, A, B, 6.0, 3))


def test_init_invariant_B_zero():
    assert check_init_invariant(O.lora_forward)


def test_forward_against_loops():
    assert check_forward_brute(O.lora_forward) < 1e-13


def test_gradients_finite_differences():
    assert check_gradients_fd(O.lora_forward, O.lora_backward) < 1e-11


def test_merge_reproduces_unmerged_output():
    assert check_merge(O.lora_forward, O.lora_merge) < 1e-12


def test_batched_matches_per_adapter():
    rng = np.random.default_rng(6)
    d, k, T = 10, 12, 9
    ranks = [1, 2, 4]
    W = rng.standard_normal((d, k))
    X = rng.standard_normal((T, k))
    As = [rng.standard_normal((r, k)) for r in ranks]
    Bs = [rng.standard_normal((d, r)) for r in ranks]
    alphas = [2.0 * r for r in ranks]
    ids = rng.integers(0, 3, size=T)
    H = O.lora_forward_batched(W, X, ids, As, Bs, alphas, ranks)
    for i in range(3):
        sel = ids == i
        if sel.any():
            ref = O.lora_forward(W, X[sel], As[i], Bs[i], alphas[i], ranks[i])
            assert rel(H[sel], ref) < 1e-13
    with pytest.raises(ValueError):
        O.lora_forward_batched(W, X, np.full(T, 3), As, Bs, alphas, ranks)


# ---------------------------------------------------------------- DoRA (R24)


def check_dora_brute(fwd):
    """Loops over a tiny layer: W' = m_j W_j / ||W_j|| row by row, then h = W' x."""
    W, X, A, B, dH = small_layer(d=5, k=4, r=2, T=3)
    mag = np.array([0.5, 1.5, 2.0, 0.25, 1.0])
    alpha, r = 3.0, 2
    H = fwd(W, X, A, B, alpha, r, mag)
    ref = np.zeros((3, 5))
    for j in range(5):
        row = [W[j, c] + (alpha / r) * sum(B[j, q] * A[q, c] for q in range(r)) for c in range(4)]
        nrm = math.sqrt(sum(x * x for x in row))
        for t in range(3):
            ref[t, j] = sum(mag[j] * row[c] / nrm * X[t, c] for c in range(4))
    return rel(H, ref)


def test_dora_against_loops():
    assert check_dora_brute(O.dora_forward) < 1e-13


def test_dora_magnitude_equal_to_norms_is_lora():
    """With m set to the row norms of W + sBA (DoRA's initialisation) the layer is LoRA."""
    W, X, A, B, dH = small_layer(d=9, k=7, r=3, T=4)
    mag = O.dora_row_norms(W, A, B, 6.0, 3)
    assert rel(O.dora_forward(W, X, A, B, 6.0, 3, mag), O.lora_forward(W, X, A, B, 6.0, 3)) < 1e-13


def test_dora_direction_is_scale_free():
    """Scaling the adapted weight (W and B together) leaves the DoRA output unchanged."""
    W, X, A, B, dH = small_layer(d=6, k=5, r=2, T=3)
    mag = np.linspace(0.5, 2.0, 6)
    h1 = O.dora_forward(W, X, A, B, 4.0, 2, mag)
    h2 = O.dora_forward(3.5 * W, X, A, 3.5 * B, 4.0, 2, mag)
    assert rel(h1, h2) < 1e-13


def check_dora_gradients_fd(bwd):
    """Largest relative gap between bwd's (dX, dA, dB, dm) and central finite differences of
    L = <dH, H> through the DoRA forward (nonlinear in A, B, m through the row norm: the
    difference quotient is exact to O(h^2); h = 1e-5 in fp64)."""
    W, X, A, B, dH = small_layer(d=5, k=6, r=2, T=3, seed=11)
    mag = np.array([0.7, 1.3, 2.0, 0.4, 1.1])
    alpha, r = 3.0, 2
    got = bwd(W, X, dH, A, B, alpha, r, mag)
    h = 1e-5

    def loss(X_, A_, B_, m_):
        return float(np.sum(dH * O.dora_forward(W, X_, A_, B_, alpha, r, m_)))

    refs = []
    for which, base in enumerate((X, A, B, mag)):
        g = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            args_p = [X.copy(), A.copy(), B.copy(), mag.copy()]
            args_m = [X.copy(), A.copy(), B.copy(), mag.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            g[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        refs.append(g)
    return max(rel(gv, rv) for gv, rv in zip(got, refs))


def test_dora_backward_against_finite_differences():
    assert check_dora_gradients_fd(O.dora_backward) < 1e-8


def test_dora_backward_reduces_to_lora_at_initialisation():
    # m = the row norms makes the forward LoRA's; the gradients of X, A, B then differ from
    # LoRA's only by the norm's term, and dm is the per-row <dH, Z> / n
    W, X, A, B, dH = small_layer(d=7, k=5, r=2, T=4, seed=12)
    n = O.dora_row_norms(W, A, B, 4.0, 2)
    dX, dA, dB, dm = O.dora_backward(W, X, dH, A, B, 4.0, 2, n)
    dXl, _, _ = O.lora_backward(W, X, dH, A, B, 4.0, 2)
    assert rel(dX, dXl) < 1e-13
    Z = O.lora_forward(W, X, A, B, 4.0, 2)
    assert rel(dm, np.sum(dH * Z, axis=0) / n) < 1e-13


# ---------------------------------------------------------------- optimizer step (R23)

ADAM = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


def check_adamw_first_step(step_fn):
    """From zero state the bias corrections make m_hat = g, v_hat = g^2 exactly:
    w1 = w0 (1 - lr wd) - lr g / (|g| + eps)."""
    rng = np.random.default_rng(21)
    w0, g = rng.standard_normal(50), rng.standard_normal(50)
    w1, m1, v1 = step_fn(w0, g, np.zeros(50), np.zeros(50), 1, **ADAM)
    h = ADAM
    ref = w0 * (1 - h["lr"] * h["weight_decay"]) - h["lr"] * g / (np.abs(g) + h["eps"])
    return max(rel(w1, ref), rel(m1, (1 - h["beta1"]) * g), rel(v1, (1 - h["beta2"]) * g * g))


def check_adamw_constant_gradient(step_fn):
    """A constant gradient keeps m_hat = g and v_hat = g^2 at every step, so with no
    decay each step moves w by exactly -lr g / (|g| + eps)."""
    rng = np.random.default_rng(22)
    w, g = rng.standard_normal(20), rng.standard_normal(20)
    m, v = np.zeros(20), np.zeros(20)
    h = dict(ADAM, weight_decay=0.0)
    w0 = w.copy()
    for t in range(1, 8):
        w, m, v = step_fn(w, g, m, v, t, **h)
    return rel(w, w0 - 7 * h["lr"] * g / (np.abs(g) + h["eps"]))


def check_adamw_decay_only(step_fn):
    """A zero gradient leaves m = v = 0 and only the decoupled decay: w_t = w0 (1 - lr wd)^t."""
    w0 = np.linspace(-2, 2, 9)
    w, m, v = w0.copy(), np.zeros(9), np.zeros(9)
    for t in range(1, 6):
        w, m, v = step_fn(w, np.zeros(9), m, v, t, **ADAM)
    return rel(w, w0 * (1 - ADAM["lr"] * ADAM["weight_decay"]) ** 5)


def test_adamw_first_step_closed_form():
    assert check_adamw_first_step(O.adamw_step) < 1e-14


def test_adamw_constant_gradient():
    assert check_adamw_constant_gradient(O.adamw_step) < 1e-13


def test_adamw_decay_only():
    assert check_adamw_decay_only(O.adamw_step) < 1e-14


def test_adamw_grad_scale_is_a_gradient_multiplier():
    rng = np.random.default_rng(23)
    w, g = rng.standard_normal(10), rng.standard_normal(10)
    a = O.adamw_step(w, g, np.zeros(10), np.zeros(10), 3, grad_scale=0.25, **ADAM)
    b = O.adamw_step(w, 0.25 * g, np.zeros(10), np.zeros(10), 3, **ADAM)
    assert all(rel(x, y) < 1e-15 for x, y in zip(a, b))


def test_gradient_accumulation_equals_full_batch():
    """dA, dB are sums over tokens, so accumulating the micro-batches' gradients gives the
    full batch's gradients (the pages' gradient accumulation before one update)."""
    W, X, A, B, dH = small_layer(d=7, k=6, r=2, T=8)
    full = O.lora_adapter_grads(X, dH, A, B, 4.0, 2)
    parts = [O.lora_adapter_grads(X[i:i + 3], dH[i:i + 3], A, B, 4.0, 2) for i in (0, 3, 6)]
    assert rel(sum(p[0] for p in parts), full[0]) < 1e-13
    assert rel(sum(p[1] for p in parts), full[1]) < 1e-13


# ---------------------------------------------------------------- FP8 (R25)


def brute_e4m3(x):
    """Nearest finite E4M3 value by scanning all 254 finite codes; ties to the
    even code; saturating at 448."""
    vals = [(c, O.e4m3_decode(np.uint8(c)).item()) for c in range(256)
            if (c & 0x7F) != 0x7F]
    out = []
    for v in np.asarray(x, np.float64).reshape(-1):
        best = None
        for c, cv in vals:
            if (c & 0x80) != (0x80 if math.copysign(1.0, v) < 0 else 0):
                continue
            d = abs(v - cv)
            if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
                best = (d, c)
        out.append(best[1])
    return np.array(out, np.uint8)


def test_e4m3_format_constants():
    # OCP 8-bit floating point, E4M3: largest finite 448, smallest normal 2^-6,
    # smallest subnormal 2^-9, 1.0 = 0x38, one NaN pattern per sign, no infinity.
    d = O.e4m3_decode
    assert d(np.uint8(0x7E)) == 448.0 and d(np.uint8(0xFE)) == -448.0
    assert d(np.uint8(0x08)) == 2.0 ** -6 and d(np.uint8(0x01)) == 2.0 ** -9
    assert d(np.uint8(0x07)) == 7 * 2.0 ** -9
    assert d(np.uint8(0x38)) == 1.0 and d(np.uint8(0x40)) == 2.0
    assert np.isnan(d(np.uint8(0x7F))) and np.isnan(d(np.uint8(0xFF)))
    pos = d(np.arange(127, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)                        # codes 0..126 increase
    assert np.sum(np.isfinite(d(np.arange(256, dtype=np.uint8)))) == 254


def e4m3_probe_values():
    rng = np.random.default_rng(11)
    mags = np.exp2(rng.uniform(-12, 10, 3000))
    x = mags * rng.choice([-1.0, 1.0], mags.size)
    pos = O.e4m3_decode(np.arange(127, dtype=np.uint8))
    mids = 0.5 * (pos[1:] + pos[:-1])                      # every tie
    extra = np.array([0.0, -0.0, 448.0, 463.99, 464.0, 1e6, -1e6, 2.0 ** -10, -2.0 ** -10, 2.0 ** -11])
    return np.concatenate([x, mids, -mids, extra]).astype(np.float32)


def check_e4m3_encode(enc):
    x = e4m3_probe_values()
    return int(np.sum(enc(x) != brute_e4m3(x)))


def test_e4m3_encode_against_brute_force():
    assert check_e4m3_encode(O.e4m3_encode) == 0


def test_e4m3_round_trip_and_error_bound():
    c = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    assert np.array_equal(O.e4m3_encode(O.e4m3_decode(c).astype(np.float32)), c)
    rng = np.random.default_rng(3)
    x = (np.exp2(rng.uniform(-6, np.log2(448), 20000)) * rng.choice([-1, 1], 20000)).astype(np.float32)
    err = np.abs(O.e4m3_decode(O.e4m3_encode(x)) - x.astype(np.float64))
    assert np.all(err <= 2.0 ** -4 * np.abs(x))            # 3 mantissa bits: half an ulp
    sub = (rng.uniform(-2.0 ** -6, 2.0 ** -6, 5000)).astype(np.float32)
    assert np.all(np.abs(O.e4m3_decode(O.e4m3_encode(sub)) - sub) <= 2.0 ** -10)


def check_pow2_scale(fn):
    bad = 0
    for amax in [4.0, 4.1, 0.06, 1e-3, 5.3, 255.0, 256.0, 300.0, 2.0 ** -20, 1e30]:
        sig = fn(amax)
        m, e = math.frexp(sig)
        bad += (m != 0.5) or not (128.0 < amax * sig <= 256.0)
    return bad + (fn(0.0) != 1.0)


def test_fp8_scale_range():
    assert check_pow2_scale(O.fp8_pow2_scale) == 0
    assert O.fp8_pow2_scale(4.0) == 64.0 and O.fp8_pow2_scale(4.1) == 32.0


def test_fp8_activation_quantizer():
    rng = np.random.default_rng(8)
    X = rng.standard_normal((37, 96)).astype(np.float32)
    X8, sig = O.fp8_quantize_act(X)
    assert X8.dtype == np.uint8 and X8.shape == X.shape
    assert 128.0 < np.max(np.abs(X)) * sig <= 256.0
    Xr = O.e4m3_decode(X8) / sig
    big = np.abs(X) * sig >= 2.0 ** -6
    assert np.all(np.abs(Xr - X)[big] <= 2.0 ** -4 * np.abs(X)[big])
    assert np.all(np.abs(Xr - X)[~big] <= 2.0 ** -10 / sig)
    # values already on the scaled E4M3 grid come back exactly
    Xg = (O.e4m3_decode(X8) / sig).astype(np.float32)
    X8g, sig_g = O.fp8_quantize_act(Xg)
    assert sig_g == sig and np.array_equal(X8g, X8)
    # an all-zero tensor: scale 1, all codes zero
    Z8, zs = O.fp8_quantize_act(np.zeros((3, 64), np.float32))
    assert zs == 1.0 and not Z8.any()


def fp8_layer(T=5, d=7, k=128, r=3, seed=21):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((d, k)) * 0.02).astype(np.float32)
    codes, q8, c2, c1 = O.nf4_quantize(W)
    X = rng.standard_normal((T, k)).astype(np.float32)
    A = rng.standard_normal((r, k)) / np.sqrt(r)
    B = rng.standard_normal((d, r)) * 0.1
    return W, codes, q8, c2, X, A, B


def check_fp8_forward_loops(fwd):
    W, codes, q8, c2, X, A, B = fp8_layer()
    d, k = W.shape
    T, r, alpha = X.shape[0], A.shape[0], 6.0
    X8, sx = O.fp8_quantize_act(X)
    sw = O.fp8_weight_scale(c2)
    W8 = O.nf4_dequantize_e4m3(codes, q8, c2, d, k, sw)
    H = fwd(X8, sx, W8, sw, A, B, alpha, r)
    ref = np.zeros((T, d))
    for t in range(T):
        for i in range(d):
            acc = 0.0
            for j in range(k):
                acc += O.e4m3_decode(X8[t, j]).item() * O.e4m3_decode(W8[i, j]).item()
            acc /= sx * sw
            for q in range(r):
                u = 0.0
                for j in range(k):
                    u += A[q, j] * O.e4m3_decode(X8[t, j]).item() / sx
                acc += (alpha / r) * B[i, q] * u
            ref[t, i] = acc
    return rel(H, ref)


def check_fp8_forward_bound(fwd):
    """The FP8 forward approximates the exact forward of the same layer: every
    element within the E4M3 rounding bound (2^-4 relative per operand in the
    normal range, 2^-10 / sigma absolute below it)."""
    W, codes, q8, c2, X, A, B = fp8_layer(T=9, d=11, k=256, r=4, seed=2)
    d, k = W.shape
    X8, sx = O.fp8_quantize_act(X)
    sw = O.fp8_weight_scale(c2)
    W8 = O.nf4_dequantize_e4m3(codes, q8, c2, d, k, sw)
    W32 = O.nf4_dequantize(codes, q8, c2, d, k, out="f32").astype(np.float64)
    H = fwd(X8, sx, W8, sw, A, B, 8.0, 4)
    exact = O.lora_forward(W32, X, A, B, 8.0, 4)
    # x~ = x + e_x with |e_x| <= 2^-4 |x| + 2^-10 / sigma_x (likewise w), so
    # |x~ w~ - x w| <= (2^-3 + 2^-8)|x||w| + (1 + 2^-4) 2^-10 (|x| / sigma_w + |w| / sigma_x)
    #                  + 2^-20 / (sigma_x sigma_w)
    aX = np.abs(X.astype(np.float64))
    aW = np.abs(W32)
    base = (2.0 ** -3 + 2.0 ** -8) * (aX @ aW.T) \
        + (1 + 2.0 ** -4) * 2.0 ** -10 * (aX @ np.ones_like(aW).T / sw + np.ones_like(aX) @ aW.T / sx) \
        + 2.0 ** -20 / (sx * sw) * k
    lowrank = (8.0 / 4) * ((2.0 ** -10 / sx + 2.0 ** -4 * aX) @ np.abs(A).T) @ np.abs(B).T
    return float(np.max(np.abs(H - exact) - (base + lowrank + 1e-12)))


def test_fp8_forward_against_loops():
    assert check_fp8_forward_loops(O.lora_forward_fp8) < 1e-12


def test_fp8_forward_within_rounding_bound_of_exact():
    assert check_fp8_forward_bound(O.lora_forward_fp8) <= 0.0


def test_fp8_weight_decode():
    W, codes, q8, c2, X, A, B = fp8_layer(d=9, k=192)
    sw = O.fp8_weight_scale(c2)
    W8 = O.nf4_dequantize_e4m3(codes, q8, c2, 9, 192, sw)
    W32 = O.nf4_dequantize(codes, q8, c2, 9, 192, out="f32").astype(np.float64)
    assert np.max(np.abs(W32)) * sw <= 256.0 * (1 + 2.0 ** -23)
    Wr = O.e4m3_decode(W8) / sw
    big = np.abs(W32) * sw >= 2.0 ** -6
    assert np.all(np.abs(Wr - W32)[big] <= 2.0 ** -4 * np.abs(W32)[big])
    # the zero level (code for |x| smallest) and the sign: W8 of -w is W8 of w with bit 7 flipped
    assert np.array_equal(O.e4m3_encode(-(W32 * sw).astype(np.float32)) ^ W8,
                          np.full_like(W8, 0x80))


# ---------------------------------------------------------------- FP8 backward (R26)


def brute_e5m2(x):
    vals = [(c, O.e5m2_decode(np.uint8(c)).item()) for c in range(256)
            if ((c >> 2) & 31) != 31]
    out = []
    for v in np.asarray(x, np.float64).reshape(-1):
        best = None
        for c, cv in vals:
            if (c & 0x80) != (0x80 if math.copysign(1.0, v) < 0 else 0):
                continue
            d = abs(v - cv)
            if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
                best = (d, c)
        out.append(best[1])
    return np.array(out, np.uint8)


def test_e5m2_format_constants():
    # OCP 8-bit floating point, E5M2: largest finite 57344, smallest normal 2^-14, smallest
    # subnormal 2^-16, 1.0 = 0x3C, infinity 0x7C, NaN 0x7D..0x7F.
    d = O.e5m2_decode
    assert d(np.uint8(0x7B)) == 57344.0 and d(np.uint8(0xFB)) == -57344.0
    assert d(np.uint8(0x04)) == 2.0 ** -14 and d(np.uint8(0x01)) == 2.0 ** -16
    assert d(np.uint8(0x3C)) == 1.0 and d(np.uint8(0x40)) == 2.0
    assert np.isinf(d(np.uint8(0x7C))) and all(np.isnan(d(np.uint8(c))) for c in (0x7D, 0x7E, 0x7F))
    pos = d(np.arange(124, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)
    assert np.sum(np.isfinite(d(np.arange(256, dtype=np.uint8)))) == 248


def e5m2_probe_values():
    rng = np.random.default_rng(13)
    mags = np.exp2(rng.uniform(-18, 17, 2000))
    x = mags * rng.choice([-1.0, 1.0], mags.size)
    pos = O.e5m2_decode(np.arange(124, dtype=np.uint8))
    mids = 0.5 * (pos[1:] + pos[:-1])
    extra = np.array([0.0, -0.0, 57344.0, 61439.0, 61440.0, 1e9, -1e9, 2.0 ** -17, -2.0 ** -17])
    return np.concatenate([x, mids, -mids, extra]).astype(np.float32)


def check_e5m2_encode(enc):
    x = e5m2_probe_values()
    return int(np.sum(enc(x) != brute_e5m2(x)))


def test_e5m2_encode_against_brute_force():
    assert check_e5m2_encode(O.e5m2_encode) == 0


def test_e5m2_round_trip_error_bound_and_scale():
    c = np.array([c for c in range(256) if ((c >> 2) & 31) != 31], np.uint8)
    assert np.array_equal(O.e5m2_encode(O.e5m2_decode(c).astype(np.float32)), c)
    rng = np.random.default_rng(5)
    x = (np.exp2(rng.uniform(-14, 15.8, 20000)) * rng.choice([-1, 1], 20000)).astype(np.float32)
    err = np.abs(O.e5m2_decode(O.e5m2_encode(x)) - x.astype(np.float64))
    assert np.all(err <= 2.0 ** -3 * np.abs(x))          # 2 mantissa bits: half an ulp
    for amax in [1e-3, 0.7, 1.0, 3.0, 6e4, 2.0 ** -30]:
        sig = O.fp8_pow2_scale_e5m2(amax)
        assert math.frexp(sig)[0] == 0.5 and 2.0 ** 14 < amax * sig <= 2.0 ** 15
    G = np.random.default_rng(2).standard_normal((9, 70)).astype(np.float32) * 1e-3
    G8, sg = O.fp8_quantize_grad(G)
    big = np.abs(G) * sg >= 2.0 ** -14
    assert np.all(np.abs(O.e5m2_decode(G8) / sg - G)[big] <= 2.0 ** -3 * np.abs(G)[big])


def fp8_bwd_case(T=4, d=6, k=128, r=2, seed=31):
    W, codes, q8, c2, X, A, B = fp8_layer(T=T, d=d, k=k, r=r, seed=seed)
    dH = (np.random.default_rng(seed + 1).standard_normal((T, d)) * 1e-2).astype(np.float32)
    X8, sx = O.fp8_quantize_act(X)
    G8, sg = O.fp8_quantize_grad(dH)
    sw = O.fp8_weight_scale(c2)
    W8 = O.nf4_dequantize_e4m3(codes, q8, c2, d, k, sw)
    W32 = O.nf4_dequantize(codes, q8, c2, d, k, out="f32").astype(np.float64)
    return X, dH, X8, sx, G8, sg, W8, sw, W32, A, B


def check_fp8_backward_loops(bwd):
    X, dH, X8, sx, G8, sg, W8, sw, W32, A, B = fp8_bwd_case()
    T, k = X.shape
    d, r = B.shape
    alpha = 4.0
    s = alpha / r
    dX, dA, dB = bwd(X8, sx, G8, sg, W8, sw, A, B, alpha, r)
    xv = lambda t, j: O.e4m3_decode(X8[t, j]).item() / sx
    gv = lambda t, i: O.e5m2_decode(G8[t, i]).item() / sg
    wv = lambda i, j: O.e4m3_decode(W8[i, j]).item() / sw
    G = [[sum(gv(t, i) * B[i, q] for i in range(d)) for q in range(r)] for t in range(T)]
    U = [[sum(xv(t, j) * A[q, j] for j in range(k)) for q in range(r)] for t in range(T)]
    rdX = np.array([[sum(gv(t, i) * wv(i, j) for i in range(d)) + s * sum(G[t][q] * A[q, j] for q in range(r))
                     for j in range(k)] for t in range(T)])
    rdA = np.array([[s * sum(G[t][q] * xv(t, j) for t in range(T)) for j in range(k)] for q in range(r)])
    rdB = np.array([[s * sum(gv(t, i) * U[t][q] for t in range(T)) for q in range(r)] for i in range(d)])
    return max(rel(dX, rdX), rel(dA, rdA), rel(dB, rdB))


def check_fp8_backward_bound(bwd):
    """The FP8 backward against the exact backward of the same layer, elementwise within the
    E4M3 / E5M2 rounding bounds (x~ = x + e_x, |e_x| <= 2^-4|x| + 2^-10/sigma_x; likewise
    |e_g| <= 2^-3|g| + 2^-17/sigma_g and the weight)."""
    X, dH, X8, sx, G8, sg, W8, sw, W32, A, B = fp8_bwd_case(T=7, d=9, k=192, r=3, seed=8)
    alpha, r = 6.0, 3
    s = alpha / r
    dX, dA, dB = bwd(X8, sx, G8, sg, W8, sw, A, B, alpha, r)
    eX, eA, eB = O.lora_backward(W32, X, dH, A, B, alpha, r)
    aX, aG, aW = np.abs(X.astype(np.float64)), np.abs(dH.astype(np.float64)), np.abs(W32)
    Ex = 2.0 ** -4 * aX + 2.0 ** -10 / sx
    Eg = 2.0 ** -3 * aG + 2.0 ** -17 / sg
    Ew = 2.0 ** -4 * aW + 2.0 ** -10 / sw
    aA, aB = np.abs(A), np.abs(B)
    bX = (aG + Eg) @ Ew + Eg @ aW + s * (Eg @ aB) @ aA
    Gt = (aG + Eg) @ aB
    bA = s * (Gt.T @ Ex + (Eg @ aB).T @ aX)
    bB = s * ((aG + Eg).T @ (Ex @ aA.T) + Eg.T @ (aX @ aA.T))
    return max(float(np.max(np.abs(dX - eX) - bX - 1e-12)), float(np.max(np.abs(dA - eA) - bA - 1e-12)),
               float(np.max(np.abs(dB - eB) - bB - 1e-12)))


def test_fp8_backward_against_loops():
    assert check_fp8_backward_loops(O.lora_backward_fp8) < 1e-12


def test_fp8_backward_within_rounding_bound_of_exact():
    assert check_fp8_backward_bound(O.lora_backward_fp8) <= 0.0


# ---------------------------------------------------------------- mutants


def test_pins_catch_planted_mistakes():
    s = O.lora_scale

    def fwd_sign(W, X, A, B, a, r):
        return np.asarray(X) @ np.asarray(W).T - s(a, r) * ((X @ A.T) @ B.T)

    def fwd_noscale(W, X, A, B, a, r):
        return X @ W.T + (X @ A.T) @ B.T

    def bwd_no_scale_dA(W, X, dH, A, B, a, r):
        dX, dA, dB = O.lora_backward(W, X, dH, A, B, a, r)
        return dX, dA / s(a, r), dB

    def bwd_dx_no_adapter(W, X, dH, A, B, a, r):
        dX, dA, dB = O.lora_backward(W, X, dH, A, B, a, r)
        return dH @ W, dA, dB

    def bwd_transposed_W(W, X, dH, A, B, a, r):
        dX, dA, dB = O.lora_backward(W, X, dH, A, B, a, r)
        return dX - dH @ W + dH @ W.T, dA, dB        # square case: W vs W^T

    def merge_noscale(W, A, B, a, r):
        return W + B @ A

    assert check_forward_brute(fwd_sign) > 1e-3
    assert check_forward_brute(fwd_noscale) > 1e-3
    assert check_gradients_fd(O.lora_forward, bwd_no_scale_dA) > 1e-3
    assert check_gradients_fd(O.lora_forward, bwd_dx_no_adapter) > 1e-3
    assert check_gradients_fd(O.lora_forward, bwd_transposed_W) > 1e-3
    assert check_merge(O.lora_forward, merge_noscale) > 1e-3

    def adam_no_bias_correction(w, g, m, v, t, lr, beta1, beta2, eps, weight_decay, grad_scale=1.0):
        m = beta1 * m + (1 - beta1) * g
        v = beta2 * v + (1 - beta2) * g * g
        return w * (1 - lr * weight_decay) - lr * m / (np.sqrt(v) + eps), m, v

    def adam_coupled_decay(w, g, m, v, t, lr, beta1, beta2, eps, weight_decay, grad_scale=1.0):
        return O.adamw_step(w, g + weight_decay * w, m, v, t, lr, beta1, beta2, eps, 0.0)

    def adam_swapped_betas(w, g, m, v, t, lr, beta1, beta2, eps, weight_decay, grad_scale=1.0):
        return O.adamw_step(w, g, m, v, t, lr, beta2, beta1, eps, weight_decay)

    assert check_adamw_first_step(adam_no_bias_correction) > 1e-3
    assert check_adamw_decay_only(adam_coupled_decay) > 1e-3
    assert check_adamw_first_step(adam_swapped_betas) > 1e-3

    def dora_no_adapter_in_norm(W, X, A, B, a, r, mag):
        Wa = W + s(a, r) * (B @ A)
        return X @ ((mag / np.sqrt(np.sum(W * W, axis=1)))[:, None] * Wa).T

    def dora_column_norms(W, X, A, B, a, r, mag):
        Wa = W + s(a, r) * (B @ A)
        return X @ (mag[:, None] * Wa / np.sqrt(np.sum(Wa * Wa, axis=0))[None, :]).T

    assert check_dora_brute(dora_no_adapter_in_norm) > 1e-3
    assert check_dora_brute(dora_column_norms) > 1e-3

    def dora_bwd_detached_norm(W, X, dH, A, B, a, r, mag):
        # the norm treated as a constant: its term dropped from dA, dB
        dX, dA, dB, dm = O.dora_backward(W, X, dH, A, B, a, r, mag)
        V = W + s(a, r) * (B @ A)
        n = np.sqrt(np.sum(V * V, axis=1))
        dZ = dH * (mag / n)[None, :]
        return dX, s(a, r) * (B.T @ (dZ.T @ X)), s(a, r) * ((dZ.T @ X) @ A.T), dm

    def dora_bwd_unscaled_dX(W, X, dH, A, B, a, r, mag):
        dX, dA, dB, dm = O.dora_backward(W, X, dH, A, B, a, r, mag)
        return dH @ (W + s(a, r) * (B @ A)), dA, dB, dm

    assert check_dora_gradients_fd(dora_bwd_detached_norm) > 1e-3
    assert check_dora_gradients_fd(dora_bwd_unscaled_dX) > 1e-3

    # FP8 mutants: ties away from zero, truncation, no saturation, a scale one power off,
    # the weight scale dropped, the low-rank branch fed the scaled activation
    def enc_ties_away(x):
        a = np.abs(np.asarray(x, np.float32).astype(np.float64))
        pos = O.e4m3_decode(np.arange(127, dtype=np.uint8))
        hi = np.minimum(np.searchsorted(pos, a), 126)
        lo = np.maximum(hi - 1, 0)
        pick = np.where(a - pos[lo] < pos[hi] - a, lo, hi)
        pick = np.where(a >= 448.0, 126, pick)
        return (pick.astype(np.uint8) | np.where(np.signbit(np.asarray(x, np.float32)), 0x80, 0)).astype(np.uint8)

    def enc_truncate(x):
        a = np.abs(np.asarray(x, np.float32).astype(np.float64))
        pos = O.e4m3_decode(np.arange(127, dtype=np.uint8))
        pick = np.maximum(np.searchsorted(pos, a, side="right") - 1, 0)
        return (pick.astype(np.uint8) | np.where(np.signbit(np.asarray(x, np.float32)), 0x80, 0)).astype(np.uint8)

    def enc_no_saturation(x):
        c = O.e4m3_encode(x)
        a = np.abs(np.asarray(x, np.float32))
        return np.where(a >= 464.0, c | 0x7F, c).astype(np.uint8)

    assert check_e4m3_encode(enc_ties_away) > 0
    assert check_e4m3_encode(enc_truncate) > 0
    assert check_e4m3_encode(enc_no_saturation) > 0
    assert check_pow2_scale(lambda a: 2.0 * O.fp8_pow2_scale(a)) > 0
    assert check_pow2_scale(lambda a: 0.5 * O.fp8_pow2_scale(a)) > 0

    def fwd8_no_wscale(X8, sx, W8, sw, A, B, a, r):
        return O.lora_forward_fp8(X8, sx, W8, 1.0, A, B, a, r)

    def fwd8_scaled_act_in_adapter(X8, sx, W8, sw, A, B, a, r):
        return O.lora_forward_fp8(X8, sx, W8, sw, A, B, a, r) + s(a, r) * (
            ((O.e4m3_decode(X8) - O.e4m3_decode(X8) / sx) @ np.asarray(A).T) @ np.asarray(B).T)

    def fwd8_transposed(X8, sx, W8, sw, A, B, a, r):
        H = O.lora_forward_fp8(X8, sx, W8, sw, A, B, a, r)
        return H[::-1]

    def enc5_ties_away(x):
        a = np.abs(np.asarray(x, np.float32).astype(np.float64))
        pos = O.e5m2_decode(np.arange(124, dtype=np.uint8))
        hi = np.minimum(np.searchsorted(pos, a), 123)
        lo = np.maximum(hi - 1, 0)
        pick = np.where(a - pos[lo] < pos[hi] - a, lo, hi)
        pick = np.where(a >= 57344.0, 123, pick)
        return (pick.astype(np.uint8) | np.where(np.signbit(np.asarray(x, np.float32)), 0x80, 0)).astype(np.uint8)

    assert check_e5m2_encode(enc5_ties_away) > 0

    def bwd8_no_gscale(X8, sx, G8, sg, W8, sw, A, B, a, r):
        dX, dA, dB = O.lora_backward_fp8(X8, sx, G8, sg, W8, sw, A, B, a, r)
        return dX * sg, dA, dB

    def bwd8_scaled_x_in_dA(X8, sx, G8, sg, W8, sw, A, B, a, r):
        dX, dA, dB = O.lora_backward_fp8(X8, sx, G8, sg, W8, sw, A, B, a, r)
        return dX, dA * sx, dB

    def bwd8_no_adapter_in_dX(X8, sx, G8, sg, W8, sw, A, B, a, r):
        dX, dA, dB = O.lora_backward_fp8(X8, sx, G8, sg, W8, sw, A, B, a, r)
        G = (O.e5m2_decode(G8) / sg) @ np.asarray(B)
        return dX - s(a, r) * (G @ np.asarray(A)), dA, dB

    for m in (bwd8_no_gscale, bwd8_scaled_x_in_dA, bwd8_no_adapter_in_dX):
        assert check_fp8_backward_loops(m) > 1e-3
        assert check_fp8_backward_bound(m) > 0.0

    for m in (fwd8_no_wscale, fwd8_scaled_act_in_adapter, fwd8_transposed):
        assert check_fp8_forward_bound(m) > 0.0
    assert check_fp8_forward_loops(fwd8_no_wscale) > 1e-3

    # quantizer mutants run through the round-trip and second-level pins: a packer that puts
    # element 2j in the high nibble, and a second stage coded on 255 steps instead of 127
    def quantize_swapped_nibbles(W):
        codes, q8, c2, c1 = O.nf4_quantize(W)
        return ((codes >> 4) | (codes << 4)).astype(np.uint8), q8, c2, c1

    def quantize_255(W):
        codes, q8, c2, c1 = O.nf4_quantize(W)
        c2b = np.repeat(c2, 256)[:c1.size]
        ratio = (c1 / np.where(c2b > 0, c2b, np.float32(1))).astype(np.float32)
        q = np.clip(np.rint((ratio * np.float32(255)).astype(np.float32)), 0, 255).astype(np.uint8)
        return codes, q, c2, c1

    assert check_round_trip(quantize_swapped_nibbles) > 0
    assert check_double_quant(quantize_255) > 0
    assert check_round_trip(quantize_255) > 0

# ------------------------------------------------------------------ helpers of the level table and the encoder


def test_normal_cdf_matches_library_routine():
    """Phi against scipy's ndtr (an independent implementation of the standard normal CDF) over
    the range the level table uses, and its exact symmetry Phi(-x) = 1 - Phi(x)."""
    from scipy.special import ndtr
    xs = np.linspace(-4.0, 4.0, 801)
    got = np.array([O.normal_cdf(float(x)) for x in xs])
    assert np.max(np.abs(got - ndtr(xs))) <= 1e-15
    assert np.max(np.abs(got + got[::-1] - 1.0)) <= 1e-15
    assert O.normal_cdf(0.0) == 0.5


def test_midpoints_separate_the_levels():
    """The 15 decision thresholds lie strictly between neighbouring levels and each is within one
    fp32 ulp of the exact midpoint."""
    L = O.nf4_levels()
    m = O.nf4_midpoints(L)
    assert m.shape == (15,) and m.dtype == np.float32
    assert np.all(L[:-1] < m) and np.all(m < L[1:])
    exact = (L[:-1].astype(np.float64) + L[1:].astype(np.float64)) / 2.0
    assert np.all(np.abs(m.astype(np.float64) - exact) <= np.spacing(np.abs(m)).astype(np.float64))


def test_codes_of_normalised_are_nearest_levels_by_brute_force():
    """The threshold encoder against an exhaustive nearest-level search: on a dense grid of [-1, 1]
    plus every threshold and its fp32 neighbours, the code is the index of the nearest level,
    and a value exactly on a threshold takes the upper level (the stated tie rule)."""
    L = O.nf4_levels()
    m = O.nf4_midpoints(L)
    grid = np.linspace(-1.0, 1.0, 20001, dtype=np.float32)
    near = np.concatenate([m, np.nextafter(m, np.float32(-2)), np.nextafter(m, np.float32(2))])
    xs = np.concatenate([grid, near]).astype(np.float32)
    got = O.nf4_codes_of_normalised(xs, m)
    dist = np.abs(xs[:, None].astype(np.float64) - L[None, :].astype(np.float64))
    best = np.argmin(dist, axis=1)
    # where the two nearest fp64 distances are too close to order (x a few ulps from a
    # threshold), decide with exact rational arithmetic
    from fractions import Fraction
    srt = np.sort(dist, axis=1)
    for i in np.nonzero(srt[:, 1] - srt[:, 0] < 1e-12)[0]:
        x = Fraction(float(xs[i]))
        best[i] = min(range(16), key=lambda j: (abs(x - Fraction(float(L[j]))), j))
    off = ~np.isin(xs, m)                      # away from a threshold: the unique nearest level
    assert np.array_equal(got[off], best[off].astype(np.uint8))
    on = np.searchsorted(m, m)                 # exactly on threshold i: the upper level i + 1
    assert np.array_equal(O.nf4_codes_of_normalised(m, m), (on + 1).astype(np.uint8))

"""CUDA path (through the C ABI) against the CPU oracle, element by element.

Integer / byte outputs (NF4 codes, absmax bytes, c2, decoded weights) must be bit-exact;
H, dX, dA, dB must be within a relative Frobenius error of 5e-3 (bf16) or 1e-5 (fp32).
Small cases span several 128x256 tiles with ragged tails in T, d_out, d_in and r; the
full-size Llama-2-7B q_proj case is checked on sampled token rows (H, dX) and in full
(dA, dB, decode).
"""
import os

import numpy as np
import pytest

import oracle as O
from qlora_parameter_efficient_b200 import synthetic as S

from parity import TOL, dev, host, oracle_weight, quantize_both, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from qlora_parameter_efficient_b200 import build
    build.build_library()
    import qlora_parameter_efficient_b200 as lib
    lib.load()
    return lib


# ------------------------------------------------------------------ NF4 storage


@pytest.mark.parametrize("d_out,d_in", [(8, 64), (3, 128), (64, 256), (256, 4096), (100, 1088)])
def test_quantize_bit_exact(q, d_out, d_in):
    rng = np.random.default_rng(d_out * 7 + d_in)
    W = (rng.standard_normal((d_out, d_in)) * 0.141).astype(np.float32)
    W[0, :64] = 0.0                      # an all-zero block
    W[-1, -1] = -3.0                      # one large block
    w = q.nf4_quantize(dev(W))
    codes, q8, c2, _ = O.nf4_quantize(W)
    assert np.array_equal(w.codes.cpu().numpy(), codes)
    assert np.array_equal(w.absmax_q.cpu().numpy(), q8)
    assert np.array_equal(w.c2.cpu().numpy().view(np.uint32), c2.view(np.uint32))


def test_quantize_bf16_input_bit_exact(q):
    import torch
    rng = np.random.default_rng(11)
    W = S.round_to_bf16((rng.standard_normal((96, 512)) * 0.141).astype(np.float32))
    w = q.nf4_quantize(dev(W, "bf16"))
    codes, q8, c2, _ = O.nf4_quantize(W)
    assert w.codes.dtype == torch.uint8
    assert np.array_equal(w.codes.cpu().numpy(), codes)
    assert np.array_equal(w.absmax_q.cpu().numpy(), q8)
    assert np.array_equal(w.c2.cpu().numpy(), c2)


@pytest.mark.parametrize("d_out,d_in", [(16, 64), (200, 192), (4096, 4096)])
def test_dequantize_bit_exact(q, d_out, d_in):
    import torch
    rng = np.random.default_rng(d_out + d_in)
    W = (rng.standard_normal((d_out, d_in)) * 0.141).astype(np.float32)
    W[1, :64] = 0.0
    w, oc = quantize_both(q, W)
    for dt, tdt in (("bf16", torch.bfloat16), ("f32", torch.float32)):
        got = host(q.nf4_dequantize(w, tdt))
        ref = O.nf4_dequantize(*oc[:3], d_out, d_in, out=dt)
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), dt


# ------------------------------------------------------------------ single-adapter layer


def run_layer(q, case, rows=None):
    """Run fwd + bwd on the GPU and compare with the oracle.  rows: sampled token rows for
    H and dX (None: all)."""
    import torch
    d_out, d_in, r, T, dt = case.d_out, case.d_in, case.r, case.T, case.dtype
    w, oc = quantize_both(q, case.W0)
    Wh = oracle_weight(oc, d_out, d_in, dt)
    X, A, B, dH = dev(case.X, dt), dev(case.A, dt), dev(case.B, dt), dev(case.dH, dt)
    H, U = q.qlora_linear_fwd(w, X, A, B, case.alpha)
    dX, dA, dB = q.qlora_linear_bwd(w, X, dH, A, B, case.alpha, U_saved=U)
    _, dA2, dB2 = q.qlora_linear_bwd(w, X, dH, A, B, case.alpha, U_saved=None, want_dx=False)
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    sel = slice(None) if rows is None else rows
    Href = O.lora_forward(Wh, case.X[sel], case.A, case.B, case.alpha, r)
    err = {"H": rel_fro(host(H)[sel], Href)}
    Uref = case.X.astype(np.float64) @ case.A.astype(np.float64).T
    err["U"] = rel_fro(host(U)[sel], Uref[sel])
    dXref, _, _ = O.lora_backward(Wh, case.X[sel], case.dH[sel], case.A, case.B, case.alpha, r)
    err["dX"] = rel_fro(host(dX)[sel], dXref)
    dAref, dBref = O.lora_adapter_grads(case.X, case.dH, case.A, case.B, case.alpha, r)
    err["dA"] = rel_fro(host(dA), dAref)
    err["dB"] = rel_fro(host(dB), dBref)
    err["dA_recomputedU"] = rel_fro(host(dA2), dAref)
    err["dB_recomputedU"] = rel_fro(host(dB2), dBref)
    tol = TOL[dt]
    bad = {k: v for k, v in err.items() if not v <= tol}
    assert not bad, f"{err} (tol {tol})"
    return err


SMALL = [
    # d_out, d_in, r, T   (several 128x256 tiles and ragged tails in every dimension)
    (256, 256, 8, 64),
    (200, 192, 5, 77),
    (64, 64, 1, 1),
    (520, 320, 16, 300),
    (256, 512, 64, 129),
    (136, 256, 100, 50),
    (1024, 1024, 128, 256),
    (768, 640, 33, 1000),
]


@pytest.mark.parametrize("d_out,d_in,r,T", SMALL)
def test_layer_bf16_small(q, d_out, d_in, r, T):
    case = S.make_layer(d_out, d_in, r, 2.0 * r, T, dtype="bf16", seed=d_out + T)
    run_layer(q, case)


# Shapes whose fused-GEMM tile count leaves a short last wave on 74 SM pairs, so that wave's
# tiles are split in two along K and reduced through the fp32 partial workspace:
#   (2048, 2048, 16, 2560): 80 tiles in forward and dX (6 split);
#   (3272, 640, 7, 1500): forward 78 tiles (4 split, ragged columns and rows);
#   (1000, 3264, 9, 1500): dX 78 tiles (4 split, ragged columns), ragged K = 1000.
@pytest.mark.parametrize("d_out,d_in,r,T", [(2048, 2048, 16, 2560), (3272, 640, 7, 1500),
                                            (1000, 3264, 9, 1500)])
def test_layer_bf16_split_tail(q, d_out, d_in, r, T):
    case = S.make_layer(d_out, d_in, r, 2.0 * r, T, dtype="bf16", seed=d_in + r)
    run_layer(q, case)


# d_out that is not a multiple of 8: the output rows are not whole 16-byte units (the GEMM
# epilogues store element by element) and the backward copies dH into padded rows for its tensor
# maps.  Token counts take the large-T route (300, 1030), the mid-size split-K route (40) and the
# decode-size stream (1, 5, 12).
@pytest.mark.parametrize("d_out,d_in,r,T", [(100, 256, 16, 300), (203, 320, 5, 1030), (203, 512, 8, 40),
                                            (100, 512, 16, 1), (203, 1024, 33, 5), (1001, 4096, 64, 12),
                                            (77, 192, 3, 130)])
def test_layer_bf16_ragged_d_out(q, d_out, d_in, r, T):
    case = S.make_layer(d_out, d_in, r, 2.0 * r, T, dtype="bf16", seed=d_out + T)
    run_layer(q, case)


@pytest.mark.parametrize("d_out,d_in,r,T", [(256, 256, 8, 64), (200, 192, 5, 77), (64, 128, 3, 1)])
def test_layer_f32(q, d_out, d_in, r, T):
    case = S.make_layer(d_out, d_in, r, 2.0 * r, T, dtype="f32", seed=3)
    run_layer(q, case)


def test_small_fp32_config(q):
    case = S.make_layer(**S.CONFIGS["small_256_r8_T64_f32"], seed=0)
    run_layer(q, case)


def test_q_proj_full_size_sampled_rows(q):
    case = S.make_layer(**S.CONFIGS["q_proj_4096x4096_r16_T4096"], seed=0)
    rows = np.sort(np.random.default_rng(0).choice(case.T, 256, replace=False))
    run_layer(q, case, rows=rows)


# The remaining full-size configurations: Llama-2-7B MLP up/gate (11008x4096, r = 64, 8192
# tokens) and the 70B-class projections (8192x8192 and 28672x8192, r = 16, 2048 and 16384
# tokens), forward and backward; H and dX on 256 sampled token rows, dA and dB in full.  The
# oracle's quantization and decode of a shape are shared by its two token counts (the weight is
# the first draw of the seed).
FULL_CONFIGS = ["mlp_up_11008x4096_r64_T8192", "proj70b_8192x8192_r16_T2048", "proj70b_8192x8192_r16_T16384",
                "proj70b_28672x8192_r16_T2048", "proj70b_28672x8192_r16_T16384"]
_ORACLE_W = {}


def oracle_weight_cached(case, seed):
    key = (case.d_out, case.d_in, seed)
    if key not in _ORACLE_W:
        _ORACLE_W.clear()
        oc = O.nf4_quantize(case.W0)
        _ORACLE_W[key] = oracle_weight(oc, case.d_out, case.d_in, "bf16")
    return _ORACLE_W[key]


@pytest.mark.parametrize("name", FULL_CONFIGS)
def test_config_full_size_sampled_rows(q, name):
    import torch
    case = S.make_layer(**S.CONFIGS[name], seed=0)
    Wh = oracle_weight_cached(case, 0)
    w = q.nf4_quantize(dev(case.W0))
    X, A, B, dH = dev(case.X, "bf16"), dev(case.A, "bf16"), dev(case.B, "bf16"), dev(case.dH, "bf16")
    H, U = q.qlora_linear_fwd(w, X, A, B, case.alpha)
    dX, dA, dB = q.qlora_linear_bwd(w, X, dH, A, B, case.alpha, U_saved=U)
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    rows = np.sort(np.random.default_rng(1).choice(case.T, 256, replace=False))
    ridx = torch.from_numpy(rows).cuda()
    Href = O.lora_forward(Wh, case.X[rows], case.A, case.B, case.alpha, case.r)
    dXref, _, _ = O.lora_backward(Wh, case.X[rows], case.dH[rows], case.A, case.B, case.alpha, case.r)
    dAref, dBref = O.lora_adapter_grads(case.X, case.dH, case.A, case.B, case.alpha, case.r)
    err = {"H": rel_fro(host(H[ridx]), Href), "dX": rel_fro(host(dX[ridx]), dXref),
           "dA": rel_fro(host(dA), dAref), "dB": rel_fro(host(dB), dBref)}
    assert all(v <= TOL["bf16"] for v in err.values()), err


@pytest.mark.parametrize("T", [3, 12])
def test_decode_size_70b_shape(q, T):
    # The 28672 x 8192 projection at decode sizes: 3 tokens (two ranks split K, 74 clusters of
    # 24-25 tiles, the tile sums kept for the end phase) and 12 tokens (four ranks, 37 clusters of
    # 48-49 tiles: more than the end phase keeps, so every finaliser finishes its tile at once).
    # Runs right after the full-size cases so that the oracle's decode of the weight is shared.
    import torch
    case = S.make_layer(**S.CONFIGS["proj70b_28672x8192_r16_T2048"], seed=0)
    Wh = oracle_weight_cached(case, 0)
    w = q.nf4_quantize(dev(case.W0))
    X, A, B = dev(case.X[:T], "bf16"), dev(case.A, "bf16"), dev(case.B, "bf16")
    H, U = q.qlora_linear_fwd(w, X, A, B, case.alpha)
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    ref = O.lora_forward(Wh, case.X[:T], case.A, case.B, case.alpha, case.r)
    assert rel_fro(host(H), ref) <= TOL["bf16"]
    assert rel_fro(host(U), case.X[:T].astype(np.float64) @ case.A.astype(np.float64).T) <= TOL["bf16"]


# ------------------------------------------------------------------ decode-size forward


@pytest.mark.parametrize("d_out,d_in,r,T", [
    (136, 192, 5, 1),        # d_in/64 not a multiple of 4: the large-T path
    (520, 320, 16, 4),
    (1000, 512, 64, 16),     # ragged last 16-row tile
    (264, 640, 33, 17),
    (2048, 1024, 128, 32),   # 32-token tile
    (264, 4352, 33, 3),      # 68 blocks per row: K split over a cluster, uneven ranks; r % 8 != 0
    (2056, 1024, 16, 24),    # 32-token tile, ragged rows
    (4096, 4096, 16, 1),     # q_proj shape
    (4096, 4096, 16, 8),
    (4096, 4096, 16, 12),    # 9..16 tokens: two ranks split K
    (1032, 11008, 1, 2),     # 172 blocks per row: three ranks, the last one partly idle; r = 1
    (4104, 8192, 100, 13),   # four ranks; r even but not a multiple of 8
    (528, 2048, 128, 9),     # the largest rank
])
def test_decode_size_forward(q, d_out, d_in, r, T):
    import torch
    case = S.make_layer(d_out, d_in, r, 2.0 * r, T, dtype="bf16", seed=T + d_out, with_grad=False)
    w, oc = quantize_both(q, case.W0)
    Wh = oracle_weight(oc, d_out, d_in, "bf16")
    H, U = q.qlora_linear_fwd(w, dev(case.X, "bf16"), dev(case.A, "bf16"), dev(case.B, "bf16"), case.alpha)
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    ref = O.lora_forward(Wh, case.X, case.A, case.B, case.alpha, r)
    e = rel_fro(host(H), ref)
    eu = rel_fro(host(U), case.X.astype(np.float64) @ case.A.astype(np.float64).T)
    assert e <= TOL["bf16"] and eu <= TOL["bf16"], (e, eu)


@pytest.mark.parametrize("T", [1, 4, 16])
def test_decode_size_mlp_shape(q, T):
    import torch
    c = S.CONFIGS["mlp_up_11008x4096_r64_T8192"]
    case = S.make_layer(c["d_out"], c["d_in"], c["r"], c["alpha"], T, dtype="bf16", seed=7, with_grad=False)
    w, oc = quantize_both(q, case.W0)
    Wh = oracle_weight(oc, c["d_out"], c["d_in"], "bf16")
    H, _ = q.qlora_linear_fwd(w, dev(case.X, "bf16"), dev(case.A, "bf16"), dev(case.B, "bf16"), case.alpha)
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    ref = O.lora_forward(Wh, case.X, case.A, case.B, case.alpha, c["r"])
    assert rel_fro(host(H), ref) <= TOL["bf16"]
    # the same call again (tile counters and partials are reused)
    H2, _ = q.qlora_linear_fwd(w, dev(case.X, "bf16"), dev(case.A, "bf16"), dev(case.B, "bf16"), case.alpha)
    torch.cuda.synchronize()
    assert torch.equal(H, H2)


# ------------------------------------------------------------------ invariants on the GPU


def test_zero_B_gives_base_output_bitwise(q):
    # With B = 0 the adapter K-steps add exact zeros, so H(B=0, A) == H(A=0, B') bit for bit.
    import torch
    case = S.make_layer(384, 512, 16, 32.0, 200, dtype="bf16", seed=5)
    w = q.nf4_quantize(dev(case.W0))
    X, A, B = dev(case.X, "bf16"), dev(case.A, "bf16"), dev(case.B, "bf16")
    H1, _ = q.qlora_linear_fwd(w, X, A, torch.zeros_like(B), 32.0)
    H2, _ = q.qlora_linear_fwd(w, X, torch.zeros_like(A), B, 32.0)
    assert torch.equal(H1, H2)
    Wh = oracle_weight(O.nf4_quantize(case.W0), 384, 512, "bf16")
    assert rel_fro(host(H1), case.X.astype(np.float64) @ Wh.T) <= TOL["bf16"]


@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_merge(q, out):
    import torch
    case = S.make_layer(520, 384, 16, 32.0, 64, dtype="bf16", seed=9)
    w, oc = quantize_both(q, case.W0)
    A, B = dev(case.A, "bf16"), dev(case.B, "bf16")
    Wf = q.lora_merge(w, A, B, 32.0, torch.bfloat16 if out == "bf16" else torch.float32)
    Wh = oracle_weight(oc, 520, 384, out)
    ref = O.lora_merge(Wh, case.A, case.B, 32.0, 16)
    assert rel_fro(host(Wf), ref) <= TOL[out]
    # the merged weight reproduces the unmerged layer output
    H, _ = q.qlora_linear_fwd(w, dev(case.X, "bf16"), A, B, 32.0)
    Hm = case.X.astype(np.float64) @ host(Wf).astype(np.float64).T
    assert rel_fro(host(H), Hm) <= TOL["bf16"]


# Tensor-core merge (bf16 adapters): ragged rows, d_in not a multiple of the 128-column tile,
# ranks that are not multiples of 16 (zero-padded K), the largest rank, and the full q_proj size.
@pytest.mark.parametrize("d_out,d_in,r", [(200, 192, 5), (136, 320, 33), (72, 64, 1),
                                          (256, 1088, 128), (4096, 4096, 16)])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_merge_shapes(q, d_out, d_in, r, out):
    import torch
    case = S.make_layer(d_out, d_in, r, 2.0 * r, 1, dtype="bf16", seed=d_out + r, with_grad=False)
    w, oc = quantize_both(q, case.W0)
    Wf = q.lora_merge(w, dev(case.A, "bf16"), dev(case.B, "bf16"), 2.0 * r,
                      torch.bfloat16 if out == "bf16" else torch.float32)
    ref = O.lora_merge(oracle_weight(oc, d_out, d_in, out), case.A, case.B, 2.0 * r, r)
    assert rel_fro(host(Wf), ref) <= TOL[out]


def test_merge_f32_adapters(q):
    import torch
    case = S.make_layer(256, 256, 8, 16.0, 16, dtype="f32", seed=2)
    w, oc = quantize_both(q, case.W0)
    Wf = q.lora_merge(w, dev(case.A), dev(case.B), 16.0, torch.float32)
    ref = O.lora_merge(oracle_weight(oc, 256, 256, "f32"), case.A, case.B, 16.0, 8)
    assert rel_fro(host(Wf), ref) <= TOL["f32"]


# ------------------------------------------------------------------ multi-adapter


def run_batched(q, mc, rows=None):
    import torch
    w, oc = quantize_both(q, mc.W0)
    Wh = oracle_weight(oc, mc.d_out, mc.d_in, mc.dtype)
    X = dev(mc.X, mc.dtype)
    ids = torch.from_numpy(mc.ids).to("cuda")
    As = [dev(a, mc.dtype) for a in mc.As]
    Bs = [dev(b, mc.dtype) for b in mc.Bs]
    H = q.qlora_linear_fwd_batched(w, X, ids, As, Bs, mc.alphas)
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    sel = slice(None) if rows is None else rows
    ref = O.lora_forward_batched(Wh, mc.X[sel], mc.ids[sel], mc.As, mc.Bs, mc.alphas, mc.ranks)
    e = rel_fro(host(H)[sel], ref)
    assert e <= TOL[mc.dtype], e


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_batched_small(q, dtype):
    mc = S.make_multi_adapter(264, 320, 150, [3, 8, 20], dtype=dtype, seed=4)
    run_batched(q, mc)


def test_batched_ragged_d_out(q):
    mc = S.make_multi_adapter(203, 320, 150, [3, 8, 20], dtype="bf16", seed=18)
    run_batched(q, mc)


def test_batched_full_uniform_and_skewed(q):
    for split in (None, [0.7, 0.1, 0.1, 0.1]):
        mc = S.make_multi_adapter(4096, 4096, 4096, [8, 16, 16, 64], split=split, seed=0)
        rows = np.sort(np.random.default_rng(1).choice(4096, 256, replace=False))
        run_batched(q, mc, rows=rows)


# ------------------------------------------------------------------ many-adapter (segmented) forward


def run_multi(q, mc, rows=None):
    import torch
    w, oc = quantize_both(q, mc.W0)
    Wh = oracle_weight(oc, mc.d_out, mc.d_in, "bf16")
    tab = q.AdapterTable([dev(a, "bf16") for a in mc.As], [dev(b, "bf16") for b in mc.Bs], mc.alphas)
    H = q.qlora_linear_fwd_multi(w, dev(mc.X, "bf16"), torch.from_numpy(mc.ids).cuda(), tab)
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    sel = slice(None) if rows is None else rows
    ref = O.lora_forward_batched(Wh, mc.X[sel], mc.ids[sel], mc.As, mc.Bs, mc.alphas, mc.ranks)
    e = rel_fro(host(H)[sel], ref)
    assert e <= TOL["bf16"], e
    return H


# mixed ranks 1..128 (odd ranks take the 16-bit B path, r > 64 two K tiles), ragged shapes
def test_multi_mixed_ranks(q):
    mc = S.make_multi_adapter(264, 320, 300, [1, 3, 8, 16, 33, 64, 100, 128, 7, 24], seed=11)
    run_multi(q, mc)


# odd and non-multiple-of-8 output widths: rows of H are not whole bf16 pairs / 16-byte units
@pytest.mark.parametrize("d_out", [203, 100])
def test_multi_ragged_d_out(q, d_out):
    mc = S.make_multi_adapter(d_out, 256, 150, [5, 16, 64], seed=17 + d_out)
    run_multi(q, mc)


# a thousand adapters, about two tokens each (many partial tiles, some empty segments)
def test_multi_many_adapters(q):
    mc = S.make_multi_adapter(512, 512, 2048, [8, 16, 32, 64] * 250, seed=12)
    run_multi(q, mc)


# one adapter with most tokens (many full 16-token tiles of one segment)
def test_multi_skewed(q):
    mc = S.make_multi_adapter(384, 256, 1000, [16, 4, 64], split=[0.9, 0.05, 0.05], seed=13)
    run_multi(q, mc)


def test_multi_full_size_sampled_rows(q):
    mc = S.make_multi_adapter(4096, 4096, 4096, [16] * 256, seed=14)
    rows = np.sort(np.random.default_rng(2).choice(4096, 256, replace=False))
    run_multi(q, mc, rows=rows)


def test_multi_matches_single_adapter_path(q):
    # one adapter for every token: the same layer as qlora_linear_fwd, within bf16 rounding
    import torch
    mc = S.make_multi_adapter(256, 384, 96, [16], seed=15)
    w, _ = quantize_both(q, mc.W0)
    X, A, B = dev(mc.X, "bf16"), dev(mc.As[0], "bf16"), dev(mc.Bs[0], "bf16")
    H1, _ = q.qlora_linear_fwd(w, X, A, B, mc.alphas[0])
    Hm = q.qlora_linear_fwd_multi(w, X, torch.from_numpy(mc.ids).cuda(), q.AdapterTable([A], [B], mc.alphas))
    assert rel_fro(host(Hm), host(H1).astype(np.float64)) <= 4e-3


def test_multi_bad_id_and_rank_report_device_error(q):
    import torch
    mc = S.make_multi_adapter(128, 128, 40, [4, 4], seed=16)
    mc.ids[7] = 5
    mc.ids[9] = -1
    w, oc = quantize_both(q, mc.W0)
    tab = q.AdapterTable([dev(a, "bf16") for a in mc.As], [dev(b, "bf16") for b in mc.Bs], mc.alphas)
    H = q.qlora_linear_fwd_multi(w, dev(mc.X, "bf16"), torch.from_numpy(mc.ids).cuda(), tab)
    assert q.get_device_error() == 5
    assert q.get_device_error() == 0
    ok = np.array([i for i in range(40) if i not in (7, 9)])
    Wh = oracle_weight(oc, 128, 128, "bf16")
    ref = O.lora_forward_batched(Wh, mc.X[ok], mc.ids[ok], mc.As, mc.Bs, mc.alphas, mc.ranks)
    assert rel_fro(host(H)[ok], ref) <= TOL["bf16"]
    # the bad tokens get the base term only
    base = mc.X[[7, 9]].astype(np.float64) @ Wh.T
    assert rel_fro(host(H)[[7, 9]], base) <= TOL["bf16"]


def test_batched_bad_id_reports_device_error(q):
    import torch
    mc = S.make_multi_adapter(128, 128, 40, [4, 4], seed=6)
    mc.ids[7] = 5
    w = q.nf4_quantize(dev(mc.W0))
    H = q.qlora_linear_fwd_batched(w, dev(mc.X, "bf16"), torch.from_numpy(mc.ids).cuda(),
                                   [dev(a, "bf16") for a in mc.As], [dev(b, "bf16") for b in mc.Bs],
                                   mc.alphas)
    assert q.get_device_error() == 5
    assert q.get_device_error() == 0          # read-and-clear
    # the other tokens are still right
    Wh = oracle_weight(O.nf4_quantize(mc.W0), 128, 128, "bf16")
    keep = np.arange(40) != 7
    ref = O.lora_forward_batched(Wh, mc.X[keep], mc.ids[keep], mc.As, mc.Bs, mc.alphas, mc.ranks)
    assert rel_fro(host(H)[keep], ref) <= TOL["bf16"]


# ------------------------------------------------------------------ failure detection


def test_bounded_wait_times_out_and_context_survives(q):
    import torch
    q.selftest_wait_timeout(20_000_000)       # 20 ms
    assert q.get_device_error() == 4
    assert q.get_device_error() == 0
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0        # the context is still usable


def test_launch_counter_moves(q):
    import torch
    n0 = q.launch_count()
    case = S.make_layer(128, 128, 4, 8.0, 16, dtype="bf16", seed=1)
    w = q.nf4_quantize(dev(case.W0))
    q.qlora_linear_fwd(w, dev(case.X, "bf16"), dev(case.A, "bf16"), dev(case.B, "bf16"), 8.0)
    torch.cuda.synchronize()
    assert q.launch_count() - n0 >= 3          # quantize, U pre-pass, weight stream


# ------------------------------------------------------------------ training-step tail


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_bwd_accumulate_matches_full_batch(q, dtype):
    """Two micro-batches with QLORA_BWD_ACCUMULATE give the full batch's dA, dB."""
    import torch
    case = S.make_layer(192, 256, 8, 16.0, 160, dtype=dtype, seed=31)
    w, oc = quantize_both(q, case.W0)
    X, A, B, dH = dev(case.X, dtype), dev(case.A, dtype), dev(case.B, dtype), dev(case.dH, dtype)
    _, dA, dB = q.qlora_linear_bwd(w, X[:96], dH[:96], A, B, case.alpha, want_dx=False)
    q.qlora_linear_bwd(w, X[96:], dH[96:], A, B, case.alpha, dA=dA, dB=dB, want_dx=False, accumulate=True)
    _, dA_full, dB_full = q.qlora_linear_bwd(w, X, dH, A, B, case.alpha, want_dx=False)
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    dAref, dBref = O.lora_adapter_grads(case.X, case.dH, case.A, case.B, case.alpha, case.r)
    assert rel_fro(host(dA), dAref) <= TOL[dtype]
    assert rel_fro(host(dB), dBref) <= TOL[dtype]
    assert rel_fro(host(dA), host(dA_full).astype(np.float64)) <= 1e-5
    assert rel_fro(host(dB), host(dB_full).astype(np.float64)) <= 1e-5


@pytest.mark.parametrize("dtype,d_out,d_in,r,T", [("bf16", 192, 256, 8, 160), ("bf16", 203, 512, 5, 77),
                                                  ("bf16", 4096, 4096, 16, 512), ("f32", 192, 256, 8, 160)])
def test_split_backward_equals_one_call(q, dtype, d_out, d_in, r, T):
    """The grads-only phase then the dX-from-workspace phase give exactly the one-call results,
    and both match the oracle."""
    import torch
    case = S.make_layer(d_out, d_in, r, 2.0 * r, T, dtype=dtype, seed=37)
    w, oc = quantize_both(q, case.W0)
    X, A, B, dH = dev(case.X, dtype), dev(case.A, dtype), dev(case.B, dtype), dev(case.dH, dtype)
    dX1, dA1, dB1 = q.qlora_linear_bwd(w, X, dH, A, B, case.alpha)
    ws = torch.empty(q.workspace_bytes(q.OP_BWD, q.BF16 if dtype == "bf16" else q.F32, T, d_out, d_in, r),
                     dtype=torch.uint8, device="cuda")
    _, dA2, dB2 = q.qlora_linear_bwd(w, X, dH, A, B, case.alpha, ws=ws, phase="grads")
    dX2, dA_none, dB_none = q.qlora_linear_bwd(w, X, dH, A, B, case.alpha, ws=ws, phase="dx")
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    assert dA_none is None and dB_none is None
    assert torch.equal(dX1, dX2) and torch.equal(dA1, dA2) and torch.equal(dB1, dB2)
    dXref, dAref, dBref = O.lora_backward(oracle_weight(oc, d_out, d_in, dtype), case.X, case.dH, case.A,
                                          case.B, case.alpha, case.r)
    assert rel_fro(host(dX2), dXref) <= TOL[dtype]
    assert rel_fro(host(dA2), dAref) <= TOL[dtype]
    assert rel_fro(host(dB2), dBref) <= TOL[dtype]


# The API takes fp32 hyperparameters; the oracle gets the same (fp32-representable) values, since
# 1 - beta2 magnifies the fp32 rounding of beta2 = 0.999 to ~1e-5 relative.
HP = {k: float(np.float32(x)) for k, x in dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8,
                                                 weight_decay=0.01).items()}


def run_adam(q, n, param_dtype, steps=4, seed=41, grad_scale=0.5):
    """`steps` AdamW steps on the GPU and in the oracle; returns the GPU state and the errors."""
    import torch
    rng = np.random.default_rng(seed)
    w0 = rng.standard_normal(n).astype(np.float32)
    grads = [rng.standard_normal(n).astype(np.float32) for _ in range(steps)]
    mk = lambda a: torch.from_numpy(a).cuda()        # noqa: E731
    m, v = mk(np.zeros(n, np.float32)), mk(np.zeros(n, np.float32))
    if param_dtype == "bf16":
        master = mk(w0.copy())
        param = torch.from_numpy(w0).cuda().bfloat16()
    else:
        master, param = None, mk(w0.copy())
    g = torch.empty(n, dtype=torch.float32, device="cuda")
    wr, mr, vr = w0.astype(np.float64), np.zeros(n), np.zeros(n)
    for t in range(1, steps + 1):
        g.copy_(torch.from_numpy(grads[t - 1]))
        q.adamw_step(param, g, m, v, t, master=master, grad_scale=grad_scale, **HP)
        wr, mr, vr = O.adamw_step(wr, grads[t - 1], mr, vr, t, grad_scale=grad_scale, **HP)
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    wg = host(master if master is not None else param)
    err = (rel_fro(wg, wr), rel_fro(host(m), mr), rel_fro(host(v), vr))
    return param, master, m, v, err


@pytest.mark.parametrize("n", [4096, 1001])        # vector path and scalar path
@pytest.mark.parametrize("param_dtype", ["bf16", "f32"])
def test_adamw_matches_oracle(q, n, param_dtype):
    import torch
    param, master, m, v, err = run_adam(q, n, param_dtype)
    assert max(err) <= 1e-6, err
    if param_dtype == "bf16":
        # the bf16 parameter is the RN-even copy of the fp32 master, bit for bit
        assert torch.equal(param, master.bfloat16())


def test_adamw_state_in_unified_memory(q):
    """Optimizer state in cudaMallocManaged memory ("paged optimizers"), paged to the GPU
    before each step and back to the host after: bit-identical to device-resident state."""
    import ctypes, torch
    import ctypes.util
    torch.zeros(1, device="cuda")           # torch's CUDA runtime is loaded from here on
    # the CUDA runtime this process already has mapped (torch's), else the loader's choice
    names = []
    with open("/proc/self/maps") as f:
        for line in f:
            path = line.split()[-1]
            if "libcudart" in os.path.basename(path) and path not in names:
                names.append(path)
    names += [n for n in (ctypes.util.find_library("cudart"), "libcudart.so.12", "libcudart.so") if n]
    rt = None
    for name in names:
        try:
            rt = ctypes.CDLL(name)
            break
        except OSError:
            continue
    if rt is None:
        pytest.skip("no CUDA runtime library to allocate unified memory with")
    rt.cudaMallocManaged.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_size_t, ctypes.c_uint]
    rt.cudaFree.argtypes = [ctypes.c_void_p]
    bufs = []

    def alloc(a):
        p = ctypes.c_void_p()
        assert rt.cudaMallocManaged(ctypes.byref(p), a.nbytes, 1) == 0
        bufs.append(p)
        arr = np.ctypeslib.as_array(ctypes.cast(p, ctypes.POINTER(ctypes.c_float)), shape=a.shape)
        arr[...] = a
        t = torch.from_numpy(arr)            # host view; the kernels take its address
        return _ManagedTensor(t, p.value)

    class _ManagedTensor:
        """Float32 unified-memory array: a host view plus the address the kernels take."""

        def __init__(self, t, addr):
            self.t, self.addr = t, addr
            self.dtype, self.shape = torch.float32, t.shape

        def data_ptr(self):
            return self.addr

        def numel(self):
            return self.t.numel()

        def is_contiguous(self):
            return True

        def prefetch(self, to_device):
            q.prefetch(self.addr, self.t.numel() * 4, to_device)

    try:
        n = 8192
        rng = np.random.default_rng(42)
        w0 = rng.standard_normal(n).astype(np.float32)
        grads = [rng.standard_normal(n).astype(np.float32) for _ in range(3)]
        mm, vm, wm = alloc(np.zeros(n, np.float32)), alloc(np.zeros(n, np.float32)), alloc(w0.copy())
        md, vd, wd = (torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda"),
                      torch.from_numpy(w0.copy()).cuda())
        pm, pd = torch.from_numpy(w0).cuda().bfloat16(), torch.from_numpy(w0).cuda().bfloat16()
        g = torch.empty(n, dtype=torch.float32, device="cuda")
        for t in range(1, 4):
            g.copy_(torch.from_numpy(grads[t - 1]))
            for s in (mm, vm, wm):
                s.prefetch(True)
            q.adamw_step(pm, g, mm, vm, t, master=wm, **HP)
            for s in (mm, vm, wm):
                s.prefetch(False)
            q.adamw_step(pd, g, md, vd, t, master=wd, **HP)
        torch.cuda.synchronize()
        assert q.get_device_error() == 0
        assert np.array_equal(mm.t.numpy(), md.cpu().numpy())
        assert np.array_equal(vm.t.numpy(), vd.cpu().numpy())
        assert np.array_equal(wm.t.numpy(), wd.cpu().numpy())
        assert torch.equal(pm, pd)
    finally:
        torch.cuda.synchronize()
        for p in bufs:
            rt.cudaFree(p)


# ------------------------------------------------------------------ DoRA (R24)


@pytest.mark.parametrize("d_out,d_in,r", [(200, 192, 5), (264, 320, 16), (256, 1088, 128)])
def test_dora_row_norms(q, d_out, d_in, r):
    import torch
    case = S.make_layer(d_out, d_in, r, 2.0 * r, 1, dtype="bf16", seed=d_out + r, with_grad=False)
    w, oc = quantize_both(q, case.W0)
    n = q.dora_row_norms(w, dev(case.A, "bf16"), dev(case.B, "bf16"), 2.0 * r)
    torch.cuda.synchronize()
    ref = O.dora_row_norms(oracle_weight(oc, d_out, d_in, "bf16"), case.A, case.B, 2.0 * r, r)
    assert rel_fro(host(n), ref) <= 1e-5


def run_dora(q, case, rows=None, seed=0):
    import torch
    w, oc = quantize_both(q, case.W0)
    Wh = oracle_weight(oc, case.d_out, case.d_in, "bf16")
    mag = np.random.default_rng(seed).uniform(0.5, 2.0, case.d_out).astype(np.float32)
    H, U = q.qlora_dora_fwd(w, dev(case.X, "bf16"), dev(case.A, "bf16"), dev(case.B, "bf16"),
                            case.alpha, torch.from_numpy(mag).cuda())
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    sel = slice(None) if rows is None else rows
    ref = O.dora_forward(Wh, case.X[sel], case.A, case.B, case.alpha, case.r, mag)
    assert rel_fro(host(H)[sel], ref) <= TOL["bf16"]
    return w, H


@pytest.mark.parametrize("d_out,d_in,r,T", [(256, 256, 8, 64), (200, 192, 5, 77), (520, 320, 16, 300),
                                            (136, 256, 100, 3), (203, 256, 8, 90)])
def test_dora_forward(q, d_out, d_in, r, T):
    run_dora(q, S.make_layer(d_out, d_in, r, 2.0 * r, T, dtype="bf16", seed=d_in + T, with_grad=False))


def test_dora_forward_q_proj_sampled_rows(q):
    case = S.make_layer(**S.CONFIGS["q_proj_4096x4096_r16_T4096"], seed=3, with_grad=False)
    rows = np.sort(np.random.default_rng(5).choice(case.T, 256, replace=False))
    run_dora(q, case, rows=rows)


def test_dora_magnitude_at_norms_is_lora(q):
    """DoRA's initialisation (m = the row norms) reproduces the LoRA layer."""
    import torch
    case = S.make_layer(384, 256, 16, 32.0, 96, dtype="bf16", seed=8, with_grad=False)
    w, _ = quantize_both(q, case.W0)
    X, A, B = dev(case.X, "bf16"), dev(case.A, "bf16"), dev(case.B, "bf16")
    mag = q.dora_row_norms(w, A, B, case.alpha)
    Hd, _ = q.qlora_dora_fwd(w, X, A, B, case.alpha, mag)
    Hl, _ = q.qlora_linear_fwd(w, X, A, B, case.alpha)
    torch.cuda.synchronize()
    assert rel_fro(host(Hd), host(Hl).astype(np.float64)) <= 4e-3


def run_dora_bwd(q, case, rows=None, seed=0):
    """DoRA backward through the C ABI against the oracle's exact chain rule: dA, dB, dm in full,
    dX on the given token rows (all by default)."""
    import torch
    w, oc = quantize_both(q, case.W0)
    Wh = oracle_weight(oc, case.d_out, case.d_in, "bf16")
    mag = np.random.default_rng(seed).uniform(0.5, 2.0, case.d_out).astype(np.float32)
    dX, dA, dB, dm = q.qlora_dora_bwd(w, dev(case.X, "bf16"), dev(case.dH, "bf16"), dev(case.A, "bf16"),
                                      dev(case.B, "bf16"), case.alpha, torch.from_numpy(mag).cuda())
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    rX, rA, rB, rm = O.dora_backward(Wh, case.X, case.dH, case.A, case.B, case.alpha, case.r, mag)
    sel = slice(None) if rows is None else rows
    err = {"dX": rel_fro(host(dX)[sel], rX[sel]), "dA": rel_fro(host(dA), rA), "dB": rel_fro(host(dB), rB),
           "dm": rel_fro(host(dm), rm)}
    assert all(v <= TOL["bf16"] for v in err.values()), err


@pytest.mark.parametrize("d_out,d_in,r,T", [(256, 256, 8, 64), (200, 192, 5, 77), (520, 320, 16, 300),
                                            (136, 256, 100, 3), (203, 256, 8, 90)])
def test_dora_backward(q, d_out, d_in, r, T):
    run_dora_bwd(q, S.make_layer(d_out, d_in, r, 2.0 * r, T, dtype="bf16", seed=d_out + T))


@pytest.mark.parametrize("d_out,d_in,r,T", [(203, 320, 5, 37), (256, 512, 16, 300), (4096, 4096, 16, 512)])
def test_dora_saved_forward_and_backward(q, d_out, d_in, r, T):
    """qlora_dora_fwd_save keeps Z (the LoRA forward, on the large-T kernels whatever T), U and the
    row norms (bit for bit the dora_row_norms result); its H matches the oracle and the
    fused-epilogue forward; the backward from those saved tensors is bit-identical to the
    backward that recomputes them."""
    import torch
    case = S.make_layer(d_out, d_in, r, 2.0 * r, T, dtype="bf16", seed=d_out + r + T)
    w, oc = quantize_both(q, case.W0)
    Wh = oracle_weight(oc, d_out, d_in, "bf16")
    X, A, B, dH = dev(case.X, "bf16"), dev(case.A, "bf16"), dev(case.B, "bf16"), dev(case.dH, "bf16")
    mag_np = np.random.default_rng(d_out).uniform(0.5, 2.0, d_out).astype(np.float32)
    mag = torch.from_numpy(mag_np).cuda()
    H1, _ = q.qlora_dora_fwd(w, X, A, B, case.alpha, mag)
    H2, saved = q.qlora_dora_fwd_save(w, X, A, B, case.alpha, mag)
    Z, U, norms = saved
    Zl, Ul = q.qlora_linear_fwd(w, X, A, B, case.alpha)
    nl = q.dora_row_norms(w, A, B, case.alpha)
    g1 = q.qlora_dora_bwd(w, X, dH, A, B, case.alpha, mag)
    g2 = q.qlora_dora_bwd(w, X, dH, A, B, case.alpha, mag, saved=saved)
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    assert torch.equal(norms, nl)
    # (for T <= 64 qlora_linear_fwd takes the decode-size or mid-size route: same values, other
    # summation orders)
    assert rel_fro(host(Z), host(Zl).astype(np.float64)) <= 4e-3
    assert rel_fro(host(U), host(Ul).astype(np.float64)) <= 4e-3
    assert rel_fro(host(Z), O.lora_forward(Wh, case.X, case.A, case.B, case.alpha, r)) <= TOL["bf16"]
    assert rel_fro(host(H2), host(H1).astype(np.float64)) <= 4e-3
    assert rel_fro(host(H2), O.dora_forward(Wh, case.X, case.A, case.B, case.alpha, r, mag_np)) <= TOL["bf16"]
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_dora_backward_q_proj_sampled_rows(q):
    case = S.make_layer(**S.CONFIGS["q_proj_4096x4096_r16_T4096"], seed=4)
    rows = np.sort(np.random.default_rng(6).choice(case.T, 256, replace=False))
    run_dora_bwd(q, case, rows=rows)


# ------------------------------------------------------------------ FP8 activations (R25)


def fp8_probe_activation(n, seed):
    """bf16 values whose scaled copies (amax 4 -> sigma 64) hit every E4M3 tie below 256, the
    subnormal range and zeros, plus normal draws."""
    rng = np.random.default_rng(seed)
    x = S.round_to_bf16((rng.standard_normal(n) * 0.8).astype(np.float32))
    x = np.clip(x, -3.875, 3.875)
    pos = O.e4m3_decode(np.arange(127, dtype=np.uint8))
    mids = 0.5 * (pos[1:] + pos[:-1])
    mids = (mids[mids < 256.0] / 64.0).astype(np.float32)
    probe = np.concatenate([mids, -mids, np.float32([0.0, 2.0 ** -20, -2.0 ** -17, 2.0 ** -110])])
    m = min(n - 1, probe.size)
    x[1:1 + m] = probe[:m]
    x[0] = 4.0
    assert np.array_equal(S.round_to_bf16(x), x)
    return x


@pytest.mark.parametrize("shape", [(12345,), (64, 4096), (3,), (7, 136)])
def test_fp8_quantize_bit_exact(q, shape):
    import torch
    n = int(np.prod(shape))
    X = fp8_probe_activation(n, seed=n).reshape(shape)
    X8, sc = q.fp8_quantize(dev(X, "bf16"))
    torch.cuda.synchronize()
    ref8, sig = O.fp8_quantize_act(X)
    assert float(sc.item()) == sig
    assert np.array_equal(X8.cpu().numpy(), ref8)


def test_fp8_quantize_zero_and_tiny_tensors(q):
    import torch
    for X in (np.zeros((5, 64), np.float32), np.full(9, 2.0 ** -100, np.float32)):
        X8, sc = q.fp8_quantize(dev(X, "bf16"))
        torch.cuda.synchronize()
        ref8, sig = O.fp8_quantize_act(S.round_to_bf16(X))
        assert float(sc.item()) == sig
        assert np.array_equal(X8.cpu().numpy(), ref8)


@pytest.mark.parametrize("d_out,d_in", [(200, 192), (4096, 4096)])
def test_fp8_weight_scale(q, d_out, d_in):
    import torch
    rng = np.random.default_rng(d_in)
    W = (rng.standard_normal((d_out, d_in)) * 0.141).astype(np.float32)
    w, oc = quantize_both(q, W)
    sw = q.fp8_weight_scale(w)
    torch.cuda.synchronize()
    assert float(sw.item()) == O.fp8_weight_scale(oc[2])


def run_fp8(q, case, rows=None):
    """FP8 forward on the oracle's E4M3 activation and scales (uploaded as inputs) against the
    oracle's FP8 forward."""
    import torch
    w, oc = quantize_both(q, case.W0)
    codes, q8, c2, _ = oc
    X8, sx = O.fp8_quantize_act(case.X)
    sw = O.fp8_weight_scale(c2)
    W8 = O.nf4_dequantize_e4m3(codes, q8, c2, case.d_out, case.d_in, sw)
    xs = torch.tensor([sx], dtype=torch.float32, device="cuda")
    wsc = torch.tensor([sw], dtype=torch.float32, device="cuda")
    H = q.qlora_linear_fwd_fp8(w, torch.from_numpy(X8).cuda(), xs, wsc, dev(case.A, "bf16"),
                               dev(case.B, "bf16"), case.alpha)
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    sel = slice(None) if rows is None else rows
    ref = O.lora_forward_fp8(X8[sel], sx, W8, sw, case.A, case.B, case.alpha, case.r)
    assert rel_fro(host(H)[sel], ref) <= TOL["bf16"]
    return w, oc, H


@pytest.mark.parametrize("d_out,d_in,r,T", [(256, 256, 8, 64), (200, 192, 5, 77), (520, 320, 16, 300),
                                            (136, 256, 100, 3), (64, 128, 16, 1), (264, 1088, 64, 520)])
def test_fp8_forward(q, d_out, d_in, r, T):
    run_fp8(q, S.make_layer(d_out, d_in, r, 2.0 * r, T, dtype="bf16", seed=d_out + T, with_grad=False))


def test_fp8_forward_q_proj_sampled_rows(q):
    case = S.make_layer(**S.CONFIGS["q_proj_4096x4096_r16_T4096"], seed=4, with_grad=False)
    rows = np.sort(np.random.default_rng(6).choice(case.T, 256, replace=False))
    run_fp8(q, case, rows=rows)


def test_fp8_end_to_end_approximates_bf16_layer(q):
    """Device quantizer -> FP8 forward stays within the E4M3 rounding of the exact layer."""
    import torch
    case = S.make_layer(384, 512, 16, 32.0, 200, dtype="bf16", seed=12, with_grad=False)
    w, oc = quantize_both(q, case.W0)
    X8, xs = q.fp8_quantize(dev(case.X, "bf16"))
    H = q.qlora_linear_fwd_fp8(w, X8, xs, q.fp8_weight_scale(w), dev(case.A, "bf16"),
                               dev(case.B, "bf16"), case.alpha)
    torch.cuda.synchronize()
    ref = O.lora_forward(oracle_weight(oc, 384, 512, "f32"), case.X, case.A, case.B, case.alpha, case.r)
    e = rel_fro(host(H), ref)
    assert 1e-3 < e < 0.06


# ------------------------------------------------------------------ FP8 backward (R26)


def fp8_probe_grad(n, seed):
    """bf16 gradient values whose scaled copies (amax 1 -> sigma 2^15) hit every E5M2 tie
    below 2^15, the subnormal range and zeros, plus small normal draws."""
    rng = np.random.default_rng(seed)
    x = S.round_to_bf16((rng.standard_normal(n) * 0.2).astype(np.float32))
    x = np.clip(x, -0.96875, 0.96875)
    pos = O.e5m2_decode(np.arange(124, dtype=np.uint8))
    mids = 0.5 * (pos[1:] + pos[:-1])
    mids = (mids[mids < 2.0 ** 15] / 2.0 ** 15).astype(np.float32)
    probe = np.concatenate([mids, -mids, np.float32([0.0, 2.0 ** -40, -2.0 ** -33])])
    m = min(n - 1, probe.size)
    x[1:1 + m] = probe[:m]
    x[0] = 1.0
    assert np.array_equal(S.round_to_bf16(x), x)
    return x


@pytest.mark.parametrize("shape", [(9999,), (64, 4096), (2,)])
def test_fp8_quantize_grad_bit_exact(q, shape):
    import torch
    n = int(np.prod(shape))
    G = fp8_probe_grad(n, seed=n + 1).reshape(shape)
    G8, sc = q.fp8_quantize_grad(dev(G, "bf16"))
    torch.cuda.synchronize()
    ref8, sig = O.fp8_quantize_grad(G)
    assert float(sc.item()) == sig
    assert np.array_equal(G8.cpu().numpy(), ref8)


def run_fp8_bwd(q, case, rows=None):
    """FP8 backward on the oracle's E4M3 activation, E5M2 gradient and scales (uploaded as
    inputs) against the oracle's FP8 backward."""
    import torch
    w, oc = quantize_both(q, case.W0)
    codes, q8, c2, _ = oc
    X8, sx = O.fp8_quantize_act(case.X)
    G8, sg = O.fp8_quantize_grad(case.dH)
    sw = O.fp8_weight_scale(c2)
    W8 = O.nf4_dequantize_e4m3(codes, q8, c2, case.d_out, case.d_in, sw)
    t = lambda v: torch.tensor([v], dtype=torch.float32, device="cuda")
    dX, dA, dB = q.qlora_linear_bwd_fp8(w, torch.from_numpy(X8).cuda(), t(sx), torch.from_numpy(G8).cuda(),
                                        t(sg), t(sw), dev(case.A, "bf16"), dev(case.B, "bf16"), case.alpha)
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    rdX, rdA, rdB = O.lora_backward_fp8(X8, sx, G8, sg, W8, sw, case.A, case.B, case.alpha, case.r)
    sel = slice(None) if rows is None else rows
    assert rel_fro(host(dX)[sel], rdX[sel]) <= TOL["bf16"]
    assert rel_fro(host(dA), rdA) <= TOL["bf16"]
    assert rel_fro(host(dB), rdB) <= TOL["bf16"]


@pytest.mark.parametrize("d_out,d_in,r,T", [(256, 256, 8, 64), (208, 192, 5, 77), (528, 320, 16, 300),
                                            (144, 256, 100, 3), (64, 128, 16, 1), (272, 1088, 64, 520)])
def test_fp8_backward(q, d_out, d_in, r, T):
    run_fp8_bwd(q, S.make_layer(d_out, d_in, r, 2.0 * r, T, dtype="bf16", seed=d_in + r))


def test_fp8_backward_q_proj_sampled_rows(q):
    case = S.make_layer(**S.CONFIGS["q_proj_4096x4096_r16_T4096"], seed=9)
    rows = np.sort(np.random.default_rng(7).choice(case.T, 256, replace=False))
    run_fp8_bwd(q, case, rows=rows)


def test_fp8_backward_accumulate(q):
    """Two FP8 micro-batches with QLORA_BWD_ACCUMULATE add their dA, dB."""
    import torch
    case = S.make_layer(272, 320, 16, 32.0, 96, dtype="bf16", seed=14)
    w, oc = quantize_both(q, case.W0)
    ws_ = q.fp8_weight_scale(w)
    A, B = dev(case.A, "bf16"), dev(case.B, "bf16")
    X8, xs = q.fp8_quantize(dev(case.X, "bf16"))
    G8, gs = q.fp8_quantize_grad(dev(case.dH, "bf16"))
    _, dA1, dB1 = q.qlora_linear_bwd_fp8(w, X8, xs, G8, gs, ws_, A, B, case.alpha)
    _, dA2, dB2 = q.qlora_linear_bwd_fp8(w, X8, xs, G8, gs, ws_, A, B, case.alpha, dA=dA1.clone(),
                                         dB=dB1.clone(), accumulate=True, want_dx=False)
    torch.cuda.synchronize()
    assert torch.equal(dA2, 2 * dA1) and torch.equal(dB2, 2 * dB1)


def test_fp8_backward_rejects_unaligned_gradient_rows(q):
    """d_out % 16 != 0: the E5M2 rows cannot be read by TMA; refused on the host."""
    import torch
    case = S.make_layer(200, 192, 8, 16.0, 10, dtype="bf16", seed=1, with_grad=False)
    w, _ = quantize_both(q, case.W0)
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    X8 = torch.zeros((10, 192), dtype=torch.uint8, device="cuda")
    G8 = torch.zeros((10, 200), dtype=torch.uint8, device="cuda")
    with pytest.raises(q.QloraError) as e:
        q.qlora_linear_bwd_fp8(w, X8, one, G8, one, one, dev(case.A, "bf16"), dev(case.B, "bf16"), 16.0)
    assert e.value.code == 2


# ------------------------------------------------------------------ row-sharded (tensor-parallel) layer


@pytest.mark.parametrize("d_out,d_in,r,T", [(600, 512, 16, 300), (600, 512, 16, 5), (1000, 1024, 8, 40)])
def test_row_shards_through_the_library(q, d_out, d_in, r, T):
    """Two row shards of W0 and B (the tensor-parallel split of tp.row_shard), each run through the
    library's own forward and backward on this GPU, combined as the ranks' exchanges would (H
    columns gathered, dX and dA partials summed, dB rows kept): equal to the unsharded layer
    within bf16 rounding, and each shard's quantization is the same rows of the whole one."""
    import torch
    from qlora_parameter_efficient_b200 import tp
    case = S.make_layer(d_out, d_in, r, 2.0 * r, T, dtype="bf16", seed=d_out + r)
    W0 = dev(case.W0)
    X, A, B, dH = dev(case.X, "bf16"), dev(case.A, "bf16"), dev(case.B, "bf16"), dev(case.dH, "bf16")
    full = q.nf4_quantize(W0)
    H_f, U_f = q.qlora_linear_fwd(full, X, A, B, case.alpha)
    dX_f, dA_f, dB_f = q.qlora_linear_bwd(full, X, dH, A, B, case.alpha, U_saved=U_f)
    world = 2
    Hs, dBs = [], []
    dX = torch.zeros((T, d_in), dtype=torch.float32, device="cuda")
    dA = torch.zeros((r, d_in), dtype=torch.float32, device="cuda")
    bpr = d_in // 64
    for p in range(world):
        b, e = tp.row_shard(d_out, d_in, world, p)
        w = q.nf4_quantize(W0[b:e].contiguous())
        assert torch.equal(w.codes.reshape(-1), full.codes.reshape(-1)[b * d_in // 2:e * d_in // 2])
        assert torch.equal(w.absmax_q, full.absmax_q[b * bpr:e * bpr])
        assert torch.equal(w.c2, full.c2[b * bpr // 256:b * bpr // 256 + w.c2.numel()])
        Bp = B[b:e].contiguous()
        H_p, U_p = q.qlora_linear_fwd(w, X, A, Bp, case.alpha)
        dX_p, dA_p, dB_p = q.qlora_linear_bwd(w, X, dH[:, b:e].contiguous(), A, Bp, case.alpha, U_saved=U_p)
        Hs.append(H_p)
        dX += dX_p.float()
        dA += dA_p
        dBs.append(dB_p)
    torch.cuda.synchronize()
    assert q.get_device_error() == 0
    H = torch.cat(Hs, dim=1)
    dB = torch.cat(dBs, dim=0)
    assert rel_fro(host(H), host(H_f)) <= 5e-3
    assert rel_fro(host(dX), host(dX_f)) <= 5e-3
    assert rel_fro(host(dA), host(dA_f)) <= 5e-3
    assert rel_fro(host(dB), host(dB_f)) <= 5e-3
    Wh = O.nf4_dequantize(*O.nf4_quantize(case.W0)[:3], d_out, d_in, out="bf16").astype(np.float64)
    Href = O.lora_forward(Wh, case.X, case.A, case.B, case.alpha, r)
    assert rel_fro(host(H), Href) <= TOL["bf16"]

"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers and rounds them to the storage dtype of
the inputs; it holds none of the layer's arithmetic.  One numpy PCG64 stream
per case, drawn in a fixed order W0 -> A -> B -> X -> dH -> adapter ids, so the
CUDA path and the CPU oracle always see identical bytes.

Distributions (the second argument of N(0, v) is a variance):
  W0 ~ N(0, 0.02) fp32, A ~ N(0, 1/r), B ~ N(0, 0.01), X ~ N(0, 1), dH ~ N(0, 1).
Shapes follow the Llama-2 projection layers named on the pages (4096x4096
q_proj, 11008x4096 MLP up/gate, 70B-class 8192x8192 and 28672x8192); no
model weights or datasets are involved.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 input values to bf16 (RN-even) and return them as fp32."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


@dataclass
class LayerCase:
    """One synthetic layer: sizes plus the drawn tensors (host, numpy)."""
    d_out: int
    d_in: int
    r: int
    alpha: float
    T: int
    dtype: str                      # "bf16" or "f32": dtype of X, dH, A, B, H, dX
    W0: np.ndarray = field(repr=False, default=None)
    A: np.ndarray = field(repr=False, default=None)
    B: np.ndarray = field(repr=False, default=None)
    X: np.ndarray = field(repr=False, default=None)
    dH: np.ndarray = field(repr=False, default=None)


def make_layer(d_out, d_in, r, alpha, T, dtype="bf16", seed=0, zero_B=False,
               with_grad=True) -> LayerCase:
    """Draw W0, A, B, X, dH for one layer (fixed draw order)."""
    g = np.random.Generator(np.random.PCG64(seed))
    W0 = g.standard_normal((d_out, d_in), dtype=np.float32) * np.float32(np.sqrt(0.02))
    A = g.standard_normal((r, d_in), dtype=np.float32) * np.float32(1.0 / np.sqrt(r))
    B = g.standard_normal((d_out, r), dtype=np.float32) * np.float32(0.1)
    X = g.standard_normal((T, d_in), dtype=np.float32)
    dH = g.standard_normal((T, d_out), dtype=np.float32) if with_grad else None
    if zero_B:
        B = np.zeros_like(B)
    if dtype == "bf16":
        A, B, X = round_to_bf16(A), round_to_bf16(B), round_to_bf16(X)
        if dH is not None:
            dH = round_to_bf16(dH)
    elif dtype != "f32":
        raise ValueError(dtype)
    return LayerCase(d_out, d_in, r, float(alpha), T, dtype,
                     W0.astype(np.float32), A, B, X, dH)


@dataclass
class MultiAdapterCase:
    d_out: int
    d_in: int
    T: int
    ranks: list
    alphas: list
    dtype: str
    W0: np.ndarray = field(repr=False, default=None)
    As: list = field(repr=False, default=None)
    Bs: list = field(repr=False, default=None)
    X: np.ndarray = field(repr=False, default=None)
    ids: np.ndarray = field(repr=False, default=None)


def make_multi_adapter(d_out, d_in, T, ranks, split=None, dtype="bf16", seed=0):
    """Shared base plus one (A_i, B_i) per adapter; alpha_i = 2 r_i.

    ``split`` is None for ids drawn uniformly from {0..n-1}, or a list of
    fractions (e.g. [0.7, 0.1, 0.1, 0.1]) giving each adapter's share of the
    tokens; ids are shuffled across token positions, not sorted.
    """
    g = np.random.Generator(np.random.PCG64(seed))
    W0 = g.standard_normal((d_out, d_in), dtype=np.float32) * np.float32(np.sqrt(0.02))
    As, Bs = [], []
    for r in ranks:
        As.append(g.standard_normal((r, d_in), dtype=np.float32) * np.float32(1.0 / np.sqrt(r)))
    for r in ranks:
        Bs.append(g.standard_normal((d_out, r), dtype=np.float32) * np.float32(0.1))
    X = g.standard_normal((T, d_in), dtype=np.float32)
    n = len(ranks)
    if split is None:
        ids = g.integers(0, n, size=T, dtype=np.int32)
    else:
        counts = [int(round(f * T)) for f in split]
        counts[0] += T - sum(counts)
        ids = np.concatenate([np.full(c, i, np.int32) for i, c in enumerate(counts)])
        g.shuffle(ids)
    if dtype == "bf16":
        As = [round_to_bf16(a) for a in As]
        Bs = [round_to_bf16(b) for b in Bs]
        X = round_to_bf16(X)
    return MultiAdapterCase(d_out, d_in, T, list(ranks), [2.0 * r for r in ranks], dtype,
                            W0, As, Bs, X, ids.astype(np.int32))


# Named workloads: the single-layer configurations of the benchmark plan.
CONFIGS = {
    # 256x256, r=8, alpha=16, 64 fp32 tokens: the small exact-fp32 case.
    "small_256_r8_T64_f32": dict(d_out=256, d_in=256, r=8, alpha=16, T=64, dtype="f32"),
    # Llama-2-7B q_proj: 4096x4096, r=16, alpha=32, 4096 bf16 tokens (4 x 1024).
    "q_proj_4096x4096_r16_T4096": dict(d_out=4096, d_in=4096, r=16, alpha=32, T=4096, dtype="bf16"),
    # Llama-2-7B MLP up/gate: 11008x4096, r=64, alpha=128, 8192 tokens.
    "mlp_up_11008x4096_r64_T8192": dict(d_out=11008, d_in=4096, r=64, alpha=128, T=8192, dtype="bf16"),
    # 70B-class projections, r=16, alpha=32.
    "proj70b_8192x8192_r16_T2048": dict(d_out=8192, d_in=8192, r=16, alpha=32, T=2048, dtype="bf16"),
    "proj70b_8192x8192_r16_T16384": dict(d_out=8192, d_in=8192, r=16, alpha=32, T=16384, dtype="bf16"),
    "proj70b_28672x8192_r16_T2048": dict(d_out=28672, d_in=8192, r=16, alpha=32, T=2048, dtype="bf16"),
    "proj70b_28672x8192_r16_T16384": dict(d_out=28672, d_in=8192, r=16, alpha=32, T=16384, dtype="bf16"),
}

"""Helpers shared by the GPU parity tests: device transfer, tolerance checks, and running
one layer through both the CUDA library (C ABI) and the CPU oracle."""
import numpy as np

import oracle as O

TOL = {"bf16": 5e-3, "f32": 1e-5}   # relative Frobenius error bounds of the acceptance bar


def rel_fro(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got))


def torch_dtype(name):
    import torch
    return torch.bfloat16 if name == "bf16" else torch.float32


def dev(a, dtype="f32"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, np.float32)).to("cuda")
    return t.to(torch_dtype(dtype)) if dtype == "bf16" else t


def host(t):
    import torch
    return t.detach().to(torch.float32).cpu().numpy()


def quantize_both(q, W0):
    """GPU quantization of W0 and the oracle's; returns (gpu NF4Weight, oracle tuple)."""
    w = q.nf4_quantize(dev(W0))
    oc = O.nf4_quantize(W0)
    return w, oc


def oracle_weight(oc, d_out, d_in, dtype):
    codes, q8, c2, _ = oc
    return O.nf4_dequantize(codes, q8, c2, d_out, d_in, out=dtype).astype(np.float64)

"""qlora_linear_fwd_noalloc: the forward for callers that cannot allocate device memory.

Some callers (an engine that owns all device memory through its own pool, or a hot path that
must not take the allocator's locks) have no workspace to lend and cannot call cudaMalloc.
The no-allocation entry point runs the same forward with its scratch in a fixed device array
inside the library.  This test calls it through the C ABI twice in a row, on different
inputs, at token counts that take each of the forward's routes (decode-size, mid-size split-K,
large-T), and checks each result against the workspace-taking qlora_linear_fwd within the
bf16 tolerance the other parity tests use; it also checks that a size beyond the array is
refused with QLORA_ERR_UNSUPPORTED before anything runs.  The file name makes pytest collect
it last.
"""
import ctypes

import numpy as np
import pytest

from qlora_parameter_efficient_b200 import synthetic as S

from parity import TOL, dev, host, rel_fro

pytestmark = pytest.mark.gpu


def _call_noalloc(L, q, w, X, A, B, alpha, H, U):
    c = w._c()
    return L.qlora_linear_fwd_noalloc(ctypes.byref(c), q._ptr(X), X.shape[0], q._ptr(A), q._ptr(B),
                                      A.shape[0], float(alpha), q.BF16, q._ptr(H), q._ptr(U),
                                      q._stream())


def test_noalloc_forward_matches_workspace_forward():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from qlora_parameter_efficient_b200 import build
    build.build_library()
    import qlora_parameter_efficient_b200 as q
    L = q.load()

    d_out, d_in, r, alpha = 4096, 4096, 16, 32.0
    # T = 1 and 16 take the decode-size route, 48 the mid-size split-K route, 1024 the large-T
    # route; each lays its scratch out differently in the shared array, and each runs twice in
    # a row on different inputs, so a byte left over from the previous call would show.
    for T in (1, 16, 48, 1024):
        assert q.workspace_bytes(q.OP_FWD, q.BF16, T, d_out, d_in, r) <= 16 << 20
        for call, seed in enumerate((21, 22)):
            case = S.make_layer(d_out, d_in, r, alpha, T, dtype="bf16", seed=seed + 10 * T)
            w = q.nf4_quantize(dev(case.W0))
            X, A, B = dev(case.X, "bf16"), dev(case.A, "bf16"), dev(case.B, "bf16")
            H_ref, U_ref = q.qlora_linear_fwd(w, X, A, B, alpha)
            H = torch.full((T, d_out), float("nan"), dtype=torch.bfloat16, device="cuda")
            U = torch.full((T, r), float("nan"), dtype=torch.bfloat16, device="cuda")
            assert _call_noalloc(L, q, w, X, A, B, alpha, H, U) == 0, f"T={T} call {call}"
            torch.cuda.synchronize()
            assert q.get_device_error() == 0
            assert rel_fro(host(H), host(H_ref)) <= TOL["bf16"], f"T={T} call {call}"
            assert rel_fro(host(U), host(U_ref)) <= TOL["bf16"], f"T={T} call {call}"

    # A problem whose scratch would not fit in the array is refused before any launch.
    # (Buffers are full size so that nothing could run out of bounds even if it were not.)
    T_big = 65536
    assert q.workspace_bytes(q.OP_FWD, q.BF16, T_big, d_out, d_in, r) > 16 << 20
    Xb = torch.zeros((T_big, d_in), dtype=torch.bfloat16, device="cuda")
    Hb = torch.empty((T_big, d_out), dtype=torch.bfloat16, device="cuda")
    Ub = torch.empty((T_big, r), dtype=torch.bfloat16, device="cuda")
    n0 = q.launch_count()
    assert _call_noalloc(L, q, w, Xb, A, B, alpha, Hb, Ub) == 2
    assert q.launch_count() == n0

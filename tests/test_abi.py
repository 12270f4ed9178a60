"""The C-ABI library loads, exports every declared symbol, and its host-only calls agree
with the oracle.  No GPU needed: nothing here launches a kernel."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
import qlora_parameter_efficient_b200 as q

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "qlora.h")


@pytest.fixture(scope="module")
def L():
    from qlora_parameter_efficient_b200 import build
    build.build_library()
    return q.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 14
    assert sorted(names) == sorted(q.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_levels_match_oracle_bitwise(L):
    lib = np.array(q.nf4_levels(), np.float32)
    assert np.array_equal(lib.view(np.uint32), O.nf4_levels().view(np.uint32))


def test_sizes_match_oracle(L):
    for d, k in [(4096, 4096), (11008, 4096), (3, 128), (256, 256)]:
        assert q.nf4_sizes(d, k) == O.nf4_sizes(d, k)
    with pytest.raises(q.QloraError):
        q.nf4_sizes(10, 100)


def test_workspace_sizes(L):
    for op in (q.OP_FWD, q.OP_BWD, q.OP_FWD_BATCHED):
        for dt in (q.BF16, q.F32):
            assert q.workspace_bytes(op, dt, 4096, 4096, 4096, 16) > 0
    for op in (q.OP_FWD_MULTI, q.OP_DORA_FWD, q.OP_FWD_FP8, q.OP_BWD_FP8, q.OP_FP8_QUANT, q.OP_DORA_BWD):
        assert q.workspace_bytes(op, q.BF16, 4096, 4096, 4096, 16) > 0
        assert q.workspace_bytes(op, q.F32, 4096, 4096, 4096, 16) == 0      # bf16 only
    # the FP8 backward needs the bf16 backward's scratch plus the exact bf16 copies of X8, dH8
    assert (q.workspace_bytes(q.OP_BWD_FP8, q.BF16, 4096, 4096, 4096, 16)
            >= q.workspace_bytes(q.OP_BWD, q.BF16, 4096, 4096, 4096, 16) + 2 * 2 * 4096 * 4096)
    assert q.workspace_bytes(q.OP_MERGE, q.BF16, 1, 64, 64, 8) == 0
    assert q.workspace_bytes(q.OP_FWD, q.BF16, 1, 64, 64, 129) == 0
    # the DoRA backward holds the pre-scale output Z and dZ besides the LoRA backward's scratch
    assert (q.workspace_bytes(q.OP_DORA_BWD, q.BF16, 4096, 4096, 4096, 16)
            >= q.workspace_bytes(q.OP_BWD, q.BF16, 4096, 4096, 4096, 16) + 2 * 2 * 4096 * 4096)
    assert q.workspace_bytes(10, q.BF16, 1, 64, 64, 8) == 0


def test_status_strings(L):
    for code, name in q.STATUS.items():
        assert L.qlora_status_string(code).decode() == name


def test_host_validation_rejects_before_launch(L):
    # Invalid arguments are refused on the host, before any CUDA call.
    nf4 = q._NF4(16, 16, 16, 64, 100)            # d_in not a multiple of 64
    r = L.qlora_linear_fwd(ctypes.byref(nf4), 16, 1, 16, 16, 8, 16.0, q.BF16, 16, None, 256, 1 << 20, None)
    assert r == 2
    nf4 = q._NF4(16, 16, 16, 64, 64)
    r = L.qlora_linear_fwd(ctypes.byref(nf4), 16, 1, 16, 16, 200, 16.0, q.BF16, 16, None, 256, 1 << 20, None)
    assert r == 2                                # r > 128
    r = L.qlora_linear_fwd(ctypes.byref(nf4), 17, 1, 16, 16, 8, 16.0, q.BF16, 16, None, 256, 1 << 20, None)
    assert r == 1                                # misaligned X
    r = L.nf4_quantize(None, q.F32, 64, 64, 16, 16, 16, None)
    assert r == 1
    r = L.qlora_linear_fwd(ctypes.byref(nf4), 16, 1, 16, 16, 8, 16.0, 7, 16, None, 256, 1 << 20, None)
    assert r == 1                                # bad dtype
    r = L.qlora_linear_fwd(ctypes.byref(nf4), 16, 1, 16, 16, 8, 16.0, q.BF16, 16, None, 256, 10, None)
    assert r == 1                                # workspace too small


def test_split_backward_flags_validated_before_launch(L):
    # the grads-only / dX-from-workspace phases of qlora_linear_bwd_ex
    nf4 = q._NF4(16, 16, 16, 64, 64)

    def bwd(flags, dX=16, dA=16, dB=16):
        return L.qlora_linear_bwd_ex(ctypes.byref(nf4), 16, 16, 8, 16, 16, 8, 16.0, None, q.BF16,
                                     dX, dA, dB, 256, 1 << 20, flags, None)
    assert bwd(q.BWD_GRADS_ONLY | q.BWD_DX_FROM_WS) == 1      # both phases at once
    assert bwd(8) == 1                                         # unknown bit
    assert bwd(q.BWD_DX_FROM_WS, dX=None) == 1                 # dX phase without dX
    assert bwd(q.BWD_GRADS_ONLY, dA=None) == 1                 # grads phase without dA
    assert bwd(q.BWD_GRADS_ONLY | q.BWD_ACCUMULATE, dB=17) == 1
    assert bwd(0, dX=None, dA=None) == 1                       # one-call backward needs dA, dB


def test_dora_save_entries_validate_before_launch(L):
    nf4 = q._NF4(16, 16, 16, 64, 64)
    # forward with saving: the norms output and Z are required
    assert L.qlora_dora_fwd_save(ctypes.byref(nf4), 16, 8, 16, 16, 8, 16.0, 16, 16, 16, 16, None,
                                 256, 1 << 20, None) == 1
    assert L.qlora_dora_fwd_save(ctypes.byref(nf4), 16, 8, 16, 16, 8, 16.0, 16, 16, None, 16, 16,
                                 256, 1 << 20, None) == 1
    # backward from saved tensors: all three are required, and must be aligned
    assert L.qlora_dora_bwd_saved(ctypes.byref(nf4), 16, 16, 8, 16, 16, 8, 16.0, 16, None, 16, 16,
                                  16, 16, 16, 16, 256, 1 << 20, None) == 1
    assert L.qlora_dora_bwd_saved(ctypes.byref(nf4), 16, 16, 8, 16, 16, 8, 16.0, 16, 17, 16, 16,
                                  16, 16, 16, 16, 256, 1 << 20, None) == 1


def test_fp8_host_validation_rejects_before_launch(L):
    nf4 = q._NF4(16, 16, 16, 64, 64)
    # forward: a missing scale, a misaligned E4M3 activation
    r = L.qlora_linear_fwd_fp8(ctypes.byref(nf4), 16, 1, None, 16, 16, 16, 8, 16.0, 16, 256, 1 << 20, None)
    assert r == 1
    r = L.qlora_linear_fwd_fp8(ctypes.byref(nf4), 17, 1, 16, 16, 16, 16, 8, 16.0, 16, 256, 1 << 20, None)
    assert r == 1
    # backward: gradient rows of d_out bytes must be whole 16-byte units (d_out = 200)
    nf4b = q._NF4(16, 16, 16, 200, 64)
    r = L.qlora_linear_bwd_fp8(ctypes.byref(nf4b), 16, 16, 16, 16, 16, 1, 16, 16, 8, 16.0, 16, 16, 16,
                               256, 1 << 20, 0, None)
    assert r == 2
    # unknown flag bits
    r = L.qlora_linear_bwd_fp8(ctypes.byref(nf4), 16, 16, 16, 16, 16, 1, 16, 16, 8, 16.0, 16, 16, 16,
                               256, 1 << 20, 4, None)
    assert r == 1
    # quantizers: empty input, misaligned input, missing weight-scale output
    assert L.qlora_fp8_quantize(16, 0, 16, 16, 256, 256, None) == 2
    assert L.qlora_fp8_quantize(18, 64, 16, 16, 256, 256, None) == 1
    assert L.qlora_fp8_quantize_grad(16, 0, 16, 16, 256, 256, None) == 2
    assert L.qlora_fp8_weight_scale(ctypes.byref(nf4), None, None) == 1


def test_debug_build_compiles_and_exports_every_symbol(tmp_path):
    """The QLORA_DEBUG=1 build (device-side index checks reporting QLORA_ERR_DEVICE) compiles for
    sm_100a and exports the same C ABI."""
    from qlora_parameter_efficient_b200 import build
    lib = build.build_library(force=True, debug=True, out=str(tmp_path / "libqlora_debug.so"))
    D = ctypes.CDLL(lib)
    for n in declared_functions():
        assert hasattr(D, n), n


def test_noalloc_host_validation_matches_workspace_forward(L):
    # The no-allocation forward checks its arguments exactly as qlora_linear_fwd does and
    # returns the same status, before any CUDA call (nothing here reaches a device).
    cases = [
        (q._NF4(16, 16, 16, 64, 100), 16, 8, q.BF16),     # d_in not a multiple of 64
        (q._NF4(16, 16, 16, 64, 64), 16, 200, q.BF16),    # r > 128
        (q._NF4(16, 16, 16, 64, 64), 17, 8, q.BF16),      # misaligned X
        (q._NF4(16, 16, 16, 64, 64), 16, 8, 7),           # unknown dtype
        (q._NF4(16, 17, 16, 64, 64), 16, 8, q.BF16),      # misaligned absmax bytes
    ]
    for nf4, x_ptr, r, dt in cases:
        ref = L.qlora_linear_fwd(ctypes.byref(nf4), x_ptr, 1, 16, 16, r, 16.0, dt, 16, None, 256, 1 << 20, None)
        got = L.qlora_linear_fwd_noalloc(ctypes.byref(nf4), x_ptr, 1, 16, 16, r, 16.0, dt, 16, None, None)
        assert ref != 0 and got == ref, (r, dt, ref, got)

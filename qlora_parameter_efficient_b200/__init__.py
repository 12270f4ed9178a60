"""Python binding of libqlora, the B200 (sm_100a) QLoRA-adapted linear layer.

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libqlora.so`` behind the C ABI declared in ``include/qlora.h``.  PyTorch
provides device memory and streams.  There is no CPU fallback: if the library
is missing or a call fails, an exception is raised.

Names follow the C ABI: ``nf4_quantize``, ``nf4_dequantize``,
``qlora_linear_fwd``, ``qlora_linear_bwd`` (``accumulate=`` for gradient
accumulation), ``lora_merge``, ``qlora_linear_fwd_batched`` (a few adapters),
``qlora_linear_fwd_multi`` with an ``AdapterTable`` (thousands of mixed-rank
adapters), ``qlora_dora_fwd`` / ``qlora_dora_bwd`` / ``dora_row_norms`` (and
``qlora_dora_fwd_save`` whose saved tensors ``qlora_dora_bwd(saved=...)`` reuses), ``adamw_step`` /
``prefetch`` (optimizer step, unified-memory state), and the FP8 path:
``fp8_quantize`` (E4M3 activation), ``fp8_quantize_grad`` (E5M2 gradient),
``fp8_weight_scale``, ``qlora_linear_fwd_fp8``, ``qlora_linear_bwd_fp8``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
# QLORA_LIB selects another build of the same library (e.g. libqlora_debug.so, whose kernels
# check their index invariants); either way a missing file raises.
LIB_PATH = os.environ.get("QLORA_LIB") or os.path.join(HERE, "libqlora.so")

QLORA_OK = 0
STATUS = {0: "QLORA_OK", 1: "QLORA_ERR_INVALID_ARG", 2: "QLORA_ERR_UNSUPPORTED",
          3: "QLORA_ERR_CUDA", 4: "QLORA_ERR_TIMEOUT", 5: "QLORA_ERR_DEVICE"}
F32, BF16 = 0, 1
OP_FWD, OP_BWD, OP_FWD_BATCHED, OP_MERGE, OP_FWD_MULTI, OP_DORA_FWD = 0, 1, 2, 3, 4, 5
OP_FWD_FP8, OP_FP8_QUANT, OP_BWD_FP8, OP_DORA_BWD = 6, 7, 8, 9

# Every symbol include/qlora.h declares.
EXPORTS = ["qlora_nf4_sizes", "qlora_nf4_levels", "nf4_quantize", "nf4_dequantize",
           "qlora_workspace_bytes", "qlora_linear_fwd", "qlora_linear_bwd", "lora_merge",
           "qlora_linear_bwd_ex", "qlora_adamw_step", "qlora_prefetch", "qlora_dora_fwd",
           "qlora_dora_bwd", "qlora_dora_fwd_save", "qlora_dora_bwd_saved", "qlora_dora_row_norms", "qlora_fp8_quantize", "qlora_fp8_weight_scale",
           "qlora_linear_fwd_fp8", "qlora_fp8_quantize_grad", "qlora_linear_bwd_fp8",
           "qlora_linear_fwd_batched", "qlora_linear_fwd_multi", "qlora_linear_fwd_noalloc",
           "qlora_get_device_error",
           "qlora_selftest_wait_timeout", "qlora_set_gemm_events", "qlora_launch_count",
           "qlora_status_string"]


class QloraError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


class _NF4(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("absmax_q", ctypes.c_void_p),
                ("c2", ctypes.c_void_p), ("d_out", ctypes.c_int64), ("d_in", ctypes.c_int64)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libqlora.so (built in-tree); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m qlora_parameter_efficient_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    pnf4 = ctypes.POINTER(_NF4)
    sig = {
        "qlora_nf4_sizes": ([i64, i64, ctypes.POINTER(sz), ctypes.POINTER(sz), ctypes.POINTER(sz)], ctypes.c_int),
        "qlora_nf4_levels": ([ctypes.POINTER(ctypes.c_float)], ctypes.c_int),
        "nf4_quantize": ([vp, ctypes.c_int, i64, i64, vp, vp, vp, vp], ctypes.c_int),
        "nf4_dequantize": ([pnf4, vp, ctypes.c_int, vp], ctypes.c_int),
        "qlora_workspace_bytes": ([ctypes.c_int, ctypes.c_int, i64, i64, i64, i32], sz),
        "qlora_linear_fwd": ([pnf4, vp, i64, vp, vp, i32, f32, ctypes.c_int, vp, vp, vp, sz, vp], ctypes.c_int),
        "qlora_linear_bwd": ([pnf4, vp, vp, i64, vp, vp, i32, f32, vp, ctypes.c_int, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "lora_merge": ([pnf4, vp, vp, i32, f32, ctypes.c_int, ctypes.c_int, vp, vp], ctypes.c_int),
        "qlora_linear_fwd_batched": ([pnf4, vp, i64, vp, i32, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                      ctypes.POINTER(i32), ctypes.POINTER(f32), ctypes.c_int, vp, vp, sz, vp],
                                     ctypes.c_int),
        "qlora_linear_fwd_multi": ([pnf4, vp, i64, vp, i32, vp, vp, vp, vp, i32, vp, vp, sz, vp],
                                   ctypes.c_int),
        "qlora_linear_bwd_ex": ([pnf4, vp, vp, i64, vp, vp, i32, f32, vp, ctypes.c_int, vp, vp, vp, vp, sz,
                                 ctypes.c_uint32, vp], ctypes.c_int),
        "qlora_adamw_step": ([vp, ctypes.c_int, vp, vp, vp, vp, i64, i32, f32, f32, f32, f32, f32, f32, vp],
                             ctypes.c_int),
        "qlora_prefetch": ([vp, sz, i32, vp], ctypes.c_int),
        "qlora_dora_fwd": ([pnf4, vp, i64, vp, vp, i32, f32, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "qlora_dora_row_norms": ([pnf4, vp, vp, i32, f32, vp, vp, sz, vp], ctypes.c_int),
        "qlora_dora_bwd": ([pnf4, vp, vp, i64, vp, vp, i32, f32, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "qlora_dora_fwd_save": ([pnf4, vp, i64, vp, vp, i32, f32, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "qlora_dora_bwd_saved": ([pnf4, vp, vp, i64, vp, vp, i32, f32, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
                                 ctypes.c_int),
        "qlora_fp8_quantize": ([vp, i64, vp, vp, vp, sz, vp], ctypes.c_int),
        "qlora_fp8_weight_scale": ([pnf4, vp, vp], ctypes.c_int),
        "qlora_linear_fwd_fp8": ([pnf4, vp, i64, vp, vp, vp, vp, i32, f32, vp, vp, sz, vp], ctypes.c_int),
        "qlora_fp8_quantize_grad": ([vp, i64, vp, vp, vp, sz, vp], ctypes.c_int),
        "qlora_linear_bwd_fp8": ([pnf4, vp, vp, vp, vp, vp, i64, vp, vp, i32, f32, vp, vp, vp, vp, sz,
                                  ctypes.c_uint32, vp], ctypes.c_int),
        "qlora_linear_fwd_noalloc": ([pnf4, vp, i64, vp, vp, i32, f32, ctypes.c_int, vp, vp, vp], ctypes.c_int),
        "qlora_get_device_error": ([vp], ctypes.c_int),
        "qlora_selftest_wait_timeout": ([ctypes.c_uint64, vp], ctypes.c_int),
        "qlora_set_gemm_events": ([vp, vp], ctypes.c_int),
        "qlora_launch_count": ([], ctypes.c_uint64),
        "qlora_status_string": ([ctypes.c_int], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def _check(fn, code):
    if code != QLORA_OK:
        raise QloraError(fn, code)


def _torch():
    import torch
    return torch


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(dt):
    torch = _torch()
    if dt == torch.bfloat16:
        return BF16
    if dt == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {dt}")


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


@dataclass
class NF4Weight:
    """Device buffers of a quantized weight (NF4 codes + double-quantized absmax)."""
    codes: object      # uint8 [d_out, d_in/2]
    absmax_q: object   # uint8 [d_out*d_in/64]
    c2: object         # float32 [ceil(d_out*d_in/16384)]
    d_out: int
    d_in: int

    def _c(self):
        return _NF4(self.codes.data_ptr(), self.absmax_q.data_ptr(), self.c2.data_ptr(),
                    self.d_out, self.d_in)


def nf4_sizes(d_out, d_in):
    L = load()
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check("qlora_nf4_sizes", L.qlora_nf4_sizes(d_out, d_in, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
    return a.value, b.value, c.value


def nf4_levels():
    L = load()
    buf = (ctypes.c_float * 16)()
    _check("qlora_nf4_levels", L.qlora_nf4_levels(buf))
    return list(buf)


def workspace_bytes(op, dtype, T, d_out, d_in, r_total):
    return int(load().qlora_workspace_bytes(op, dtype, T, d_out, d_in, r_total))


def nf4_quantize(W, stream=None) -> NF4Weight:
    """Quantize a device fp32/bf16 weight W[d_out, d_in] to NF4 + double quant."""
    torch = _torch()
    _contig(W)
    d_out, d_in = W.shape
    nc, na, n2 = nf4_sizes(d_out, d_in)
    codes = torch.empty((d_out, d_in // 2), dtype=torch.uint8, device=W.device)
    absmax = torch.empty(na, dtype=torch.uint8, device=W.device)
    c2 = torch.empty(n2 // 4, dtype=torch.float32, device=W.device)
    _check("nf4_quantize", load().nf4_quantize(_ptr(W), _dtype_code(W.dtype), d_out, d_in,
                                               _ptr(codes), _ptr(absmax), _ptr(c2), _stream(stream)))
    return NF4Weight(codes, absmax, c2, d_out, d_in)


def nf4_dequantize(w: NF4Weight, dtype, out=None, stream=None):
    torch = _torch()
    if out is None:
        out = torch.empty((w.d_out, w.d_in), dtype=dtype, device=w.codes.device)
    c = w._c()
    _check("nf4_dequantize", load().nf4_dequantize(ctypes.byref(c), _ptr(out), _dtype_code(dtype), _stream(stream)))
    return out


def _ws(op, dtype_code, T, d_out, d_in, r, device, ws):
    torch = _torch()
    need = workspace_bytes(op, dtype_code, T, d_out, d_in, r)
    if ws is None or ws.numel() < need:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
    return ws


def qlora_linear_fwd(w: NF4Weight, X, A, B, alpha, H=None, U_save=None, ws=None, stream=None,
                     save_u=True):
    """H = X W^T + (alpha/r) (X A^T) B^T.  Returns (H, U_save)."""
    torch = _torch()
    _contig(X, A, B, H, U_save)
    T = X.shape[0]
    r = A.shape[0]
    dt = _dtype_code(X.dtype)
    if H is None:
        H = torch.empty((T, w.d_out), dtype=X.dtype, device=X.device)
    if U_save is None and save_u:
        U_save = torch.empty((T, r), dtype=X.dtype, device=X.device)
    ws = _ws(OP_FWD, dt, T, w.d_out, w.d_in, r, X.device, ws)
    c = w._c()
    _check("qlora_linear_fwd", load().qlora_linear_fwd(
        ctypes.byref(c), _ptr(X), T, _ptr(A), _ptr(B), r, float(alpha), dt, _ptr(H), _ptr(U_save),
        _ptr(ws), ws.numel(), _stream(stream)))
    return H, U_save


BWD_ACCUMULATE = 1
BWD_GRADS_ONLY = 2
BWD_DX_FROM_WS = 4
_BWD_PHASES = {"all": 0, "grads": BWD_GRADS_ONLY, "dx": BWD_DX_FROM_WS}


def qlora_linear_bwd(w: NF4Weight, X, dH, A, B, alpha, U_saved=None, dX=None, dA=None, dB=None,
                     ws=None, stream=None, want_dx=True, accumulate=False, phase="all"):
    """Returns (dX, dA, dB); dA, dB fp32.  accumulate=True adds into the given dA, dB.

    phase="grads" computes dA and dB only and leaves bf16(s G) in ws; phase="dx" then computes
    dX only from that ws (pass the same ws and operands); phase="all" does both in one call."""
    torch = _torch()
    _contig(X, dH, A, B, U_saved, dX, dA, dB)
    if phase not in _BWD_PHASES:
        raise ValueError(f"phase must be one of {sorted(_BWD_PHASES)}")
    if phase == "dx" and ws is None:
        raise ValueError('phase="dx" reads the workspace of the preceding phase="grads" call')
    T = X.shape[0]
    r = A.shape[0]
    dt = _dtype_code(X.dtype)
    if dX is None and want_dx and phase != "grads":
        dX = torch.empty((T, w.d_in), dtype=X.dtype, device=X.device)
    if dA is None and phase != "dx":
        dA = torch.empty((r, w.d_in), dtype=torch.float32, device=X.device)
    if dB is None and phase != "dx":
        dB = torch.empty((w.d_out, r), dtype=torch.float32, device=X.device)
    ws = _ws(OP_BWD, dt, T, w.d_out, w.d_in, r, X.device, ws)
    c = w._c()
    flags = _BWD_PHASES[phase] | (BWD_ACCUMULATE if accumulate else 0)
    if flags:
        _check("qlora_linear_bwd_ex", load().qlora_linear_bwd_ex(
            ctypes.byref(c), _ptr(X), _ptr(dH), T, _ptr(A), _ptr(B), r, float(alpha), _ptr(U_saved),
            dt, _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(), flags, _stream(stream)))
    else:
        _check("qlora_linear_bwd", load().qlora_linear_bwd(
            ctypes.byref(c), _ptr(X), _ptr(dH), T, _ptr(A), _ptr(B), r, float(alpha), _ptr(U_saved),
            dt, _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(), _stream(stream)))
    return dX, dA, dB


def adamw_step(param, grad, m, v, step, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0,
               master=None, grad_scale=1.0, stream=None):
    """One AdamW step in place: param (bf16 with an fp32 master, or fp32), grad, m, v fp32."""
    torch = _torch()
    _contig(param, grad, m, v, master)
    n = param.numel()
    _check("qlora_adamw_step", load().qlora_adamw_step(
        _ptr(param), _dtype_code(param.dtype), _ptr(master), _ptr(grad), _ptr(m), _ptr(v), n,
        int(step), float(lr), float(beta1), float(beta2), float(eps), float(weight_decay),
        float(grad_scale), _stream(stream)))
    return param


def dora_row_norms(w: NF4Weight, A, B, alpha, norms=None, ws=None, stream=None):
    """n_j = ||(W^ + (alpha/r) B A)[j, :]||_2 for every output row (fp32 [d_out])."""
    torch = _torch()
    _contig(A, B, norms)
    r = A.shape[0]
    if norms is None:
        norms = torch.empty(w.d_out, dtype=torch.float32, device=A.device)
    if ws is None:
        ws = torch.empty(w.d_out * (w.d_in // 64) * 4, dtype=torch.uint8, device=A.device)
    _check("qlora_dora_row_norms", load().qlora_dora_row_norms(
        ctypes.byref(w._c()), _ptr(A), _ptr(B), r, float(alpha), _ptr(norms), _ptr(ws), ws.numel(),
        _stream(stream)))
    return norms


def qlora_dora_fwd(w: NF4Weight, X, A, B, alpha, magnitude, H=None, U_save=None, save_u=True,
                   ws=None, stream=None):
    """DoRA forward (bf16): H = (m / ||W^ + sBA||_rows) * (X W^T + s U B^T); returns (H, U)."""
    torch = _torch()
    _contig(X, A, B, magnitude, H, U_save)
    T = X.shape[0]
    r = A.shape[0]
    if H is None:
        H = torch.empty((T, w.d_out), dtype=X.dtype, device=X.device)
    if U_save is None and save_u:
        U_save = torch.empty((T, r), dtype=X.dtype, device=X.device)
    ws = _ws(OP_DORA_FWD, BF16, T, w.d_out, w.d_in, r, X.device, ws)
    c = w._c()
    _check("qlora_dora_fwd", load().qlora_dora_fwd(
        ctypes.byref(c), _ptr(X), T, _ptr(A), _ptr(B), r, float(alpha), _ptr(magnitude), _ptr(H),
        _ptr(U_save), _ptr(ws), ws.numel(), _stream(stream)))
    return H, U_save


def qlora_dora_fwd_save(w: NF4Weight, X, A, B, alpha, magnitude, H=None, Z=None, U=None, norms=None,
                        ws=None, stream=None):
    """DoRA forward that keeps what the backward needs: returns (H, saved) with saved = (Z, U,
    norms), the pre-scale output, U and the row norms, for qlora_dora_bwd(..., saved=saved)."""
    torch = _torch()
    _contig(X, A, B, magnitude, H, Z, U, norms)
    T = X.shape[0]
    r = A.shape[0]
    dev = X.device
    if H is None:
        H = torch.empty((T, w.d_out), dtype=X.dtype, device=dev)
    if Z is None:
        Z = torch.empty((T, w.d_out), dtype=X.dtype, device=dev)
    if U is None:
        U = torch.empty((T, r), dtype=X.dtype, device=dev)
    if norms is None:
        norms = torch.empty((w.d_out,), dtype=torch.float32, device=dev)
    ws = _ws(OP_DORA_FWD, BF16, T, w.d_out, w.d_in, r, dev, ws)
    c = w._c()
    _check("qlora_dora_fwd_save", load().qlora_dora_fwd_save(
        ctypes.byref(c), _ptr(X), T, _ptr(A), _ptr(B), r, float(alpha), _ptr(magnitude), _ptr(H),
        _ptr(Z), _ptr(U), _ptr(norms), _ptr(ws), ws.numel(), _stream(stream)))
    return H, (Z, U, norms)


def qlora_dora_bwd(w: NF4Weight, X, dH, A, B, alpha, magnitude, dX=None, dA=None, dB=None, dm=None,
                   want_dx=True, ws=None, stream=None, saved=None):
    """DoRA backward (bf16), the chain rule through the row norm: returns (dX, dA, dB, dm).
    saved: the (Z, U, norms) of qlora_dora_fwd_save for the same operands (else recomputed)."""
    torch = _torch()
    _contig(X, dH, A, B, magnitude, dX, dA, dB, dm)
    if saved is not None:
        _contig(*saved)
    T = X.shape[0]
    r = A.shape[0]
    dev = X.device
    if dX is None and want_dx:
        dX = torch.empty((T, w.d_in), dtype=X.dtype, device=dev)
    if dA is None:
        dA = torch.empty((r, w.d_in), dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty((w.d_out, r), dtype=torch.float32, device=dev)
    if dm is None:
        dm = torch.empty((w.d_out,), dtype=torch.float32, device=dev)
    ws = _ws(OP_DORA_BWD, BF16, T, w.d_out, w.d_in, r, dev, ws)
    c = w._c()
    if saved is None:
        _check("qlora_dora_bwd", load().qlora_dora_bwd(
            ctypes.byref(c), _ptr(X), _ptr(dH), T, _ptr(A), _ptr(B), r, float(alpha), _ptr(magnitude),
            _ptr(dX), _ptr(dA), _ptr(dB), _ptr(dm), _ptr(ws), ws.numel(), _stream(stream)))
    else:
        Z, U, norms = saved
        _check("qlora_dora_bwd_saved", load().qlora_dora_bwd_saved(
            ctypes.byref(c), _ptr(X), _ptr(dH), T, _ptr(A), _ptr(B), r, float(alpha), _ptr(magnitude),
            _ptr(Z), _ptr(U), _ptr(norms), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(dm), _ptr(ws), ws.numel(),
            _stream(stream)))
    return dX, dA, dB, dm


def fp8_quantize(X, X8=None, scale=None, ws=None, stream=None):
    """E4M3 bytes of a bf16 tensor with its power-of-two scale: returns (X8 uint8, scale fp32[1]),
    X ~ E4M3value(X8) / scale."""
    torch = _torch()
    _contig(X, X8)
    if X.dtype != torch.bfloat16:
        raise TypeError("fp8_quantize takes a bf16 tensor")
    if X8 is None:
        X8 = torch.empty(X.shape, dtype=torch.uint8, device=X.device)
    if scale is None:
        scale = torch.empty(1, dtype=torch.float32, device=X.device)
    if ws is None:
        ws = torch.empty(256, dtype=torch.uint8, device=X.device)
    _check("qlora_fp8_quantize", load().qlora_fp8_quantize(
        _ptr(X), X.numel(), _ptr(X8), _ptr(scale), _ptr(ws), ws.numel(), _stream(stream)))
    return X8, scale


def fp8_weight_scale(w: NF4Weight, out=None, stream=None):
    """sigma_w (fp32[1], device) of a stored weight for the FP8 forward."""
    torch = _torch()
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=w.codes.device)
    _check("qlora_fp8_weight_scale", load().qlora_fp8_weight_scale(ctypes.byref(w._c()), _ptr(out),
                                                                   _stream(stream)))
    return out


def qlora_linear_fwd_fp8(w: NF4Weight, X8, x_scale, w_scale, A, B, alpha, H=None, ws=None, stream=None):
    """H = (X8 W8^T) / (sigma_x sigma_w) + (alpha/r) (X~ A^T) B^T with an E4M3 activation (bf16 H)."""
    torch = _torch()
    _contig(X8, A, B, H)
    if X8.dtype != torch.uint8:
        raise TypeError("X8 holds E4M3 bytes (uint8)")
    T = X8.shape[0]
    r = A.shape[0]
    if H is None:
        H = torch.empty((T, w.d_out), dtype=torch.bfloat16, device=X8.device)
    ws = _ws(OP_FWD_FP8, BF16, T, w.d_out, w.d_in, r, X8.device, ws)
    c = w._c()
    _check("qlora_linear_fwd_fp8", load().qlora_linear_fwd_fp8(
        ctypes.byref(c), _ptr(X8), T, _ptr(x_scale), _ptr(w_scale), _ptr(A), _ptr(B), r, float(alpha),
        _ptr(H), _ptr(ws), ws.numel(), _stream(stream)))
    return H


def fp8_quantize_grad(dH, dH8=None, scale=None, ws=None, stream=None):
    """E5M2 bytes of a bf16 gradient with its power-of-two scale: (dH8 uint8, scale fp32[1])."""
    torch = _torch()
    _contig(dH, dH8)
    if dH.dtype != torch.bfloat16:
        raise TypeError("fp8_quantize_grad takes a bf16 tensor")
    if dH8 is None:
        dH8 = torch.empty(dH.shape, dtype=torch.uint8, device=dH.device)
    if scale is None:
        scale = torch.empty(1, dtype=torch.float32, device=dH.device)
    if ws is None:
        ws = torch.empty(256, dtype=torch.uint8, device=dH.device)
    _check("qlora_fp8_quantize_grad", load().qlora_fp8_quantize_grad(
        _ptr(dH), dH.numel(), _ptr(dH8), _ptr(scale), _ptr(ws), ws.numel(), _stream(stream)))
    return dH8, scale


def qlora_linear_bwd_fp8(w: NF4Weight, X8, x_scale, dH8, g_scale, w_scale, A, B, alpha, dX=None,
                         dA=None, dB=None, ws=None, accumulate=False, want_dx=True, stream=None):
    """Backward from the E4M3 activation and the E5M2 gradient: returns (dX bf16, dA, dB fp32)."""
    torch = _torch()
    _contig(X8, dH8, A, B, dX, dA, dB)
    T = X8.shape[0]
    r = A.shape[0]
    if dX is None and want_dx:
        dX = torch.empty((T, w.d_in), dtype=torch.bfloat16, device=X8.device)
    if dA is None:
        dA = torch.zeros((r, w.d_in), dtype=torch.float32, device=X8.device)
    if dB is None:
        dB = torch.zeros((w.d_out, r), dtype=torch.float32, device=X8.device)
    ws = _ws(OP_BWD_FP8, BF16, T, w.d_out, w.d_in, r, X8.device, ws)
    c = w._c()
    _check("qlora_linear_bwd_fp8", load().qlora_linear_bwd_fp8(
        ctypes.byref(c), _ptr(X8), _ptr(x_scale), _ptr(dH8), _ptr(g_scale), _ptr(w_scale), T, _ptr(A),
        _ptr(B), r, float(alpha), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(),
        BWD_ACCUMULATE if accumulate else 0, _stream(stream)))
    return dX, dA, dB


def prefetch(ptr: int, nbytes: int, to_device: bool, stream=None):
    """Page a unified-memory range to the current device or back to the host."""
    _check("qlora_prefetch", load().qlora_prefetch(ctypes.c_void_p(ptr), nbytes, 1 if to_device else 0,
                                                   _stream(stream)))


def lora_merge(w: NF4Weight, A, B, alpha, out_dtype, out=None, stream=None):
    torch = _torch()
    _contig(A, B, out)
    r = A.shape[0]
    if out is None:
        out = torch.empty((w.d_out, w.d_in), dtype=out_dtype, device=A.device)
    c = w._c()
    _check("lora_merge", load().lora_merge(ctypes.byref(c), _ptr(A), _ptr(B), r, float(alpha),
                                           _dtype_code(A.dtype), _dtype_code(out_dtype), _ptr(out),
                                           _stream(stream)))
    return out


def qlora_linear_fwd_batched(w: NF4Weight, X, adapter_id, As, Bs, alphas, H=None, ws=None,
                             stream=None):
    torch = _torch()
    _contig(X, adapter_id, H, *As, *Bs)
    T = X.shape[0]
    n = len(As)
    ranks = [a.shape[0] for a in As]
    dt = _dtype_code(X.dtype)
    if H is None:
        H = torch.empty((T, w.d_out), dtype=X.dtype, device=X.device)
    ws = _ws(OP_FWD_BATCHED, dt, T, w.d_out, w.d_in, sum(ranks), X.device, ws)
    Ap = (ctypes.c_void_p * n)(*[a.data_ptr() for a in As])
    Bp = (ctypes.c_void_p * n)(*[b.data_ptr() for b in Bs])
    rp = (ctypes.c_int32 * n)(*ranks)
    ap = (ctypes.c_float * n)(*[float(a) for a in alphas])
    c = w._c()
    _check("qlora_linear_fwd_batched", load().qlora_linear_fwd_batched(
        ctypes.byref(c), _ptr(X), T, _ptr(adapter_id), n, Ap, Bp, rp, ap, dt, _ptr(H), _ptr(ws),
        ws.numel(), _stream(stream)))
    return H


class AdapterTable:
    """Device-resident adapter table for qlora_linear_fwd_multi: pointer arrays, ranks and
    alphas uploaded once from lists of bf16 tensors A_i [r_i, d_in], B_i [d_out, r_i] (the
    library forms alpha_i / r_i itself)."""

    def __init__(self, As, Bs, alphas):
        torch = _torch()
        _contig(*As, *Bs)
        dev = As[0].device
        self.As, self.Bs = list(As), list(Bs)        # keep the tensors alive
        self.ranks_host = [int(a.shape[0]) for a in As]
        self.n = len(As)
        self.r_max = max(self.ranks_host)
        self.A_ptrs = torch.tensor([a.data_ptr() for a in As], dtype=torch.int64, device=dev)
        self.B_ptrs = torch.tensor([b.data_ptr() for b in Bs], dtype=torch.int64, device=dev)
        self.ranks = torch.tensor(self.ranks_host, dtype=torch.int32, device=dev)
        self.alphas = torch.tensor([float(al) for al in alphas], dtype=torch.float32, device=dev)


def qlora_linear_fwd_multi(w: NF4Weight, X, adapter_id, table: AdapterTable, H=None, ws=None,
                           stream=None):
    torch = _torch()
    _contig(X, adapter_id, H)
    T = X.shape[0]
    if H is None:
        H = torch.empty((T, w.d_out), dtype=X.dtype, device=X.device)
    ws = _ws(OP_FWD_MULTI, BF16, T, w.d_out, w.d_in, table.r_max, X.device, ws)
    c = w._c()
    _check("qlora_linear_fwd_multi", load().qlora_linear_fwd_multi(
        ctypes.byref(c), _ptr(X), T, _ptr(adapter_id), table.n, _ptr(table.A_ptrs),
        _ptr(table.B_ptrs), _ptr(table.ranks), _ptr(table.alphas), table.r_max, _ptr(H),
        _ptr(ws), ws.numel(), _stream(stream)))
    return H


def get_device_error(stream=None) -> int:
    return int(load().qlora_get_device_error(_stream(stream)))


def selftest_wait_timeout(limit_ns, stream=None):
    _check("qlora_selftest_wait_timeout", load().qlora_selftest_wait_timeout(int(limit_ns), _stream(stream)))


def set_gemm_events(start=None, stop=None):
    """Make the fused NF4 GEMM record torch.cuda.Event objects around itself."""
    s = ctypes.c_void_p(start.cuda_event) if start is not None else None
    e = ctypes.c_void_p(stop.cuda_event) if stop is not None else None
    _check("qlora_set_gemm_events", load().qlora_set_gemm_events(s, e))


def launch_count() -> int:
    return int(load().qlora_launch_count())

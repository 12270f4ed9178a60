"""Benchmark of the QLoRA-adapted linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--extra]

A step is one forward + backward pass of the layer (NF4 W0 decoded on the fly inside the
tensor-core GEMM, LoRA branch fused; dX, dA, dB) over one batch of synthetic tokens shaped
like Llama-2-7B q_proj: W0 4096x4096 NF4 + double quant, r = 16, alpha = 32, 4096 bf16
tokens.  With N > 1 (one process per GPU under torchrun) every rank runs its own batch
(weak scaling, data parallel) and the adapter gradients dA, dB are all-reduced over NCCL
inside the step.  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (the plain fp64 implementation the tests check
against) on this host's cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "q_proj_4096x4096_r16_T4096"
METRIC = "QLoRA linear fwd+bwd tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def cfg():
    from qlora_parameter_efficient_b200 import synthetic as S
    return dict(S.CONFIGS[WORKLOAD])


def flops_fwd(T, d, k, r):
    return 2 * T * d * k + 2 * T * r * (d + k)


def flops_bwd(T, d, k, r):
    return 2 * T * d * k + 4 * T * r * (d + k)


def w_bytes(d, k):
    """Stored NF4 weight: codes + uint8 absmax + fp32 second-level constants (0.5159 B/param)."""
    return d * k * (0.5 + 1 / 64) + 4 * ((d * k // 64 + 255) // 256)


def bytes_fwd(T, d, k, r):
    """Forward call: W, X read, H written, A and B read, U saved (bf16)."""
    return w_bytes(d, k) + 2 * T * k + 2 * T * d + 2 * r * (d + k) + 2 * T * r


def bytes_bwd(T, d, k, r):
    """Backward call: W, X, dH, U, A, B read; dX (bf16), dA and dB (fp32) written."""
    return w_bytes(d, k) + 2 * T * k + 2 * T * d + 2 * T * k + 2 * T * r + 2 * r * (d + k) + 4 * r * (d + k)


def t_roof(flops, byts, peaks):
    """max(FLOPs at the measured burst bf16 tensor peak, bytes at the measured HBM peak), s."""
    return max(flops / (peaks["bf16_tflops"] * 1e12), byts / (peaks["hbm_gbs"] * 1e9))


# ---------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                       "-i", str(self.index), "-lms", "200"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.p:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()

    def summary(self):
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------- oracle timing


def oracle_sample(n_tokens, seed=0):
    """One bounded-sample step of the oracle: decode W^ and fwd + bwd over n_tokens tokens."""
    import oracle as O
    from qlora_parameter_efficient_b200 import synthetic as S
    c = cfg()
    case = S.make_layer(c["d_out"], c["d_in"], c["r"], c["alpha"], n_tokens, dtype="bf16", seed=seed)
    codes, q8, c2, _ = O.nf4_quantize(case.W0)         # storage prepared outside the timing
    t0 = time.perf_counter()
    Wh = O.nf4_dequantize(codes, q8, c2, c["d_out"], c["d_in"], out="bf16")
    O.lora_forward(Wh, case.X, case.A, case.B, case.alpha, case.r)
    O.lora_backward(Wh, case.X, case.dH, case.A, case.B, case.alpha, case.r)
    return time.perf_counter() - t0


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return len(os.sched_getaffinity(0))


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_baseline(target_s=10.0):
    """The oracle timed on this host: all of its BLAS threads on a sample sized for about
    target_s seconds, and one thread on a smaller sample (tokens/s is per-token work, so the
    rates compare)."""
    t_small = oracle_sample(256)
    n = int(min(cfg()["T"], max(256, 256 * target_s / max(t_small, 1e-3))))
    n = max(256, (n // 256) * 256)
    t = oracle_sample(n, seed=1)
    out = {"value": n / t, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
           "cpu_model": cpu_model(),
           "sample": f"{n} of {cfg()['T']} tokens of {WORKLOAD}: NF4 decode + fp64 fwd + bwd "
                     f"({t:.1f} s)"}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            n1 = 128
            t1 = oracle_sample(n1, seed=2)
        out["value_1core"] = n1 / t1
        out["sample_1core"] = f"{n1} tokens on 1 thread ({t1:.1f} s)"
    except Exception as e:          # threadpoolctl missing: report the all-core figure only
        out["value_1core"] = None
        out["sample_1core"] = f"not measured: {type(e).__name__}"
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    c = cfg()
    n = 512
    oracle_sample(256)                                   # warm import / caches
    for _ in range(args.warmup):
        oracle_sample(n)
    times = [oracle_sample(n, seed=i + 1) for i in range(args.steps)]
    total = sum(times)
    value = n * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD + " fwd+bwd", "d_out": c["d_out"], "d_in": c["d_in"],
                   "r": c["r"], "alpha": c["alpha"], "tokens_per_step": n,
                   "note": "each step is a bounded sample of the workload"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "kind": "oracle",
                         "cores": oracle_threads(),
                         "sample": f"{n} of {c['T']} tokens per step: NF4 decode + fp64 fwd + bwd"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------- GPU arm


def run_gpu(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import qlora_parameter_efficient_b200 as q
    from qlora_parameter_efficient_b200 import build as qb
    from qlora_parameter_efficient_b200 import dp
    from qlora_parameter_efficient_b200 import synthetic as S

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.only == "decode":
        return run_decode_only(args, q, qb, S, torch, dev)
    if args.only == "multi":
        return run_multi_only(args, q, qb, torch, dev)
    if args.only in ("fp8", "fp8bwd"):
        return run_fp8_only(args, q, qb, S, torch, dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    if rank == 0:
        qb.build_library()
    if world > 1:
        dist.barrier()
    q.load()
    peaks, peak_src = load_peaks()
    c = cfg()
    d, k, r, T, alpha = c["d_out"], c["d_in"], c["r"], c["T"], c["alpha"]
    bf = torch.bfloat16

    # Rotating input sets so the working set (about 4 x 75 MB) exceeds 2 x the 126 MB L2.
    NSETS = 4
    sets = []
    for i in range(NSETS):
        case = S.make_layer(d, k, r, alpha, T, dtype="bf16", seed=1000 * rank + i)
        w = q.nf4_quantize(torch.from_numpy(case.W0).to(dev))
        sets.append(dict(
            w=w, X=torch.from_numpy(case.X).to(dev).to(bf), dH=torch.from_numpy(case.dH).to(dev).to(bf),
            A=torch.from_numpy(case.A).to(dev).to(bf), B=torch.from_numpy(case.B).to(dev).to(bf)))
        del case
    H = torch.empty((T, d), dtype=bf, device=dev)
    U = torch.empty((T, r), dtype=bf, device=dev)
    dX = torch.empty((T, k), dtype=bf, device=dev)
    # dA and dB in one flat buffer: one all-reduce per step when the data-parallel ranks sum them
    grads = torch.empty(r * k + d * r, dtype=torch.float32, device=dev)
    dA = grads[: r * k].view(r, k)
    dB = grads[r * k:].view(d, r)
    ws = torch.empty(max(q.workspace_bytes(q.OP_FWD, q.BF16, T, d, k, r),
                         q.workspace_bytes(q.OP_BWD, q.BF16, T, d, k, r)), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def backward(w, X_, dH_, A_, B_):
        if world == 1:
            q.qlora_linear_bwd(w, X_, dH_, A_, B_, alpha, U_saved=U, dX=dX, dA=dA, dB=dB, ws=ws)
            return
        # dA, dB first, then their sum over ranks on NCCL's stream beside the dX GEMM
        dp.backward_overlapped(
            lambda: q.qlora_linear_bwd(w, X_, dH_, A_, B_, alpha, U_saved=U, dA=dA, dB=dB, ws=ws,
                                       phase="grads"),
            lambda: q.qlora_linear_bwd(w, X_, dH_, A_, B_, alpha, U_saved=U, dX=dX, ws=ws, phase="dx"),
            grads)

    def step(i):
        s = sets[i % NSETS]
        q.qlora_linear_fwd(s["w"], s["X"], s["A"], s["B"], alpha, H=H, U_save=U, ws=ws)
        backward(s["w"], s["X"], s["dH"], s["A"], s["B"])

    def timed(fn, K, W, with_gemm_events=False):
        for i in range(W):
            fn(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        gev = []
        n0 = q.launch_count()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(K):
            if with_gemm_events:
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                b.record(stream)      # materialise the events before handing them over
                q.set_gemm_events(a, b)
                gev.append((a, b))
            fn(i)
            if with_gemm_events:
                q.set_gemm_events(None, None)
        e1.record(stream)
        torch.cuda.synchronize()
        launches = q.launch_count() - n0
        ms = dp.max_over_ranks(e0.elapsed_time(e1), device=dev)
        g_ms = [a.elapsed_time(b) for a, b in gev]
        return ms, launches, g_ms

    W = max(3, args.warmup)

    def fn_fwd(i):
        s = sets[i % NSETS]
        q.qlora_linear_fwd(s["w"], s["X"], s["A"], s["B"], alpha, H=H, U_save=U, ws=ws)

    def fn_bwd(i):
        s = sets[i % NSETS]
        q.qlora_linear_bwd(s["w"], s["X"], s["dH"], s["A"], s["B"], alpha, U_saved=U, dX=dX, dA=dA,
                           dB=dB, ws=ws)

    if args.only != "step":
        # One part of the step alone (for profiling a single kernel on the same workload).
        ms, launches, _ = timed(fn_fwd if args.only == "fwd" else fn_bwd, args.steps, W)
        if rank == 0:
            print(json.dumps({"only": args.only, "ms_per_call": ms / args.steps,
                              "launches": launches, "workload": WORKLOAD}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0
    with ClockSampler(local) as clk:
        ms, launches, _ = timed(step, args.steps, W)
    clocks = clk.summary()
    # Dominant kernel: the fused NF4-decode GEMM of the forward (its last launch in each
    # step is the dX GEMM, the first the forward one; the hook records the latest launch,
    # so time the forward alone with the hook on).
    _, _, g_ms = timed(fn_fwd, args.steps, W, with_gemm_events=True)
    # forward alone and backward alone (device time)
    fwd_ms, _, _ = timed(fn_fwd, args.steps, W)
    bwd_ms, _, _ = timed(fn_bwd, args.steps, W)

    # ------------------------------------------------------------------ end to end
    # Each step: pinned host X, dH -> device, fwd + bwd through the C ABI, dA, dB -> host.  The
    # next step's inputs are copied on a second stream into the other of two device buffers
    # while this step computes (a data loader's prefetch); every copy of every step lies inside
    # the timed region, and a buffer is refilled only after the step that read it has finished.
    hX = [sets[i]["X"].cpu().pin_memory() for i in range(2)]
    hdH = [sets[i]["dH"].cpu().pin_memory() for i in range(2)]
    hdA = torch.empty_like(dA, device="cpu").pin_memory()
    hdB = torch.empty_like(dB, device="cpu").pin_memory()
    Xd = [torch.empty_like(sets[0]["X"]) for _ in range(2)]
    dHd = [torch.empty_like(sets[0]["dH"]) for _ in range(2)]
    copy_stream = torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_free = [torch.cuda.Event() for _ in range(2)]

    def copy_in(i):
        bi = i % 2
        with torch.cuda.stream(copy_stream):
            if i >= 2:
                copy_stream.wait_event(ev_free[bi])
            Xd[bi].copy_(hX[i % 2], non_blocking=True)
            dHd[bi].copy_(hdH[i % 2], non_blocking=True)
            ev_in[bi].record(copy_stream)

    def e2e_run(K):
        copy_stream.wait_stream(stream)
        copy_in(0)
        for i in range(K):
            bi = i % 2
            if i + 1 < K:
                copy_in(i + 1)
            stream.wait_event(ev_in[bi])
            s = sets[i % NSETS]
            q.qlora_linear_fwd(s["w"], Xd[bi], s["A"], s["B"], alpha, H=H, U_save=U, ws=ws)
            backward(s["w"], Xd[bi], dHd[bi], s["A"], s["B"])
            ev_free[bi].record(stream)
            hdA.copy_(dA, non_blocking=True)
            hdB.copy_(dB, non_blocking=True)

    e2e_run(W)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ee0, ee1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ee0.record(stream)
    e2e_run(args.steps)
    ee1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = dp.max_over_ranks(ee0.elapsed_time(ee1), device=dev)

    # CUDA-graph timing of the step, the forward and the backward (median and min per call over
    # 5 replays of 20 captured calls on the rotating input sets); one GPU only (no NCCL capture)
    graph = None
    if world == 1:
        gs = _graph_time(torch, [(lambda i=i: step(i)) for i in range(NSETS)], reps=5)
        gf = _graph_time(torch, [(lambda i=i: fn_fwd(i)) for i in range(NSETS)], reps=5)
        gb = _graph_time(torch, [(lambda i=i: fn_bwd(i)) for i in range(NSETS)], reps=5)
        graph = {"step_us_median": gs[0], "step_us_min": gs[1], "fwd_us_median": gf[0],
                 "fwd_us_min": gf[1], "bwd_us_median": gb[0], "bwd_us_min": gb[1],
                 "calls_per_graph": 20}

    rows = {}
    if world == 1 and rank == 0 and not args.no_rows:
        rows = extra_rows(q, torch, S, dev, peaks, args)

    toks = T * args.steps * world
    value = toks / (ms / 1e3)
    gemm_flops = 2 * T * d * k + 2 * T * r * d           # base GEMM + adapter K-extension
    g_avg = statistics.mean(g_ms) if g_ms else None
    achieved = gemm_flops / (g_avg / 1e3) / 1e12 if g_avg else None
    # the fused GEMM is timed alone (each launch bracketed by events, a few ms of work at full
    # clock): the measured burst bf16 peak applies; the sustained one is given beside it
    peak = peaks["bf16_tflops"]
    peak_sus = peaks.get("bf16_tflops_sustained")
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": (achieved / peak) if achieved else None,
                "traffic": GEMM_FWD_DRAM_BYTES, "traffic_unit": "bytes per launch",
                "kernel": "k_nf4_gemm2<0> (fused NF4 decode + adapter K-extension, 2-SM tcgen05)",
                "peak_source": f"{peak_src} bf16_tflops (burst: the kernel is timed alone)",
                "frac_of_sustained": (achieved / peak_sus) if (achieved and peak_sus) else None,
                "kernel_ms": g_avg, "algorithmic_flops_per_launch": gemm_flops}
    step_flops = flops_fwd(T, d, k, r) + flops_bwd(T, d, k, r)
    tr_f = t_roof(flops_fwd(T, d, k, r), bytes_fwd(T, d, k, r), peaks)
    tr_b = t_roof(flops_bwd(T, d, k, r), bytes_bwd(T, d, k, r), peaks)
    call_roof = {"t_roof_fwd_us": tr_f * 1e6, "t_roof_bwd_us": tr_b * 1e6,
                 "fwd": tr_f / (fwd_ms / args.steps / 1e3), "bwd": tr_b / (bwd_ms / args.steps / 1e3),
                 "step": (tr_f + tr_b) / (ms / args.steps / 1e3),
                 "definition": "t_roof / t_measured, t_roof = max(FLOPs / bf16_tflops (burst), "
                               "bytes / hbm_gbs); eager timing"}
    if graph:
        call_roof["fwd_graph"] = tr_f * 1e6 / graph["fwd_us_median"]
        call_roof["bwd_graph"] = tr_b * 1e6 / graph["bwd_us_median"]
        call_roof["step_graph"] = (tr_f + tr_b) * 1e6 / graph["step_us_median"]
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": W, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD + " fwd+bwd", "d_out": d, "d_in": k, "r": r, "alpha": alpha,
                   "tokens_per_rank": T, "parallelism": f"dp{world}",
                   "l2": "4 rotating input sets (~300 MB) > 2x L2"},
        "tflops": step_flops * args.steps * world / (ms / 1e3) / 1e12,
        "fwd_ms": fwd_ms / args.steps, "bwd_ms": bwd_ms / args.steps,
        "roofline": roofline,
        "call_roofline": call_roof,
        "e2e": {"value": toks / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(Xd[0].numel() * 2 + dHd[0].numel() * 2),
                "d2h_bytes_per_step": int(dA.numel() * 4 + dB.numel() * 4)},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if graph:
        line["graph"] = graph
    if rows:
        line["rows"] = rows
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_decode_only(args, q, qb, S, torch, dev):
    """The decode-size forward alone on the 11008 x 4096 MLP shape (r = 64): W warm-up and K
    timed eager calls over 8 rotating NF4 weights (> L2), for profiling its kernels."""
    qb.build_library()
    q.load()
    bf = torch.bfloat16
    c3 = S.CONFIGS["mlp_up_11008x4096_r64_T8192"]
    d, k, r, alpha, T = c3["d_out"], c3["d_in"], c3["r"], c3["alpha"], args.tokens
    base = S.make_layer(d, k, r, alpha, T, dtype="bf16", seed=7, with_grad=False)
    W0 = torch.from_numpy(base.W0).to(dev)
    wl = [q.nf4_quantize(W0) for _ in range(8)]
    del W0
    X = torch.from_numpy(base.X).to(dev).to(bf)
    A = torch.from_numpy(base.A).to(dev).to(bf)
    B = torch.from_numpy(base.B).to(dev).to(bf)
    H = torch.empty((T, d), dtype=bf, device=dev)
    ws = torch.empty(q.workspace_bytes(q.OP_FWD, q.BF16, T, d, k, r), dtype=torch.uint8, device=dev)
    W = max(3, args.warmup)
    for i in range(W):
        q.qlora_linear_fwd(wl[i % 8], X, A, B, alpha, H=H, ws=ws, save_u=False)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        q.qlora_linear_fwd(wl[i % 8], X, A, B, alpha, H=H, ws=ws, save_u=False)
    e1.record()
    torch.cuda.synchronize()
    err = q.get_device_error()
    print(json.dumps({"only": "decode", "tokens": T, "ms_per_call": e0.elapsed_time(e1) / args.steps,
                      "device_error": err, "workload": "mlp_up_11008x4096_r64 decode-size forward"}),
          flush=True)
    return 0 if err == 0 else 1


def make_multi_workload(q, torch, dev, n_ad=1024, r_ad=16, T=4096, seed=7, n_w=4):
    """Many-adapter forward workload: 4096^2 NF4 base (n_w rotating copies), n_ad adapters of
    rank r_ad drawn on the device, T tokens with uniform ids."""
    bf = torch.bfloat16
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    W0 = torch.randn((4096, 4096), generator=gen, device=dev) * 0.02 ** 0.5
    wl = [q.nf4_quantize(W0) for _ in range(n_w)]
    del W0
    X = torch.randn((T, 4096), generator=gen, device=dev).to(bf)
    ids = torch.randint(0, n_ad, (T,), generator=gen, device=dev, dtype=torch.int32)
    As = [(torch.randn((r_ad, 4096), generator=gen, device=dev) / r_ad ** 0.5).to(bf) for _ in range(n_ad)]
    Bs = [(torch.randn((4096, r_ad), generator=gen, device=dev) * 0.1).to(bf) for _ in range(n_ad)]
    tab = q.AdapterTable(As, Bs, [2.0 * r_ad] * n_ad)
    H = torch.empty((T, 4096), dtype=bf, device=dev)
    ws = torch.empty(q.workspace_bytes(q.OP_FWD_MULTI, q.BF16, T, 4096, 4096, r_ad),
                     dtype=torch.uint8, device=dev)
    return wl, X, ids, tab, H, ws


def run_multi_only(args, q, qb, torch, dev):
    """The many-adapter forward alone (4096^2, 1024 adapters of rank 16, 4096 tokens): W warm-up
    and K timed eager calls over 4 rotating NF4 weights, for profiling its kernels."""
    qb.build_library()
    q.load()
    wl, X, ids, tab, H, ws = make_multi_workload(q, torch, dev)
    W = max(3, args.warmup)
    for i in range(W):
        q.qlora_linear_fwd_multi(wl[i % 4], X, ids, tab, H=H, ws=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        q.qlora_linear_fwd_multi(wl[i % 4], X, ids, tab, H=H, ws=ws)
    e1.record()
    torch.cuda.synchronize()
    err = q.get_device_error()
    print(json.dumps({"only": "multi", "ms_per_call": e0.elapsed_time(e1) / args.steps,
                      "device_error": err,
                      "workload": "4096x4096 NF4 base, 1024 adapters r=16, T=4096 uniform ids"}), flush=True)
    return 0 if err == 0 else 1


def make_fp8_workload(q, S, torch, dev, n_weights=4, seed=19):
    """The q_proj shape (4096^2, r = 16, T = 4096) with an E4M3 activation: n_weights NF4 copies
    of one weight, their sigma_w, the bf16 and E4M3 activation, adapters, output, workspace."""
    c = S.CONFIGS["q_proj_4096x4096_r16_T4096"]
    bf = torch.bfloat16
    case = S.make_layer(c["d_out"], c["d_in"], c["r"], c["alpha"], c["T"], dtype="bf16", seed=seed,
                        with_grad=False)
    wl = [q.nf4_quantize(torch.from_numpy(case.W0).to(dev)) for _ in range(n_weights)]
    wsc = [q.fp8_weight_scale(w) for w in wl]
    Xb = torch.from_numpy(case.X).to(dev).to(bf)
    X8, xs = q.fp8_quantize(Xb)
    A = torch.from_numpy(case.A).to(dev).to(bf)
    B = torch.from_numpy(case.B).to(dev).to(bf)
    H = torch.empty((c["T"], c["d_out"]), dtype=bf, device=dev)
    ws = torch.empty(q.workspace_bytes(q.OP_FWD_FP8, q.BF16, c["T"], c["d_out"], c["d_in"], c["r"]),
                     dtype=torch.uint8, device=dev)
    return c, wl, wsc, Xb, X8, xs, A, B, H, ws


def run_fp8_only(args, q, qb, S, torch, dev):
    """The FP8 forward alone on the q_proj shape (4096^2, r = 16, T = 4096): W warm-up and K timed
    eager calls over 4 rotating NF4 weights, for profiling its kernels."""
    qb.build_library()
    q.load()
    c, wl, wsc, Xb, X8, xs, A, B, H, ws = make_fp8_workload(q, S, torch, dev)
    if args.only == "fp8bwd":
        G8, gs, dX, dA, dB, wsb = make_fp8_bwd_buffers(q, torch, dev, c)

        def call(i):
            q.qlora_linear_bwd_fp8(wl[i % 4], X8, xs, G8, gs, wsc[i % 4], A, B, c["alpha"], dX=dX, dA=dA,
                                   dB=dB, ws=wsb)
    else:
        def call(i):
            q.qlora_linear_fwd_fp8(wl[i % 4], X8, xs, wsc[i % 4], A, B, c["alpha"], H=H, ws=ws)
    W = max(3, args.warmup)
    for i in range(W):
        call(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        call(i)
    e1.record()
    torch.cuda.synchronize()
    err = q.get_device_error()
    print(json.dumps({"only": args.only, "ms_per_call": e0.elapsed_time(e1) / args.steps,
                      "device_error": err,
                      "workload": "4096x4096 NF4, r=16, T=4096, E4M3 activation"
                                  + (", E5M2 gradient" if args.only == "fp8bwd" else "")}), flush=True)
    return 0 if err == 0 else 1


def make_fp8_bwd_buffers(q, torch, dev, c, seed=23):
    """E5M2 upstream gradient of the q_proj workload and the FP8 backward's outputs and workspace."""
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    dH = torch.randn((c["T"], c["d_out"]), generator=gen, device=dev).to(torch.bfloat16)
    G8, gs = q.fp8_quantize_grad(dH)
    dX = torch.empty((c["T"], c["d_in"]), dtype=torch.bfloat16, device=dev)
    dA = torch.empty((c["r"], c["d_in"]), dtype=torch.float32, device=dev)
    dB = torch.empty((c["d_out"], c["r"]), dtype=torch.float32, device=dev)
    wsb = torch.empty(q.workspace_bytes(q.OP_BWD_FP8, q.BF16, c["T"], c["d_out"], c["d_in"], c["r"]),
                      dtype=torch.uint8, device=dev)
    return G8, gs, dX, dA, dB, wsb


def _graph_time(torch, calls, reps=20):
    """Per-call device time of `calls` (a list of zero-argument launches) captured in one CUDA
    graph and replayed `reps` times: (median, min) microseconds per call over 5 measurements."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for fn in calls:       # warm-up (and one-time host setup) outside the capture
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for fn in calls:
                fn()
    torch.cuda.synchronize()
    for _ in range(3):
        g.replay()
    samples = []
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        samples.append(a.elapsed_time(b) * 1e3 / (reps * len(calls)))
    del g
    return statistics.median(samples), min(samples)


def _kernel_us(torch, q, calls, n_warm):
    """Median device time of the library's main kernel over eager calls (events recorded by the
    library right around that kernel's launch), after n_warm calls."""
    kev = []
    for fn in calls:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        e1.record()
        q.set_gemm_events(e0, e1)
        fn()
        q.set_gemm_events(None, None)
        kev.append((e0, e1))
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) * 1e3 for a, b in kev[n_warm:])


def extra_rows(q, torch, S, dev, peaks, args):
    """The other rows of the hot path, each timed on the device by CUDA-graph replay over
    rotating weight copies whose working set exceeds the 126 MB L2 (median and min per call).
    Fractions: "roof_frac" = t_roof / t, t_roof = max(FLOPs at the measured burst bf16 peak,
    algorithmic bytes at the measured HBM peak) -- the same definition as the headline's
    call_roofline; "tc_frac" is against the burst peak and "tc_frac_sustained" against the
    sustained one (calls that run for seconds settle near it under the power cap)."""
    out = {}
    bf = torch.bfloat16
    hbm = peaks["hbm_gbs"]
    tc = peaks["bf16_tflops"]
    tcs = peaks.get("bf16_tflops_sustained", tc)

    def guarded(name, fn):
        try:
            fn()
        except Exception as e:          # one row failing must not lose the others
            out[name] = {"error": f"{type(e).__name__}: {e}"[:300]}
        torch.cuda.synchronize()
        torch.cuda.empty_cache()

    def fwd_bwd_row(name, d, k, r, alpha, T, wl, X, dH, A, B, reps):
        H = torch.empty((T, d), dtype=bf, device=dev)
        U = torch.empty((T, r), dtype=bf, device=dev)
        dX = torch.empty((T, k), dtype=bf, device=dev)
        dA = torch.empty((r, k), dtype=torch.float32, device=dev)
        dB = torch.empty((d, r), dtype=torch.float32, device=dev)
        ws = torch.empty(max(q.workspace_bytes(q.OP_FWD, q.BF16, T, d, k, r),
                             q.workspace_bytes(q.OP_BWD, q.BF16, T, d, k, r)), dtype=torch.uint8, device=dev)
        fwd = [(lambda w=w: q.qlora_linear_fwd(w, X, A, B, alpha, H=H, U_save=U, ws=ws)) for w in wl]
        bwd = [(lambda w=w: q.qlora_linear_bwd(w, X, dH, A, B, alpha, U_saved=U, dX=dX, dA=dA, dB=dB,
                                               ws=ws)) for w in wl]
        fmed, fmin = _graph_time(torch, fwd, reps=reps)
        bmed, bmin = _graph_time(torch, bwd, reps=reps)
        ff, fb = flops_fwd(T, d, k, r), flops_bwd(T, d, k, r)
        trf, trb = t_roof(ff, bytes_fwd(T, d, k, r), peaks), t_roof(fb, bytes_bwd(T, d, k, r), peaks)
        out[name] = {"fwd_us": fmed, "fwd_us_min": fmin, "bwd_us": bmed, "bwd_us_min": bmin,
                     "fwd_tflops": ff / (fmed * 1e-6) / 1e12, "bwd_tflops": fb / (bmed * 1e-6) / 1e12,
                     "t_roof_fwd_us": trf * 1e6, "t_roof_bwd_us": trb * 1e6,
                     "fwd_roof_frac": trf / (fmed * 1e-6), "bwd_roof_frac": trb / (bmed * 1e-6),
                     "fwd_tc_frac_sustained": ff / (fmed * 1e-6) / 1e12 / tcs,
                     "bwd_tc_frac_sustained": fb / (bmed * 1e-6) / 1e12 / tcs}

    # ---- decode-size forward (T = 1, 4, 16) on the 11008 x 4096 MLP shape, r = 64: an HBM
    # stream of the 4-bit weight (8 rotating copies, 8 x 25 MB > 2 x L2)
    def decode_rows():
        c3 = S.CONFIGS["mlp_up_11008x4096_r64_T8192"]
        d, k, r, alpha = c3["d_out"], c3["d_in"], c3["r"], c3["alpha"]
        NW = 8
        base = S.make_layer(d, k, r, alpha, 16, dtype="bf16", seed=7, with_grad=False)
        W0 = torch.from_numpy(base.W0).to(dev)
        wl = [q.nf4_quantize(W0) for _ in range(NW)]
        del W0
        A = torch.from_numpy(base.A).to(dev).to(bf)
        B = torch.from_numpy(base.B).to(dev).to(bf)
        for T in (1, 4, 16):
            X = torch.from_numpy(base.X[:T]).to(dev).to(bf)
            H = torch.empty((T, d), dtype=bf, device=dev)
            ws = torch.empty(q.workspace_bytes(q.OP_FWD, q.BF16, T, d, k, r), dtype=torch.uint8, device=dev)
            calls = [(lambda w=w: q.qlora_linear_fwd(w, X, A, B, alpha, H=H, ws=ws, save_u=False)) for w in wl]
            med, mn = _graph_time(torch, calls)
            kus = _kernel_us(torch, q, calls * 3, NW)
            byts = w_bytes(d, k) + 2 * T * (k + d) + 2 * r * (d + k)
            out[f"decode_11008x4096_r64_T{T}"] = {
                "call_us": med, "call_us_min": min(mn, med), "kernel_us": kus,
                "GB/s": byts / (med * 1e-6) / 1e9, "hbm_frac": byts / (med * 1e-6) / 1e9 / hbm,
                "kernel_hbm_frac": byts / (kus * 1e-6) / 1e9 / hbm, "bytes": byts,
                "t_roof_us": t_roof(flops_fwd(T, d, k, r), byts, peaks) * 1e6,
                "hbm_peak_gbs": hbm, "device_error": q.get_device_error()}

    # ---- large-T forward and backward on the MLP shape, T = 8192
    def mlp_row():
        c3 = S.CONFIGS["mlp_up_11008x4096_r64_T8192"]
        d, k, r, alpha, T = c3["d_out"], c3["d_in"], c3["r"], c3["alpha"], c3["T"]
        case = S.make_layer(d, k, r, alpha, T, dtype="bf16", seed=11)
        wl = [q.nf4_quantize(torch.from_numpy(case.W0).to(dev)) for _ in range(2)]
        X = torch.from_numpy(case.X).to(dev).to(bf)
        dH = torch.from_numpy(case.dH).to(dev).to(bf)
        A = torch.from_numpy(case.A).to(dev).to(bf)
        B = torch.from_numpy(case.B).to(dev).to(bf)
        del case
        fwd_bwd_row("mlp_11008x4096_r64_T8192", d, k, r, alpha, T, wl, X, dH, A, B, reps=5)

    # ---- 70B-class projections (8192x8192 and 28672x8192, r = 16) at 2048 and 16384 tokens;
    # inputs drawn on the device (W0 ~ N(0, 0.02), X, dH ~ N(0, 1), A ~ N(0, 1/r), B ~ N(0, 0.01)),
    # 2 NF4 copies of the weight
    def proj70b_rows():
        gen = torch.Generator(device=dev)
        gen.manual_seed(7)
        for shape in ("8192x8192", "28672x8192"):
            for T4 in (2048, 16384):
                name = f"proj70b_{shape}_r16_T{T4}"
                cc = S.CONFIGS[name]
                d4, k4, r4, a4 = cc["d_out"], cc["d_in"], cc["r"], cc["alpha"]
                wl = [q.nf4_quantize(torch.randn((d4, k4), generator=gen, device=dev) * (0.02 ** 0.5))
                      for _ in range(2)]
                X = torch.randn((T4, k4), generator=gen, device=dev).to(bf)
                dH = torch.randn((T4, d4), generator=gen, device=dev).to(bf)
                A = (torch.randn((r4, k4), generator=gen, device=dev) / r4 ** 0.5).to(bf)
                B = (torch.randn((d4, r4), generator=gen, device=dev) * 0.1).to(bf)
                fwd_bwd_row(name, d4, k4, r4, a4, T4, wl, X, dH, A, B, reps=3 if T4 > 4096 else 10)
                del wl, X, dH, A, B
                torch.cuda.empty_cache()

    # ---- multi-adapter forward: 4096^2 base, 4 adapters r = 8, 16, 16, 64 (alpha = 2r), T = 4096
    def batched_rows():
        for split_name, split in (("uniform", None), ("skewed", [0.7, 0.1, 0.1, 0.1])):
            mc = S.make_multi_adapter(4096, 4096, 4096, [8, 16, 16, 64], split=split, dtype="bf16", seed=5)
            wl = [q.nf4_quantize(torch.from_numpy(mc.W0).to(dev)) for _ in range(4)]
            X = torch.from_numpy(mc.X).to(dev).to(bf)
            ids = torch.from_numpy(mc.ids).to(dev)
            As = [torch.from_numpy(a).to(dev).to(bf) for a in mc.As]
            Bs = [torch.from_numpy(b).to(dev).to(bf) for b in mc.Bs]
            H = torch.empty((4096, 4096), dtype=bf, device=dev)
            ws = torch.empty(q.workspace_bytes(q.OP_FWD_BATCHED, q.BF16, 4096, 4096, 4096, sum(mc.ranks)),
                             dtype=torch.uint8, device=dev)
            calls = [(lambda w=w: q.qlora_linear_fwd_batched(w, X, ids, As, Bs, mc.alphas, H=H, ws=ws))
                     for w in wl]
            med, mn = _graph_time(torch, calls, reps=10)
            counts = np.bincount(mc.ids, minlength=len(mc.ranks))
            fl = 2 * 4096 * 4096 * 4096 + sum(int(c) * 2 * rr * (4096 + 4096) for c, rr in zip(counts, mc.ranks))
            byts = w_bytes(4096, 4096) + 2 * 4096 * 4096 * 2 + sum(2 * rr * 8192 for rr in mc.ranks)
            tr = t_roof(fl, byts, peaks)
            out[f"batched_4096x4096_4x_{split_name}_T4096"] = {
                "fwd_us": med, "fwd_us_min": mn, "tflops": fl / (med * 1e-6) / 1e12,
                "t_roof_us": tr * 1e6, "roof_frac": tr / (med * 1e-6), "device_error": q.get_device_error()}
            del wl, X, ids, As, Bs, H, ws

    # ---- many-adapter (segmented) forward: 4096^2 base, 1024 adapters of rank 16, T = 4096,
    # ids uniform (about 4 tokens per adapter); adapters drawn on the device (268 MB > L2)
    def multi_row():
        n_ad, r_ad, T_ad = 1024, 16, 4096
        wl, X, ids, tab, H, ws = make_multi_workload(q, torch, dev, n_ad, r_ad, T_ad)
        calls = [(lambda w=w: q.qlora_linear_fwd_multi(w, X, ids, tab, H=H, ws=ws)) for w in wl]
        med, mn = _graph_time(torch, calls, reps=10)
        fl = 2 * T_ad * 4096 * 4096 + 2 * T_ad * r_ad * (4096 + 4096)
        byts = w_bytes(4096, 4096) + 2 * T_ad * 4096 * 3 + n_ad * r_ad * (4096 + 4096) * 2
        tr = t_roof(fl, byts, peaks)
        out["multi_4096x4096_1024xr16_T4096"] = {
            "fwd_us": med, "fwd_us_min": mn, "tokens/s": T_ad / (med * 1e-6),
            "tflops": fl / (med * 1e-6) / 1e12, "t_roof_us": tr * 1e6, "roof_frac": tr / (med * 1e-6),
            "adapter_MB": n_ad * r_ad * 8192 * 2 / 1e6, "device_error": q.get_device_error()}

    # ---- DoRA forward on the q_proj shape (4096^2, r = 16, T = 4096): row norms of W^ + sBA
    # (recomputed every call) + the fused forward with the m / n column scale
    def dora_row():
        c2d = S.CONFIGS["q_proj_4096x4096_r16_T4096"]
        d, k, r, al, T = c2d["d_out"], c2d["d_in"], c2d["r"], c2d["alpha"], c2d["T"]
        case = S.make_layer(d, k, r, al, T, dtype="bf16", seed=17, with_grad=True)
        wl = [q.nf4_quantize(torch.from_numpy(case.W0).to(dev)) for _ in range(4)]
        X = torch.from_numpy(case.X).to(dev).to(bf)
        dH = torch.from_numpy(case.dH).to(dev).to(bf)
        A = torch.from_numpy(case.A).to(dev).to(bf)
        B = torch.from_numpy(case.B).to(dev).to(bf)
        del case
        mag = torch.ones(d, dtype=torch.float32, device=dev)
        H = torch.empty((T, d), dtype=bf, device=dev)
        ws = torch.empty(q.workspace_bytes(q.OP_DORA_FWD, q.BF16, T, d, k, r), dtype=torch.uint8, device=dev)
        calls = [(lambda w=w: q.qlora_dora_fwd(w, X, A, B, al, mag, H=H, save_u=False, ws=ws)) for w in wl]
        med, mn = _graph_time(torch, calls, reps=10)
        fl = flops_fwd(T, d, k, r) + 2 * d * r * k
        tr = t_roof(fl, bytes_fwd(T, d, k, r), peaks)
        row = {"fwd_us": med, "fwd_us_min": mn, "tflops": fl / (med * 1e-6) / 1e12, "t_roof_us": tr * 1e6,
               "roof_frac": tr / (med * 1e-6)}
        # the backward (exact chain rule through the row norm): algorithmic work = the LoRA
        # backward + the norms (2dkr) + the norm's two weight products A W^T and (B^T e) W^
        # (4dkr); the call also recomputes the pre-scale output Z (not counted)
        del H, ws
        dX = torch.empty((T, k), dtype=bf, device=dev)
        dA = torch.empty((r, k), dtype=torch.float32, device=dev)
        dB = torch.empty((d, r), dtype=torch.float32, device=dev)
        dm = torch.empty((d,), dtype=torch.float32, device=dev)
        wsb = torch.empty(q.workspace_bytes(q.OP_DORA_BWD, q.BF16, T, d, k, r), dtype=torch.uint8, device=dev)
        bcalls = [(lambda w=w: q.qlora_dora_bwd(w, X, dH, A, B, al, mag, dX=dX, dA=dA, dB=dB, dm=dm, ws=wsb))
                  for w in wl]
        # eager launches between CUDA events (this call is not captured into a graph here)
        for c_ in bcalls:
            c_()
        torch.cuda.synchronize()
        times = []
        for _ in range(3):
            b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            b0.record()
            for c_ in bcalls:
                c_()
            b1.record()
            torch.cuda.synchronize()
            times.append(b0.elapsed_time(b1) * 1e3 / len(bcalls))
        bmed, bmn = sorted(times)[1], min(times)
        bfl = flops_bwd(T, d, k, r) + 6 * d * k * r
        btr = t_roof(bfl, bytes_bwd(T, d, k, r), peaks)
        row.update({"bwd_us": bmed, "bwd_us_min": bmn, "bwd_tflops": bfl / (bmed * 1e-6) / 1e12,
                    "t_roof_bwd_us": btr * 1e6, "bwd_roof_frac": btr / (bmed * 1e-6)})
        # training form: the forward keeps Z, U and the norms (qlora_dora_fwd_save) and the backward
        # reuses them; one weight's saved tensors serve every timed call (the same arithmetic)
        H2 = torch.empty((T, d), dtype=bf, device=dev)
        wsf = torch.empty(q.workspace_bytes(q.OP_DORA_FWD, q.BF16, T, d, k, r), dtype=torch.uint8, device=dev)
        fcalls = [(lambda w=w: q.qlora_dora_fwd_save(w, X, A, B, al, mag, H=H2, ws=wsf)) for w in wl]
        fmed, _ = _graph_time(torch, fcalls, reps=10)
        _, saved = q.qlora_dora_fwd_save(wl[0], X, A, B, al, mag, H=H2, ws=wsf)
        del wsf
        scalls = [(lambda w=w: q.qlora_dora_bwd(w, X, dH, A, B, al, mag, dX=dX, dA=dA, dB=dB, dm=dm, ws=wsb,
                                                saved=saved)) for w in wl]
        for c_ in scalls:
            c_()
        torch.cuda.synchronize()
        stimes = []
        for _ in range(3):
            b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            b0.record()
            for c_ in scalls:
                c_()
            b1.record()
            torch.cuda.synchronize()
            stimes.append(b0.elapsed_time(b1) * 1e3 / len(scalls))
        smed = sorted(stimes)[1]
        row.update({"fwd_save_us": fmed, "bwd_saved_us": smed, "bwd_saved_roof_frac": btr / (smed * 1e-6),
                    "device_error": q.get_device_error()})
        out["dora_4096x4096_r16_T4096"] = row

    # ---- FP8 forward and backward on the q_proj shape (4096^2, r = 16, T = 4096): E4M3
    # activation, E5M2 gradient, the weight decoded to E4M3 for kind::f8f6f4 tensor cores, the
    # adapter term in bf16.  FP8 peak = measured burst bf16 x 2 (the part's dense fp8 : bf16
    # ratio, 4.5 : 2.25 PFLOP/s).
    def fp8_row():
        c, wl, wsc, Xb, X8, xs, A, B, H, ws = make_fp8_workload(q, S, torch, dev)
        calls = [(lambda w=w, sw=sw: q.qlora_linear_fwd_fp8(w, X8, xs, sw, A, B, c["alpha"], H=H, ws=ws))
                 for w, sw in zip(wl, wsc)]
        med, mn = _graph_time(torch, calls, reps=10)
        kus = _kernel_us(torch, q, calls * 3, 4)
        qws = torch.empty(256, dtype=torch.uint8, device=dev)
        qcalls = [(lambda: q.fp8_quantize(Xb, X8=X8, scale=xs, ws=qws))] * 4
        qmed, _ = _graph_time(torch, qcalls, reps=10)
        T, d, k, r = c["T"], c["d_out"], c["d_in"], c["r"]
        fl = flops_fwd(T, d, k, r)
        tc8 = 2 * tc
        G8, gs, dX, dA, dB, wsb = make_fp8_bwd_buffers(q, torch, dev, c)
        bcalls = [(lambda w=w, sw=sw: q.qlora_linear_bwd_fp8(w, X8, xs, G8, gs, sw, A, B, c["alpha"], dX=dX,
                                                             dA=dA, dB=dB, ws=wsb)) for w, sw in zip(wl, wsc)]
        bmed, bmn = _graph_time(torch, bcalls, reps=10)
        bkus = _kernel_us(torch, q, bcalls * 3, 4)
        bfl = flops_bwd(T, d, k, r)
        dxfl = 2 * T * d * k + 2 * T * r * k
        out["fp8_4096x4096_r16_T4096"] = {
            "fwd_us": med, "fwd_us_min": mn, "tflops": fl / (med * 1e-6) / 1e12,
            "tc_frac_fp8": fl / (med * 1e-6) / 1e12 / tc8, "gemm_us": kus,
            "gemm_tc_frac_fp8": fl / (kus * 1e-6) / 1e12 / tc8, "fp8_peak_tflops": tc8,
            "quantize_us": qmed, "quantize_hbm_frac": 3 * T * k / (qmed * 1e-6) / 1e9 / hbm,
            "bwd_us": bmed, "bwd_us_min": bmn, "bwd_tflops": bfl / (bmed * 1e-6) / 1e12,
            "dx_gemm_us": bkus, "dx_gemm_tc_frac_fp8": dxfl / (bkus * 1e-6) / 1e12 / tc8}

    # ---- AdamW step over the adapters of a 32-layer d = 4096 model with rank 16 on q, k, v, o:
    # 32 * 4 * 16 * (4096 + 4096) = 16.8 M parameters, bf16 params + fp32 master, m, v, grad
    # (30 bytes per parameter, 503 MB > L2)
    def adamw_row():
        n_p = 32 * 4 * 16 * 8192
        gen = torch.Generator(device=dev)
        gen.manual_seed(3)
        master = torch.randn(n_p, generator=gen, device=dev)
        param = master.to(bf)
        grad = torch.randn(n_p, generator=gen, device=dev)
        m_s = torch.zeros(n_p, device=dev)
        v_s = torch.zeros(n_p, device=dev)
        calls = [(lambda t=t: q.adamw_step(param, grad, m_s, v_s, t, 1e-4, weight_decay=0.01, master=master))
                 for t in range(1, 5)]
        med, mn = _graph_time(torch, calls, reps=10)
        byts = 30 * n_p
        out["adamw_16.8M_params"] = {"us": med, "us_min": mn, "GB/s": byts / (med * 1e-6) / 1e9,
                                     "hbm_frac": byts / (med * 1e-6) / 1e9 / hbm}

    # ---- merge W_final = W^ + s B A on the 4096^2 shape, bf16 out
    def merge_row():
        c2_ = S.CONFIGS["q_proj_4096x4096_r16_T4096"]
        d, k, r, alpha = c2_["d_out"], c2_["d_in"], c2_["r"], c2_["alpha"]
        case = S.make_layer(d, k, r, alpha, 1, dtype="bf16", seed=13, with_grad=False)
        wl = [q.nf4_quantize(torch.from_numpy(case.W0).to(dev)) for _ in range(8)]
        A = torch.from_numpy(case.A).to(dev).to(bf)
        B = torch.from_numpy(case.B).to(dev).to(bf)
        outs = [torch.empty((d, k), dtype=bf, device=dev) for _ in range(8)]
        calls = [(lambda w=w, o=o: q.lora_merge(w, A, B, alpha, bf, out=o)) for w, o in zip(wl, outs)]
        med, mn = _graph_time(torch, calls, reps=10)
        byts = w_bytes(d, k) + 2 * d * k + 2 * r * (d + k)
        out["merge_4096x4096_r16_bf16"] = {"us": med, "us_min": mn, "GB/s": byts / (med * 1e-6) / 1e9,
                                           "hbm_frac": byts / (med * 1e-6) / 1e9 / hbm}

    for name, fn in (("decode", decode_rows), ("mlp", mlp_row), ("proj70b", proj70b_rows),
                     ("batched", batched_rows), ("multi", multi_row), ("dora", dora_row),
                     ("fp8", fp8_row), ("adamw", adamw_row), ("merge", merge_row)):
        guarded(name, fn)
    return out


# dram__bytes_read.sum + dram__bytes_write.sum of one k_nf4_gemm2<0> launch at this workload,
# from an ncu capture of the forward call on the q_proj shape
# (44.11 MB read + 16.15 MB written; H is still partly in L2 when the kernel ends).  Set to
# None whenever the kernel changes until it is captured again.
GEMM_FWD_DRAM_BYTES = 44107776 + 16151552


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-rows", action="store_true",
                    help="skip the other hot-path rows (decode-size sweep, 7B MLP, 70B-class, "
                         "multi-adapter, DoRA, FP8, AdamW, merge) that a 1-GPU run reports")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--only", default="step", choices=["step", "fwd", "bwd", "decode", "multi", "fp8", "fp8bwd"],
                    help="time only the forward, only the backward, the decode-size forward "
                         "(11008x4096, r = 64, --tokens T) or the many-adapter forward (4096^2, "
                         "1024 adapters of rank 16), the FP8 forward or the FP8 backward (4096^2, "
                         "r = 16, T = 4096) alone, for profiling its kernels")
    ap.add_argument("--tokens", type=int, default=1, help="tokens of the --only decode run")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())

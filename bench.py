#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 hot path on B200.

The measured step is the largest single-GPU workload: the seven linears of a
70B-shaped decoder layer (q, o 8192 x 8192; k, v 1024 x 8192 (GQA); gate, up
28672 x 8192; down 8192 x 28672), NF4 + double quant, 2048 tokens, LoRA r = 16,
alpha = 32.  One step is one pass of the whole hot path over one batch, for
each linear in turn:
  nf4_quantize (bf16 W -> NF4 codes + fp32 absmax)
  nf4_double_quant (absmax -> E4M3 codes + group scales + mean)
  qlora_linear_fwd (U = X A^T, Y = X dequant(W)^T + s U B^T; dequant fused)
  qlora_linear_bwd (V, dX = dY dequant(W) + s V A, dA, dB)
Throughput counts the GEMM work 4 M N K + 6 M r (K + N) per linear per step
(dequantization and quantization are not counted as FLOPs).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun (N > 1) every rank runs its own batch of 2048 tokens (weak
scaling) and the adapter gradients of all seven linears, held in one flat
buffer, are summed over NCCL by one all-reduce per step (the data-parallel
exchange).  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s & small-M weight GB/s vs B200 roofline"
WORKLOAD = "layer_70b_linears"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=30)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-secondary", action="store_true", help="skip the secondary workloads")
    p.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    p.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) measurement")
    p.add_argument("--leg", choices=["layer", "projection", "smallm", "codec", "merge", "fp4gemm", "mxfp4gemm"], default="layer",
                   help="with --profile: which workload to run")
    p.add_argument("--profile", action="store_true",
                   help="fixed launch sequence for profilers: exactly --warmup then --steps steps of --leg, "
                        "no clock-sampling warm-up, no e2e, secondary or CPU legs")
    a = p.parse_args()
    if a.profile:
        a.no_secondary = a.no_cpu = a.no_e2e = True
    return a


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def config(world: int) -> dict:
    return {"workload": "70B-shaped decoder layer linears (q, o 8192x8192; k, v 1024x8192; gate, up 28672x8192; "
                        "down 8192x28672), bf16 weights quantized to NF4 + double quant each step, 2048 tokens/GPU, "
                        "LoRA r=16 alpha=32 on all seven: quantize + double quant + fwd + bwd (dX, dA, dB)",
            "global_batch": 2048 * world, "tokens_per_gpu": 2048, "linears": 7, "r": 16,
            "parallelism": f"dp{world}", "l2": "flushed between steps (256 MiB write, untimed); inputs > L2",
            "outputs": "Y, dX bf16; dA, dB fp32",
            "schedule": "the seven linears on 3 streams, longest first to the least-loaded stream",
            "launch": "stream order" if os.environ.get("QL_PDL", "1") == "0" else "programmatic dependent launch"}


def gemm_traffic(workload: str = WORKLOAD):
    """Mean DRAM bytes per launch of the fused GEMM on `workload` from the
    committed ncu capture, or None when the kernel source has changed since."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            d = json.load(f)["qlora_gemm_kernel"][workload]
        with open(os.path.join(ROOT, "bit_nf4_quantized_10_b200", "csrc", "gemm.cu"), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
        return float(d["dram_bytes_per_launch"]) if d["gemm_cu_sha256"] == sha else None
    except Exception:
        return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------- the workloads
def _lin_flops(M, N, K, r):
    return 4.0 * M * N * K + 6.0 * M * r * (K + N)


class LinearSet:
    """A list of QLoRA linears resident on one device, each with its bf16 (or
    fp32) master weight, the NF4 + double-quant buffers it is quantized into,
    its batch (X, dY), adapters and outputs.  The adapter gradients of all the
    linears live in one flat buffer (GradBucket), so the data-parallel exchange
    is one all-reduce.  step() runs the whole hot path once."""

    def __init__(self, q, dev, wl, rank=0, w_dtype=None, M=None, streams=1):
        import torch
        from synthetic import inputs as S
        from bit_nf4_quantized_10_b200.dp import GradBucket
        self.q, self.dev, self.wl = q, dev, wl
        self.M = wl.M if M is None else M
        self.r, self.s = wl.r, wl.s
        M, r = self.M, self.r
        self.items = []
        ws = 16
        for j, lin in enumerate(wl.linears):
            d = S.linear_inputs(wl, j, M=M, device=dev)
            W = d["W"] if w_dtype is None else d["W"].to(w_dtype)
            if rank:     # a different batch per rank, same weights and adapters
                d["X"] = S.normal((M, lin.K), 1.0, 100000 + 100 * rank + j, device=dev, dtype=torch.bfloat16)
                d["dY"] = S.normal((M, lin.N), 1.0, 200000 + 100 * rank + j, device=dev, dtype=torch.bfloat16)
            n = lin.N * lin.K
            it = dict(N=lin.N, K=lin.K, W=W, X=d["X"], A=d["A"], B=d["B"], dY=d["dY"],
                      wq=q.NF4Weight.allocate(lin.N, lin.K, dev, dq=True),
                      absmax=torch.empty(-(-n // 64), dtype=torch.float32, device=dev),
                      Y=torch.empty(M, lin.N, dtype=torch.bfloat16, device=dev),
                      U=torch.empty(M, r, dtype=torch.bfloat16, device=dev),
                      dX=torch.empty(M, lin.K, dtype=torch.bfloat16, device=dev))
            it["ws_dq"] = torch.empty(q.qlora_workspace_size(q.QL_OP_DOUBLE_QUANT, it["absmax"].numel()),
                                      dtype=torch.uint8, device=dev)
            ws = max(ws, q.qlora_workspace_size(q.QL_OP_FWD, M, lin.N, lin.K, r),
                     q.qlora_workspace_size(q.QL_OP_BWD, M, lin.N, lin.K, r))
            self.items.append(it)
            del d
        # the linears are independent: with several streams each runs on one of
        # them (each stream with its own workspace), so that one GEMM's last,
        # partly filled wave of tiles overlaps the next linear's work
        self.streams = [torch.cuda.Stream(dev) for _ in range(streams)] if streams > 1 else []
        # longest first, each to the least-loaded stream, so the streams end
        # together and the small linears fill the last waves
        order = sorted(range(len(wl.linears)), key=lambda j: -wl.linears[j].N * wl.linears[j].K)
        load = [0] * max(1, streams)
        self.plan = []
        for j in order:
            k = load.index(min(load))
            load[k] += wl.linears[j].N * wl.linears[j].K
            self.plan.append((j, k))
        self.ws_list = [torch.empty(ws, dtype=torch.uint8, device=dev) for _ in range(max(1, streams))]
        self.ws = self.ws_list[0]
        self.fork = torch.cuda.Event()
        self.joins = [torch.cuda.Event() for _ in self.streams]
        shapes = []
        for it in self.items:
            shapes += [(r, it["K"]), (it["N"], r)]
        self.bucket = GradBucket(shapes, device=dev)
        for i, it in enumerate(self.items):
            it["dA"], it["dB"] = self.bucket.views[2 * i], self.bucket.views[2 * i + 1]

    @property
    def flops(self) -> float:
        return sum(_lin_flops(self.M, it["N"], it["K"], self.r) for it in self.items)

    def gemm_flops(self) -> tuple[float, float]:
        """Algorithmic flop of the forward and backward GEMM launches of one
        step: 2MNK + 2MrN (forward, main product + adapter K-steps) and
        2MNK + 2MrK (backward)."""
        M, r = self.M, self.r
        f = sum(2.0 * M * it["N"] * it["K"] + 2.0 * M * r * it["N"] for it in self.items)
        b = sum(2.0 * M * it["N"] * it["K"] + 2.0 * M * r * it["K"] for it in self.items)
        return f, b

    def _linear(self, it, ws, quantize):
        q, r, s = self.q, self.r, self.s
        wq = it["wq"]
        if quantize:
            q.nf4_quantize(it["W"], wq.codes, it["absmax"])
            q.nf4_double_quant(it["absmax"], wq.absmax_q, wq.scale2, wq.offset, it["ws_dq"])
        q.qlora_linear_fwd(wq, it["X"], it["A"], it["B"], r, s, it["Y"], U_out=it["U"], ws=ws)
        q.qlora_linear_bwd(wq, it["X"], it["dY"], it["A"], it["B"], r, s, it["U"], it["dX"], it["dA"],
                           it["dB"], ws=ws)

    def step(self, allreduce=False, quantize=True, concurrent=True):
        import torch
        if not self.streams or not concurrent:
            for it in self.items:
                self._linear(it, self.ws, quantize)
        else:
            cur = torch.cuda.current_stream(self.dev)
            self.fork.record(cur)
            for st in self.streams:
                st.wait_event(self.fork)
            for j, k in self.plan:
                with torch.cuda.stream(self.streams[k]):
                    self._linear(self.items[j], self.ws_list[k], quantize)
            for st, ev in zip(self.streams, self.joins):
                ev.record(st)
                cur.wait_event(ev)
        if allreduce:
            self.bucket.allreduce()

    def inputs(self):
        """The step's inputs, in a fixed order (the e2e copies)."""
        out = []
        for it in self.items:
            out += [it["W"], it["X"], it["A"], it["B"], it["dY"]]
        return out

    def outputs(self):
        out = [it[k] for it in self.items for k in ("Y", "dX")]
        return out + [self.bucket.buffer]


def trace_read(q):
    import ctypes
    L = q._lib.LIB
    L.qlora_trace_read.restype = ctypes.c_int
    L.qlora_trace_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int), ctypes.c_int]
    L.qlora_trace_kind_name.restype = ctypes.c_char_p
    L.qlora_trace_kind_name.argtypes = [ctypes.c_int]
    ms = (ctypes.c_double * 32)()
    cnt = (ctypes.c_int * 32)()
    n = L.qlora_trace_read(ms, cnt, 32)
    return {L.qlora_trace_kind_name(k).decode(): (ms[k], cnt[k]) for k in range(n) if cnt[k]}


def trace_enable(q, on):
    import ctypes
    L = q._lib.LIB
    L.qlora_trace_enable.argtypes = [ctypes.c_int]
    L.qlora_trace_enable.restype = None
    L.qlora_trace_enable(1 if on else 0)


def trace_enable_kinds(q, names):
    """Trace only the named kernel kinds (an event pair around a launch keeps it
    from overlapping the previous kernel, so the timed steps trace only the
    dominant kernel)."""
    import ctypes
    L = q._lib.LIB
    L.qlora_trace_kind_name.restype = ctypes.c_char_p
    L.qlora_trace_kind_name.argtypes = [ctypes.c_int]
    L.qlora_trace_enable_kinds.argtypes = [ctypes.c_uint]
    L.qlora_trace_enable_kinds.restype = None
    mask = 0
    for k in range(32):
        if L.qlora_trace_kind_name(k).decode() in names:
            mask |= 1 << k
    L.qlora_trace_enable_kinds(mask)


def gemm_roofline(q, ls, run_steps, n_steps, bf16_peak, peak_src, workload):
    """Time `n_steps` steps with only the GEMM launches traced: algorithmic
    flop of those launches / their summed device time, against the bf16 peak."""
    trace_enable_kinds(q, ("qlora_gemm_fwd", "qlora_gemm_bwd"))
    run_steps()
    kern = trace_read(q)
    trace_enable(q, False)
    f_fwd, f_bwd = ls.gemm_flops()
    ms_f, n_f = kern.get("qlora_gemm_fwd", (0.0, 0))
    ms_b, n_b = kern.get("qlora_gemm_bwd", (0.0, 0))
    gemm_ms = ms_f + ms_b
    launches = n_f + n_b
    per_step = len(ls.items)
    achieved = (n_steps * (f_fwd + f_bwd)) / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 and n_f == n_b == n_steps * per_step else 0.0
    return {"bound": "tensor", "kernel": "qlora_gemm (fused NF4 dequant + tcgen05 GEMM + LoRA K-steps)",
            "achieved": achieved, "peak": bf16_peak, "unit": "TFLOP/s", "frac": achieved / bf16_peak,
            "peak_source": f"{peak_src} bf16 burst", "traffic": gemm_traffic(workload),
            "algorithmic_flop_per_launch": (f_fwd + f_bwd) / (2 * per_step), "launches": launches,
            "avg_launch_us": gemm_ms / max(launches, 1) * 1e3}


# --------------------------------------------------------------- CPU oracle
_ORACLE_INPUTS = {}


def cpu_oracle_sample(rows: int = 512, tokens: int = 256):
    """The oracle on a bounded sample of the measured step: linear q of the
    70B-shaped layer (8192 x 8192): quantize + double quant + dequant of `rows`
    weight rows, forward + backward for `tokens` tokens."""
    import torch
    from oracle import lora, nf4
    from synthetic import inputs as S
    w = S.WORKLOADS["c4"]
    if "c4q" not in _ORACLE_INPUTS:
        d = S.linear_inputs(w, 0)
        d["W"] = d["W"].to(torch.bfloat16)
        _ORACLE_INPUTS["c4q"] = d
    d = _ORACLE_INPUTS["c4q"]
    W = d["W"][:rows]
    X, dY = d["X"][:tokens], d["dY"][:tokens, :rows]
    A, B = d["A"], d["B"][:rows]
    K = W.shape[1]
    t0 = time.perf_counter()
    packed, c, _ = nf4.quantize(W)
    e, s2, mu = nf4.double_quant(c)
    What = nf4.dequant(packed, rows * K, nf4.dq_constants(e, s2, mu)).reshape(rows, K)
    Y, U = lora.forward(X, What, A, B, w.s)
    lora.backward(X, What, A, B, w.s, dY, U=U)
    dt = time.perf_counter() - t0
    return _lin_flops(tokens, rows, K, w.r), dt, (f"linear q (8192x8192) of the 70B-shaped layer: weight rows {rows} "
                                                 f"of 8192 (quantize, double quant, dequant), fwd+bwd on {tokens} "
                                                 f"of 2048 tokens")


def cpu_baseline_leg(min_s: float = 10.0, max_reps: int = 30) -> dict:
    """The oracle as it stands on the host cores: the same bounded sample of the
    measured step repeated until at least `min_s` seconds of CPU work."""
    tf, tt, reps, desc = 0.0, 0.0, 0, ""
    while tt < min_s and reps < max_reps:
        f, t, desc = cpu_oracle_sample()
        tf += f
        tt += t
        reps += 1
    return {"value": tf / tt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "host_cores": host_cores(),
            "kind": "oracle", "sample": f"{desc}; {reps} repetitions, {tt:.1f} s (numpy float64: BLAS products on "
                                        f"{blas_threads()} threads, elementwise steps on one)"}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------ end to end
def e2e_leg(q, dev, wl, flops_of, world, rank, n_steps, allreduce):
    """The measured step through the public API with host buffers: every step
    copies its inputs (bf16 weights, X, A, B, dY of the seven linears) in from
    pinned host memory and its results (Y, dX, dA, dB) back out.  Two device
    buffer sets and separate copy streams let step i's input copy and step
    i-1's output copy overlap step i's compute (double buffering, ordered by
    events).  Also measures the copy-only ceiling of the same bytes."""
    import torch
    import torch.distributed as dist
    sets = [LinearSet(q, dev, wl, rank, w_dtype=torch.bfloat16, streams=3) for _ in range(2)]
    h_in = [torch.empty(t.shape, dtype=t.dtype).pin_memory().copy_(t) for t in sets[0].inputs()]
    h_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in sets[0].outputs()]
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = sum(t.numel() * t.element_size() for t in h_out)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    s_comp = torch.cuda.current_stream(dev)

    def run(n):
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_comp = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        for i in range(n):
            st = sets[i % 2]
            if i >= 2:
                s_in.wait_event(ev_comp[i - 2])          # set reused: its last compute read the inputs
            with torch.cuda.stream(s_in):
                for d, h in zip(st.inputs(), h_in):
                    d.copy_(h, non_blocking=True)
                ev_in[i].record(s_in)
            s_comp.wait_event(ev_in[i])
            if i >= 2:
                s_comp.wait_event(ev_out[i - 2])         # its outputs have been read out
            st.step(allreduce)
            ev_comp[i].record(s_comp)
            s_out.wait_event(ev_comp[i])
            with torch.cuda.stream(s_out):
                for h, d in zip(h_out, st.outputs()):
                    h.copy_(d, non_blocking=True)
                ev_out[i].record(s_out)
        s_comp.wait_event(ev_out[n - 1])

    run(3)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_comp)
    run(n_steps)
    e1.record(s_comp)
    torch.cuda.synchronize(dev)
    t = e0.elapsed_time(e1) / 1e3
    if world > 1:
        tt = torch.tensor([t], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        t = float(tt.item())

    # copy-only ceiling: the same bytes each way, no compute
    def copies(n):
        for _ in range(n):
            with torch.cuda.stream(s_in):
                for d, h in zip(sets[0].inputs(), h_in):
                    d.copy_(h, non_blocking=True)
            with torch.cuda.stream(s_out):
                for h, d in zip(h_out, sets[1].outputs()):
                    h.copy_(d, non_blocking=True)
    torch.cuda.synchronize(dev)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(s_comp)
    s_in.wait_event(c0)
    s_out.wait_event(c0)
    copies(3)
    ea, eb = torch.cuda.Event(), torch.cuda.Event()
    ea.record(s_in)
    eb.record(s_out)
    s_comp.wait_event(ea)
    s_comp.wait_event(eb)
    c1.record(s_comp)
    torch.cuda.synchronize(dev)
    t_copy = c0.elapsed_time(c1) / 1e3 / 3
    fl = flops_of(sets[0])
    out = {"value": world * n_steps * fl / t / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "steps": n_steps, "ms_per_step": t / n_steps * 1e3,
           "pipeline": "double-buffered: input copies, compute and output copies on three streams",
           "copy_only_ms_per_step": t_copy * 1e3, "copy_bound_value": world * fl / t_copy / 1e12}
    del sets
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------- secondary lines
def _time_calls(fn, flush, n_warm=2, n=5):
    import torch
    for _ in range(n_warm):
        fn()
    times = []
    for _ in range(n):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times) / 1e3


def secondary_legs(q, dev, hbm_peak, bf16_peak, peak_src, layer_set):
    import torch
    from synthetic import inputs as S
    out = {}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    # the measured layer without the per-step quantization (fwd + bwd only)
    t = _time_calls(lambda: layer_set.step(quantize=False), flush, n_warm=2, n=10)
    out["layer_70b_linears_fwd_bwd_only"] = {"ms": round(t * 1e3, 3), "TFLOPs": round(layer_set.flops / t / 1e12, 1)}
    t_own = t
    t = _time_calls(lambda: layer_set.step(concurrent=False), flush, n_warm=2, n=10)
    out["layer_70b_linears_one_stream"] = {"ms": round(t * 1e3, 3), "TFLOPs": round(layer_set.flops / t / 1e12, 1)}
    out.update(dense_context_leg(layer_set, flush, t_own))
    # the 4096^2 projection: quantize + double quant + fwd + bwd, with its GEMM roofline
    proj = LinearSet(q, dev, S.WORKLOADS["c2"])
    t = _time_calls(proj.step, flush, n_warm=3, n=20)

    def proj_steps():
        for _ in range(10):
            flush.zero_()
            proj.step()
        torch.cuda.synchronize()
    proj_steps()
    rf = gemm_roofline(q, proj, proj_steps, 10, bf16_peak, peak_src, "projection_4096")
    out["projection_4096"] = {"ms": round(t * 1e3, 3), "TFLOPs": round(proj.flops / t / 1e12, 1),
                              "gemm_avg_launch_us": round(rf["avg_launch_us"], 2), "gemm_frac": round(rf["frac"], 3),
                              "gemm_traffic": rf["traffic"]}
    del proj
    torch.cuda.empty_cache()
    out.update(fp4_gemm_leg(q, dev, flush, bf16_peak, layer_set))
    out.update(mlp_leg(q, dev, flush))
    out.update(small_m_and_codec(q, dev, hbm_peak, flush))
    out.update(adamw_leg(q, dev, hbm_peak, layer_set, flush))
    return out


def dense_context_leg(layer_set, flush, t_nf4):
    """Same-box context, not the product: the layer's forward and dX GEMMs with
    the unquantized bf16 weights through torch.matmul (cuBLAS), next to the
    NF4 path's fwd + bwd on the same shapes.  The pages put the cost of
    dequantizing on the fly at under 15% of unquantized throughput
    ("QLoRA: Quantize Base Weights to 4-Bit", Section 3)."""
    import torch
    outs = [(torch.empty_like(it["Y"]), torch.empty_like(it["dX"])) for it in layer_set.items]

    def dense():
        for it, (y, dx) in zip(layer_set.items, outs):
            torch.matmul(it["X"], it["W"].t(), out=y)
            torch.matmul(it["dY"], it["W"], out=dx)

    t = _time_calls(dense, flush, n_warm=2, n=10)
    flop = sum(4.0 * layer_set.M * it["N"] * it["K"] for it in layer_set.items)
    del outs
    return {"torch_bf16_dense_layer_70b": {
        "ms": round(t * 1e3, 3), "TFLOPs": round(flop / t / 1e12, 1),
        "what": "Y = X W^T and dX = dY W per linear, bf16 dense weights, torch.matmul (context only)",
        "nf4_fwd_bwd_over_dense": round(t_nf4 / t, 3)}}


def fp4_gemm_leg(q, dev, flush, bf16_peak, layer_set):
    """The next row's native 4-bit product: the gate linear's shape (2048
    tokens x 28672 x 8192) as NVFP4 x NVFP4 and MXFP4 x MXFP4 GEMMs on the
    block-scaled tensor cores (both operands quantized on the GPU from the
    layer's bf16 tensors), beside the NF4 path's forward GEMM on the same shape
    (no adapter).  The FP4 peak is the measured bf16 peak times the nominal 4x."""
    import torch
    it = layer_set.items[4]
    M, N, K = layer_set.M, it["N"], it["K"]

    def operand(x, rows):
        n = x.numel()
        codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
        sc = torch.empty(n // 16, dtype=torch.uint8, device=dev)
        ts = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.empty(max(256, q.qlora_workspace_size(q.QL_OP_NVFP4, n)), dtype=torch.uint8, device=dev)
        q.nvfp4_quantize(x, codes, sc, ts, ws)
        atoms = torch.empty(q.nvfp4_scale_atoms_bytes(rows, K), dtype=torch.uint8, device=dev)
        q.nvfp4_scale_atoms(sc, rows, K, atoms)
        return codes, atoms, ts

    def mx_operand(x, rows):
        n = x.numel()
        codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
        sc = torch.empty(n // 32, dtype=torch.uint8, device=dev)
        q.mxfp4_quantize(x, codes, sc)
        atoms = torch.empty(q.mxfp4_scale_atoms_bytes(rows, K), dtype=torch.uint8, device=dev)
        q.mxfp4_scale_atoms(sc, rows, K, atoms)
        return codes, atoms

    a, b = operand(it["X"], M), operand(it["W"], N)
    Y = torch.empty(M, N, dtype=torch.float32, device=dev)
    t = _time_calls(lambda: q.nvfp4_gemm(a[0], a[1], a[2], b[0], b[1], b[2], M, N, K, Y), flush, n_warm=3, n=10)
    del a, b
    am, bm = mx_operand(it["X"], M), mx_operand(it["W"], N)
    t_mx = _time_calls(lambda: q.mxfp4_gemm(am[0], am[1], bm[0], bm[1], M, N, K, Y), flush, n_warm=3, n=10)
    del am, bm
    flop = 2.0 * M * N * K
    Yb = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(16, q.qlora_workspace_size(q.QL_OP_FWD, M, N, K, 0)), dtype=torch.uint8, device=dev)
    A0 = torch.empty(0, K, dtype=torch.bfloat16, device=dev)
    B0 = torch.empty(N, 0, dtype=torch.bfloat16, device=dev)
    t_nf4 = _time_calls(lambda: q.qlora_linear_fwd(it["wq"], it["X"], A0, B0, 0, 1.0, Yb, ws=ws), flush, n_warm=3, n=10)
    st = q.qlora_get_status()
    if st != q.QL_OK:
        raise RuntimeError(f"device status: {q.status_string(st)}")
    peak = 4 * bf16_peak
    res = {"nvfp4_gemm_gate_shape": {"us": round(t * 1e6, 2), "TFLOPs": round(flop / t / 1e12, 1),
                                     "frac_fp4_peak": round(flop / t / 1e12 / peak, 3),
                                     "fp4_peak_TFLOPs": round(peak, 1), "shape": [M, N, K],
                                     "nf4_fwd_same_shape_us": round(t_nf4 * 1e6, 2),
                                     "speedup_over_nf4_fwd": round(t_nf4 / t, 2)},
           "mxfp4_gemm_gate_shape": {"us": round(t_mx * 1e6, 2), "TFLOPs": round(flop / t_mx / 1e12, 1),
                                     "frac_fp4_peak": round(flop / t_mx / 1e12 / peak, 3), "shape": [M, N, K],
                                     "speedup_over_nf4_fwd": round(t_nf4 / t_mx, 2)}}
    del Y, Yb
    torch.cuda.empty_cache()
    return res


def mlp_leg(q, dev, flush):
    """The 7B MLP block (gate/up 11008 x 4096, down 4096 x 11008, 8192 tokens,
    r = 64, SiLU-gated), forward + backward."""
    import torch
    from synthetic import inputs as S
    from bit_nf4_quantized_10_b200.mlp import QLoRAMLP
    w3 = S.WORKLOADS["c3"]
    D, H, M, r, s = 4096, 11008, w3.M, w3.r, w3.s
    ws = [q.quantize_weight(S.custom_weight(n, k, w3.wstd, 3000 + i, device=dev), dq=True)
          for i, (n, k) in enumerate(((H, D), (H, D), (D, H)))]
    Ag = S.uniform((r, D), 1 / D ** 0.5, 3003, device=dev)
    Au = S.uniform((r, D), 1 / D ** 0.5, 3004, device=dev)
    Ad = S.uniform((r, H), 1 / H ** 0.5, 3005, device=dev)
    Bg = S.normal((H, r), 0.01, 3006, device=dev, dtype=torch.bfloat16)
    Bu = S.normal((H, r), 0.01, 3007, device=dev, dtype=torch.bfloat16)
    Bd = S.normal((D, r), 0.01, 3008, device=dev, dtype=torch.bfloat16)
    X = S.normal((M, D), 1.0, 3009, device=dev, dtype=torch.bfloat16)
    dy = S.normal((M, D), 1.0, 3010, device=dev, dtype=torch.bfloat16)
    mlp = QLoRAMLP(ws[0], ws[1], ws[2], Ag, Bg, Au, Bu, Ad, Bd, r, s, M)
    y = torch.empty(M, D, dtype=torch.bfloat16, device=dev)

    def mlp_step():
        mlp.forward(X, y)
        mlp.backward(X, dy)

    t = _time_calls(mlp_step, flush)
    res = {"mlp_7b": {"ms": round(t * 1e3, 3), "TFLOPs": round(mlp.flops() / t / 1e12, 1), "tokens": M, "r": r}}
    del mlp, ws, X, dy, y
    torch.cuda.empty_cache()
    return res


def small_m_and_codec(q, dev, hbm_peak, flush):
    """Small-token forward on the 28672 x 8192 weight (HBM-bound on the packed
    weight), the adapter merge of that weight, and the standalone codecs over
    4 Gi bf16 elements (NF4 + double quant; NVFP4; MXFP4)."""
    import torch
    from synthetic import inputs as S
    out = {}
    w5 = S.WORKLOADS["c5"]
    lin = w5.linears[0]
    N, K, r, s = lin.N, lin.K, w5.r, w5.s
    W = S.normal((N, K), w5.wstd, S.seed_of(5, 0, "W"), device=dev)
    wq = q.quantize_weight(W, dq=True)
    del W
    A = S.uniform((r, K), 1.0 / K ** 0.5, S.seed_of(5, 0, "A"), device=dev)
    B = S.normal((N, r), 0.01, S.seed_of(5, 0, "B"), device=dev, dtype=torch.bfloat16)
    wbytes = q.nf4_storage_bytes(N * K, True)
    for M in w5.Ms:
        X = S.normal((M, K), 1.0, S.seed_of(5, 0, "X") + M, device=dev, dtype=torch.bfloat16)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(max(16, q.qlora_workspace_size(q.QL_OP_FWD, M, N, K, r)), dtype=torch.uint8, device=dev)
        t = _time_calls(lambda: q.qlora_linear_fwd(wq, X, A, B, r, s, Y, ws=ws), flush, n_warm=3, n=20)
        gbs = wbytes / t / 1e9
        out[f"M{M}"] = {"us": round(t * 1e6, 2), "weight_GBps": round(gbs, 1), "frac_hbm": round(gbs / hbm_peak, 3)}
    # adapter merge, bf16 output and re-quantized codes + fp32 constants
    n5 = N * K
    W_out = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
    codes_out = torch.empty(n5 // 2, dtype=torch.uint8, device=dev)
    absmax_out = torch.empty(n5 // 64, dtype=torch.float32, device=dev)
    t = _time_calls(lambda: q.qlora_merge(wq, A, B, r, s, W_out=W_out, codes_out=codes_out, absmax_out=absmax_out),
                    flush, n_warm=3, n=10)
    moved = n5 // 2 + n5 // 64 + 4 * (n5 // 16384) + 2 * r * (N + K) + 2 * n5 + n5 // 2 + 4 * (n5 // 64)
    out[f"merge_{N}x{K}_r{r}"] = {"us": round(t * 1e6, 2), "GBps": round(moved / t / 1e9, 1),
                                 "frac_hbm": round(moved / t / 1e9 / hbm_peak, 3), "bytes": moved,
                                 "fma_per_element": r}
    del W_out, codes_out, absmax_out, wq
    torch.cuda.empty_cache()
    # codecs over 4 Gi bf16 elements
    n = w5.codec_n
    x = S.codec_tensor(n, 0.02, S.seed_of(5, 9, "W"), device=dev)
    codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    absmax = torch.empty(n // 64, dtype=torch.float32, device=dev)
    aq = torch.empty(n // 64, dtype=torch.uint8, device=dev)
    s2 = torch.empty(-(-n // 64 // 256), dtype=torch.float32, device=dev)
    mu = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.empty(q.qlora_workspace_size(q.QL_OP_DOUBLE_QUANT, n // 64), dtype=torch.uint8, device=dev)

    def nf4_codec():
        q.nf4_quantize(x, codes, absmax)
        q.nf4_double_quant(absmax, aq, s2, mu, ws)
    t = _time_calls(nf4_codec, flush, n_warm=2, n=5)
    nb = n // 64
    # read x, write codes + absmax, read absmax twice (mean, encode), write E4M3 + scales
    moved = 2 * n + n // 2 + 4 * nb + 2 * 4 * nb + nb + 4 * (nb // 256)
    out["codec_4Gi_bf16"] = {"ms": round(t * 1e3, 3), "GBps": round(moved / t / 1e9, 1),
                             "frac_hbm": round(moved / t / 1e9 / hbm_peak, 3), "bytes": moved}
    del absmax, aq
    sc = torch.empty(n // 16, dtype=torch.uint8, device=dev)
    ts = torch.empty(4, dtype=torch.float32, device=dev)
    wsn = torch.empty(256, dtype=torch.uint8, device=dev)
    t = _time_calls(lambda: q.nvfp4_quantize(x, codes, sc, ts, wsn), flush, n_warm=2, n=5)
    moved = 2 * 2 * n + n // 2 + n // 16         # x read twice (tensor maximum, then codes)
    out["nvfp4_4Gi_bf16"] = {"ms": round(t * 1e3, 3), "GBps": round(moved / t / 1e9, 1),
                             "frac_hbm": round(moved / t / 1e9 / hbm_peak, 3), "bytes": moved}
    t = _time_calls(lambda: q.mxfp4_quantize(x, codes, sc[: n // 32]), flush, n_warm=2, n=5)
    moved = 2 * n + n // 2 + n // 32
    out["mxfp4_4Gi_bf16"] = {"ms": round(t * 1e3, 3), "GBps": round(moved / t / 1e9, 1),
                             "frac_hbm": round(moved / t / 1e9 / hbm_peak, 3), "bytes": moved}
    st = q.qlora_get_status()
    if st != q.QL_OK:
        raise RuntimeError(f"device status after the codec legs: {q.status_string(st)}")
    del x, codes, sc
    torch.cuda.empty_cache()
    return out


def adamw_leg(q, dev, hbm_peak, layer_set, flush):
    """One fused AdamW step over every adapter parameter of the measured layer
    (fp32 parameters and states in device memory; gradients from the bucket)."""
    import torch
    g = layer_set.bucket.buffer
    n = g.numel()
    p = torch.randn(n, device=dev) * 0.01
    m = torch.zeros(n, device=dev)
    v = torch.zeros(n, device=dev)
    pb = torch.empty(n, dtype=torch.bfloat16, device=dev)
    step = [0]

    def upd():
        step[0] += 1
        q.qlora_adamw_step(p, g, m, v, n, step[0], 2e-4, weight_decay=0.01, p_bf16=pb)
    t = _time_calls(upd, flush, n_warm=3, n=20)
    moved = n * (4 * 4 + 3 * 4 + 2)
    return {"adamw_adapters_70b_layer": {"us": round(t * 1e6, 2), "params": n, "GBps": round(moved / t / 1e9, 1),
                                         "frac_hbm": round(moved / t / 1e9 / hbm_peak, 3)}}


# ------------------------------------------------------------------- arms
def run_reference(args, rank):
    """The oracle (CPU, float64 numpy) as the reference arm, rank 0 only."""
    if rank != 0:
        return
    for _ in range(max(0, min(args.warmup, 1))):
        cpu_oracle_sample(64, 64)
    total_f, total_t = 0.0, 0.0
    desc = ""
    for _ in range(args.steps):
        f, t, desc = cpu_oracle_sample()
        total_f += f
        total_t += t
    v = total_f / total_t / 1e12
    line = {"metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_t / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": config(max(1, args.gpus)),
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": blas_threads(), "host_cores": host_cores(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def profile_leg(args, q, dev):
    """A fixed launch sequence of one workload for profilers: layer = the
    measured step (one stream); projection = the 4096^2 step; smallm = the
    16-token forward on the 28672 x 8192 weight; merge = the adapter merge of
    that weight (bf16 output and re-quantized codes); codec = quantize + double
    quant of 256 Mi bf16 elements; fp4gemm / mxfp4gemm = the NVFP4 x NVFP4 /
    MXFP4 x MXFP4 GEMM at 2048 x 4096 x 8192.  Prints per-call device times."""
    import torch
    from synthetic import inputs as S
    w5 = S.WORKLOADS["c5"]
    if args.leg in ("layer", "projection"):
        ls = LinearSet(q, dev, S.WORKLOADS["c4" if args.leg == "layer" else "c2"],
                       w_dtype=torch.bfloat16 if args.leg == "layer" else None)
        call = lambda: ls.step(concurrent=False)
    elif args.leg == "merge":
        lin = w5.linears[0]
        N, K, r = lin.N, lin.K, w5.r
        W = S.normal((N, K), w5.wstd, S.seed_of(5, 0, "W"), device=dev)
        wq = q.quantize_weight(W, dq=True)
        del W
        A = S.uniform((r, K), 1.0 / K ** 0.5, S.seed_of(5, 0, "A"), device=dev)
        B = S.normal((N, r), 0.01, S.seed_of(5, 0, "B"), device=dev, dtype=torch.bfloat16)
        W_out = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
        codes_out = torch.empty(N * K // 2, dtype=torch.uint8, device=dev)
        absmax_out = torch.empty(N * K // 64, dtype=torch.float32, device=dev)
        call = lambda: q.qlora_merge(wq, A, B, r, w5.s, W_out=W_out, codes_out=codes_out, absmax_out=absmax_out)
    elif args.leg == "fp4gemm":
        # NVFP4 x NVFP4 on the block-scaled tensor cores, 2048 x 4096 x 8192
        M, N, K = 2048, 4096, 8192
        fp = []
        for rows, std, seed in ((M, 1.0, 950), (N, 0.015, 951)):
            x = S.normal((rows, K), std, seed, device=dev, dtype=torch.bfloat16)
            codes = torch.empty(rows * K // 2, dtype=torch.uint8, device=dev)
            sc = torch.empty(rows * K // 16, dtype=torch.uint8, device=dev)
            ts = torch.empty(1, dtype=torch.float32, device=dev)
            ws = torch.empty(max(256, q.qlora_workspace_size(q.QL_OP_NVFP4, rows * K)), dtype=torch.uint8, device=dev)
            q.nvfp4_quantize(x, codes, sc, ts, ws)
            atoms = torch.empty(q.nvfp4_scale_atoms_bytes(rows, K), dtype=torch.uint8, device=dev)
            q.nvfp4_scale_atoms(sc, rows, K, atoms)
            fp.append((codes, atoms, ts))
        Yf = torch.empty(M, N, dtype=torch.float32, device=dev)
        (ac, aa, at), (bc, ba, bt) = fp
        call = lambda: q.nvfp4_gemm(ac, aa, at, bc, ba, bt, M, N, K, Yf)
    elif args.leg == "mxfp4gemm":
        # MXFP4 x MXFP4 on the block-scaled tensor cores, 2048 x 4096 x 8192
        M, N, K = 2048, 4096, 8192
        fp = []
        for rows, std, seed in ((M, 1.0, 950), (N, 0.015, 951)):
            x = S.normal((rows, K), std, seed, device=dev, dtype=torch.bfloat16)
            codes = torch.empty(rows * K // 2, dtype=torch.uint8, device=dev)
            sc = torch.empty(rows * K // 32, dtype=torch.uint8, device=dev)
            q.mxfp4_quantize(x, codes, sc)
            atoms = torch.empty(q.mxfp4_scale_atoms_bytes(rows, K), dtype=torch.uint8, device=dev)
            q.mxfp4_scale_atoms(sc, rows, K, atoms)
            fp.append((codes, atoms))
        Ym = torch.empty(M, N, dtype=torch.float32, device=dev)
        (ac, aa), (bc, ba) = fp
        call = lambda: q.mxfp4_gemm(ac, aa, bc, ba, M, N, K, Ym)
    elif args.leg == "smallm":
        lin = w5.linears[0]
        N, K, r, s, M = lin.N, lin.K, w5.r, w5.s, 16
        W = S.normal((N, K), w5.wstd, S.seed_of(5, 0, "W"), device=dev)
        wq = q.quantize_weight(W, dq=True)
        del W
        A = S.uniform((r, K), 1.0 / K ** 0.5, S.seed_of(5, 0, "A"), device=dev)
        B = S.normal((N, r), 0.01, S.seed_of(5, 0, "B"), device=dev, dtype=torch.bfloat16)
        X = S.normal((M, K), 1.0, S.seed_of(5, 0, "X") + M, device=dev, dtype=torch.bfloat16)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(max(16, q.qlora_workspace_size(q.QL_OP_FWD, M, N, K, r)), dtype=torch.uint8, device=dev)
        call = lambda: q.qlora_linear_fwd(wq, X, A, B, r, s, Y, ws=ws)
    else:
        n = 1 << 28
        x = S.codec_tensor(n, 0.02, S.seed_of(5, 9, "W"), device=dev)
        codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
        absmax = torch.empty(n // 64, dtype=torch.float32, device=dev)
        aq = torch.empty(n // 64, dtype=torch.uint8, device=dev)
        s2 = torch.empty(-(-n // 64 // 256), dtype=torch.float32, device=dev)
        mu = torch.empty(1, dtype=torch.float32, device=dev)
        wsq = torch.empty(q.qlora_workspace_size(q.QL_OP_DOUBLE_QUANT, n // 64), dtype=torch.uint8, device=dev)

        def call():
            q.nf4_quantize(x, codes, absmax)
            q.nf4_double_quant(absmax, aq, s2, mu, wsq)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        call()
    times = []
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
    st = q.qlora_get_status()
    if st != q.QL_OK:
        raise RuntimeError(f"device status: {q.status_string(st)}")
    print(json.dumps({"leg": args.leg, "us_per_call": [round(t, 2) for t in times]}), flush=True)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import bit_nf4_quantized_10_b200 as q
    from synthetic import inputs as S

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if args.profile:
        profile_leg(args, q, dev)
        return
    hbm_peak, bf16_peak, bf16_sus, peak_src = peaks()
    wl = S.WORKLOADS["c4"]
    ls = LinearSet(q, dev, wl, rank, w_dtype=torch.bfloat16, streams=3)
    allreduce = world > 1
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > L2 (126 MB)

    clocks = ClockSampler(local_rank)
    clocks.start()
    t_warm = time.time()
    for _ in range(args.warmup):
        ls.step(allreduce)
    torch.cuda.synchronize()
    # clock samples under load: a wall-clock bound, so the step count differs
    # between ranks; these steps therefore skip the collective (every rank must
    # issue the same all-reduces in the same order)
    while time.time() - t_warm < 0.5:
        ls.step(False)
        torch.cuda.synchronize()
    st = q.qlora_get_status()
    if st != q.QL_OK:
        raise RuntimeError(f"device status after warm-up: {q.status_string(st)}")

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record()
        ls.step(allreduce)
        ev[i][1].record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_s = sum(step_ms) / 1e3
    if world > 1:
        tt = torch.tensor([total_s], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        total_s = float(tt.item())
    st = q.qlora_get_status()
    if st != q.QL_OK:
        raise RuntimeError(f"device status after timing: {q.status_string(st)}")
    value = world * args.steps * ls.flops / total_s / 1e12

    # dominant kernel: the fused dequant GEMM, its launches timed by events on
    # the launching stream over the same number of steps (only its kind traced)
    n_rf = args.steps

    # (one stream here: the event pairs time each launch alone)
    def rf_steps():
        for _ in range(n_rf):
            flush.zero_()
            ls.step(allreduce, concurrent=False)
        torch.cuda.synchronize()
    roofline = gemm_roofline(q, ls, rf_steps, n_rf, bf16_peak, peak_src, WORKLOAD)

    # per-kernel breakdown: more steps (untimed, one stream) with every kind traced
    trace_enable(q, True)
    n_br = min(args.steps, 5)
    for _ in range(n_br):
        flush.zero_()
        ls.step(allreduce, concurrent=False)
    torch.cuda.synchronize()
    breakdown = trace_read(q)
    trace_enable(q, False)
    launches_per_step = sum(c for _, c in breakdown.values()) / n_br
    gpu_launches = int(round(launches_per_step * args.steps))

    e2e = None
    if not args.no_e2e:
        e2e = e2e_leg(q, dev, wl, lambda s: s.flops, world, rank, max(5, args.steps // 3), allreduce)

    secondary = None
    if rank == 0 and not args.no_secondary:
        del flush
        torch.cuda.empty_cache()
        secondary = secondary_legs(q, dev, hbm_peak, bf16_peak, peak_src, ls)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline_leg()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_s / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config(world),
            "roofline": roofline,
            "kernels": {k: {"us_per_launch": round(v[0] / v[1] * 1e3, 2), "launches_per_step": v[1] / n_br,
                            "ms_per_step": round(v[0] / n_br, 4)}
                        for k, v in breakdown.items()},
            "gpu_launches": gpu_launches,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "clocks": clk,
            "secondary": secondary,
        }
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Throughput of the outlier-aware W4A8 quantized linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--op forward|backward] [--tokens M]

One step = one pass of the whole hot path -- targeted momentum update,
per-token INT8 quantization, tcgen05 INT8 GEMM with the fused dequant and
outlier compensation -- over every linear of the workload at every token
count, on NL distinct copies of the packed weights (so the weights streamed
in one step exceed the 126 MB L2 and come from HBM).  Default workload:
LLaMA-2-7B-shaped linears (q, k, v, o 4096x4096; gate, up 4096->11008; down
11008->4096), W4A8 per-channel, M in {1, 4, 16, 64}, 1% outlier channels
x100, synthetic seeded data.

metric / unit: effective GB/s = algorithmic bytes of the step / step time
(weights K*N/2, scales 4N, W_O 2*n_O*N, X 2MK, Xq written and read 2MK,
a 4M, outlier codes M*n_O, Y 2MN); TOPS (2MNK) are reported beside it.

N > 1 (torchrun): data-parallel over tokens, weak scaling: every rank runs
the same step on its own token batch with replicated weights; the outlier
column maxima of all linears are combined with one all-reduce(MAX) per step
so every replica keeps the same momentum state.

The forwards of a step are independent (every linear at every token
count), so on one GPU they are spread round-robin over --streams compute
streams (default 4): one GEMM's tail then overlaps the next one's weight
streaming on other SMs.  The roofline line times the GEMMs one after
another on a single stream, so its per-launch figure is unaffected.

``--impl reference`` times the CPU oracle (single thread) on a bounded
sample of the same workload and prints the same JSON line.

``--op backward`` measures the fine-tuning input gradient instead: one step
is qlin_backward_dx on every linear of the workload (default: the Phi-3-mini
W8A8 linears of the Quaff notes) at --tokens tokens; metric TFLOP/s
(2 M N K per linear) against the tensor-core roofline.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_linear_layers_token_b200 import synth  # noqa: E402

METRIC = "W4A8/W8A8 quantized-linear effective TOPS, GB/s and % of INT8/HBM roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def algorithmic_bytes(M, K, N, nO, fmt):
    wbytes = K * N // 2 if fmt != synth.W8_PERCHANNEL else K * N
    gemm = wbytes + 4 * N + (2 * (K // 128) * N if fmt == synth.W4_G128 else 0) + 2 * nO * N \
        + M * K + 4 * M + M * nO + 2 * M * N
    act = 2 * M * K + M * K + 4 * M + M * nO
    return gemm, act


GEMM_SOURCES = ["quantized_linear_layers_token_b200/csrc/gemm.cuh", "quantized_linear_layers_token_b200/csrc/sm100.cuh",
                "quantized_linear_layers_token_b200/csrc/qlin.cu"]


def gemm_sources_sha256():
    """Hash of the GEMM sources' code: comments and blank lines are dropped,
    so a comment edit does not retire the recorded traffic."""
    import hashlib
    import re
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        with open(os.path.join(ROOT, rel)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        code = "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())
        h.update(code.encode())
    return h.hexdigest()


def recorded_traffic(workload, copies):
    """DRAM bytes (read + write) of the GEMM launches of one step, from the
    ncu launch list summarised in profiles/gemm_traffic.json -- only while
    the GEMM sources are the ones that capture was taken with."""
    try:
        with open(os.path.join(ROOT, "profiles", "gemm_traffic.json")) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("sources_sha256") != gemm_sources_sha256():
        return None
    if rec.get("workload") != workload or rec.get("weight_copies") != copies:
        return None
    return rec.get("dram_bytes_per_step")


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


class ClockSampler:
    """SM clocks and clock-event reasons sampled through NVML by a host
    thread every few milliseconds while the timed region runs (reading only;
    no setting of the GPU is changed).  The device is found by its UUID so
    CUDA_VISIBLE_DEVICES remapping does not matter."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.device_index = device_index
        self.period = period_s
        self.samples = []
        self.error = None
        self._stop = None
        self._thread = None

    def _run(self, ready):
        import pynvml as nv
        try:
            import torch
            nv.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(self.device_index).uuid)
            h = nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            masks = [(name, getattr(nv, attr)) for name, attr in self.REASONS]
            while True:
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((mhz, [n for n, m in masks if bits & m]))
                ready.set()
                if self._stop.wait(self.period):
                    break
        except Exception as e:  # sampling is evidence, never a reason to fail the run
            self.error = f"{type(e).__name__}: {e}"
        finally:
            ready.set()
            try:
                nv.nvmlShutdown()
            except Exception:
                pass

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        ready = threading.Event()
        self._thread = threading.Thread(target=self._run, args=(ready,), daemon=True)
        self._thread.start()
        ready.wait(10.0)
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._thread.join(5.0)
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable: " + str(self.error)],
                    "samples": 0}
        reasons = sorted({r for _, rs in self.samples for r in rs})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle on a bounded sample
# ---------------------------------------------------------------------------

class OracleSample:
    """The CPU oracle on a bounded sample of the workload: every linear at
    ``sample_m`` tokens (one weight copy).  Packing is offline and untimed."""

    def __init__(self, wl, sample_m):
        from oracle import oracle
        self.o = oracle
        self.wl = wl
        self.m = sample_m
        self.items = []
        for si, (name, K, N) in enumerate(wl.shapes):
            L = synth.layer(wl, si, M=sample_m)
            Xb = np.ascontiguousarray(L["X"]).view(np.uint16)
            Wb = np.ascontiguousarray(L["W"]).view(np.uint16)
            pk = oracle.pack_layer(Wb, L["O"], wl.fmt)
            self.items.append((Xb, Wb, pk, len(L["O"]), K, N))
        self.bytes = sum(sum(algorithmic_bytes(sample_m, K, N, nO, wl.fmt)) for _, _, _, nO, K, N in self.items)
        self.ops = sum(2 * sample_m * K * N for *_, K, N in self.items)

    def step(self):
        t0 = time.perf_counter()
        for Xb, Wb, pk, nO, K, N in self.items:
            self.o.forward(Xb, Wb, pk, np.ones(nO, np.float32), self.wl.gamma, update_momentum=True)
        return time.perf_counter() - t0

    def describe(self, seconds):
        return (f"every linear of {self.wl.name} ({len(self.items)}) at M={self.m}, one weight copy: "
                f"momentum update, quantization, int64 GEMM, fp64 dequant; {seconds:.1f} s of "
                f"single-threaded CPU time; host has {os.cpu_count()} cores")


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    sample = OracleSample(wl, 4)
    for _ in range(args.warmup):
        sample.step()
    t = sum(sample.step() for _ in range(args.steps))
    gbs = args.steps * sample.bytes / t / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64/f64",
        "data": "synthetic", "tops": args.steps * sample.ops / t / 1e12,
        "config": {"workload": wl.name, "sample": f"all {len(wl.shapes)} linears at M={sample.m}",
                   "parallelism": "single thread"},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample.describe(t / args.steps) + " (per step)"},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def build_problem(wl, copies, device):
    import torch
    from quantized_linear_layers_token_b200 import qlin
    layers = []  # per shape: list of PackedLayer copies
    meta = []
    for si, (name, K, N) in enumerate(wl.shapes):
        L = synth.layer(wl, si, M=1)
        W = torch.from_numpy(L["W"]).to(device)
        base = qlin.PackedLayer.pack(W, L["O"], wl.fmt)
        del W
        cps = [base] + [base.clone() for _ in range(copies - 1)]
        layers.append(cps)
        meta.append({"name": name, "K": K, "N": N, "O": L["O"]})
    inputs = {}
    for M in wl.ms:
        for si, (name, K, N) in enumerate(wl.shapes):
            L = synth.layer(wl, si, M=M, with_weights=False)
            inputs[(M, si)] = L["X"]
    return layers, meta, inputs


def run_profile_case(args, wl):
    """A few qlin_forward calls on one linear of the workload (one weight
    copy), launched eagerly so a profiler sees every kernel: W warm-up
    calls, then K calls timed with CUDA events."""
    import torch
    from quantized_linear_layers_token_b200 import qlin
    name, m = args.profile_case.split(":")
    M = int(m)
    si = [n for n, _, _ in wl.shapes].index(name)
    _, K, N = wl.shapes[si]
    L = synth.layer(wl, si, M=M)
    layer = qlin.PackedLayer.pack(torch.from_numpy(L["W"]).cuda(), L["O"], wl.fmt)
    X = torch.from_numpy(L["X"]).cuda()
    s = torch.ones(max(len(L["O"]), 1), dtype=torch.float32, device="cuda")
    Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    nws = qlin.qlin_forward_workspace(M, layer.w)
    ws = qlin.empty_workspace(nws)
    for _ in range(args.warmup):
        qlin.qlin_forward(X, M, layer.w, s, wl.gamma, True, Y, ws, nws)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        qlin.qlin_forward(X, M, layer.w, s, wl.gamma, True, Y, ws, nws)
    e1.record()
    torch.cuda.synchronize()
    qlin.qlin_poll_device_status()
    us = e0.elapsed_time(e1) * 1e3 / max(args.steps, 1)
    print(json.dumps({"profile_case": args.profile_case, "workload": wl.name, "K": K, "N": N, "M": M,
                      "us_per_forward_eager": us}), flush=True)
    return 0


# ---------------------------------------------------------------------------
# --op backward: the input gradient under the straight-through estimator
# ---------------------------------------------------------------------------

BWD_METRIC = "input-gradient (straight-through estimator) TFLOP/s of the quantized linear layers"


def bwd_flops(M, shapes):
    return sum(2 * M * K * N for _, K, N in shapes)


class OracleBackwardSample:
    """The oracle's dX = (dY Weff^T) on a bounded sample: every linear of
    the workload at ``rows`` token rows (the rows are independent)."""

    def __init__(self, wl, rows):
        from oracle import oracle
        self.o = oracle
        self.wl = wl
        self.rows = rows
        self.items = []
        for si, (name, K, N) in enumerate(wl.shapes):
            L = synth.layer(wl, si, M=1)
            Wb = np.ascontiguousarray(L["W"]).view(np.uint16)
            pk = oracle.pack_layer(Wb, L["O"], wl.fmt)
            dY = np.ascontiguousarray(synth.grad_output(wl.index, si, rows, N)).view(np.uint16)
            s = synth.outlier_scales(wl.index, si, len(L["O"]))
            self.items.append((dY, Wb, pk, s))
        self.flops = bwd_flops(rows, wl.shapes)

    def step(self):
        t0 = time.perf_counter()
        for dY, Wb, pk, s in self.items:
            self.o.backward_dx(dY, Wb, pk, s)
        return time.perf_counter() - t0

    def describe(self, seconds):
        return (f"oracle backward_dx (fp64, single thread) on every linear of {self.wl.name} "
                f"({len(self.items)}) at {self.rows} token rows; {seconds:.1f} s of CPU time; "
                f"host has {os.cpu_count()} cores")


def run_backward_reference(args, wl):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    sample = OracleBackwardSample(wl, 2)
    for _ in range(args.warmup):
        sample.step()
    t = sum(sample.step() for _ in range(args.steps))
    v = args.steps * sample.flops / t / 1e12
    line = {
        "impl": "reference", "metric": BWD_METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "op": "backward", "sample": f"all {len(wl.shapes)} linears at 2 token rows",
                   "parallelism": "single thread"},
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                         "sample": sample.describe(t / args.steps) + " (per step)"},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_backward(args, wl):
    """One step = qlin_backward_dx on every linear of the workload at
    ``--tokens`` tokens (the fine-tuning backward through the frozen
    quantized weights).  N > 1: every rank runs its own token batch, no
    collective (the input gradient has no exchange step)."""
    import torch
    from quantized_linear_layers_token_b200 import qlin

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    M = args.tokens
    if args.profile_case:
        # one linear, eager launches, so a profiler sees each kernel
        si = [n for n, _, _ in wl.shapes].index(args.profile_case)
        _, K, N = wl.shapes[si]
        L = synth.layer(wl, si, M=1)
        lay = qlin.PackedLayer.pack(torch.from_numpy(L["W"]).to(device), L["O"], wl.fmt)
        dY = torch.from_numpy(synth.grad_output(wl.index, si, M, N)).to(device)
        s = torch.from_numpy(synth.outlier_scales(wl.index, si, len(L["O"]))).to(device) if len(L["O"]) else None
        dX = torch.empty((M, K), dtype=torch.float16, device=device)
        nws = qlin.qlin_backward_dx_workspace(M, lay.w)
        ws = qlin.empty_workspace(nws) if nws else None
        for _ in range(args.warmup):
            qlin.qlin_backward_dx(lay.w, dY, M, s, dX, ws, nws)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            qlin.qlin_backward_dx(lay.w, dY, M, s, dX, ws, nws)
        e1.record()
        torch.cuda.synchronize()
        qlin.qlin_poll_device_status()
        us = e0.elapsed_time(e1) * 1e3 / max(args.steps, 1)
        print(json.dumps({"profile_case": args.profile_case, "op": "backward", "workload": wl.name, "K": K, "N": N,
                          "M": M, "us_per_call_eager": us, "tflops": 2 * M * N * K / us / 1e6}), flush=True)
        return 0
    slots = []
    for si, (name, K, N) in enumerate(wl.shapes):
        L = synth.layer(wl, si, M=1)
        lay = qlin.PackedLayer.pack(torch.from_numpy(L["W"]).to(device), L["O"], wl.fmt)
        dY_np = synth.grad_output(wl.index, si, M, N)
        s_np = synth.outlier_scales(wl.index, si, len(L["O"]))
        nws = qlin.qlin_backward_dx_workspace(M, lay.w)
        slots.append({"layer": lay, "K": K, "N": N, "nO": len(L["O"]), "dY_np": dY_np,
                      "ws": qlin.empty_workspace(nws) if nws else None, "nws": nws,
                      "dY": torch.from_numpy(dY_np).to(device),
                      "s": torch.from_numpy(s_np).to(device) if len(L["O"]) else None,
                      "dX": torch.empty((M, K), dtype=torch.float16, device=device)})
    stream = torch.cuda.Stream(device)

    def step():
        for sl in slots:
            qlin.qlin_backward_dx(sl["layer"].w, sl["dY"], M, sl["s"], sl["dX"], sl["ws"], sl["nws"], stream)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    for _ in range(args.warmup):
        with torch.cuda.stream(stream):
            graph.replay()
    torch.cuda.synchronize()
    qlin.qlin_poll_device_status()

    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            with torch.cuda.stream(stream):
                graph.replay()
        ev1.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms_step = ev0.elapsed_time(ev1) / args.steps
    if dist is not None:
        t = torch.tensor([ms_step], device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_step = float(t.item())
    clocks = clk.summary()
    flops = bwd_flops(M, wl.shapes)
    value = world * flops / (ms_step * 1e-3) / 1e12

    # the step is nothing but backward_dx_kernel launches: their average
    # duration is the step time over the launches of a step
    hbm, bf16, bf16_sus, peak_kind = read_peaks()
    achieved = flops / (ms_step * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": achieved, "peak": bf16_sus, "unit": "TFLOP/s",
                "frac": achieved / bf16_sus, "frac_of_burst": achieved / bf16, "traffic": None,
                "peak_source": f"bf16_tflops_sustained of {peak_kind} peaks (fp16 and bf16 have the same "
                               f"dense tensor rate; kernel timed inside a seconds-long loop)",
                "kernel": "backward_dx_kernel, all launches of one step", "flops_per_step": flops,
                "launches_per_step": len(slots)}

    e2e = None
    if world == 1:
        host_dy = [torch.from_numpy(sl["dY_np"]).pin_memory() for sl in slots]
        host_dx = [torch.empty(sl["dX"].shape, dtype=torch.float16).pin_memory() for sl in slots]
        h2d = sum(x.numel() * 2 for x in host_dy)
        d2h = sum(y.numel() * 2 for y in host_dx)
        h2d_stream = torch.cuda.Stream(device)
        d2h_stream = torch.cuda.Stream(device)

        def e2e_step():
            h2d_stream.wait_stream(stream)
            d2h_stream.wait_stream(stream)
            ready = []
            with torch.cuda.stream(h2d_stream):
                for sl, hy in zip(slots, host_dy):
                    sl["dY"].copy_(hy, non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(h2d_stream)
                    ready.append(ev)
            for sl, hx, ev in zip(slots, host_dx, ready):
                stream.wait_event(ev)
                qlin.qlin_backward_dx(sl["layer"].w, sl["dY"], M, sl["s"], sl["dX"], sl["ws"], sl["nws"], stream)
                done = torch.cuda.Event()
                done.record(stream)
                d2h_stream.wait_event(done)
                with torch.cuda.stream(d2h_stream):
                    hx.copy_(sl["dX"], non_blocking=True)
            stream.wait_stream(h2d_stream)
            stream.wait_stream(d2h_stream)

        with torch.cuda.stream(stream):
            e2e_step()
        torch.cuda.synchronize()
        g3 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g3, stream=stream):
            e2e_step()
        with torch.cuda.stream(stream):
            g3.replay()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            with torch.cuda.stream(stream):
                g3.replay()
        ev1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = ev0.elapsed_time(ev1) / args.steps
        e2e = {"value": flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "note": "per linear: pinned host dY -> device (copy stream), qlin_backward_dx (compute stream), "
                       "device -> pinned host dX (second copy stream); one CUDA graph per step"}

    cpu = None
    if rank == 0 and world == 1:
        sample = OracleBackwardSample(wl, 48)
        t = sample.step()
        cpu = {"value": sample.flops / t / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
               "sample": sample.describe(t)}

    if rank == 0:
        dy_bytes = sum(sl["dY"].numel() * 2 for sl in slots)
        line = {
            "metric": BWD_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16 (f32 accumulate)", "data": "synthetic",
            "config": {"workload": wl.name, "op": "backward", "tokens": M,
                       "shapes": [[n, K, N] for n, K, N in wl.shapes], "outlier_frac": wl.outlier_frac,
                       "format": "W4A8 per-channel" if wl.fmt == 0 else ("W4A8 g128" if wl.fmt == 1 else "W8A8"),
                       "l2": f"inputs larger than L2 (dY of one step {dy_bytes / 1e6:.0f} MB)",
                       "parallelism": f"dp{world}",
                       "timing": "CUDA graph of one step, CUDA events on the launch stream"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps * len(slots),
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                       "reasons": clocks["reasons"], "samples": clocks["samples"]},
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama7b_w4_decode")
    ap.add_argument("--copies", type=int, default=4)
    ap.add_argument("--streams", type=int, default=4,
                    help="compute streams the independent forwards of a step are spread over (N = 1)")
    ap.add_argument("--op", default="forward", choices=["forward", "backward"],
                    help="backward: the input gradient of every linear (default workload phi3_w8_quaff)")
    ap.add_argument("--tokens", type=int, default=4096, help="--op backward: tokens per step")
    ap.add_argument("--profile-case", default=None,
                    help="NAME:M -- run only that linear of the workload at M tokens (for ncu captures)")
    args = ap.parse_args()
    if args.op == "backward":
        wl = synth.WORKLOADS["phi3_w8_quaff" if args.workload == "llama7b_w4_decode" else args.workload]
        return run_backward_reference(args, wl) if args.impl == "reference" else run_backward(args, wl)
    wl = synth.WORKLOADS[args.workload]

    if args.impl == "reference":
        return run_reference(args, wl)
    if args.profile_case:
        return run_profile_case(args, wl)

    import torch
    from quantized_linear_layers_token_b200 import qlin

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    layers, meta, inputs_np = build_problem(wl, args.copies, device)
    ms = wl.ms
    nshape = len(wl.shapes)

    # per (M, shape, copy): device input, output, momentum state, workspace
    slots = []
    for M in ms:
        for c in range(args.copies):
            for si in range(nshape):
                lay = layers[si][c]
                X = torch.from_numpy(inputs_np[(M, si)]).to(device)
                Y = torch.empty((M, meta[si]["N"]), dtype=torch.float16, device=device)
                s = torch.ones(max(len(meta[si]["O"]), 1), dtype=torch.float32, device=device)
                nws = qlin.qlin_forward_workspace(M, lay.w)
                ws = qlin.empty_workspace(nws)
                slots.append({"M": M, "si": si, "c": c, "layer": lay, "X": X, "Y": Y, "s": s, "ws": ws,
                              "nws": nws})
    stream = torch.cuda.Stream(device)

    # DP exchange (N > 1): all outlier column maxima of a step in one vector
    from quantized_linear_layers_token_b200.dp import ColmaxExchange
    xchg = ColmaxExchange([len(meta[sl["si"]]["O"]) for sl in slots], device)

    # Independent forwards of a step go round-robin to --streams compute
    # streams forked from (and joined back into) the launch stream, so one
    # GEMM's tail overlaps the next one's weight streaming on other SMs.
    nstreams = max(1, args.streams) if world == 1 else 1
    side = [torch.cuda.Stream(device) for _ in range(nstreams - 1)]

    def step_single():
        if nstreams == 1:
            for sl in slots:
                qlin.qlin_forward(sl["X"], sl["M"], sl["layer"].w, sl["s"], wl.gamma, True, sl["Y"], sl["ws"],
                                  sl["nws"], stream)
            return
        streams = [stream] + side
        fork = torch.cuda.Event()
        fork.record(stream)
        for st in side:
            st.wait_event(fork)
        for j, sl in enumerate(slots):
            qlin.qlin_forward(sl["X"], sl["M"], sl["layer"].w, sl["s"], wl.gamma, True, sl["Y"], sl["ws"],
                              sl["nws"], streams[j % nstreams])
        for st in side:
            done = torch.cuda.Event()
            done.record(st)
            stream.wait_event(done)

    def step_dp():
        for j, sl in enumerate(slots):
            if xchg.n_outliers[j]:
                qlin.qlin_outlier_colmax(sl["X"], sl["M"], sl["layer"].w, xchg.view(j), stream)
        with torch.cuda.stream(stream):
            xchg.allreduce()
        for j, sl in enumerate(slots):
            lay = sl["layer"]
            if xchg.n_outliers[j]:
                qlin.qlin_momentum_update(lay.w, xchg.view(j), sl["s"], wl.gamma, stream)
            # quantization with the already-updated state, then the GEMM
            qlin.qlin_forward(sl["X"], sl["M"], lay.w, sl["s"], wl.gamma, False, sl["Y"], sl["ws"], sl["nws"],
                              stream)

    step = step_single if world == 1 else step_dp

    # warm-up (eager; sets kernel attributes and resolves the driver entry point)
    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()

    graph = None
    if world == 1:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()

    def run_steps(k):
        for _ in range(k):
            if graph is not None:
                with torch.cuda.stream(stream):
                    graph.replay()
            else:
                step()

    # ---------------------------------------------------------------- timed region
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        ev0.record(stream)
        run_steps(args.steps)
        ev1.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms_step = ev0.elapsed_time(ev1) / args.steps
    if dist is not None:
        t = torch.tensor([ms_step], device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_step = float(t.item())
    clocks = clk.summary()

    step_bytes = 0
    step_ops = 0
    gemm_bytes = 0
    for sl in slots:
        m = meta[sl["si"]]
        g, a = algorithmic_bytes(sl["M"], m["K"], m["N"], len(m["O"]), wl.fmt)
        step_bytes += g + a
        gemm_bytes += g
        step_ops += 2 * sl["M"] * m["K"] * m["N"]
    value = world * step_bytes / (ms_step * 1e-3) / 1e9

    # ---------------------------------------------------------------- GEMM-only timing (roofline)
    gemm_slots = []
    for sl in slots:
        M, lay = sl["M"], sl["layer"]
        K, nO = meta[sl["si"]]["K"], len(meta[sl["si"]]["O"])
        Xq = torch.empty((M, K), dtype=torch.int8, device=device)
        a = torch.empty(M, dtype=torch.float32, device=device)
        XqO = torch.empty((M, max(nO, 1)), dtype=torch.int8, device=device)
        naws = qlin.qlin_quant_act_workspace(M, lay.w)
        aws = qlin.empty_workspace(naws)
        qlin.qlin_quant_act(sl["X"], M, lay.w, sl["s"], wl.gamma, False, Xq, a, XqO, aws, naws, stream)
        gemm_slots.append((sl, Xq, a, XqO, aws, naws))
    torch.cuda.synchronize()

    def gemm_pass():
        # qlin_gemm = the compensation-operand kernel (when n_O > 0) + the tcgen05 GEMM kernel
        for sl, Xq, a, XqO, _, _ in gemm_slots:
            qlin.qlin_gemm(sl["layer"].w, Xq, a, XqO, sl["s"], sl["M"], sl["Y"], None, sl["ws"], sl["nws"], stream)

    gemm_pass()
    torch.cuda.synchronize()
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, stream=stream):
        gemm_pass()
    for _ in range(3):
        with torch.cuda.stream(stream):
            g2.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    reps = max(5, args.steps)
    e0.record(stream)
    for _ in range(reps):
        with torch.cuda.stream(stream):
            g2.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    gemm_ms = e0.elapsed_time(e1) / reps
    n_gemm_launches = len(gemm_slots)

    # ---------------------------------------------------------------- activation quantization alone
    # (momentum update + per-token INT8 codes, the forward's own path; one
    # stream, CUDA graph).  Evidence only: an error is reported in the line,
    # it does not fail the run.
    act_quant = None
    try:
        def quant_pass():
            for sl, Xq, a, XqO, aws, naws in gemm_slots:
                qlin.qlin_quant_act(sl["X"], sl["M"], sl["layer"].w, sl["s"], wl.gamma, True, Xq, a, XqO, aws,
                                    naws, stream)

        quant_pass()
        torch.cuda.synchronize()
        g4 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g4, stream=stream):
            quant_pass()
        for _ in range(3):
            with torch.cuda.stream(stream):
                g4.replay()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            with torch.cuda.stream(stream):
                g4.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        qlin.qlin_poll_device_status()
        act_ms = e0.elapsed_time(e1) / reps
        act_bytes = sum(algorithmic_bytes(sl["M"], meta[sl["si"]]["K"], meta[sl["si"]]["N"],
                                          len(meta[sl["si"]]["O"]), wl.fmt)[1] for sl, *_ in gemm_slots)
        act_gbs = act_bytes / (act_ms * 1e-3) / 1e9
        act_quant = {"bound": "hbm", "achieved": act_gbs, "unit": "GB/s", "algorithmic_bytes": act_bytes,
                     "ms_per_step": act_ms, "calls_per_step": len(gemm_slots),
                     "kernel": "qlin_quant_act (colmax above 16 tokens, then quant_kernel), one stream"}
    except Exception as ex:  # evidence only
        act_quant = {"error": f"{type(ex).__name__}: {ex}"[:300]}

    hbm, bf16, bf16_sus, peak_kind = read_peaks()
    achieved = gemm_bytes / (gemm_ms * 1e-3) / 1e9
    if act_quant is not None and "achieved" in act_quant:
        act_quant["peak"] = hbm
        act_quant["frac"] = act_quant["achieved"] / hbm
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": recorded_traffic(wl.name, args.copies),
                "traffic_unit": "bytes per step (all GEMM launches), ncu dram__bytes_read.sum + dram__bytes_write.sum",
                "algorithmic_bytes": gemm_bytes,
                "peak_source": f"hbm_gbs of {peak_kind} peaks (copy burst)",
                "kernel": "qlin_gemm (comp operand + tcgen05 GEMM), all launches of one step",
                "ms_per_step": gemm_ms, "launches_per_step": n_gemm_launches}

    # ---------------------------------------------------------------- end to end through the API
    e2e = None
    if world == 1:
        host_x = [torch.from_numpy(inputs_np[(sl["M"], sl["si"])]).pin_memory() for sl in slots]
        host_y = [torch.empty(sl["Y"].shape, dtype=torch.float16).pin_memory() for sl in slots]
        h2d = sum(x.numel() * 2 for x in host_x)
        d2h = sum(y.numel() * 2 for y in host_y)

        # copies overlap compute: every X goes up on its own stream, each
        # forward waits only for its own input, each Y comes down on a third
        # stream as soon as its forward has finished
        h2d_stream = torch.cuda.Stream(device)
        d2h_stream = torch.cuda.Stream(device)

        def e2e_step():
            h2d_stream.wait_stream(stream)
            d2h_stream.wait_stream(stream)
            ready = []
            with torch.cuda.stream(h2d_stream):
                for sl, hx in zip(slots, host_x):
                    sl["X"].copy_(hx, non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(h2d_stream)
                    ready.append(ev)
            streams = [stream] + side
            fork = torch.cuda.Event()
            fork.record(stream)
            for st in side:
                st.wait_event(fork)
            for j, (sl, hy, ev) in enumerate(zip(slots, host_y, ready)):
                cs = streams[j % nstreams]
                cs.wait_event(ev)
                qlin.qlin_forward(sl["X"], sl["M"], sl["layer"].w, sl["s"], wl.gamma, True, sl["Y"], sl["ws"],
                                  sl["nws"], cs)
                done = torch.cuda.Event()
                done.record(cs)
                d2h_stream.wait_event(done)
                with torch.cuda.stream(d2h_stream):
                    hy.copy_(sl["Y"], non_blocking=True)
            for st in side:
                joined = torch.cuda.Event()
                joined.record(st)
                stream.wait_event(joined)
            stream.wait_stream(h2d_stream)
            stream.wait_stream(d2h_stream)

        with torch.cuda.stream(stream):
            e2e_step()
        torch.cuda.synchronize()
        g3 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g3, stream=stream):
            e2e_step()
        with torch.cuda.stream(stream):
            g3.replay()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            with torch.cuda.stream(stream):
                g3.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / args.steps
        e2e = {"value": step_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "note": "per linear: pinned host X -> device (copy stream), qlin_forward (the step's compute "
                       "streams, round-robin), device -> pinned host Y (second copy stream); copies overlap other "
                       "linears' compute; one CUDA graph per step"}

    # ---------------------------------------------------------------- CPU baseline (rank 0, N = 1)
    cpu = None
    if rank == 0 and world == 1:
        sample = OracleSample(wl, 16)
        t = sample.step()
        cpu = {"value": sample.bytes / t / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": sample.describe(t)}

    # per forward: quantization (+ the column-max kernel when the library
    # does not fuse the momentum update into quantization, above 16 tokens)
    # and the GEMM; data-parallel steps run the column-max and momentum
    # kernels separately around the all-reduce
    def forward_launches(sl):
        has_o = len(meta[sl["si"]]["O"]) > 0
        if world > 1:
            return 2 + (2 if has_o else 0)
        return 2 + (1 if has_o and sl["M"] > 16 else 0)
    gpu_launches = args.steps * sum(forward_launches(sl) for sl in slots)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "tops": world * step_ops / (ms_step * 1e-3) / 1e12,
            "config": {"workload": wl.name, "shapes": [[n, K, N] for n, K, N in wl.shapes], "M": ms,
                       "weight_copies": args.copies,
                       "weight_bytes_per_step": int(sum(layers[si][0].nbytes for si in range(nshape)) * args.copies
                                                    * len(ms)),
                       "l2": "inputs larger than L2 (distinct packed-weight copies rotated each step)",
                       "outlier_frac": wl.outlier_frac, "gamma": wl.gamma, "format": "W4A8 per-channel"
                       if wl.fmt == 0 else ("W4A8 g128" if wl.fmt == 1 else "W8A8"),
                       "parallelism": f"dp{world}", "forwards_per_step": len(slots),
                       "timing": "CUDA graph of one step, CUDA events on the launch stream",
                       "streams": nstreams},
            "roofline": roofline, "act_quant": act_quant, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": gpu_launches,
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                       "reasons": clocks["reasons"], "samples": clocks["samples"]},
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

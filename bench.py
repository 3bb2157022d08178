"""Throughput of the outlier-aware W4A8 / W8A8 quantized linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--extras LIST] [--op forward|backward]

One step = one pass of the whole hot path -- targeted momentum update,
per-token INT8 quantization, tcgen05 INT8 GEMM with the fused dequant and
outlier compensation -- over every linear of the workload at every token
count.  Default workload: LLaMA-2-70B-shaped linears (q 8192x8192, kv
8192->1024, up 8192->28672, down 28672->8192), W4A8 with g = 128 group
scales, M in {1, 16, 128, 1024, 8192} tokens, 1% outlier channels x100,
synthetic seeded data (no weights or datasets are used).

metric / unit: effective TOPS = 2 M N K of every linear of the step / step
time.  The line also carries the step's effective GB/s over the fused
layer's algorithmic bytes (X 2MK, packed weights, scales, W_O, Y 2MN), and
per token count a bucket timed on its own (median of >= 20 CUDA-graph
replays) with its roofline: the bound is whichever of HBM bytes / measured
copy bandwidth and INT8 ops / INT8 peak takes longer (decode buckets are
HBM-bound, prefill buckets tensor-bound).  The INT8 peak is twice the
measured dense bf16 figure (the nominal INT8 : bf16 ratio of B200).

``roofline`` is the dominant kernel's: the GEMM calls of the prefill
buckets (INT4 widened once per call, then the INT8 tcgen05 GEMM), timed
alone on one stream.

``workloads`` holds the other workloads the layer is specified on, each
measured the same way: the LLaMA-2-7B decode set (W4A8 per-channel, M in
{1, 4, 16, 64}, four weight copies so weights come from HBM), the 7B
prefill set (W4A8 g128, M in {512, 2048, 4096}), the Phi-3-mini W8A8 Quaff
step (M = 4096, momentum update on) and the fine-tuning input gradient of
the Phi-3-mini linears.

N > 1 (torchrun): data-parallel over tokens, weak scaling: every rank runs
the same step on its own token batch with replicated weights; the outlier
column maxima of all linears are combined with one all-reduce(MAX) per step
so every replica keeps the same momentum state.

``--impl reference`` times the CPU oracle (single thread) on a bounded
sample of the same workload and prints the same JSON line.

``--op backward`` measures only the fine-tuning input gradient: one step is
qlin_backward_dx on every linear of the workload (default: the Phi-3-mini
W8A8 linears of the Quaff notes) at --tokens tokens; metric TFLOP/s.
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
INT8_PER_BF16 = 2.0  # nominal dense INT8 : bf16 tensor rate of B200 (4.5 : 2.25 PFLOP/s)
DEFAULT_WORKLOAD = "llama70b_w4g128"
DEFAULT_EXTRAS = "llama7b_w4_decode,llama7b_w4g128_prefill,phi3_w8_quaff,backward,gptq,smooth_search,offq"


# ---------------------------------------------------------------------------
# algorithmic work
# ---------------------------------------------------------------------------

def weight_bytes(K, N, nO, fmt):
    """Packed weights a forward must read once: codes, channel scales, the
    g128 ratios, the fp16 outlier rows W_O, wmax_O, O and the state s."""
    codes = K * N // 2 if fmt != synth.W8_PERCHANNEL else K * N
    ratios = 2 * (K // 128) * N if fmt == synth.W4_G128 else 0
    return codes + 4 * N + ratios + 2 * nO * N + 4 * nO + 4 * nO + 8 * nO


def layer_bytes(M, K, N, nO, fmt):
    """The fused layer's algorithmic bytes: X in, packed weights, Y out."""
    return 2 * M * K + weight_bytes(K, N, nO, fmt) + 2 * M * N


def algorithmic_bytes(M, K, N, nO, fmt):
    """(GEMM call, quantization call): the bytes each of the two stages must
    move at least once when they run as separate kernels (the GEMM reads the
    INT8 codes, token scales and outlier codes the quantization wrote)."""
    wbytes = K * N // 2 if fmt != synth.W8_PERCHANNEL else K * N
    gemm = wbytes + 4 * N + (2 * (K // 128) * N if fmt == synth.W4_G128 else 0) + 2 * nO * N \
        + M * K + 4 * M + M * nO + 2 * M * N
    act = 2 * M * K + M * K + 4 * M + M * nO
    return gemm, act


# The GEMM kernels' sources, and the part of the host file that plans and
# launches them (between its "TMA maps" and "act quant" section markers).
TRAFFIC_SOURCES = ("quantized_linear_layers_token_b200/csrc/gemm.cuh",
                   "quantized_linear_layers_token_b200/csrc/gemm_pair.cuh",
                   "quantized_linear_layers_token_b200/csrc/sm100.cuh",
                   "quantized_linear_layers_token_b200/csrc/qlin.cu:TMA maps:act quant")


def gemm_sources_sha256():
    """sha256 of the GEMM sources with // comments and blank lines removed, so
    a recorded DRAM-traffic figure is used only while the code it was taken
    on is unchanged."""
    import hashlib
    import re
    h = hashlib.sha256()
    for spec in TRAFFIC_SOURCES:
        rel, *section = spec.split(":")
        with open(os.path.join(ROOT, rel)) as f:
            lines = f.readlines()
        if section:
            start = next(i for i, l in enumerate(lines) if l.startswith("// ---") and l.rstrip().endswith(section[0]))
            end = next(i for i, l in enumerate(lines) if l.startswith("// ---") and l.rstrip().endswith(section[1]))
            lines = lines[start:end]
        for line in lines:
            line = re.sub(r"//.*", "", line).rstrip()
            if line:
                h.update(line.encode() + b"\n")
    return h.hexdigest()


def recorded_traffic(workload):
    """DRAM bytes of the headline roofline's launch set from the ncu capture
    recorded under profiles/, or None if there is none for these sources."""
    p = os.path.join(ROOT, "profiles", f"gemm_traffic_{workload}.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d if d.get("sources_sha256") == gemm_sources_sha256() else None
    except Exception:
        return None


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm": float(d["hbm_gbs"]), "bf16": float(d["bf16_tflops"]),
                "bf16_sus": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "kind": "measured"}
    except Exception:
        return {"hbm": FALLBACK_HBM_GBS, "bf16": FALLBACK_BF16_TFLOPS, "bf16_sus": 1400.0, "kind": "fallback"}


def roofline_of(ops, nbytes, seconds, peaks):
    """Roofline of work that moves `nbytes` and does `ops` INT8 operations in
    `seconds`: the bound is whichever of the HBM time (bytes / measured copy
    bandwidth) and the tensor time (ops / INT8 peak) is longer; frac is that
    time over the measured one."""
    int8 = INT8_PER_BF16 * peaks["bf16"]
    t_hbm = nbytes / (peaks["hbm"] * 1e9)
    t_tc = ops / (int8 * 1e12)
    if t_hbm >= t_tc:
        ach = nbytes / seconds / 1e9
        return {"bound": "hbm", "achieved": ach, "peak": peaks["hbm"], "unit": "GB/s", "frac": ach / peaks["hbm"],
                "peak_source": f"hbm_gbs of {peaks['kind']} peaks (copy)"}
    ach = ops / seconds / 1e12
    return {"bound": "tensor", "achieved": ach, "peak": int8, "unit": "TOPS", "frac": ach / int8,
            "frac_of_sustained": ach / (INT8_PER_BF16 * peaks["bf16_sus"]),
            "peak_source": f"INT8 = {INT8_PER_BF16:g} x bf16_tflops (burst) of {peaks['kind']} peaks"}


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
        self.max_mhz = None

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


def fmt_name(fmt):
    return "W4A8 per-channel" if fmt == 0 else ("W4A8 g128" if fmt == 1 else "W8A8")


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle on a bounded sample
# ---------------------------------------------------------------------------

class OracleSample:
    """The CPU oracle on a bounded sample of the workload: the linears
    ``shape_ids`` at ``sample_m`` tokens each (one weight copy).  Packing is
    offline and untimed."""

    def __init__(self, wl, sample_m, shape_ids=None):
        from oracle import oracle
        self.o = oracle
        self.wl = wl
        self.m = sample_m
        self.items = []
        ids = list(range(len(wl.shapes))) if shape_ids is None else shape_ids
        for si in ids:
            name, K, N = wl.shapes[si]
            L = synth.layer(wl, si, M=sample_m)
            Xb = np.ascontiguousarray(L["X"]).view(np.uint16)
            Wb = np.ascontiguousarray(L["W"]).view(np.uint16)
            pk = oracle.pack_layer(Wb, L["O"], wl.fmt)
            pk["Bt"] = np.ascontiguousarray(pk["B"].T)
            self.items.append((name, Xb, Wb, pk, len(L["O"]), K, N))
        self.bytes = sum(layer_bytes(sample_m, K, N, nO, wl.fmt) for *_, nO, K, N in self.items)
        self.ops = sum(2 * sample_m * K * N for *_, K, N in self.items)

    def step(self):
        t0 = time.perf_counter()
        for _, Xb, Wb, pk, nO, K, N in self.items:
            self.o.forward(Xb, Wb, pk, np.ones(nO, np.float32), self.wl.gamma, update_momentum=True)
        return time.perf_counter() - t0

    def describe(self, seconds):
        names = ", ".join(it[0] for it in self.items)
        return (f"{names} of {self.wl.name} at M={self.m}, one weight copy: momentum update, quantization, "
                f"int64 GEMM, fp64 dequant; {seconds:.2f} s of single-threaded CPU time; "
                f"host has {os.cpu_count()} cores")


def oracle_sample_for(wl):
    """Bounded oracle sample of a workload (about 10-30 s of CPU time in
    all, packing included): for the 70B set the two square-ish linears at
    one token, else every linear at four tokens."""
    if wl.name == "llama70b_w4g128":
        return OracleSample(wl, 1, shape_ids=[0, 1])
    if wl.name == "phi3_w8_quaff":
        return OracleSample(wl, 2)
    return OracleSample(wl, 4)


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    sample = oracle_sample_for(wl)
    for _ in range(args.warmup):
        sample.step()
    t = sum(sample.step() for _ in range(args.steps))
    tops = args.steps * sample.ops / t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": tops, "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64/f64",
        "data": "synthetic", "gbs": args.steps * sample.bytes / t / 1e9,
        "config": {"workload": wl.name, "sample": sample.describe(t / args.steps),
                   "parallelism": "single thread"},
        "cpu_baseline": {"value": tops, "unit": "TOPS", "cores": 1, "kind": "oracle",
                         "sample": sample.describe(t / args.steps) + " (per step)"},
        "e2e": {"value": tops, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm: timing helpers
# ---------------------------------------------------------------------------

def graph_of(fn, stream):
    import torch
    with torch.cuda.stream(stream):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def replay_median_ms(graph, stream, reps, warm=3):
    """Median over `reps` replays, each bracketed by its own CUDA events on
    the launch stream."""
    import torch
    for _ in range(warm):
        with torch.cuda.stream(stream):
            graph.replay()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for e0, e1 in evs:
        e0.record(stream)
        with torch.cuda.stream(stream):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)


class ForwardWorkload:
    """Packed weights, inputs, outputs and workspaces of one forward workload
    on one device: slot = (M, copy, linear)."""

    GROUP_MAX_M = 64     # token counts the grouped entry point takes
    GROUP_MAX_COUNT = 32  # problems per grouped call

    def __init__(self, wl, copies, device, ms=None, grouped=True):
        import torch
        from quantized_linear_layers_token_b200 import qlin
        self.q = qlin
        self.wl = wl
        self.copies = copies
        self.grouped = grouped
        self.device = device
        self._group_ws = {}
        self.ms = list(wl.ms if ms is None else ms)
        self.meta = []
        layers = []
        for si, (name, K, N) in enumerate(wl.shapes):
            L = synth.layer(wl, si, M=1)
            W = torch.from_numpy(L["W"]).to(device)
            base = qlin.PackedLayer.pack(W, L["O"], wl.fmt)
            del W
            layers.append([base] + [base.clone() for _ in range(copies - 1)])
            self.meta.append({"name": name, "K": K, "N": N, "nO": len(L["O"])})
        self.layers = layers
        self.x_np = {}
        self.slots = []
        for M in self.ms:
            for si, (name, K, N) in enumerate(wl.shapes):
                self.x_np[(M, si)] = synth.layer(wl, si, M=M, with_weights=False)["X"]
            for c in range(copies):
                for si in range(len(wl.shapes)):
                    lay = layers[si][c]
                    nO = self.meta[si]["nO"]
                    nws = qlin.qlin_forward_workspace(M, lay.w)
                    self.slots.append({
                        "M": M, "si": si, "c": c, "layer": lay,
                        "X": torch.from_numpy(self.x_np[(M, si)]).to(device),
                        "Y": torch.empty((M, self.meta[si]["N"]), dtype=torch.float16, device=device),
                        "s": torch.ones(max(nO, 1), dtype=torch.float32, device=device),
                        "ws": qlin.empty_workspace(nws, device), "nws": nws})

    def ops(self, slots=None):
        return sum(2 * sl["M"] * self.meta[sl["si"]]["K"] * self.meta[sl["si"]]["N"] for sl in (slots or self.slots))

    def bytes(self, slots=None):
        return sum(layer_bytes(sl["M"], self.meta[sl["si"]]["K"], self.meta[sl["si"]]["N"], self.meta[sl["si"]]["nO"],
                               self.wl.fmt) for sl in (slots or self.slots))

    def forward(self, sl, stream, update=True):
        self.q.qlin_forward(sl["X"], sl["M"], sl["layer"].w, sl["s"], self.wl.gamma, update, sl["Y"], sl["ws"],
                            sl["nws"], stream)

    def units(self, slots):
        """Launch units of a list of slots: decode-sized token counts go in
        groups of up to 32 independent linears (one qlin_forward_grouped
        call each), larger ones one qlin_forward call per linear."""
        out, pend = [], {}
        for sl in slots:
            if self.grouped and sl["M"] <= self.GROUP_MAX_M:
                pend.setdefault(sl["M"], []).append(sl)
            else:
                out.append([sl])
        for M, sls in pend.items():
            for i in range(0, len(sls), self.GROUP_MAX_COUNT):
                out.append(sls[i:i + self.GROUP_MAX_COUNT])
        return out

    def run_unit(self, unit, stream, update=True):
        if len(unit) == 1 and not (self.grouped and unit[0]["M"] <= self.GROUP_MAX_M):
            self.forward(unit[0], stream, update)
            return
        key = tuple(id(sl) for sl in unit)
        if key not in self._group_ws:
            n = self.q.qlin_forward_grouped_workspace([sl["layer"].w for sl in unit], unit[0]["M"])
            self._group_ws[key] = (n, self.q.empty_workspace(n, self.device))
        n, ws = self._group_ws[key]
        self.q.qlin_forward_grouped([sl["layer"].w for sl in unit], [sl["X"] for sl in unit], [sl["s"] for sl in unit],
                                    [sl["Y"] for sl in unit], unit[0]["M"], self.wl.gamma, update, ws, n, stream)

    def run(self, slots, stream, side=()):
        """Independent launch units round-robin over the launch stream and
        the side streams (forked from and joined back into the launch
        stream)."""
        import torch
        units = self.units(slots)
        if not side:
            for u in units:
                self.run_unit(u, stream)
            return
        streams = [stream, *side]
        fork = torch.cuda.Event()
        fork.record(stream)
        for st in side:
            st.wait_event(fork)
        for j, u in enumerate(units):
            self.run_unit(u, streams[j % len(streams)])
        for st in side:
            done = torch.cuda.Event()
            done.record(st)
            stream.wait_event(done)

    def bucket(self, M):
        return [sl for sl in self.slots if sl["M"] == M]

    def measure_buckets(self, stream, side, reps, peaks):
        """Per token count: the forwards of that bucket (one graph, median of
        replays) and its GEMM calls alone on one stream."""
        import torch
        q = self.q
        out = []
        for M in self.ms:
            sls = self.bucket(M)
            g = graph_of(lambda: self.run(sls, stream, side), stream)
            ms = replay_median_ms(g, stream, reps)
            del g
            ops, nbytes = self.ops(sls), self.bytes(sls)
            rec = {"M": M, "forwards": len(sls), "ms": ms, "tops": ops / (ms * 1e-3) / 1e12,
                   "gbs": nbytes / (ms * 1e-3) / 1e9, "algorithmic_bytes": nbytes, "ops": ops,
                   "roofline": roofline_of(ops, nbytes, ms * 1e-3, peaks)}
            # GEMM calls alone (quantized inputs prepared once, untimed)
            gsl = []
            for sl in sls:
                K, nO = self.meta[sl["si"]]["K"], self.meta[sl["si"]]["nO"]
                Xq = torch.empty((M, K), dtype=torch.int8, device=stream.device)
                a = torch.empty(M, dtype=torch.float32, device=stream.device)
                XqO = torch.empty((M, max(nO, 1)), dtype=torch.int8, device=stream.device)
                naws = q.qlin_quant_act_workspace(M, sl["layer"].w)
                aws = q.empty_workspace(naws, stream.device)
                q.qlin_quant_act(sl["X"], M, sl["layer"].w, sl["s"], self.wl.gamma, False, Xq, a, XqO, aws, naws,
                                 stream)
                gsl.append((sl, Xq, a, XqO))

            def gemms():
                for sl, Xq, a, XqO in gsl:
                    q.qlin_gemm(sl["layer"].w, Xq, a, XqO, sl["s"], M, sl["Y"], None, sl["ws"], sl["nws"], stream)
            g = graph_of(gemms, stream)
            gms = replay_median_ms(g, stream, reps)
            del g
            gbytes = sum(algorithmic_bytes(M, self.meta[sl["si"]]["K"], self.meta[sl["si"]]["N"],
                                           self.meta[sl["si"]]["nO"], self.wl.fmt)[0] for sl, *_ in gsl)
            # qlin_gemm: the compensation operand (layers with outliers), the
            # widening of INT4 weights (from 512 tokens), the GEMM
            widen = 1 if (self.wl.fmt != synth.W8_PERCHANNEL and M >= 512) else 0
            nl = sum(1 + widen + (1 if self.meta[sl["si"]]["nO"] > 0 else 0) for sl, *_ in gsl)
            rec["gemm"] = {"ms": gms, "calls": len(gsl), "launches": nl, "algorithmic_bytes": gbytes,
                           "roofline": roofline_of(ops, gbytes, gms * 1e-3, peaks)}
            q.qlin_poll_device_status(stream)
            out.append(rec)
            del gsl
        return out

    def describe(self):
        return {"workload": self.wl.name, "shapes": [[n, K, N] for n, K, N in self.wl.shapes], "M": self.ms,
                "format": fmt_name(self.wl.fmt), "outlier_frac": self.wl.outlier_frac, "gamma": self.wl.gamma,
                "weight_copies": self.copies, "forwards_per_step": len(self.slots)}


def measure_workload_record(wl, copies, device, stream, side, reps, peaks, grouped=True):
    """Sub-record of a further workload: one step (all its forwards) as the
    median of graph replays, and its buckets."""
    fw = ForwardWorkload(wl, copies, device, grouped=grouped)
    g = graph_of(lambda: fw.run(fw.slots, stream, side), stream)
    ms = replay_median_ms(g, stream, reps)
    del g
    ops, nbytes = fw.ops(), fw.bytes()
    rec = {"ms_per_step": ms, "tops": ops / (ms * 1e-3) / 1e12, "gbs": nbytes / (ms * 1e-3) / 1e9,
           "roofline": roofline_of(ops, nbytes, ms * 1e-3, peaks), "config": fw.describe(),
           "buckets": fw.measure_buckets(stream, side, reps, peaks),
           "timing": f"median of {reps} CUDA-graph replays, CUDA events on the launch stream"}
    fw.q.qlin_poll_device_status(stream)
    return rec


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


class BackwardWorkload:
    def __init__(self, wl, M, device):
        import torch
        from quantized_linear_layers_token_b200 import qlin
        self.q = qlin
        self.wl = wl
        self.M = M
        self.slots = []
        for si, (name, K, N) in enumerate(wl.shapes):
            L = synth.layer(wl, si, M=1)
            lay = qlin.PackedLayer.pack(torch.from_numpy(L["W"]).to(device), L["O"], wl.fmt)
            dY_np = synth.grad_output(wl.index, si, M, N)
            s_np = synth.outlier_scales(wl.index, si, len(L["O"]))
            nws = qlin.qlin_backward_dx_workspace(M, lay.w)
            self.slots.append({"layer": lay, "K": K, "N": N, "nO": len(L["O"]), "dY_np": dY_np,
                               "ws": qlin.empty_workspace(nws, device) if nws else None, "nws": nws,
                               "dY": torch.from_numpy(dY_np).to(device),
                               "s": torch.from_numpy(s_np).to(device) if len(L["O"]) else None,
                               "dX": torch.empty((M, K), dtype=torch.float16, device=device)})
        self.flops = bwd_flops(M, wl.shapes)

    def call(self, sl, stream):
        self.q.qlin_backward_dx(sl["layer"].w, sl["dY"], self.M, sl["s"], sl["dX"], sl["ws"], sl["nws"], stream)

    def step(self, stream):
        for sl in self.slots:
            self.call(sl, stream)


def backward_roofline(flops, ms, peaks):
    achieved = flops / (ms * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_sus"], "unit": "TFLOP/s",
            "frac": achieved / peaks["bf16_sus"], "frac_of_burst": achieved / peaks["bf16"], "traffic": None,
            "peak_source": f"bf16_tflops_sustained of {peaks['kind']} peaks (fp16 and bf16 have the same "
                           f"dense tensor rate)"}


def run_backward(args, wl):
    """One step = qlin_backward_dx on every linear of the workload at
    ``--tokens`` tokens (the fine-tuning backward through the frozen
    quantized weights).  N > 1: every rank runs its own token batch, no
    collective (the input gradient has no exchange step)."""
    import torch

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
    bw = BackwardWorkload(wl, M, device)
    stream = torch.cuda.Stream(device)
    if args.profile_case:
        sl = bw.slots[[n for n, _, _ in wl.shapes].index(args.profile_case)]
        for _ in range(args.warmup):
            bw.call(sl, stream)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            bw.call(sl, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        bw.q.qlin_poll_device_status()
        us = e0.elapsed_time(e1) * 1e3 / max(args.steps, 1)
        print(json.dumps({"profile_case": args.profile_case, "op": "backward", "workload": wl.name, "K": sl["K"],
                          "N": sl["N"], "M": M, "us_per_call_eager": us,
                          "tflops": 2 * M * sl["N"] * sl["K"] / us / 1e6}), flush=True)
        return 0
    for _ in range(max(1, args.warmup)):
        with torch.cuda.stream(stream):
            bw.step(stream)
    torch.cuda.synchronize()
    graph = graph_of(lambda: bw.step(stream), stream)
    for _ in range(args.warmup):
        with torch.cuda.stream(stream):
            graph.replay()
    torch.cuda.synchronize()
    bw.q.qlin_poll_device_status()

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
    peaks = read_peaks()
    value = world * bw.flops / (ms_step * 1e-3) / 1e12
    roofline = backward_roofline(bw.flops, ms_step, peaks)
    roofline.update({"kernel": "backward_dx_kernel, all launches of one step", "flops_per_step": bw.flops,
                     "launches_per_step": len(bw.slots)})

    e2e = None
    if world == 1:
        host_dy = [torch.from_numpy(sl["dY_np"]).pin_memory() for sl in bw.slots]
        host_dx = [torch.empty(sl["dX"].shape, dtype=torch.float16).pin_memory() for sl in bw.slots]
        h2d = sum(x.numel() * 2 for x in host_dy)
        d2h = sum(y.numel() * 2 for y in host_dx)
        h2d_stream = torch.cuda.Stream(device)
        d2h_stream = torch.cuda.Stream(device)

        def e2e_step():
            h2d_stream.wait_stream(stream)
            d2h_stream.wait_stream(stream)
            ready = []
            with torch.cuda.stream(h2d_stream):
                for sl, hy in zip(bw.slots, host_dy):
                    sl["dY"].copy_(hy, non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(h2d_stream)
                    ready.append(ev)
            for sl, hx, ev in zip(bw.slots, host_dx, ready):
                stream.wait_event(ev)
                bw.call(sl, stream)
                done = torch.cuda.Event()
                done.record(stream)
                d2h_stream.wait_event(done)
                with torch.cuda.stream(d2h_stream):
                    hx.copy_(sl["dX"], non_blocking=True)
            stream.wait_stream(h2d_stream)
            stream.wait_stream(d2h_stream)

        g3 = graph_of(e2e_step, stream)
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
        e2e = {"value": bw.flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
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
        dy_bytes = sum(sl["dY"].numel() * 2 for sl in bw.slots)
        line = {
            "metric": BWD_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16 (f32 accumulate)", "data": "synthetic",
            "config": {"workload": wl.name, "op": "backward", "tokens": M,
                       "shapes": [[n, K, N] for n, K, N in wl.shapes], "outlier_frac": wl.outlier_frac,
                       "format": fmt_name(wl.fmt),
                       "l2": f"inputs larger than L2 (dY of one step {dy_bytes / 1e6:.0f} MB)",
                       "parallelism": f"dp{world}",
                       "timing": "CUDA graph of one step, CUDA events on the launch stream"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps * len(bw.slots),
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                       "reasons": clocks["reasons"], "samples": clocks["samples"]},
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def gptq_bytes(K, N):
    """Bytes the Hessian-compensated quantization must move at least once
    per step of its three phases, fp64: the Gauss-Jordan step c reads and
    writes the K x (K - c) active part of the eliminated matrix and all of
    the inverse; the compensation step i reads and writes the N x (K - i - 1)
    not-yet-quantized weights and the (K - i - 1)^2 remaining inverse."""
    gj = sum(16 * K * ((K - c) + K) for c in range(K))
    steps = sum(16 * (N * (K - i - 1) + (K - i - 1) ** 2) for i in range(K))
    return gj, steps


def gptq_record(device, stream, peaks, K=4096, N=4096, ns=8192, reps=2):
    """Hessian-compensated quantization of a 7B q_proj-shaped layer (K = N =
    4096, INT4 grid, per-channel steps) from 8192 synthetic calibration
    tokens: H = 2 X^T X, Gauss-Jordan inverse, column-sequential
    compensation.  HBM-bound streaming kernels (fp64)."""
    import torch
    from quantized_linear_layers_token_b200 import qlin
    rng = synth.rng_for(9, 0)
    X = torch.from_numpy(rng.standard_normal((ns, K))).to(device)
    W0 = torch.from_numpy(rng.standard_normal((K, N)) * 0.02).to(device)
    scale = (W0.abs().amax(dim=0) / 7).contiguous()
    W = torch.empty_like(W0)
    codes = torch.empty((K, N), dtype=torch.int8, device=device)
    Hinv = torch.empty((K, K), dtype=torch.float64, device=device)
    sing = torch.zeros(1, dtype=torch.int32, device=device)
    n = qlin.qlin_gptq_workspace(K, N)
    ws = qlin.empty_workspace(n, device)
    times = []
    for r in range(reps + 1):
        W.copy_(W0)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        qlin.qlin_gptq_quantize(X, ns, K, N, W, scale, 7, codes, Hinv, sing, ws, n, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        if r:
            times.append(e0.elapsed_time(e1))
    qlin.qlin_poll_device_status(stream)
    ms = statistics.median(times)
    gj, st = gptq_bytes(K, N)
    nbytes = gj + st + 8 * ns * K + 16 * K * N
    ach = nbytes / (ms * 1e-3) / 1e9
    return {"op": "gptq", "K": K, "N": N, "calibration_tokens": ns, "ms": ms, "singular": int(sing.item()),
            "hessian_flops": 2 * ns * K * K, "launches": 4 * K + 3,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm"], "unit": "GB/s",
                         "frac": ach / peaks["hbm"], "algorithmic_bytes": nbytes,
                         "peak_source": f"hbm_gbs of {peaks['kind']} peaks (copy)"},
            "timing": f"median of {reps} calls, CUDA events on the launch stream"}


FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # 148 SMs x 128 FP32 lanes x FMA x max SM clock


def smooth_record(device, stream, peaks, M=512, G=10, reps=3):
    """QQQ adaptive-smoothing threshold search on a 7B q_proj-shaped layer
    (K = N = 4096, W4A8 per-channel) with 512 calibration tokens of the 7B
    recipe (1% outlier channels x100), 10 thresholds.  Per candidate: the
    smoothed tensors, the layer's packer, quantization and tcgen05 GEMM, the
    fp32 reference product on the smoothed channels and the loss.  The
    reference product (CUDA-core fp32 FMA) dominates: reported against the
    FP32 FMA peak from the unit counts and the maximum clock."""
    import torch
    from quantized_linear_layers_token_b200 import qlin
    wl = synth.WORKLOADS["llama7b_w4_decode"]
    L = synth.layer(wl, 0, M=M)
    K, N = L["K"], L["N"]
    X = torch.from_numpy(L["X"]).to(device)
    W = torch.from_numpy(L["W"]).to(device)
    loss = torch.zeros(G, dtype=torch.float64, device=device)
    best = torch.zeros(1, dtype=torch.int32, device=device)
    n = qlin.qlin_smooth_search_workspace(M, K, N, G)
    ws = qlin.empty_workspace(n, device)
    times = []
    for r in range(reps + 1):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        qlin.qlin_smooth_search(X, M, K, W, N, G, loss, best, None, ws, n, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        if r:
            times.append(e0.elapsed_time(e1))
    qlin.qlin_poll_device_status(stream)
    ms = statistics.median(times)
    ref_flops = 2 * M * N * K * G
    ach = ref_flops / (ms * 1e-3) / 1e12
    return {"op": "smooth_search", "M": M, "K": K, "N": N, "candidates": G, "ms": ms, "best": int(best.item()),
            "int8_ops": 2 * M * N * K * G,
            "roofline": {"bound": "alu", "achieved": ach, "peak": FP32_PEAK_TFLOPS, "unit": "TFLOP/s",
                         "frac": ach / FP32_PEAK_TFLOPS,
                         "peak_source": "148 SMs x 128 FP32 lanes x 2 (FMA) x 1.965 GHz (unit counts x max clock)",
                         "note": "the whole call's time against the fp32 reference product's FLOPs"},
            "timing": f"median of {reps} calls, CUDA events on the launch stream"}


# OffQ reports on Llama-3-8B; its linears (hidden 4096, 8 KV heads of 128,
# intermediate 14336) at 4096 prefill tokens.
OFFQ_LAYERS = (("q_proj", 4096, 4096), ("k_proj", 4096, 1024), ("v_proj", 4096, 1024), ("o_proj", 4096, 4096),
               ("gate_proj", 4096, 14336), ("up_proj", 4096, 14336), ("down_proj", 14336, 4096))


def offq_bytes(M, K, N):
    """(quantization, GEMM) algorithmic bytes of one OffQ linear: X fp16 in,
    one code byte per value and two fp32 per (token, group) out; then the
    codes and group scales in, the packed INT4 weights, channel scales and
    per-group column sums, and Y fp16 out."""
    G = K // 128
    quant = 2 * M * K + M * K + 8 * M * G
    gemm = M * K + 8 * M * G + K * N // 2 + 4 * N + 4 * G * N + 2 * M * N
    return quant, gemm


def offq_record(device, stream, peaks, reps, M=4096):
    """OffQ W4A4 prefill (Hadamard offset, per-group asymmetric INT4
    activations, per-channel INT4 rotated weights) on the Llama-3-8B linears
    at 4096 tokens: qlin_offq_forward per linear, and its two stages timed
    apart.  Synthetic inputs of the OffQ recipe (each group's outlier energy
    in its first channel, x U[20, 60])."""
    import torch
    from quantized_linear_layers_token_b200 import qlin
    d = synth.offq_signs(0)
    xs, layers = {}, []
    for i, (name, K, N) in enumerate(OFFQ_LAYERS):
        if K not in xs:
            xs[K] = torch.from_numpy(synth.offq_activations(M, K, seed=K).view(np.uint16)).to(device)
        W = torch.from_numpy(synth.offq_weights(K, N, seed=i).view(np.uint16)).to(device)
        codes = torch.zeros(qlin.qlin_offq_codes_bytes(K, N), dtype=torch.uint8, device=device)
        cs = torch.zeros(N, dtype=torch.float32, device=device)
        colsum = torch.zeros((K // 128, N), dtype=torch.float32, device=device)
        Wr = torch.empty((K, N), dtype=torch.float32, device=device)
        qlin.qlin_offq_pack(W, K, N, d, codes, cs, colsum, Wr, stream)
        del Wr, W
        nf = qlin.qlin_offq_forward_workspace(M, K, N)
        ng = qlin.qlin_offq_gemm_workspace(M, K, N)
        layers.append({"K": K, "N": N, "codes": codes, "cs": cs, "colsum": colsum,
                       "Y": torch.empty((M, N), dtype=torch.int16, device=device),
                       "Xq": torch.empty((M, K), dtype=torch.int8, device=device),
                       "sc": torch.empty((M, K // 128), dtype=torch.float32, device=device),
                       "off": torch.empty((M, K // 128), dtype=torch.float32, device=device),
                       "nf": nf, "wsf": qlin.empty_workspace(nf, device), "ng": ng,
                       "wsg": qlin.empty_workspace(ng, device)})

    def fwd():
        for L in layers:
            qlin.qlin_offq_forward(xs[L["K"]], M, L["K"], L["N"], d, L["codes"], L["cs"], L["colsum"], L["Y"],
                                   L["wsf"], L["nf"], stream)

    def quant():
        for L in layers:
            qlin.qlin_offq_quant_act(xs[L["K"]], M, L["K"], d, L["Xq"], L["sc"], L["off"], stream)

    def gemm():
        for L in layers:
            qlin.qlin_offq_gemm(L["Xq"], L["sc"], L["off"], M, L["K"], L["N"], L["codes"], L["cs"], L["colsum"],
                                L["Y"], L["wsg"], L["ng"], stream)
    times = {}
    for key, fn in (("forward", fwd), ("quant", quant), ("gemm", gemm)):
        g = graph_of(fn, stream)
        times[key] = replay_median_ms(g, stream, reps)
        del g
    qlin.qlin_poll_device_status(stream)
    ops = sum(2 * M * K * N for _, K, N in OFFQ_LAYERS)
    qb = sum(offq_bytes(M, K, N)[0] for _, K, N in OFFQ_LAYERS)
    gb = sum(offq_bytes(M, K, N)[1] for _, K, N in OFFQ_LAYERS)
    fb = sum(2 * M * K + K * N // 2 + 4 * N + 4 * (K // 128) * N + 2 * M * N for _, K, N in OFFQ_LAYERS)
    ms = times["forward"]
    return {"op": "offq_forward", "model": "llama3_8b linears (q, k, v, o, gate, up, down)", "tokens": M,
            "ms_per_step": ms, "tops": ops / (ms * 1e-3) / 1e12,
            "roofline": roofline_of(ops, fb, ms * 1e-3, peaks),
            "quant": {"ms": times["quant"], "roofline": roofline_of(0, qb, times["quant"] * 1e-3, peaks)},
            "gemm": {"ms": times["gemm"], "tops": ops / (times["gemm"] * 1e-3) / 1e12,
                     "roofline": roofline_of(ops, gb, times["gemm"] * 1e-3, peaks),
                     "note": "includes the per-call widening of the INT4 codes to INT8"},
            "launches_per_step": 3 * len(OFFQ_LAYERS),
            "timing": f"median of {reps} CUDA-graph replays of the 7 linears"}


def backward_record(device, stream, reps, peaks):
    import torch  # noqa: F401
    wl = synth.WORKLOADS["phi3_w8_quaff"]
    bw = BackwardWorkload(wl, 4096, device)
    g = graph_of(lambda: bw.step(stream), stream)
    ms = replay_median_ms(g, stream, reps)
    del g
    bw.q.qlin_poll_device_status(stream)
    return {"op": "backward", "workload": wl.name, "tokens": bw.M, "ms_per_step": ms,
            "tflops": bw.flops / (ms * 1e-3) / 1e12, "roofline": backward_roofline(bw.flops, ms, peaks),
            "launches_per_step": len(bw.slots),
            "timing": f"median of {reps} CUDA-graph replays of qlin_backward_dx on every linear"}


# ---------------------------------------------------------------------------
# --profile-case: one linear, eager launches (for ncu)
# ---------------------------------------------------------------------------

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


def run_profile_tensor_buckets(args, wl):
    """tensor-buckets -- one qlin_forward per linear at each token count of
    the workload's tensor-bound buckets (the launch set of the headline
    roofline), eager and in order, for an ncu DRAM-traffic capture."""
    import torch
    from quantized_linear_layers_token_b200 import qlin
    peaks = read_peaks()
    ms = [M for M in wl.ms if roofline_of(2 * M * sum(K * N for _, K, N in wl.shapes),
                                          sum(layer_bytes(M, K, N, 0, wl.fmt) for _, K, N in wl.shapes),
                                          1.0, peaks)["bound"] == "tensor"]
    for M in ms:
        for si, (name, K, N) in enumerate(wl.shapes):
            L = synth.layer(wl, si, M=M)
            layer = qlin.PackedLayer.pack(torch.from_numpy(L["W"]).cuda(), L["O"], wl.fmt)
            X = torch.from_numpy(L["X"]).cuda()
            s = torch.ones(max(len(L["O"]), 1), dtype=torch.float32, device="cuda")
            Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
            nws = qlin.qlin_forward_workspace(M, layer.w)
            ws = qlin.empty_workspace(nws)
            qlin.qlin_forward(X, M, layer.w, s, wl.gamma, True, Y, ws, nws)
            torch.cuda.synchronize()
            del layer, X, Y, ws
            torch.cuda.empty_cache()
    qlin.qlin_poll_device_status()
    print(json.dumps({"profile_case": "tensor-buckets", "workload": wl.name, "M": ms,
                      "linears": [n for n, _, _ in wl.shapes]}), flush=True)
    return 0


def run_profile_grouped(args, wl):
    """grouped:M -- every linear of the workload (one weight copy) as one
    qlin_forward_grouped call at M <= 64 tokens, launched eagerly (for ncu)."""
    import torch
    from quantized_linear_layers_token_b200 import qlin
    M = int(args.profile_case.split(":")[1])
    layers, Xs, ss, Ys = [], [], [], []
    for si, (_, K, N) in enumerate(wl.shapes):
        L = synth.layer(wl, si, M=M)
        layers.append(qlin.PackedLayer.pack(torch.from_numpy(L["W"]).cuda(), L["O"], wl.fmt))
        Xs.append(torch.from_numpy(L["X"]).cuda())
        ss.append(torch.ones(max(len(L["O"]), 1), dtype=torch.float32, device="cuda"))
        Ys.append(torch.empty((M, N), dtype=torch.float16, device="cuda"))
    ws = [l.w for l in layers]
    n = qlin.qlin_forward_grouped_workspace(ws, M)
    wsp = qlin.empty_workspace(n)
    for _ in range(args.warmup):
        qlin.qlin_forward_grouped(ws, Xs, ss, Ys, M, wl.gamma, True, wsp, n)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        qlin.qlin_forward_grouped(ws, Xs, ss, Ys, M, wl.gamma, True, wsp, n)
    e1.record()
    torch.cuda.synchronize()
    qlin.qlin_poll_device_status()
    us = e0.elapsed_time(e1) * 1e3 / max(args.steps, 1)
    nbytes = sum(layer_bytes(M, K, N, l.n_outlier, wl.fmt) for (_, K, N), l in zip(wl.shapes, layers))
    print(json.dumps({"profile_case": args.profile_case, "workload": wl.name, "M": M, "problems": len(ws),
                      "us_per_call_eager": us, "algorithmic_bytes": nbytes,
                      "gbs": nbytes / (us * 1e-6) / 1e9}), flush=True)
    return 0


def run_profile_offq(args):
    """offq:NAME:M -- W warm-up and K timed qlin_offq_forward calls on one
    Llama-3-8B linear, launched eagerly (for ncu)."""
    import torch
    from quantized_linear_layers_token_b200 import qlin
    _, name, m = args.profile_case.split(":")
    M = int(m)
    i = [n for n, _, _ in OFFQ_LAYERS].index(name)
    _, K, N = OFFQ_LAYERS[i]
    d = synth.offq_signs(0)
    X = torch.from_numpy(synth.offq_activations(M, K, seed=K).view(np.uint16)).cuda()
    W = torch.from_numpy(synth.offq_weights(K, N, seed=i).view(np.uint16)).cuda()
    codes = torch.zeros(qlin.qlin_offq_codes_bytes(K, N), dtype=torch.uint8, device="cuda")
    cs = torch.zeros(N, dtype=torch.float32, device="cuda")
    colsum = torch.zeros((K // 128, N), dtype=torch.float32, device="cuda")
    Wr = torch.empty((K, N), dtype=torch.float32, device="cuda")
    qlin.qlin_offq_pack(W, K, N, d, codes, cs, colsum, Wr)
    del Wr
    Y = torch.empty((M, N), dtype=torch.int16, device="cuda")
    n = qlin.qlin_offq_forward_workspace(M, K, N)
    ws = qlin.empty_workspace(n)
    for _ in range(args.warmup):
        qlin.qlin_offq_forward(X, M, K, N, d, codes, cs, colsum, Y, ws, n)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        qlin.qlin_offq_forward(X, M, K, N, d, codes, cs, colsum, Y, ws, n)
    e1.record()
    torch.cuda.synchronize()
    qlin.qlin_poll_device_status()
    us = e0.elapsed_time(e1) * 1e3 / max(args.steps, 1)
    print(json.dumps({"profile_case": args.profile_case, "K": K, "N": N, "M": M, "us_per_forward_eager": us,
                      "tops": 2 * M * K * N / (us * 1e-6) / 1e12}), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm: the forward step
# ---------------------------------------------------------------------------

def run_forward(args, wl):
    import torch
    from quantized_linear_layers_token_b200 import qlin
    from quantized_linear_layers_token_b200.dp import ColmaxExchange

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
    peaks = read_peaks()
    copies = args.copies if args.copies else (4 if wl.name == "llama7b_w4_decode" else 1)
    fw = ForwardWorkload(wl, copies, device, grouped=bool(args.grouped))
    meta = fw.meta
    stream = torch.cuda.Stream(device)
    xchg = ColmaxExchange([meta[sl["si"]]["nO"] for sl in fw.slots], device)
    nstreams = max(1, args.streams) if world == 1 else 1
    side = [torch.cuda.Stream(device) for _ in range(nstreams - 1)]

    def step_single():
        fw.run(fw.slots, stream, side)

    def step_dp():
        for j, sl in enumerate(fw.slots):
            if xchg.n_outliers[j]:
                qlin.qlin_outlier_colmax(sl["X"], sl["M"], sl["layer"].w, xchg.view(j), stream)
        with torch.cuda.stream(stream):
            xchg.allreduce()
        for j, sl in enumerate(fw.slots):
            lay = sl["layer"]
            if xchg.n_outliers[j]:
                qlin.qlin_momentum_update(lay.w, xchg.view(j), sl["s"], wl.gamma, stream)
            fw.forward(sl, stream, update=False)  # quantize with the already-updated state, then the GEMM

    step = step_single if world == 1 else step_dp
    for _ in range(max(1, args.warmup)):
        with torch.cuda.stream(stream):
            step()
    torch.cuda.synchronize()
    graph = None
    if world == 1:
        graph = graph_of(step, stream)
        for _ in range(args.warmup):
            with torch.cuda.stream(stream):
                graph.replay()
        torch.cuda.synchronize()

    def run_steps(k):
        for _ in range(k):
            with torch.cuda.stream(stream):
                if graph is not None:
                    graph.replay()
                else:
                    step()

    # ------------------------------------------------------------ timed region
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
    qlin.qlin_poll_device_status(stream)
    step_ops, step_bytes = fw.ops(), fw.bytes()
    value = world * step_ops / (ms_step * 1e-3) / 1e12

    line = None
    if rank == 0:
        reps = max(20, args.reps)
        buckets = fw.measure_buckets(stream, side, reps, peaks) if world == 1 else None
        # the dominant kernel: the GEMM calls of the tensor-bound buckets
        roofline = None
        if buckets:
            tb = [b for b in buckets if b["gemm"]["roofline"]["bound"] == "tensor"] or buckets
            g_ms = sum(b["gemm"]["ms"] for b in tb)
            g_ops = sum(b["ops"] for b in tb)
            g_bytes = sum(b["gemm"]["algorithmic_bytes"] for b in tb)
            roofline = roofline_of(g_ops, g_bytes, g_ms * 1e-3, peaks)
            tr = recorded_traffic(wl.name)
            roofline.update({
                "kernel": "qlin_gemm (INT4 widened once per call, then the tcgen05 INT8 GEMM with the fused "
                          "dequant and compensation), all calls of the buckets M in "
                          f"{[b['M'] for b in tb]}, one stream",
                "ms": g_ms, "launches": sum(b["gemm"]["launches"] for b in tb),
                "ops": g_ops, "algorithmic_bytes": g_bytes,
                "traffic": tr["dram_bytes"] if tr else None,
                "traffic_source": tr["how"] if tr else "no capture recorded for these GEMM sources",
                "timing": f"sum over the buckets of the median of {reps} CUDA-graph replays"})

        # ------------------------------------------------------------ end to end through the API
        e2e = None
        if world == 1:
            host_x = [torch.from_numpy(fw.x_np[(sl["M"], sl["si"])]).pin_memory() for sl in fw.slots]
            host_y = [torch.empty(sl["Y"].shape, dtype=torch.float16).pin_memory() for sl in fw.slots]
            h2d = sum(x.numel() * 2 for x in host_x)
            d2h = sum(y.numel() * 2 for y in host_y)
            h2d_stream = torch.cuda.Stream(device)
            d2h_stream = torch.cuda.Stream(device)

            hx_of = {id(sl): hx for sl, hx in zip(fw.slots, host_x)}
            hy_of = {id(sl): hy for sl, hy in zip(fw.slots, host_y)}
            units = fw.units(fw.slots)

            def e2e_step():
                h2d_stream.wait_stream(stream)
                d2h_stream.wait_stream(stream)
                ready = []
                with torch.cuda.stream(h2d_stream):
                    for u in units:
                        for sl in u:
                            sl["X"].copy_(hx_of[id(sl)], non_blocking=True)
                        ev = torch.cuda.Event()
                        ev.record(h2d_stream)
                        ready.append(ev)
                streams = [stream, *side]
                fork = torch.cuda.Event()
                fork.record(stream)
                for st in side:
                    st.wait_event(fork)
                for j, (u, ev) in enumerate(zip(units, ready)):
                    cs = streams[j % len(streams)]
                    cs.wait_event(ev)
                    fw.run_unit(u, cs)
                    done = torch.cuda.Event()
                    done.record(cs)
                    d2h_stream.wait_event(done)
                    with torch.cuda.stream(d2h_stream):
                        for sl in u:
                            hy_of[id(sl)].copy_(sl["Y"], non_blocking=True)
                for st in side:
                    joined = torch.cuda.Event()
                    joined.record(st)
                    stream.wait_event(joined)
                stream.wait_stream(h2d_stream)
                stream.wait_stream(d2h_stream)

            g3 = graph_of(e2e_step, stream)
            with torch.cuda.stream(stream):
                g3.replay()
            torch.cuda.synchronize()
            e2e_steps = max(3, min(args.steps, 10))
            ev0.record(stream)
            for _ in range(e2e_steps):
                with torch.cuda.stream(stream):
                    g3.replay()
            ev1.record(stream)
            torch.cuda.synchronize()
            e2e_ms = ev0.elapsed_time(ev1) / e2e_steps
            del g3
            e2e = {"value": step_ops / (e2e_ms * 1e-3) / 1e12, "unit": "TOPS", "h2d_bytes_per_step": h2d,
                   "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps,
                   "note": "per linear: pinned host X -> device (copy stream), qlin_forward (the step's compute "
                           "streams), device -> pinned host Y (second copy stream); one CUDA graph per step"}

        # ------------------------------------------------------------ further workloads
        workloads = {}
        if world == 1 and args.extras:
            for name in [x for x in args.extras.split(",") if x and x != wl.name]:
                try:
                    if name == "backward":
                        workloads[name] = backward_record(device, stream, reps, peaks)
                    elif name == "gptq":
                        workloads[name] = gptq_record(device, stream, peaks)
                    elif name == "smooth_search":
                        workloads[name] = smooth_record(device, stream, peaks)
                    elif name == "offq":
                        workloads[name] = offq_record(device, stream, peaks, reps)
                    else:
                        w2 = synth.WORKLOADS[name]
                        workloads[name] = measure_workload_record(w2, 4 if name == "llama7b_w4_decode" else 1,
                                                                  device, stream, side, reps, peaks,
                                                                  grouped=bool(args.grouped))
                except Exception as ex:  # evidence only: recorded, the headline stands
                    workloads[name] = {"error": f"{type(ex).__name__}: {ex}"[:400]}
                torch.cuda.empty_cache()

        # ------------------------------------------------------------ CPU baseline
        cpu = None
        if world == 1:
            sample = oracle_sample_for(wl)
            t = sample.step()
            cpu = {"value": sample.ops / t / 1e12, "unit": "TOPS", "cores": 1, "kind": "oracle",
                   "gbs": sample.bytes / t / 1e9, "sample": sample.describe(t)}

        def unit_launches(u):
            M = u[0]["M"]
            if world > 1:  # colmax + momentum per linear, then quant + GEMM per linear
                return sum(2 + (2 if meta[sl["si"]]["nO"] > 0 else 0) +
                           (1 if (wl.fmt != synth.W8_PERCHANNEL and M >= 512) else 0) for sl in u)
            colmax = sum(1 for sl in u if meta[sl["si"]]["nO"] > 0 and M > 64)
            if len(u) > 1 or (fw.grouped and M <= fw.GROUP_MAX_M):
                return 2 + colmax  # one quantization launch, one GEMM launch for the group
            widen = 1 if (wl.fmt != synth.W8_PERCHANNEL and M >= 512) else 0
            return 2 + widen + colmax

        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "gbs": world * step_bytes / (ms_step * 1e-3) / 1e9, "algorithmic_bytes_per_step": step_bytes,
            "ops_per_step": step_ops,
            "config": {**fw.describe(), "parallelism": f"dp{world}", "streams": nstreams,
                       "l2": "inputs larger than L2 (one step streams "
                             f"{sum(l[0].nbytes for l in fw.layers) * copies / 1e6:.0f} MB of packed weights and "
                             f"{sum(x.nbytes for x in fw.x_np.values()) / 1e6:.0f} MB of activations)",
                       "timing": "CUDA graph of one step, CUDA events on the launch stream",
                       "grouped": "decode token counts (<= 64): the step's linears at that count go through "
                                  "qlin_forward_grouped, up to 32 per call" if args.grouped else "off"},
            "roofline": roofline, "buckets": buckets, "workloads": workloads, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps * sum(unit_launches(u) for u in (fw.units(fw.slots) if world == 1 else
                                                                          [[sl] for sl in fw.slots])),
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                       "reasons": clocks["reasons"], "samples": clocks["samples"]},
        }
    if line is not None:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--extras", default=DEFAULT_EXTRAS,
                    help="further workloads measured into the line's `workloads` (comma list; '' for none)")
    ap.add_argument("--copies", type=int, default=0,
                    help="distinct packed-weight copies per linear (0: 4 for the 7B decode set, else 1)")
    ap.add_argument("--streams", type=int, default=4,
                    help="compute streams the independent forwards of a step are spread over (N = 1)")
    ap.add_argument("--reps", type=int, default=20, help="graph replays per bucket (median)")
    ap.add_argument("--grouped", type=int, default=1,
                    help="1: decode-sized token counts (<= 64) run the step's linears through qlin_forward_grouped "
                         "(up to 32 per call); 0: one qlin_forward per linear")
    ap.add_argument("--op", default="forward", choices=["forward", "backward"],
                    help="backward: the input gradient of every linear (default workload phi3_w8_quaff)")
    ap.add_argument("--tokens", type=int, default=4096, help="--op backward: tokens per step")
    ap.add_argument("--profile-case", default=None,
                    help="NAME:M -- run only that linear of the workload at M tokens (for ncu captures); "
                         "offq:NAME:M -- one OffQ linear of the Llama-3-8B set")
    args = ap.parse_args()
    if args.op == "backward":
        wl = synth.WORKLOADS["phi3_w8_quaff" if args.workload == DEFAULT_WORKLOAD else args.workload]
        return run_backward_reference(args, wl) if args.impl == "reference" else run_backward(args, wl)
    wl = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    if args.profile_case and args.profile_case.startswith("offq:"):
        return run_profile_offq(args)
    if args.profile_case and args.profile_case.startswith("grouped:"):
        return run_profile_grouped(args, wl)
    if args.profile_case and args.profile_case.startswith("tensor-buckets"):
        return run_profile_tensor_buckets(args, wl)
    if args.profile_case:
        return run_profile_case(args, wl)
    return run_forward(args, wl)


if __name__ == "__main__":
    sys.exit(main())

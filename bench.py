"""Benchmark of the MoE expert layer on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config NAME]

A step is one pass of the whole layer -- router, dispatch/permutation, W1/W3
grouped GEMM + SwiGLU, W2 grouped GEMM, shared experts when the workload has
them, combine -- over one batch of N synthetic tokens (seeded, inputs resident
in HBM before timing).  The headline workload is the largest single-GPU one, the
skewed Qwen3-235B-shaped layer (N=16384, tensor-bound); the same run also times
every other workload shape (`other_workloads`, skipped with --no-others).  Under
torchrun every rank runs its own batch against its own copy of the weights (the
layer shards by tokens with no exchange step: weak scaling); time is the max
over ranks of CUDA-event time.

`--impl reference` times the plain CPU oracle (test infrastructure, never tuned)
on rank 0 on a bounded sample of tokens of the same workload, on the host's
cores (its OpenMP build: tokens and rows spread over threads, same arithmetic).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from expert_ffn_layer_moe_b200.inputs import CONFIGS, QWEN3_30B_TOKEN_SWEEP, make_inputs  # noqa: E402

METRIC = "MoE-layer tokens/s; grouped-GEMM TFLOP/s and % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PHASES = ("route", "permute", "gemm13", "gemm2", "shared", "combine")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(cfg):
    s = f"{cfg.name}: N={cfg.N} H={cfg.H} I={cfg.I} E={cfg.E} top-{cfg.k}"
    if cfg.Is:
        s += f" shared Is={cfg.Is}"
    if cfg.skew:
        s += f" skew bias x{cfg.bias_scale}"
    return s + ", bf16, SwiGLU experts"


def layer_flops(cfg):
    """Algorithmic FLOPs: router 2NHE + routed experts 6RHI + shared 6NHIs."""
    return 2 * cfg.N * cfg.H * cfg.E + 6 * cfg.R * cfg.H * cfg.I + 6 * cfg.N * cfg.H * cfg.Is


def gemm13_bytes(cfg, touched, wbytes=2, abytes=2):
    """W1+W3 tiles of the touched experts (wbytes per weight; fp8 adds a 4-byte scale
    per row), x_perm read (abytes per value; fp8 adds a scale per row), h written."""
    scales = touched * 2 * cfg.I * 4 if wbytes == 1 else 0
    ascales = cfg.R * 4 if abytes == 1 else 0
    return (touched * 2 * cfg.I * cfg.H * wbytes + scales + cfg.R * cfg.H * abytes + ascales
            + cfg.R * cfg.I * 2)


def gemm2_bytes(cfg, touched, wbytes=2, abytes=2):
    scales = touched * cfg.H * 4 if wbytes == 1 else 0
    ascales = cfg.R * 4 if abytes == 1 else 0
    return touched * cfg.H * cfg.I * wbytes + scales + cfg.R * cfg.I * abytes + ascales + cfg.R * cfg.H * 2


def layer_bytes(cfg, touched, wbytes=2):
    """Touched expert weights (+ their scales for fp8) + shared weights + router weights
    + x in + out."""
    scales = touched * (2 * cfg.I + cfg.H) * 4 if wbytes == 1 else 0  # one per weight row
    return (touched * 3 * cfg.H * cfg.I * wbytes + scales + 3 * cfg.H * cfg.Is * 2 + cfg.H * cfg.E * 4
            + 2 * cfg.N * cfg.H * 2)


def l2_bytes(dev):
    try:
        return int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0)) or 126 << 20
    except (AttributeError, RuntimeError):
        return 126 << 20


def rotation_copies(weight_bytes, l2):
    """Independent weight copies to cycle through so that consecutive steps read
    different weights and their total is at least twice the L2 size (1: the touched
    weights alone exceed it)."""
    return 1 if weight_bytes > 2 * l2 else int(math.ceil(2 * l2 / max(1, weight_bytes)))


def l2_note(weight_bytes, touched, l2, copies):
    """How the timed steps stand to L2."""
    if copies <= 1:
        return (f"inputs larger than L2: {touched} touched experts' weights ({weight_bytes / 1e9:.2f} GB, L2 "
                f"{l2 / 1e6:.0f} MB) streamed from HBM every step")
    return (f"weight rotation: {touched} touched experts' weights ({weight_bytes / 1e6:.1f} MB) are under twice "
            f"the L2 size ({l2 / 1e6:.0f} MB), so the steps cycle through {copies} independent copies of every "
            f"weight tensor ({copies * weight_bytes / 1e6:.0f} MB of touched weights in the cycle)")


def kernel_source_digest(path):
    """sha256[:12] of a CUDA source with its comments and blank lines removed (a comment
    edit leaves the compiled kernel, and so its measured traffic, unchanged)."""
    import re
    text = open(path, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    code = "\n".join(l.rstrip() for l in text.splitlines() if l.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:12]


def kernel_traffic(kernel, workload, path=None, src=None):
    """DRAM bytes per launch recorded from an ncu capture in profiles/traffic.txt,
    valid only while the kernel source is unchanged (its sha256 prefix matches)."""
    path = path or os.path.join(ROOT, "profiles", "traffic.txt")
    src = src or os.path.join(ROOT, "expert_ffn_layer_moe_b200", "csrc", "grouped_gemm.cu")
    if not os.path.exists(path):
        return None
    digest = kernel_source_digest(src)
    for line in open(path):
        f = line.split()
        if len(f) >= 4 and not line.startswith("#") and f[0] == kernel and f[1] == workload and f[3] == digest:
            return float(f[2])
    return None


CLOCK_SAMPLER = r"""
import sys, time
import pynvml as N
bus, period = sys.argv[1], float(sys.argv[2])
N.nvmlInit()
try:
    h = N.nvmlDeviceGetHandleByPciBusId(bus)
except Exception:
    h = N.nvmlDeviceGetHandleByIndex(int(sys.argv[3]))
mx = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
get_reasons = getattr(N, "nvmlDeviceGetCurrentClocksEventReasons", None) or N.nvmlDeviceGetCurrentClocksThrottleReasons
print("ready", flush=True)
while True:
    t = time.time()
    print(t, N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM), mx, N.nvmlDeviceGetPowerUsage(h), get_reasons(h), flush=True)
    time.sleep(max(0.0, period - (time.time() - t)))
"""


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons sampled through NVML every
    2 ms by a helper process (no GIL shared with the launching thread), kept for the
    samples whose host timestamps fall inside the timed region [enter, exit]."""

    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}
    PERIOD_S = 0.002

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.t0 = self.t1 = None
        self.lines = []

    def start(self):
        """Start the helper before the region (it needs a moment to initialise NVML)."""
        try:
            p = torch.cuda.get_device_properties(self.dev)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        except (AttributeError, RuntimeError):
            bus = ""
        try:
            self.proc = subprocess.Popen([sys.executable, "-c", CLOCK_SAMPLER, bus, str(self.PERIOD_S),
                                          str(self.dev)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            if self.proc.stdout.readline().strip() != "ready":
                self.stop()
        except OSError:
            self.proc = None
        return self

    def __enter__(self):
        self.t0 = time.time()
        return self

    def __exit__(self, *a):
        self.t1 = time.time()
        self._read_until(self.t1, timeout_s=1.0)
        self.stop()

    def _read_until(self, t, timeout_s):
        """Keep the helper's lines until one is stamped at or after t (at most timeout_s),
        so a region shorter than the helper's first query still has a sample."""
        import select
        if self.proc is None:
            return
        deadline = time.time() + timeout_s
        while True:
            left = deadline - time.time()
            if left <= 0 or not select.select([self.proc.stdout], [], [], left)[0]:
                return
            line = self.proc.stdout.readline()
            if not line:
                return
            self.lines.append(line)
            f = line.split()
            try:
                if len(f) == 5 and float(f[0]) >= t:
                    return
            except ValueError:
                pass

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
                self.lines += out.splitlines()
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.proc = None

    def summary(self):
        rows = []
        for l in self.lines:
            f = l.split()
            if len(f) == 5:
                try:
                    rows.append((float(f[0]), float(f[1]), float(f[2]), float(f[3]) / 1e3, int(f[4])))
                except ValueError:
                    pass
        if not rows or self.t0 is None:
            return None
        inside = [r for r in rows if self.t0 <= r[0] <= self.t1]
        if not inside:  # region shorter than one period: the first sample after it began
            later = [r for r in rows if r[0] >= self.t0]
            inside = later[:1] or rows[-1:]
        reasons = sorted(n for n, b in self.REASON_BITS.items() if any(r[4] & b for r in inside))
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "power_w_max": max(r[3] for r in inside), "reasons": reasons, "samples": len(inside),
                "sampler": f"NVML every {self.PERIOD_S * 1e3:.0f} ms, samples inside the timed region"}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def oracle_sample_rate(cfg, t_host, tokens, seed=0):
    """Tokens/s of the CPU oracle on `tokens` seeded tokens of the workload (whole
    layer from x: logits, top-k, dispatch, experts, combine), on the thread count the
    oracle is set to."""
    import oracle
    rng = np.random.default_rng(seed)
    sel = np.sort(rng.choice(cfg.N, tokens, replace=False))
    x = t_host["x"][sel]
    t0 = time.perf_counter()
    oracle.layer(x, t_host["W_gate"], t_host["W1"], t_host["W3"], t_host["W2"], cfg.k, bias=t_host["bias"],
                 Ws1=t_host["Ws1"], Ws3=t_host["Ws3"], Ws2=t_host["Ws2"])
    dt = time.perf_counter() - t0
    return tokens / dt, dt


def host_inputs(cfg):
    """Oracle-side copies (numpy, bf16 as uint16) of the seeded inputs."""
    gen = "cuda" if torch.cuda.is_available() else "cpu"
    t = make_inputs(cfg, seed=0, device=gen)
    out = {}
    for n, v in t.items():
        if v is None:
            out[n] = None
        elif v.dtype == torch.bfloat16:
            out[n] = v.cpu().view(torch.int16).numpy().view(np.uint16)
        else:
            out[n] = v.cpu().numpy()
    del t
    if torch.cuda.is_available():
        torch.cuda.empty_cache()
    return out


def sample_size(cfg, rate, target_s, cores):
    """Tokens the oracle gets through in about target_s at `rate` tokens/s: the whole
    batch when it fits, else a multiple of the thread count (whole rounds of rows)."""
    n = int(rate * target_s)
    if n >= cfg.N:
        return cfg.N
    return max(cores, n - n % cores) if n >= cores else max(1, n)


def cpu_baseline(cfg, th, target_s):
    """The oracle, as it stands, on the host's cores (its OpenMP build, one thread per
    core): the whole layer when one run fits in about target_s, else a seeded token
    sample of that size (tokens are independent once routed), reported per token.  A
    small single-thread sample is timed beside it."""
    import oracle
    oracle.build()
    oracle.set_threads(1)
    st_tokens = max(1, min(cfg.N, int(round(2.0 * oracle_sample_rate(cfg, th, 1, seed=7)[0]))))
    st_rate, st_dt = oracle_sample_rate(cfg, th, st_tokens, seed=8)
    cores = oracle.set_threads(os.cpu_count() or 1)
    try:
        probe = min(cfg.N, cores)
        rate, _ = oracle_sample_rate(cfg, th, probe, seed=0)
        n = sample_size(cfg, rate, target_s, cores)
        rate, dt = oracle_sample_rate(cfg, th, n, seed=1)
    finally:
        oracle.set_threads(1)
    whole = n == cfg.N
    sample = (f"the whole {cfg.N}-token layer from x" if whole else
              f"{n} seeded tokens of the {cfg.N}-token batch, whole layer from x (scaled per token)")
    return {"value": rate, "unit": "tokens/s", "cores": cores, "threads": cores, "kind": "oracle",
            "sample": f"{sample}, {cores} threads (OpenMP build), {dt:.1f} s",
            "nproc": os.cpu_count(),
            "single_thread": {"value": st_rate, "unit": "tokens/s",
                              "sample": f"{st_tokens} seeded tokens, serial build, {st_dt:.1f} s"}}


def run_reference(args, cfg, world, rank):
    if rank != 0:
        return
    import oracle
    oracle.build()
    th = host_inputs(cfg)
    cores = oracle.set_threads(os.cpu_count() or 1)
    # each step is a bounded sample of the workload: as many tokens as the threads get
    # through in about --ref-seconds (a multiple of the thread count)
    rate0, _ = oracle_sample_rate(cfg, th, min(cfg.N, cores), seed=0)
    per_step = sample_size(cfg, rate0, args.ref_seconds, cores)
    for i in range(args.warmup):
        oracle_sample_rate(cfg, th, min(cfg.N, cores), seed=100 + i)
    total_tok, total_t = 0, 0.0
    for i in range(args.steps):
        r, dt = oracle_sample_rate(cfg, th, per_step, seed=i + 1)
        total_tok += per_step
        total_t += dt
    oracle.set_threads(1)
    value = total_tok / total_t
    sample = (f"{per_step} seeded tokens of the {cfg.N}-token batch per step, whole layer from x, "
              f"{cores} threads (OpenMP build of the oracle)")
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * cfg.N / value, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": workload_desc(cfg), "global_batch": cfg.N, "parallelism": "rank 0 only"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


class Workload:
    """One workload's inputs on the device, its workspace, and the step function (one
    whole-layer call through the C ABI).  With `copies` > 1 the weights are held that
    many times and consecutive steps cycle through the copies, so a shape whose touched
    weights fit in L2 still reads them from HBM every step."""

    def __init__(self, cfg, args, dev, stream, rank, world):
        from expert_ffn_layer_moe_b200 import moe
        self.moe, self.cfg, self.dev, self.stream = moe, cfg, dev, stream
        t = make_inputs(cfg, seed=0, device=dev)
        if world > 1:  # every rank its own token batch
            t["x"] = make_inputs(cfg, seed=rank, device=dev, weights=False)["x"]
        self.t = t
        N, H, I, E, k = cfg.N, cfg.H, cfg.I, cfg.E, cfg.k
        self.fp8 = args.weights == "fp8"
        self.a8 = args.acts == "fp8"
        self.wbytes, self.abytes = (1 if self.fp8 else 2), (1 if self.a8 else 2)
        ws_bytes = (moe.moe_workspace_bytes_w8a8 if self.a8 else moe.moe_workspace_bytes)(N, H, I, E, k, cfg.Is)
        self.ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        self.out = torch.empty((N, H), dtype=torch.bfloat16, device=dev)
        counts = moe.moe_permute(t["x"], moe.moe_route(t["x"], t["W_gate"], k, bias=t["bias"])[0], E)["counts"]
        self.touched = int((counts > 0).sum().item())
        self.max_load = int(counts.max().item())
        self.l2 = l2_bytes(dev)
        touched_w = self.touched * 3 * H * I * self.wbytes
        self.copies = rotation_copies(touched_w, self.l2) if not args.no_rotate else 1
        self.l2_note = l2_note(touched_w, self.touched, self.l2, self.copies)
        names = ("W_gate", "W1", "W3", "W2", "Ws1", "Ws3", "Ws2")
        sets = [{n: t[n] for n in names}]
        for _ in range(self.copies - 1):
            sets.append({n: (None if t[n] is None else t[n].clone()) for n in names})
        if self.fp8:
            # weight preparation, once, outside every timed region: e4m3 codes + row scales
            for w in sets:
                w["q"] = {n: moe.moe_quantize_fp8(w[n], stream=stream) for n in ("W1", "W3", "W2")}
        self.sets = sets
        torch.cuda.synchronize()
        self.i = 0

    def step(self, events=None, x=None, o=None, st=None, copy=None):
        moe, t = self.moe, self.t
        w = self.sets[(self.i if copy is None else copy) % self.copies]
        if copy is None:
            self.i += 1
        xx = t["x"] if x is None else x
        oo = self.out if o is None else o
        ss = self.stream if st is None else st
        if self.fp8:
            q = w["q"]
            fn = moe.moe_layer_forward_w8a8_ex if self.a8 else moe.moe_layer_forward_fp8_ex
            fn(xx, w["W_gate"], *q["W1"], *q["W3"], *q["W2"], self.cfg.k, bias=t["bias"], Ws1=w["Ws1"],
               Ws3=w["Ws3"], Ws2=w["Ws2"], ws=self.ws, out=oo, stream=ss, phase_events=events)
        else:
            moe.moe_layer_forward_ex(xx, w["W_gate"], w["W1"], w["W3"], w["W2"], self.cfg.k, bias=t["bias"],
                                     Ws1=w["Ws1"], Ws3=w["Ws3"], Ws2=w["Ws2"], ws=self.ws, out=oo, stream=ss,
                                     phase_events=events)

    def capture_graphs(self, warmup):
        """One captured layer step per weight copy (the library only enqueues kernels on
        the stream it is given); returns the kernel launches one step captures."""
        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize()
        self.graphs = []
        n0 = self.moe.moe_kernel_launches()
        for c in range(self.copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.step(st=torch.cuda.current_stream(), copy=c)
            self.graphs.append(g)
        torch.cuda.synchronize()
        return (self.moe.moe_kernel_launches() - n0) // self.copies

    def release(self):
        self.graphs = []
        self.sets = self.t = self.ws = self.out = None


def time_steps(W, steps, warmup, world, graph, clock=None):
    """Device time of `steps` layer steps on the launching stream (max over ranks is
    taken by the caller), the library's launch count over them, and the mean per-phase
    times from a second pass with events between the phases."""
    moe, stream = W.moe, W.stream
    graph_launches = W.capture_graphs(warmup) if graph else 0
    for _ in range(warmup):
        W.step()
    torch.cuda.synchronize()
    if moe.moe_get_device_error(stream) != 0:
        raise RuntimeError("device error reported during warm-up")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    ctx = clock if clock is not None else _NullCtx()
    with ctx:
        n0 = moe.moe_kernel_launches()
        start.record(stream)
        for i in range(steps):
            if graph:
                W.graphs[i % W.copies].replay()
            else:
                W.step()
        end.record(stream)
        launches = moe.moe_kernel_launches() - n0 if not graph else graph_launches * steps
        torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = start.elapsed_time(end)
    # per-kernel times: the same steps again with an event between consecutive phases
    # (an event between two kernels also stops the second from launching early, so this
    # pass is timed separately from the one above)
    phase_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(PHASES) + 1)] for _ in range(steps)]
    for evs in phase_ev:  # materialise the events before handing their handles to C
        for e in evs:
            e.record(stream)
    barrier(world)
    torch.cuda.synchronize()
    for i in range(steps):
        W.step(phase_ev[i])
    torch.cuda.synchronize()
    barrier(world)
    phase_ms = {p: statistics.mean(evs[j].elapsed_time(evs[j + 1]) for evs in phase_ev)
                for j, p in enumerate(PHASES)}
    if moe.moe_get_device_error(stream) != 0:
        raise RuntimeError("device error reported during the timed steps")
    return elapsed_ms, launches, phase_ms


class _NullCtx:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def summarise(cfg, touched, step_s, phase_ms, pk, wbytes, abytes, a8):
    """Layer floor and fraction, grouped-GEMM rates, and the W1/W3 kernel's roofline."""
    H, I = cfg.H, cfg.I
    hbm = pk["hbm_gbs"]
    g13_s = phase_ms["gemm13"] / 1e3
    g2_s = phase_ms["gemm2"] / 1e3
    g13_b = gemm13_bytes(cfg, touched, wbytes, abytes)
    flops = layer_flops(cfg)
    gemm_flops = 6 * cfg.R * H * I
    lbytes = layer_bytes(cfg, touched, wbytes)
    # tensor floor: the routed experts' FLOPs at their operands' peak (e4m3 x e4m3: the bf16
    # peak times the nominal 2x), the router's and the shared experts' at the bf16 peak
    routed_flops = 6 * cfg.R * H * I
    tensor_s = (routed_flops / (2.0 if a8 else 1.0) + (flops - routed_flops)) / (pk["bf16_tflops"] * 1e12)
    floor_s = max(tensor_s, lbytes / (hbm * 1e9))
    # the W1/W3 kernel's bound: weight streaming (HBM) at decode sizes, the tensor cores
    # once the token tiles are long enough (its FLOPs at the tensor peak outlast its
    # bytes).  An e4m3 x e4m3 contraction takes the measured bf16 peak times the nominal
    # fp8 : bf16 ratio (4.5 : 2.25 PFLOP/s dense).
    g13_flops = 4 * cfg.R * H * I
    tratio = 2.0 if a8 else 1.0
    tpeak = pk["bf16_tflops"] * tratio
    if g13_flops / (tpeak * 1e12) > g13_b / (hbm * 1e9):
        roofline = {"bound": "tensor", "achieved": g13_flops / g13_s / 1e12, "peak": tpeak,
                    "unit": "TFLOP/s", "frac": g13_flops / g13_s / 1e12 / tpeak,
                    "alg_flops_per_launch": g13_flops}
        if a8:
            roofline["peak_note"] = "measured bf16 peak x 2 (nominal e4m3 : bf16 dense ratio)"
        if "bf16_tflops_sustained" in pk:
            roofline["frac_of_sustained_peak"] = (g13_flops / g13_s / 1e12 /
                                                  (pk["bf16_tflops_sustained"] * tratio))
    else:
        roofline = {"bound": "hbm", "achieved": g13_b / g13_s / 1e9, "peak": hbm, "unit": "GB/s",
                    "frac": g13_b / g13_s / 1e9 / hbm, "alg_bytes_per_launch": g13_b}
    layer = {"tflops": flops / step_s / 1e12, "alg_bytes": lbytes, "gb_s": lbytes / step_s / 1e9,
             "roofline_floor_us": floor_s * 1e6, "roofline_frac": floor_s / step_s,
             "useful_flop_fraction_k_over_E": cfg.k / cfg.E}
    g2_b = gemm2_bytes(cfg, touched, wbytes, abytes)
    gg = {"tflops": gemm_flops / (g13_s + g2_s) / 1e12, "gb_s": (g13_b + g2_b) / (g13_s + g2_s) / 1e9,
          "gemm13_tflops": g13_flops / g13_s / 1e12, "gemm2_tflops": 2 * cfg.R * H * I / g2_s / 1e12,
          "gemm2_frac_hbm": g2_b / g2_s / 1e9 / hbm}
    return layer, gg, roofline


def other_workload_line(cfg, args, dev, stream, rank, world, graph, pk):
    """Tokens/s, step time, layer fraction and phase times of one more workload, with
    the clocks sampled over its timed steps."""
    W = Workload(cfg, args, dev, stream, rank, world)
    try:
        time.sleep(1.0)  # let the power draw of the previous workload settle
        clk = ClockSampler(dev.index if dev.index is not None else 0).start()
        elapsed_ms, launches, phase_ms = time_steps(W, args.other_steps, args.warmup, world, graph, clock=clk)
        cs = clk.summary()
        elapsed_ms = max_over_ranks(elapsed_ms, world)
        step_s = elapsed_ms / 1e3 / args.other_steps
        layer, gg, roof = summarise(cfg, W.touched, step_s, phase_ms, pk, W.wbytes, W.abytes, W.a8)
        return {"workload": workload_desc(cfg), "tokens_per_s": world * cfg.N / step_s,
                "ms_per_step": elapsed_ms / args.other_steps, "layer_floor_us": layer["roofline_floor_us"],
                "layer_frac": layer["roofline_frac"], "gemm_tflops": gg["tflops"], "gemm_gb_s": gg["gb_s"],
                "gemm13_roofline": {k: roof[k] for k in ("bound", "achieved", "unit", "frac")},
                "phase_us": {p: 1e3 * v for p, v in phase_ms.items()},
                "launch_mode": "cuda graph replay" if graph else "stream launches", "gpu_launches": launches,
                "touched_experts": W.touched, "max_expert_rows": W.max_load, "l2": W.l2_note,
                "clocks": ({k: cs[k] for k in ("sm_mhz", "power_w_max", "reasons", "samples")} if cs else None)}
    finally:
        W.release()
        del W
        torch.cuda.empty_cache()


def other_workloads(args, headline, dev, stream, rank, world, pk):
    """Every workload shape other than the headline, timed in the same run (steps
    --other-steps each).  The launch-bound decode shapes are also timed replayed from a
    CUDA graph."""
    names = [("mixtral_8x22b_decode", None, False), ("deepseek_v2", None, False),
             ("qwen3_235b_a22b_skew", None, False), ("qwen3_235b_a22b_skew4x", None, False)]
    names += [("qwen3_30b_a3b", n, False) for n in QWEN3_30B_TOKEN_SWEEP]
    names += [("qwen3_30b_a3b", 1, True), ("qwen3_30b_a3b", 16, True), ("tiny", None, False), ("tiny", None, True)]
    out = []
    for name, n, graph in names:
        if name not in CONFIGS:
            continue
        cfg = CONFIGS[name] if n is None else CONFIGS[name].with_tokens(n)
        if cfg.name == headline.name and not graph:
            continue
        out.append(other_workload_line(cfg, args, dev, stream, rank, world, graph, pk))
    return out


def run_ours(args, cfg, world, rank, local):
    from expert_ffn_layer_moe_b200 import moe
    moe.moe_set_gather_mode({"auto": moe.MOE_GATHER_AUTO, "on": moe.MOE_GATHER_ON,
                             "off": moe.MOE_GATHER_OFF}[args.gather])
    moe.moe_set_microbatches(args.microbatches)
    moe.moe_set_shared_stream(bool(args.shared_stream))
    moe.moe_set_decode_gemv({"auto": moe.MOE_DECODE_AUTO, "off": moe.MOE_DECODE_OFF,
                             "on": moe.MOE_DECODE_ON}[args.decode])
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    W = Workload(cfg, args, dev, stream, rank, world)
    moe, t = W.moe, W.t
    N, H, I, E, k = cfg.N, cfg.H, cfg.I, cfg.E, cfg.k
    fp8, a8 = W.fp8, W.a8

    fp8_err = None
    if fp8:
        # the experiment's numerical cost: the fp8 layer against the bf16 layer, same inputs
        ref = moe.moe_layer_forward_ex(t["x"], t["W_gate"], t["W1"], t["W3"], t["W2"], k, bias=t["bias"],
                                       Ws1=t["Ws1"], Ws3=t["Ws3"], Ws2=t["Ws2"], ws=W.ws, stream=stream)
        W.step(copy=0)
        torch.cuda.synchronize()
        d = (W.out.float() - ref.float()).norm() / ref.float().norm()
        fp8_err = {"rel_l2_vs_bf16_layer": float(d),
                   "max_abs_vs_bf16_layer": float((W.out.float() - ref.float()).abs().max())}
        del ref

    clk = ClockSampler(local).start()
    elapsed_ms, launches, phase_ms = time_steps(W, args.steps, args.warmup, world, args.graph, clock=clk)

    # end to end through the public API, host x in and host out back every step, both
    # inside the timed region.  The headline form runs the explicit call on its stream
    # with the copies on two copy streams, double-buffered: step i+1's input copy and
    # step i's output copy overlap the neighbouring steps' layers, as in a serving loop.
    # The short form (which takes host pointers, copies them itself and returns when
    # out is on the host) is timed as well, where it covers the workload.
    x_host = t["x"].cpu().pin_memory()
    out_host = [torch.empty((N, H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_buf = [torch.empty_like(t["x"]) for _ in range(2)]
    o_buf = [torch.empty_like(W.out) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_pipelined(steps):
        """Returns the device time (ms) from the first input copy to the last output copy."""
        ev_in = [torch.cuda.Event() for _ in range(steps)]
        ev_done = [torch.cuda.Event() for _ in range(steps)]
        ev_out = [torch.cuda.Event() for _ in range(steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def h2d(i):
            if i >= 2:
                s_in.wait_event(ev_done[i - 2])  # the layer of step i-2 has read this buffer
            with torch.cuda.stream(s_in):
                x_buf[i % 2].copy_(x_host, non_blocking=True)
            ev_in[i].record(s_in)

        t0.record(s_in)
        h2d(0)
        for i in range(steps):
            if i + 1 < steps:
                h2d(i + 1)
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_out[i - 2])  # the output copy of step i-2 has read this buffer
            W.step(x=x_buf[i % 2], o=o_buf[i % 2])
            ev_done[i].record(stream)
            s_out.wait_event(ev_done[i])
            with torch.cuda.stream(s_out):
                out_host[i % 2].copy_(o_buf[i % 2], non_blocking=True)
            ev_out[i].record(s_out)
        stream.wait_event(ev_out[steps - 1])
        t1.record(stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    e2e_pipelined(args.warmup)
    barrier(world)
    e2e_ms = max_over_ranks(e2e_pipelined(args.steps), world)
    call = "moe_layer_forward_w8a8_ex" if a8 else ("moe_layer_forward_fp8_ex" if fp8 else "moe_layer_forward_ex")
    e2e = {"value": world * N * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": N * H * 2, "d2h_bytes_per_step": N * H * 2,
           "how": (f"{call} on its stream; each step's x copied in from pinned host memory and its out copied "
                   "back to pinned host memory on two copy streams, double-buffered (copies overlap the "
                   "neighbouring steps' layers); timed from the first copy in to the last copy out")}
    if not fp8 and cfg.Is == 0 and cfg.bias_scale == 1.0 and not cfg.skew and W.copies == 1:
        def short_step():
            moe.moe_layer_forward(x_host, t["W_gate"], t["W1"], t["W3"], t["W2"], k, out=out_host[0])
        for _ in range(args.warmup):
            short_step()
        barrier(world)
        torch.cuda.synchronize()
        d = torch.cuda.default_stream(dev)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(d)
        for _ in range(args.steps):
            short_step()
        s1.record(d)
        torch.cuda.synchronize()
        short_ms = max_over_ranks(s0.elapsed_time(s1), world)
        e2e["short_form"] = {"value": world * N * args.steps / (short_ms / 1e3), "unit": "tokens/s",
                             "how": "moe_layer_forward with host x and out, one synchronous call per step"}
    del x_buf, o_buf

    elapsed_ms = max_over_ranks(elapsed_ms, world)
    pk, pk_kind = peaks()
    step_s = elapsed_ms / 1e3 / args.steps
    value = world * N / step_s
    layer, gg, roofline = summarise(cfg, W.touched, step_s, phase_ms, pk, W.wbytes, W.abytes, a8)
    workload = cfg.name
    kdesc = ", e4m3 weights and activations" if a8 else (", e4m3 weights" if fp8 else "")
    roofline.update({"kernel": "grouped_gemm SwiGLU W1/W3 (gemm13)" + kdesc,
                     "peak_kind": pk_kind,
                     "traffic": (kernel_traffic("gemm13_w8a8", workload) if a8 else
                                 None if fp8 else kernel_traffic("gemm13", workload)),
                     "avg_launch_ms": phase_ms["gemm13"]})
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if a8 else "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(cfg), "global_batch": world * N, "tokens_per_gpu": N,
                   "parallelism": f"dp{world} (token batches, replicated weights, no exchange)",
                   "l2": W.l2_note, "touched_experts": W.touched, "max_expert_rows": W.max_load,
                   "expert_weights": (("e4m3, one fp32 scale per output channel (quantized once before "
                                       "timing; " + ("multiplied as e4m3" if a8 else "widened to bf16 on chip")
                                       + ")") if fp8 else "bf16"),
                   "expert_activations": ("e4m3, one fp32 scale per row (x_perm and h quantized on the device "
                                          "every step)") if a8 else "bf16",
                   "w13_rows": f"gather mode {args.gather}", "microbatches": args.microbatches,
                   "shared_experts_stream": "second stream" if args.shared_stream else "caller's stream",
                   "decode_gemv": args.decode},
        "roofline": roofline,
        "layer": layer,
        "grouped_gemm": gg,
        "phase_ms": phase_ms,
        "phase_ms_note": "mean per-phase CUDA-event times from a second timed pass with events between phases",
        "gpu_launches": launches,
        "gpu_launches_note": ("the library's own host-side count of its kernel launches over the timed steps" +
                              (" (counted once at graph capture, times the replays)" if args.graph else "")),
        "launch_mode": "cuda graph replay of one captured step" if args.graph else "stream launches",
        "e2e": e2e,
    }
    if fp8_err is not None:
        line["fp8_error"] = fp8_err
    clk_sum = clk.summary()
    if clk_sum:
        line["clocks"] = clk_sum
    W.release()
    del W, t
    torch.cuda.empty_cache()
    if not args.no_others:
        line["other_workloads"] = other_workloads(args, cfg, dev, stream, rank, world, pk)
        line["other_workloads_note"] = (f"each workload timed in this run: {args.warmup} warm-up and "
                                        f"{args.other_steps} timed steps, CUDA events on the launching stream; "
                                        "phase_us from a second pass with events between phases")
    if world == 1 and not args.no_cpu_baseline and rank == 0:
        th = host_inputs(cfg)
        line["cpu_baseline"] = cpu_baseline(cfg, th, args.cpu_seconds)
        del th
    if rank == 0:
        print(json.dumps(line), flush=True)


def ep_local_inputs(cfg, rank, world, device):
    """Expert-parallel inputs of one rank: its own token batch (seed = rank), the whole
    router, and its slice [rank*L, (rank+1)*L) of every expert stack (L = E / world)."""
    from expert_ffn_layer_moe_b200 import ep
    if cfg.E % world:
        raise ValueError(f"{cfg.E} experts do not split over {world} ranks")
    t = make_inputs(cfg, seed=0, device=device)
    x = make_inputs(cfg, seed=rank, device=device, weights=False)["x"]
    local = {n: ep.local_experts(t[n], rank, world).contiguous() for n in ("W1", "W3", "W2")}
    del t["W1"], t["W3"], t["W2"]
    return x, t["W_gate"], t["bias"], local


def ep_line(cfg, world, steps, warmup, step_ms_max, exchange, rows_sent, rows_recv, e2e_ms_max=None):
    """The expert-parallel JSON line: value = all ranks' tokens / the slowest rank's time."""
    line = {"metric": METRIC, "value": world * cfg.N / (step_ms_max / 1e3), "unit": "tokens/s", "n_gpus": world,
            "steps": steps, "warmup": warmup, "ms_per_step": step_ms_max, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload_desc(cfg), "global_batch": world * cfg.N, "tokens_per_gpu": cfg.N,
                       "parallelism": (f"ep{world}: experts split {cfg.E}/{world} per rank, token rows exchanged "
                                       f"by {exchange}, one token batch per rank"),
                       "rows_sent_per_rank": rows_sent, "rows_received_per_rank": rows_recv}}
    if e2e_ms_max is not None:
        line["e2e"] = {"value": world * cfg.N / (e2e_ms_max / 1e3), "unit": "tokens/s",
                       "h2d_bytes_per_step": cfg.N * cfg.H * 2, "d2h_bytes_per_step": cfg.N * cfg.H * 2,
                       "how": "each step's x copied in from pinned host memory and its out read back, synchronous"}
    return line


def run_ep(args, cfg, world, rank, local):
    """Expert parallelism: every rank holds E/world experts and its own batch; a step is
    route, permute, the row exchange to the experts' ranks, the local grouped GEMMs,
    the exchange back and the combine (moe_layer_forward_ep).  One rank works too (the
    exchange then stays on the GPU)."""
    import datetime
    import socket
    import torch.distributed as dist
    from expert_ffn_layer_moe_b200 import ep, moe
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    own_group = False
    if not dist.is_initialized():  # one rank: a group of one
        sk = socket.socket()
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
        sk.close()
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=120))
        own_group = True
    try:
        x, Wg, bias, W = ep_local_inputs(cfg, rank, world, dev)
        tr = None
        if args.exchange == "peer_copy":
            tr = ep.PeerCopyTransport(ep.CudaPeers(device=dev), max_rows=cfg.N * cfg.k, words_in=cfg.H // 2,
                                      words_out=cfg.H)
        stats = []

        def step(xx=None, record=None):
            return ep.moe_layer_forward_ep(x if xx is None else xx, Wg, W["W1"], W["W3"], W["W2"], cfg.k, bias=bias,
                                           transport=tr, stats=record)

        for _ in range(args.warmup):
            step()
        step(record=stats)  # one step with per-phase records (rows moved)
        torch.cuda.synchronize()
        if moe.moe_get_device_error() != 0:
            raise RuntimeError("device error reported during warm-up")
        s = torch.cuda.current_stream(dev)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dist.barrier()
        torch.cuda.synchronize()
        t0.record(s)
        for _ in range(args.steps):
            step()
        t1.record(s)
        torch.cuda.synchronize()
        dist.barrier()
        ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world)
        # end to end: x from pinned host memory in, out back to the host, every step
        xh = x.cpu().pin_memory()
        oh = torch.empty((cfg.N, cfg.H), dtype=torch.bfloat16).pin_memory()
        dist.barrier()
        torch.cuda.synchronize()
        t0.record(s)
        for _ in range(args.steps):
            xd = xh.to(dev, non_blocking=True)
            oh.copy_(step(xd), non_blocking=True)
        t1.record(s)
        torch.cuda.synchronize()
        dist.barrier()
        e2e_ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world)
        if tr is not None:
            tr.close()
        if moe.moe_get_device_error() != 0:
            raise RuntimeError("device error reported during the timed steps")
        line = ep_line(cfg, world, args.steps, args.warmup, ms, args.exchange, stats[0].rows_sent,
                       stats[0].rows_received, e2e_ms)
        line["ep_phase_s"] = stats[0].seconds
        line["gpu_launches_note"] = "not counted for the expert-parallel step"
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if own_group:
            dist.destroy_process_group()


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    tt = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="qwen3_235b_a22b_skew", choices=sorted(CONFIGS))
    ap.add_argument("--tokens", type=int, default=0, help="override N (a smaller case for profiling)")
    ap.add_argument("--experts", type=int, default=0, help="override E (a smaller case for profiling)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="about this much multi-threaded oracle time for cpu_baseline")
    ap.add_argument("--ref-seconds", type=float, default=10.0,
                    help="--impl reference: about this much oracle time per step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-others", action="store_true", help="time the headline workload only")
    ap.add_argument("--other-steps", type=int, default=10)
    ap.add_argument("--no-rotate", action="store_true",
                    help="do not cycle through weight copies on shapes whose touched weights fit in L2")
    ap.add_argument("--graph", action="store_true",
                    help="time replays of one layer step captured as a CUDA graph (launch-bound decode sizes)")
    ap.add_argument("--weights", choices=["bf16", "fp8"], default="bf16",
                    help="routed-expert weight format (fp8: e4m3 with per-channel scales, a separate experiment)")
    ap.add_argument("--acts", choices=["bf16", "fp8"], default="bf16",
                    help="routed-expert activation format (fp8: e4m3 with per-row scales; needs --weights fp8)")
    ap.add_argument("--microbatches", type=int, choices=[1, 2], default=1,
                    help="run large layers as two micro-batches on two streams (moe_set_microbatches)")
    ap.add_argument("--decode", choices=["auto", "off", "on"], default="auto",
                    help="decode batches: expert FFN as CUDA-core GEMVs with the combine folded in "
                         "(moe_set_decode_gemv)")
    ap.add_argument("--shared-stream", type=int, choices=[0, 1], default=1,
                    help="run the shared experts on a second stream beside the dispatch (moe_set_shared_stream)")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism: the experts split over the ranks, token rows exchanged")
    ap.add_argument("--exchange", choices=["collective", "peer_copy"], default="collective",
                    help="--ep: rows moved by NCCL all-to-all or by copies into the peers' buffers (CUDA IPC)")
    ap.add_argument("--gather", choices=["auto", "on", "off"], default="auto",
                    help="W1/W3 token rows: gathered from x (on), the permuted copy (off), or by shape (auto)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.acts == "fp8" and args.weights != "fp8":
        ap.error("--acts fp8 needs --weights fp8")
    cfg = CONFIGS[args.config]
    if args.tokens:
        cfg = cfg.with_tokens(args.tokens)
    if args.experts:
        cfg = dataclasses.replace(cfg, name=f"{cfg.name}@E={args.experts}", E=args.experts,
                                  k=min(cfg.k, args.experts))
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, cfg, world, rank)
        elif args.ep:
            run_ep(args, cfg, world, rank, local)
        else:
            run_ours(args, cfg, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

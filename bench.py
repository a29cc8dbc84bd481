"""Benchmark of the DBF layer forward on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload attn_1b] [--batch 1] [--sweep OUT.json]
                    [--profile-calls N [--flags F]]   (plain calls for ncu captures)

Workload (default): the Llama-8B-shaped attention projection n = m_in = 4096,
k = 2048 (1.0 bit/weight), batch 1 (config attn_1b of dbf_inputs).  A step is
the forward of one batch through R distinct copies of that layer (each copy in
its own HBM buffers, R * bytes >= 4 * L2), so every layer's weights stream from
HBM; the R forwards are captured once as a CUDA graph and the graph is replayed
once per step.  Metric: tokens/s through one DBF layer (= batch / time per
layer forward), with us/layer and achieved HBM GB/s reported alongside.

Multi-GPU (torchrun, N > 1): replicas only - every rank runs the same workload
on its own GPU with no data-path collective; the timed region is bracketed by
barriers and the slowest rank's time is used.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import dbf_inputs as gen  # noqa: E402

METRIC = "DBF layer fwd µs, HBM GB/s (% of peak) & tokens/s at 1/2 bit, batch 1–2048"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ------------------------------------------------------------------ helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def layer_bytes(n, k, m_in, batch):
    """Algorithmic HBM bytes of one layer forward: packed signs, fp16 scales, x in, y out."""
    return n * k / 8 + k * m_in / 8 + 2 * (n + k + m_in) + 2 * batch * (m_in + n)


def layer_flops(n, k, m_in, batch):
    """Signed additions of the two sign products, counted as multiply-adds (2 flops)."""
    return 2.0 * batch * k * (m_in + n)


# Sources each path's kernels and their launches are built from (the others
# do not change what that path runs).
DECODE_SOURCES = ("dbf_api.cu", "dbf_device.cuh", "dbf_internal.h", "decode.cu")
PREFILL_SOURCES = ("dbf_api.cu", "dbf_device.cuh", "dbf_internal.h", "prefill.cu")


def kernel_source_hash(files=None):
    """Hash of the kernel sources (all of csrc, or the named files of it)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "binary_factorized_weight_b200", "csrc")
    for name in sorted(files if files is not None else os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def graph_kernel_launches(graph):
    """Kernel nodes of a captured CUDA graph: the launches one replay makes
    (None when the graph cannot be inspected)."""
    try:
        from cuda.bindings import runtime as rt

        handle = rt.cudaGraph_t(init_value=graph.raw_cuda_graph())
        err, _, count = rt.cudaGraphGetNodes(handle, 0)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        err, nodes, count = rt.cudaGraphGetNodes(handle, count)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        kernels = 0
        for node in nodes[:count]:
            err, kind = rt.cudaGraphNodeGetType(node)
            if err != rt.cudaError_t.cudaSuccess:
                return None
            kernels += kind == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
        return kernels
    except Exception:
        return None


def traffic_for(workload_key):
    """DRAM bytes per forward from the committed ncu summary, if the kernels are unchanged since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        entry = t[workload_key]
        if entry.get("source_hash") != kernel_source_hash(entry.get("source_files")):
            return None
        return entry["dram_bytes_per_forward"]
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"], "samples": 0}
        inside = [r for r in rows if t0 <= r[0] <= t1]
        window = "timed region"
        if not inside:
            inside = sorted(rows, key=lambda r: min(abs(r[0] - t0), abs(r[0] - t1)))[:3]
            window = "nearest samples (timed region shorter than the sampling period)"
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside), "window": window}


def max_over_ranks(value_ms, world, device=None):
    """The slowest rank's time (every rank takes part; a no-op on one rank)."""
    if world <= 1:
        return float(value_ms)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, elapsed_ms):
    """Units all ranks processed per second (weak scaling: every rank does the same work)."""
    return world * units_per_rank / (elapsed_ms * 1e-3)


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    return world, rank, local


# ------------------------------------------------------------------ reference arm (the fp64 oracle)
def oracle_rate(shape, batch, seconds, rotation=0):
    """Time the oracle as it stands on host cores: tokens/s through one layer."""
    import oracle

    L = gen.make_layer(shape, batch, rotation)
    oracle.forward_staged(L["x"][:1], L["A"], L["B"], L["a"], L["mid"], L["b"])  # load + page in
    calls, t0 = 0, time.perf_counter()
    while True:
        oracle.forward_staged(L["x"], L["A"], L["B"], L["a"], L["mid"], L["b"])
        calls += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return batch * calls / el, calls, el, oracle.num_threads()


def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


REFERENCE_MIN_SECONDS = 8.0


def run_reference(args, shape, batch):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return
    import oracle

    L = gen.make_layer(shape, batch)
    oracle.forward_staged(L["x"], L["A"], L["B"], L["a"], L["mid"], L["b"])  # warm
    for _ in range(args.warmup):
        oracle.forward_staged(L["x"], L["A"], L["B"], L["a"], L["mid"], L["b"])
    # K steps of one layer forward each, continued until at least a few seconds
    # are timed, so that the rate is stable whatever K the caller asks for
    calls, t0 = 0, time.perf_counter()
    while True:
        oracle.forward_staged(L["x"], L["A"], L["B"], L["a"], L["mid"], L["b"])
        calls += 1
        el = time.perf_counter() - t0
        if calls >= args.steps and el >= REFERENCE_MIN_SECONDS:
            break
    value = batch * calls / el
    sample = (f"{calls} fp64 oracle forwards of one {shape.name} layer at batch {batch} ({el:.1f} s; each the unit "
              f"of the GPU arm's R-layer step); CPU: {cpu_model()}")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / calls,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(shape, batch), "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def workload_name(shape, batch):
    bpw = shape.k * (shape.n + shape.m_in) / (shape.n * shape.m_in)
    return f"{shape.name}: n={shape.n} m_in={shape.m_in} k={shape.k} ({bpw:.3f} bit/weight), batch {batch}"


# ------------------------------------------------------------------ our arm
class Workload:
    """R rotated copies of one layer on the device plus everything a step needs."""

    def __init__(self, dbf, torch, shape, batch, device, copies=None, flags=None):
        self.dbf, self.torch = dbf, torch
        self.shape, self.batch = shape, batch
        n, k, m_in = shape.n, shape.k, shape.m_in
        L = gen.make_layer(shape, batch)
        self.host = L
        d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        pA = dbf.dbf_pack_signs(d(L["A"]))
        pB = dbf.dbf_pack_signs(d(L["B"]))
        a, mid, b = d(L["a"]), d(L["mid"]), d(L["b"])
        self.bytes = layer_bytes(n, k, m_in, batch)
        l2 = torch.cuda.get_device_properties(device).L2_cache_size
        weight_bytes = (pA.numel() + pB.numel()) * 4 + 2 * (n + k + m_in)
        self.copies = copies or max(2, int(math.ceil(4 * l2 / weight_bytes)))
        self.pA = [pA] + [pA.clone() for _ in range(self.copies - 1)]
        self.pB = [pB] + [pB.clone() for _ in range(self.copies - 1)]
        self.sc = [(a, mid, b)] + [(a.clone(), mid.clone(), b.clone()) for _ in range(self.copies - 1)]
        self.x = d(L["x"])
        self.y = torch.empty((batch, n), dtype=torch.float16, device=device)
        self.ws = dbf.dbf_new_workspace(n, k, m_in, batch, device=device)
        self.flags = dbf.DBF_FWD_WEIGHTS_STATIC if flags is None else flags
        self.weight_bytes_total = self.copies * weight_bytes
        decode = batch <= 16 and not (self.flags & dbf.DBF_FWD_FORCE_PREFILL)
        two_stage = self.flags & (dbf.DBF_FWD_DECODE_TWO_STAGE | dbf.DBF_FWD_DECODE_SHIFT_EXPAND)
        self.launches_per_forward = ((1 if not two_stage else 2) * math.ceil(batch / 16)) if decode else 2
        self.path = "decode" if decode else "prefill (tcgen05, 2 GEMMs)"

    def forward_all(self, x=None, y=None):
        x = self.x if x is None else x
        y = self.y if y is None else y
        s = self.shape
        for i in range(self.copies):
            a, mid, b = self.sc[i]
            self.dbf.dbf_forward(x, self.pA[i], self.pB[i], a, mid, b, s.n, s.k, s.m_in, y=y, workspace=self.ws,
                                 flags=self.flags)

    def capture(self):
        torch = self.torch
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.forward_all()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph(keep_graph=True)  # kept so that its launches can be counted
        with torch.cuda.graph(g):
            self.forward_all()
        g.instantiate()
        torch.cuda.synchronize()
        return g


class TransposedWorkload(Workload):
    """The same R layer copies run as the transpose product dx = dy W (dy: batch x n)."""

    def __init__(self, dbf, torch, shape, batch, device, copies=None):
        super().__init__(dbf, torch, shape, batch, device, copies=copies)
        n, k, m_in = shape.n, shape.k, shape.m_in
        self.pAT = [dbf.dbf_transpose_signs(pA, n, k) for pA in self.pA]
        self.pBT = [dbf.dbf_transpose_signs(pB, k, m_in) for pB in self.pB]
        rng = np.random.default_rng(7)
        self.dy = torch.from_numpy(gen.normal_activations(rng, batch, n)).to(device)
        self.dx = torch.empty((batch, m_in), dtype=torch.float16, device=device)
        self.ws = dbf.dbf_new_workspace(m_in, k, n, batch, device=device)
        self.bytes = layer_bytes(m_in, k, n, batch)
        self.path = "transposed " + self.path

    def forward_all(self, x=None, y=None):
        s = self.shape
        for i in range(self.copies):
            a, mid, b = self.sc[i]
            self.dbf.dbf_forward_transposed(self.dy, self.pAT[i], self.pBT[i], a, mid, b, s.n, s.k, s.m_in,
                                            dx=self.dx, workspace=self.ws, flags=self.flags)


GROUPS = {"qkv": ("q", "k", "v"), "gate_up": ("gate", "up")}


class GroupWorkload(Workload):
    """R rotated copies of layers that share their input, run through dbf_forward_grouped."""

    def __init__(self, dbf, torch, shapes, batch, device, copies=None):
        self.dbf, self.torch = dbf, torch
        self.batch = batch
        self.m_in = shapes[0].m_in
        d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        Ls = [gen.make_layer(s, batch) for s in shapes]
        self.host = Ls
        base = [dict(packedA=dbf.dbf_pack_signs(d(L["A"])), packedB=dbf.dbf_pack_signs(d(L["B"])), a=d(L["a"]),
                     m=d(L["mid"]), b=d(L["b"]), n=s.n, k=s.k) for s, L in zip(shapes, Ls)]
        self.bytes = sum(layer_bytes(s.n, s.k, s.m_in, batch) for s in shapes) - 2 * batch * self.m_in * (
            len(shapes) - 1)  # x is read once
        self.flops = sum(layer_flops(s.n, s.k, s.m_in, batch) for s in shapes)
        weight_bytes = sum((L["packedA"].numel() + L["packedB"].numel()) * 4 + 2 * (L["n"] + L["k"] + self.m_in)
                           for L in base)
        l2 = torch.cuda.get_device_properties(device).L2_cache_size
        self.copies = copies or max(2, int(math.ceil(4 * l2 / weight_bytes)))
        self.groups = [base] + [[{k: (v.clone() if hasattr(v, "clone") else v) for k, v in L.items()} for L in base]
                                for _ in range(self.copies - 1)]
        self.x = d(Ls[0]["x"])
        self.ys = [torch.empty((batch, s.n), dtype=torch.float16, device=device) for s in shapes]
        self.ws = dbf.dbf_new_grouped_workspace(base, self.m_in, batch, device=device)
        self.flags = dbf.DBF_FWD_WEIGHTS_STATIC
        self.path = "decode (grouped)" if batch <= 16 else "prefill (per layer)"

    def forward_all(self, x=None, y=None):
        for grp in self.groups:
            self.dbf.dbf_forward_grouped(self.x, grp, self.m_in, ys=self.ys, workspace=self.ws, flags=self.flags)


def time_replays(torch, graph, reps, rounds=1):
    """Device time (ms) of `reps` replays of a captured graph, CUDA events on
    the current stream; the median over `rounds` rounds."""
    times = []
    for _ in range(rounds):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def path_name(wl, launches_per_layer):
    if wl.batch <= 16 and not (wl.flags & wl.dbf.DBF_FWD_FORCE_PREFILL):
        if launches_per_layer is not None and launches_per_layer <= math.ceil(wl.batch / 16):
            return "decode: one launch per layer (int8 mma.sync sign products, V handed over inside the cluster)"
        return "decode: two PDL-chained launches per layer (fp16 mma.sync sign-GEMV)"
    return "prefill: tcgen05 GEMMs (two or three launches per layer)"


def roofline_for(wl, shape, batch, us, peaks, traffic, peak_kind="burst"):
    """The roofline object of one layer forward timed at `us` per layer."""
    if batch > 16:
        fl = layer_flops(shape.n, shape.k, shape.m_in, batch)
        tf = fl / (us * 1e-6) / 1e12
        peak = peaks["bf16_tflops"] if peak_kind == "burst" else peaks["bf16_tflops_sustained"]
        return {"bound": "tensor", "kernel": "dbf_forward prefill (GEMM1 + GEMM2, one layer)", "achieved": tf,
                "peak": peak, "unit": "TFLOP/s", "frac": tf / peak, "traffic": traffic,
                "peak_source": f"{peaks['source']} dense bf16 {peak_kind} of measured (fp16 runs at the bf16 rate)",
                "algorithmic_flops_per_layer": fl}
    gbs = wl.bytes / (us * 1e-6) / 1e9
    return {"bound": "hbm", "kernel": "dbf_forward decode (one layer)", "achieved": gbs, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "traffic": traffic,
            "peak_source": f"{peaks['source']} STREAM-style copy of measured (MEASURED_PEAKS.json)",
            "algorithmic_bytes_per_layer": wl.bytes}


def measure_workload(dbf, torch, shape, batch, device, peaks, rounds=5):
    """One more configuration of the metric in the same run: R rotated copies in
    one CUDA graph, device-timed; its own roofline and clock record.  A
    tensor-core configuration whose timed rounds run back to back for 100 ms or
    more is a kernel timed inside a long step: its fraction is taken of the
    sustained dense peak (the burst fraction is given beside it)."""
    wl = Workload(dbf, torch, shape, batch, device)
    g = wl.capture()
    launches = graph_kernel_launches(g)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    reps = max(3, int(400 / wl.copies))
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)  # nvidia-smi's first samples (outside the timed region)
    t0 = time.time()
    ms = time_replays(torch, g, reps, rounds)
    t1 = time.time()
    sampler.stop()
    us = 1e3 * ms / reps / wl.copies
    ok = dbf.dbf_workspace_status(wl.ws) == 0
    long_run = (t1 - t0) >= 0.1
    roof = roofline_for(wl, shape, batch, us, peaks, traffic_for(f"{shape.name}_b{batch}"),
                        peak_kind="sustained" if (batch > 16 and long_run) else "burst")
    if batch > 16:
        roof["frac_of_burst"] = roof["achieved"] / peaks["bf16_tflops"]
        roof["timed_seconds"] = round(t1 - t0, 3)
    out = {"workload": workload_name(shape, batch), "path": path_name(wl, None if launches is None else
                                                                         launches / wl.copies),
           "us_per_layer": us, "tokens_per_s": batch / (us * 1e-6), "layers_per_replay": wl.copies,
           "launches_per_layer": None if launches is None else launches / wl.copies,
           "roofline": roof, "clocks": sampler.summary(t0, t1), "status_ok": ok}
    del g, wl
    torch.cuda.empty_cache()
    return out


def e2e_per_call(dbf, torch, wl, steps, warmup):
    """End to end through the public C ABI, one call per layer: every step copies
    x from pinned host memory, calls dbf_forward for each of the R layers (no
    graph: the host cost of every call is inside the timed region) and reads y
    back into pinned host memory.  Returns (tokens/s, h2d bytes, d2h bytes)."""
    import ctypes

    lib = dbf.load_library()
    s = wl.shape
    x_host = torch.from_numpy(np.ascontiguousarray(wl.host["x"])).pin_memory()
    y_host = torch.empty((wl.batch, s.n), dtype=torch.float16).pin_memory()
    x_dev = torch.empty_like(wl.x)
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)
    vp = ctypes.c_void_p
    ws_bytes = wl.ws.numel()
    calls = []
    for i in range(wl.copies):
        a, mid, b = wl.sc[i]
        calls.append((vp(x_dev.data_ptr()), vp(wl.pA[i].data_ptr()), vp(wl.pB[i].data_ptr()), vp(a.data_ptr()),
                      vp(mid.data_ptr()), vp(b.data_ptr()), s.n, s.k, s.m_in, wl.batch, vp(wl.y.data_ptr()), 1,
                      vp(wl.ws.data_ptr()), ws_bytes, wl.flags, sp))
    fwd = lib.dbf_forward

    def step():
        x_dev.copy_(x_host, non_blocking=True)
        bad = 0
        for c in calls:
            bad |= fwd(*c)
        y_host.copy_(wl.y, non_blocking=True)
        return bad

    for _ in range(max(3, warmup)):
        if step() != 0:
            raise RuntimeError("dbf_forward failed in the end-to-end loop")
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    bad = 0
    for _ in range(steps):
        bad |= step()
    e1.record()
    torch.cuda.synchronize()
    if bad != 0:
        raise RuntimeError("dbf_forward failed in the end-to-end loop")
    ms = e0.elapsed_time(e1)
    return ms, int(x_host.numel() * 2), int(y_host.numel() * 2)


def run_ours(args, shape, batch):
    import torch

    world, rank, local = dist_setup(args)
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    device = torch.device("cuda", local)

    from binary_factorized_weight_b200 import build as lib_build

    lib_build.build()
    import binary_factorized_weight_b200 as dbf

    dbf.load_library()
    peaks = load_peaks()
    wl = Workload(dbf, torch, shape, batch, device)
    graph = wl.capture()
    # launches per step, counted in the captured graph (the planner may split a
    # product into more than one launch); the per-path formula if it cannot be read
    step_launches = graph_kernel_launches(graph)
    launches_source = "counted in the captured graph"
    if step_launches is None:
        step_launches = wl.copies * wl.launches_per_forward
        launches_source = "per-path formula"

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    # ---------------------------------------------------------- device-timed steps
    sampler = ClockSampler(local)
    sampler.start()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    ev0.record()
    for _ in range(args.steps):
        graph.replay()
    ev1.record()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, device)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)

    ms_per_step = ms / args.steps
    us_per_layer = 1e3 * ms_per_step / wl.copies
    tokens_per_s = whole_job_rate(batch * wl.copies * args.steps, world, ms)
    hbm_gbs = wl.bytes / (us_per_layer * 1e-6) / 1e9

    # cold single launch: one layer forward after writing a buffer of 2 x L2
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(2 * l2 // 4, dtype=torch.float32, device=device)
    cold = []
    for _ in range(5):
        flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dbf.dbf_forward(wl.x, wl.pA[0], wl.pB[0], *wl.sc[0], shape.n, shape.k, shape.m_in, y=wl.y, workspace=wl.ws,
                        flags=wl.flags)
        e1.record()
        torch.cuda.synchronize()
        cold.append(1e3 * e0.elapsed_time(e1))
    del flush

    # ---------------------------------------------------------- end to end: host buffers, one C-ABI call per layer
    e2e_steps = max(3, min(args.steps, 200))
    e2e_ms, h2d, d2h = e2e_per_call(dbf, torch, wl, e2e_steps, args.warmup)
    e2e_ms = max_over_ranks(e2e_ms, world, device)
    e2e_value = whole_job_rate(batch * wl.copies * e2e_steps, world, e2e_ms)
    status_ok = dbf.dbf_workspace_status(wl.ws) == 0

    # the metric's other regimes in the same run (rank 0 reports them)
    extra = []
    if args.extra:
        for name, b in (("mlp_up", 2048), ("attn_2b", 16)):
            extra.append(measure_workload(dbf, torch, gen.CONFIGS[name], b, device, peaks))

    # output check of the timed configuration (every token, against the oracle)
    check = None
    if rank == 0 and args.check:
        import oracle

        torch.cuda.synchronize()
        ref = oracle.forward_staged(wl.host["x"], wl.host["A"], wl.host["B"], wl.host["a"], wl.host["mid"],
                                    wl.host["b"])
        y = wl.y.float().cpu().numpy().astype(np.float64)
        check = float(np.linalg.norm(y - ref) / np.linalg.norm(ref))

    if world > 1:
        torch.distributed.barrier()
        del graph
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    # ---------------------------------------------------------- CPU baseline (oracle), rank 0 at N = 1 only
    cpu = None
    if world == 1 and args.cpu_seconds > 0:
        import oracle

        rate, calls, el, cores = oracle_rate(shape, batch, args.cpu_seconds)
        oracle.set_num_threads(1)
        rate1, calls1, el1, _ = oracle_rate(shape, batch, max(1.0, args.cpu_seconds / 4))
        oracle.set_num_threads(cores)
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{calls} fp64 oracle forwards of one {shape.name} layer at batch {batch} "
                         f"({el:.1f} s on {cores} host threads)",
               "one_thread": {"value": rate1, "unit": "tokens/s", "cores": 1,
                              "sample": f"{calls1} forwards in {el1:.1f} s on one thread"},
               "cpu_model": cpu_model()}

    key = f"{shape.name}_b{batch}"
    traffic = traffic_for(key)
    launches_per_layer = step_launches / wl.copies
    result = {
        "metric": METRIC,
        "value": tokens_per_s,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic",
        "config": {
            "workload": workload_name(shape, batch),
            "path": path_name(wl, launches_per_layer),
            "layers_per_step": wl.copies,
            "l2": f"inputs larger than L2: {wl.copies} distinct weight copies, "
                  f"{wl.weight_bytes_total / 1e6:.0f} MB >= 4 x L2",
            "parallelism": "replicas" if world > 1 else "single GPU",
            "graph": "one CUDA graph of the step's dbf_forward calls, replayed once per step",
        },
        "us_per_layer": us_per_layer,
        "us_cold_single_launch": statistics.median(cold),
        "hbm_gbs": hbm_gbs,
        "hbm_frac": hbm_gbs / peaks["hbm_gbs"],
        "roofline": roofline_for(wl, shape, batch, us_per_layer, peaks, traffic),
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "how": f"{e2e_steps} steps; per step: x from pinned host memory, {wl.copies} dbf_forward calls "
                       "through the C ABI (ctypes, no graph), y back to pinned host memory; CUDA events"},
        "gpu_launches": args.steps * step_launches,
        "gpu_launches_source": launches_source,
        "clocks": clocks,
        "workspace_status_ok": status_ok,
        "also": extra,
    }
    if check is not None:
        result["output_check_rel_fro"] = check
    print(json.dumps(result))


# ------------------------------------------------------------------ sweep (all configs, one GPU)
def dense_fp16_us(torch, shape, batch, device):
    """Context only (not the product): torch.matmul of x with a dense fp16 W of the
    same shape, W rotated over copies larger than 4x L2 like the DBF layers."""
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    wbytes = 2 * shape.n * shape.m_in
    copies = max(2, int(math.ceil(4 * l2 / wbytes)))
    Ws = [torch.randn(shape.n, shape.m_in, device=device, dtype=torch.float16) for _ in range(copies)]
    x = torch.randn(batch, shape.m_in, device=device, dtype=torch.float16)
    y = torch.empty(batch, shape.n, device=device, dtype=torch.float16)
    for W in Ws[:3]:
        torch.matmul(x, W.t(), out=y)
    torch.cuda.synchronize()
    times = []
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for W in Ws:
            torch.matmul(x, W.t(), out=y)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / copies * 1e3)
    del Ws
    torch.cuda.empty_cache()
    return statistics.median(times)


def run_sweep(args):
    import torch

    torch.cuda.set_device(0)
    from binary_factorized_weight_b200 import build as lib_build

    lib_build.build()
    import binary_factorized_weight_b200 as dbf

    dbf.load_library()
    peaks = load_peaks()
    device = torch.device("cuda", 0)
    cases = [(gen.CONFIGS["attn_1b"], 1)]
    cases += [(gen.CONFIGS["attn_2b"], b) for b in (1, 4, 16)]
    cases += [(gen.CONFIGS["mlp_up"], b) for b in (1, 2048)]
    for bits in (1, 2):
        for s in gen.LAYER_SET[bits]:
            cases += [(s, b) for b in (1, 16, 128, 2048)]
    rows = []
    for shape, batch in cases:
        wl = Workload(dbf, torch, shape, batch, device)
        g = wl.capture()
        for _ in range(5):
            g.replay()
        torch.cuda.synchronize()
        reps = max(3, int(200 / max(1, wl.copies)))
        times = []
        for _ in range(7):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) / reps / wl.copies * 1e3)
        us = statistics.median(times)
        gbs = wl.bytes / (us * 1e-6) / 1e9
        tf = layer_flops(shape.n, shape.k, shape.m_in, batch) / (us * 1e-6) / 1e12
        dense_us = dense_fp16_us(torch, shape, batch, device)
        dense_bytes = 2 * shape.n * shape.m_in + 2 * batch * (shape.n + shape.m_in)  # fp16 W, x and y once
        dense_floor_us = dense_bytes / (peaks["hbm_gbs"] * 1e9) * 1e6
        row = {"layer": shape.name, "n": shape.n, "k": shape.k, "m_in": shape.m_in, "batch": batch,
               "bpw": shape.k * (shape.n + shape.m_in) / (shape.n * shape.m_in), "us": us,
               "us_p10": sorted(times)[0], "us_p90": sorted(times)[-1], "tokens_per_s": batch / (us * 1e-6),
               "hbm_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"], "tflops": tf,
               "tensor_frac": tf / peaks["bf16_tflops"], "copies": wl.copies, "path": wl.path,
               "context_torch_fp16_dense_us": dense_us,
               "context_dense_hbm_frac": dense_bytes / (dense_us * 1e-6) / 1e9 / peaks["hbm_gbs"],
               "speedup_vs_dense_fp16": dense_us / us,
               "dense_fp16_hbm_floor_us": dense_floor_us,
               "speedup_vs_dense_hbm_floor": dense_floor_us / us}
        rows.append(row)
        print(json.dumps(row), flush=True)
        del g, wl
        torch.cuda.empty_cache()
    # the transpose product dx = dy W on the same layers
    for shape, batch in [(gen.CONFIGS["attn_1b"], 1), (gen.CONFIGS["attn_1b"], 2048), (gen.CONFIGS["mlp_up"], 1),
                         (gen.CONFIGS["mlp_up"], 2048)]:
        wl = TransposedWorkload(dbf, torch, shape, batch, device)
        g = wl.capture()
        for _ in range(5):
            g.replay()
        torch.cuda.synchronize()
        reps = max(3, int(200 / max(1, wl.copies)))
        times = []
        for _ in range(7):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) / reps / wl.copies * 1e3)
        us = statistics.median(times)
        gbs = wl.bytes / (us * 1e-6) / 1e9
        tf = layer_flops(shape.n, shape.k, shape.m_in, batch) / (us * 1e-6) / 1e12
        row = {"layer": f"{shape.name} (transposed: dx = dy W)", "n": shape.n, "k": shape.k, "m_in": shape.m_in,
               "batch": batch, "us": us, "us_p10": sorted(times)[0], "us_p90": sorted(times)[-1],
               "tokens_per_s": batch / (us * 1e-6), "hbm_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"], "tflops": tf,
               "tensor_frac": tf / peaks["bf16_tflops"], "copies": wl.copies, "path": wl.path}
        rows.append(row)
        print(json.dumps(row), flush=True)
        del g, wl
        torch.cuda.empty_cache()
    # layers that share their input, as one grouped forward, against the same
    # layers run one by one (the rows above)
    by_name = {(r["layer"], r["batch"]): r["us"] for r in rows}
    for bits in (1, 2):
        set_ = {s.name.split("_")[0]: s for s in gen.LAYER_SET[bits]}
        for gname, members in GROUPS.items():
            shapes = [set_[m] for m in members]
            for batch in (1, 16):
                wl = GroupWorkload(dbf, torch, shapes, batch, device)
                g = wl.capture()
                for _ in range(5):
                    g.replay()
                torch.cuda.synchronize()
                reps = max(3, int(200 / max(1, wl.copies)))
                times = []
                for _ in range(7):
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    for _ in range(reps):
                        g.replay()
                    e1.record()
                    torch.cuda.synchronize()
                    times.append(e0.elapsed_time(e1) / reps / wl.copies * 1e3)
                us = statistics.median(times)
                sep = sum(by_name.get((s.name, batch), float("nan")) for s in shapes)
                gbs = wl.bytes / (us * 1e-6) / 1e9
                row = {"layer": f"{gname}_{bits}b (grouped)", "members": [s.name for s in shapes], "batch": batch,
                       "us": us, "us_p10": sorted(times)[0], "us_p90": sorted(times)[-1],
                       "tokens_per_s": batch / (us * 1e-6), "hbm_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
                       "tflops": wl.flops / (us * 1e-6) / 1e12, "copies": wl.copies, "path": wl.path,
                       "separate_layers_us": sep, "speedup_vs_separate": sep / us}
                rows.append(row)
                print(json.dumps(row), flush=True)
                del g, wl
                torch.cuda.empty_cache()
    with open(args.sweep, "w") as f:
        json.dump({"peaks": peaks, "rows": rows}, f, indent=1)


def run_profile_calls(args, shape, batch):
    """For ncu captures: `--profile-calls N` plain dbf_forward calls of one layer
    (no graph, no timing), with the given flags; exits non-zero on a wrong status."""
    import torch

    torch.cuda.set_device(0)
    from binary_factorized_weight_b200 import build as lib_build

    lib_build.build()
    import binary_factorized_weight_b200 as dbf

    dbf.load_library()
    L = gen.make_layer(shape, batch)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    pA, pB = dbf.dbf_pack_signs(d(L["A"])), dbf.dbf_pack_signs(d(L["B"]))
    a, mid, b, x = d(L["a"]), d(L["mid"]), d(L["b"]), d(L["x"])
    ws = dbf.dbf_new_workspace(shape.n, shape.k, shape.m_in, batch)
    y = None
    for _ in range(args.profile_calls):
        y = dbf.dbf_forward(x, pA, pB, a, mid, b, shape.n, shape.k, shape.m_in, workspace=ws, flags=args.flags)
    torch.cuda.synchronize()
    if dbf.dbf_workspace_status(ws) != 0:
        raise SystemExit("device status word set")
    print(json.dumps({"profile_calls": args.profile_calls, "workload": workload_name(shape, batch), "flags": args.flags,
                      "mean_abs_y": float(y.float().abs().mean())}))


def run_factorize(args):
    """Offline factorisation timing: one 4096 x 4096 fp32 weight (Gaussian, column
    scales falling from 2 to 0.2), k from --fact-k, the start and --fact-passes
    alternating passes of 20 ADMM steps per factor, each pass timed with CUDA
    events.  Dense products are cuBLAS SGEMM (fp32): the flops of one pass are
    counted as its GEMMs' 2*M*N*K and reported against the fp32 rate."""
    import torch

    torch.cuda.set_device(0)
    from binary_factorized_weight_b200 import build as lib_build

    lib_build.build()
    import binary_factorized_weight_b200 as dbf

    dbf.load_library()
    n = m = 4096
    k = args.fact_k
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((n, m)) * np.linspace(2.0, 0.2, m)[None, :]).astype(np.float32)
    Om = gen.projection_signs(rng, m, k)
    Wd, Omd = torch.from_numpy(W).cuda(), torch.from_numpy(Om).cuda()
    ws = torch.empty(dbf.load_library().dbf_factorize_workspace_bytes(n, m, k), dtype=torch.uint8, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dbf.dbf_factorize_start(Wd, Omd, workspace=ws)  # untimed: the first call creates the cuBLAS handle
    torch.cuda.synchronize()
    e0.record()
    L, R, err = dbf.dbf_factorize_start(Wd, Omd, workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    start_ms = e0.elapsed_time(e1)
    errors, times = [float(err.item())], []
    for _ in range(args.fact_passes):
        e0.record()
        err = dbf.dbf_factorize_pass(Wd, L, R, admm_steps=20, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
        errors.append(float(err.item()))
    steps = 20
    # GEMMs of one pass: per factor G (k*k*inner), the right-hand product (rows*k*inner), the Cholesky factor and
    # inverse (k^3 flops together), per ADMM step one (rows x k x k) product; the error product n*m*k
    fl = 2.0 * (k * k * m + n * k * m + 0.5 * k ** 3 + steps * n * k * k) + 2.0 * (k * k * n + k * m * n + 0.5 * k ** 3 +
                                                                                   steps * k * m * k) + 2.0 * n * m * k
    ms = statistics.median(times)
    print(json.dumps({"factorize": {"n": n, "m": m, "k": k, "bits_per_weight": k * (n + m) / (n * m),
                                    "start_ms": start_ms, "ms_per_pass": ms, "pass_ms": times,
                                    "gemm_tflops": fl / (ms * 1e-3) / 1e12, "relative_errors": errors}}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    layer_set = {s.name: s for bits in (1, 2) for s in gen.LAYER_SET[bits]}
    ap.add_argument("--workload", default="attn_1b", choices=sorted(gen.CONFIGS) + sorted(layer_set),
                    help="a configuration, or one layer of the decoder-layer set (e.g. k_1b)")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-check", dest="check", action="store_false")
    ap.add_argument("--no-extra", dest="extra", action="store_false",
                    help="skip the batch-2048 and batch-16 configurations timed beside the main one")
    ap.add_argument("--sweep", default=None, help="run every config and write a JSON table here")
    ap.add_argument("--profile-calls", type=int, default=0,
                    help="only run this many dbf_forward calls of one layer (for ncu captures)")
    ap.add_argument("--flags", type=int, default=1, help="dbf_forward flags for --profile-calls (default: weights static)")
    ap.add_argument("--factorize", action="store_true", help="time the offline factorisation of a 4096^2 weight")
    ap.add_argument("--fact-k", type=int, default=2048)
    ap.add_argument("--fact-passes", type=int, default=3)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    shape = gen.CONFIGS[args.workload] if args.workload in gen.CONFIGS else layer_set[args.workload]
    if args.factorize:
        run_factorize(args)
    elif args.profile_calls > 0:
        run_profile_calls(args, shape, args.batch)
    elif args.sweep:
        run_sweep(args)
    elif args.impl == "reference":
        run_reference(args, shape, args.batch)
    else:
        run_ours(args, shape, args.batch)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""SGMV benchmark: LoRA-delta tokens/s and achieved HBM bandwidth on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Default workload ("distinct"): Llama-7B-shaped decode with the Distinct
adapter distribution of the throughput benchmark on page “Punica：多 LoRA 模型统一服务框架” (the Punica
README): 32 tokens,
each on its own rank-16 adapter, H1 = H2 = 4096, fp16. One step is one decoder
layer's LoRA work: four SGMV calls (q, k, v, o projections), each with its
own adapters, input and output. Steps rotate over 32 layers, each with its own
weights and activations (1.1 GiB in all, far above the 126 MB L2), so every
step reads cold data, as a model's layers would.

Each layer's four projections share one token grouping, so a step is one
lora_sgmv_apply_batched launch. The timed region replays CUDA graphs: one
graph holding a whole rotation of layers back to back (consecutive launches
overlap through programmatic dependent launch, as a captured decode step
would), plus single-layer graphs for a remainder, so host launch latency does
not stand in for kernel time. ``e2e`` repeats the measurement through the
public calls with host buffers: each step groups the token batch on the host,
copies the segment arrays and the four projections' X and Y from pinned host
memory, runs one lora_sgmv_apply_batched launch, and reads Y back. Other
workloads (--workload) run one lora_sgmv_apply per step, the dispatcher
choosing the kernels.

Multi-GPU (torchrun): every rank runs its own replica of the workload (the
path has no cross-GPU data exchange); value = all ranks' tokens / max time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from adapter_matmul_b200 import inputs  # noqa: E402

METRIC = "LoRA-delta tokens/s (SGMV)"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024


# DRAM bytes (read + write) of one launch of the dominant kernel, from one ncu capture of the
# same launch (summaries under profiles/). A figure holds only while the kernel's sources are
# those it was taken from: their SHA-256 is stored with it and checked here, else "traffic"
# is null. (The 70B-shaped decode runs two kernels per call, the split form, and has no
# capture of both yet.)
TRAFFIC = {
    "distinct": {"bytes": 35724288 + 2048, "profile": "profiles/fused_kernel_distinct_decode.md",
                 "sources": ["sgmv_common.cuh", "sgmv_fused.cuh"],
                 "sha256": "e2d41ed385c1ba3b023529a9127f563df5317aa29af52d1bb8a4398c386b2c2b"},
    "prefill": {"bytes": 168609024 + 21820416, "profile": "profiles/grouped_kernel_prefill.md",
                "sources": ["sgmv_common.cuh", "sgmv_fused.cuh", "sgmv_tmap.cuh", "sgmv_grouped_tc.cuh"],
                "sha256": "ac9d51d05a761e2b4057b75a73f86a10c89895e1982478c529ca7b3a8ff7df66"},
}


def kernel_sources_sha(files) -> str:
    import hashlib

    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "adapter_matmul_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(name: str):
    e = TRAFFIC.get(name)
    if e is None or kernel_sources_sha(e["sources"]) != e["sha256"]:
        return None
    return e["bytes"]


NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, the vendor's figure


def make_roofline(bytes_launch: float, flops_launch: float, launch_s: float, hbm_gbs: float, bf16_tflops: float,
                  which: str, traffic, kernel_name: str) -> dict:
    """The roofline object of the JSON line: algorithmic bytes (and FLOPs) of one launch over
    its measured duration, against the measured copy peak (frac), the nominal HBM figure
    (frac_nominal) and, for the tensor pipe, the measured dense bf16 peak (tensor_frac)."""
    achieved = bytes_launch / launch_s / 1e9
    tflops = flops_launch / launch_s / 1e12
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_gbs, "unit": "GB/s",
            "frac": round(achieved / hbm_gbs, 4), "traffic": traffic, "kernel": kernel_name,
            "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)" if which == "measured" else which,
            "frac_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
            "algorithmic_bytes_per_launch": int(bytes_launch),
            "launch_us": round(launch_s * 1e6, 3),
            "tflops": round(tflops, 3),
            "tensor_frac": round(tflops / bf16_tflops, 4)}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------------------------

class Spec:
    def __init__(self, name, workload, projections, layers, desc):
        self.name, self.w, self.P, self.L, self.desc = name, workload, projections, layers, desc


def make_spec(name: str) -> Spec:
    if name == "distinct":
        w = inputs.distinct()
        return Spec(name, w, 4, 32, "Distinct decode, Llama-7B shape: H1=H2=4096, r=16, fp16, 32 tokens each on "
                                    "its own adapter; step = one layer = 4 SGMV calls (q,k,v,o)")
    w = inputs.make(name)
    per_call = w.algorithmic_bytes()
    layers = max(1, min(64, math.ceil(3 * L2_BYTES / per_call)))
    return Spec(name, w, 1, layers, f"{name}: H1={w.H1}, H2={w.H2}, r={w.r}, {w.dtype}, T={w.T}, "
                                    f"{len(w.touched_adapters())} adapters touched; step = 1 SGMV call")


VARIANT_NAMES = {1: "SPLIT", 2: "GROUPED_TC", 3: "FUSED", 4: "FUSED_TC", 5: "SPLIT_TC"}


def dispatch_name(spec: Spec, n_segments: int, max_len: int, dt: int, device):
    """The kernels of one step, as the library's dispatcher chooses them (None if unknown)."""
    try:
        import torch

        from adapter_matmul_b200 import sgmv

        w = spec.w
        if spec.P > 1:  # one batched launch: the fused kernel, on tcgen05 where the rule allows
            tc = max_len > 2 and w.r >= 32 and w.r <= 64 and w.H1 % 64 == 0 and w.H2 % 64 == 0
            return f"batched {'FUSED_TC' if tc else 'FUSED'} ({spec.P} projections per launch)"
        sms = torch.cuda.get_device_properties(device).multi_processor_count
        v = sgmv.lora_sgmv_auto_variant(w.T, n_segments, w.H1, w.r, w.H2, dt, max_len, sms)
        return VARIANT_NAMES.get(v)
    except Exception:
        return None


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest of every rank's x (the slowest replica sets a multi-GPU time)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank: int, world: int, seconds_max: float) -> float:
    """Whole-job throughput of `world` replicas: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world / seconds_max


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ---------------------------------------------------------------------------------------------
# clocks (NVML, sampled during the timed region)
# ---------------------------------------------------------------------------------------------

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
            0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            self._nv = pynvml
            pr = torch.cuda.get_device_properties(index)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            try:
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _sample(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        try:
            self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
        except Exception:
            self.reasons |= int(nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h))

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self._period)

    def __enter__(self):
        if self._nv:
            self._sample()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._nv:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self):
        if not self._nv or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for bit, n in _REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------------
# the CPU oracle as a baseline (host cores)
# ---------------------------------------------------------------------------------------------

class OracleSampler:
    """The oracle (single-threaded C, as it stands) on bounded samples of one workload.

    The host inputs (grouping, the touched adapters, X and Y) are made once; every sample
    then runs for about the time it is given: whole SGMV calls repeated when a call fits in
    half of it, else the first rows of one call in segment order (whole segments, then part
    of the next, at least one row)."""

    def __init__(self, spec: Spec):
        import oracle

        self.oracle, self.spec = oracle, spec
        w = spec.w
        self.seg, self.idx, _ = oracle.group_segments(w.ids, w.num_adapters)
        touched = set(int(i) for i in w.touched_adapters())
        zA = np.zeros((w.H1, w.r), np.uint16)  # shared by every untouched adapter
        zB = np.zeros((w.r, w.H2), np.uint16)
        self.A = [w.adapter_a(i) if i in touched else zA for i in range(w.num_adapters)]
        self.B = [w.adapter_b(i) if i in touched else zB for i in range(w.num_adapters)]
        self.X, self.Y = w.x(), w.y0()
        # seconds per token row, from up to 4 rows of the first segment
        rows = max(1, min(4, int(self.seg[1] - self.seg[0])))
        t0 = time.perf_counter()
        self._run_rows(rows)
        self.per_row = (time.perf_counter() - t0) / rows

    @staticmethod
    def first_rows(seg, idx, n: int):
        """Segment bounds and adapter ids of the first n rows (segment order) of a call: the
        segments that end at or before row n, then the part of the next one below n."""
        whole = int(np.searchsorted(seg, n, side="right")) - 1
        cut = [int(v) for v in seg[: whole + 1]]
        if cut[-1] < n:
            cut.append(n)
        return np.array(cut, np.int32), np.asarray(idx[: len(cut) - 1], np.int32)

    def _run_rows(self, n: int) -> None:
        """The first n rows (segment order) of one call."""
        sub_seg, sub_idx = self.first_rows(self.seg, self.idx, n)
        w = self.spec.w
        self.oracle.apply_f32(self.Y[:n], self.X[:n], self.A, self.B, sub_seg, sub_idx, w.scale, w.dtype)

    def sample(self, seconds: float) -> dict:
        w = self.spec.w
        t_start = time.perf_counter()
        if self.per_row * w.T <= seconds / 2:
            what = f"whole SGMV calls of the workload ({w.T} tokens each), repeated for ~{seconds:.3g} s"
            calls, tokens = 0, 0
            while calls == 0 or time.perf_counter() - t_start < seconds:
                self.oracle.apply_f32(self.Y, self.X, self.A, self.B, self.seg, self.idx, w.scale, w.dtype)
                calls += 1
                tokens += w.T
        else:
            n = max(1, min(w.T, int(seconds / self.per_row)))
            what = f"first {n} of {w.T} token rows of one call (segment order)"
            self._run_rows(n)
            calls, tokens = 1, n
        elapsed = time.perf_counter() - t_start
        # tokens/s of whole steps: a step holds spec.P calls over the same T tokens
        return {"value": tokens / self.spec.P / elapsed, "unit": UNIT, "cores": 1, "kind": "oracle",
                "sample": what, "seconds": round(elapsed, 6), "calls": calls}


def oracle_baseline(spec: Spec, seconds: float):
    """Time the oracle (single-threaded C, as it stands) on a bounded sample of the workload."""
    return OracleSampler(spec).sample(seconds)


def rows_share(seg, idx, a: int, b: int):
    """Segment bounds (relative to row a) and adapter ids of rows [a, b) of a call."""
    seg = np.asarray(seg, np.int64)
    cut, ids = [0], []
    for s in range(len(seg) - 1):
        lo, hi = max(int(seg[s]), a), min(int(seg[s + 1]), b)
        if lo < hi:
            cut.append(hi - a)
            ids.append(int(idx[s]))
    return np.array(cut, np.int32), np.array(ids, np.int32)


def _all_cores_worker(name: str, a: int, b: int, seconds: float, barrier, queue) -> None:
    """One process of the all-cores baseline: the oracle on rows [a, b) of one call."""
    try:
        import oracle

        w = make_spec(name).w
        seg, idx, _ = oracle.group_segments(w.ids, w.num_adapters)
        sub_seg, sub_idx = rows_share(seg, idx, a, b)
        need = set(int(i) for i in sub_idx)
        zA, zB = np.zeros((w.H1, w.r), np.uint16), np.zeros((w.r, w.H2), np.uint16)
        A = [w.adapter_a(i) if i in need else zA for i in range(w.num_adapters)]
        B = [w.adapter_b(i) if i in need else zB for i in range(w.num_adapters)]
        X, Y = w.x()[a:b], w.y0()[a:b]
        n = b - a
        t0 = time.perf_counter()
        probe = min(n, 4)
        ps, pi = rows_share(sub_seg, sub_idx, 0, probe)
        oracle.apply_f32(Y[:probe], X[:probe], A, B, ps, pi, w.scale, w.dtype)
        per_row = (time.perf_counter() - t0) / probe
        barrier.wait(timeout=120)
        t_start = time.perf_counter()
        tokens = 0
        if per_row * n <= seconds / 2:
            while tokens == 0 or time.perf_counter() - t_start < seconds:
                oracle.apply_f32(Y, X, A, B, sub_seg, sub_idx, w.scale, w.dtype)
                tokens += n
        else:
            m = max(1, min(n, int(seconds / per_row)))
            ps, pi = rows_share(sub_seg, sub_idx, 0, m)
            oracle.apply_f32(Y[:m], X[:m], A, B, ps, pi, w.scale, w.dtype)
            tokens = m
        queue.put((tokens, time.perf_counter() - t_start, None))
    except Exception as e:  # reported by the parent; the run goes on without this figure
        queue.put((0, 0.0, f"{type(e).__name__}: {e}"))


def oracle_all_cores(spec: Spec, seconds: float, max_procs: int = 64) -> dict:
    """The same oracle, unchanged, on every host core: one process per core, each on its own
    contiguous share of one call's rows (with only the adapters its rows use), started
    together; throughput = all processes' tokens over the slowest one's time. Processes are
    spawned (never forked: the parent may hold a CUDA context). On any failure the figure is
    replaced by the reason and the run goes on."""
    import multiprocessing as mp

    try:
        cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
        w = spec.w
        procs_n = max(1, min(cores, max_procs, w.T))
        bounds = [round(k * w.T / procs_n) for k in range(procs_n + 1)]
        ctx = mp.get_context("spawn")
        barrier = ctx.Barrier(procs_n)
        queue = ctx.Queue()
        procs = [ctx.Process(target=_all_cores_worker,
                             args=(spec.name, bounds[k], bounds[k + 1], seconds, barrier, queue), daemon=True)
                 for k in range(procs_n)]
        for p in procs:
            p.start()
        results = [queue.get(timeout=180 + 4 * seconds) for _ in procs]
        for p in procs:
            p.join(timeout=30)
        errors = [e for _, _, e in results if e]
        if errors:
            return {"unavailable": errors[0]}
        tokens = sum(t for t, _, _ in results)
        slowest = max(el for _, el, _ in results)
        return {"value": round(tokens / spec.P / slowest, 3), "unit": UNIT, "cores": procs_n, "kind": "oracle",
                "sample": f"{procs_n} processes of the single-threaded oracle, each on its own share of the "
                          f"rows of one call (about {w.T // procs_n} rows each), run for ~{seconds:.3g} s or "
                          f"its first rows"}
    except Exception as e:
        return {"unavailable": f"{type(e).__name__}: {e}"}


# ---------------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------------

def run_ours(args, spec: Spec, rank: int, world: int, local: int):
    import torch
    import torch.distributed as dist

    from adapter_matmul_b200 import sgmv

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    w = spec.w
    dt = sgmv.F16 if w.dtype == "f16" else sgmv.BF16
    tdt = torch.float16 if w.dtype == "f16" else torch.bfloat16
    seg, idx, _ = sgmv.lora_sgmv_group_segments(w.ids, w.num_adapters)
    n = len(idx)
    max_len = int(np.max(np.diff(seg)))
    touched = w.touched_adapters()

    def dev_bits(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(tdt).to(dev)

    # per (layer, projection): adapters (pool), X, Y; adapters drawn from the seeded generator
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234 + rank)
    calls = []
    keep = []
    for l in range(spec.L):
        for p in range(spec.P):
            proj = l * spec.P + p
            A_pool = torch.empty((w.num_adapters, w.H1, w.r), dtype=tdt, device=dev)
            B_pool = torch.empty((w.num_adapters, w.r, w.H2), dtype=tdt, device=dev)
            if len(touched) < w.num_adapters:  # resident but unused by this batch
                A_pool.normal_(0.0, 1.0 / math.sqrt(w.H1), generator=gen)
                B_pool.normal_(0.0, 1.0 / math.sqrt(w.r), generator=gen)
            for i in touched:
                A_pool[i] = dev_bits(w.adapter_a(i, proj))
                B_pool[i] = dev_bits(w.adapter_b(i, proj))
            A_ptrs = torch.tensor([A_pool[i].data_ptr() for i in range(w.num_adapters)], dtype=torch.int64, device=dev)
            B_ptrs = torch.tensor([B_pool[i].data_ptr() for i in range(w.num_adapters)], dtype=torch.int64, device=dev)
            X = dev_bits(w.x(proj))
            Y = torch.zeros((w.T, w.H2), dtype=tdt, device=dev)
            keep += [A_pool, B_pool]
            calls.append((l, p, X, Y, A_ptrs, B_ptrs))
    d_seg = torch.from_numpy(seg).to(dev)
    d_idx = torch.from_numpy(idx).to(dev)
    ws_bytes = sgmv.lora_sgmv_workspace_bytes(w.T, w.r)
    ws = torch.empty(ws_bytes // 4, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    stream = torch.cuda.Stream(device=dev)
    sh = stream.cuda_stream

    # one launch per step: the layer's projections share the token grouping
    batched = {}
    for l in range(spec.L):
        batched[l] = [sgmv.Problem(Y.data_ptr(), X.data_ptr(), A_ptrs.data_ptr(), B_ptrs.data_ptr(),
                                   w.num_adapters, w.H1, w.H2, w.scale)
                      for (ll, p, X, Y, A_ptrs, B_ptrs) in calls[l * spec.P:(l + 1) * spec.P]]

    def enqueue_layer(l):
        if spec.P > 1:
            sgmv.lora_sgmv_apply_batched(batched[l], d_seg, d_idx, n, w.T, w.r, dt, max_len, status, sh)
            return
        for (ll, p, X, Y, A_ptrs, B_ptrs) in calls[l * spec.P:(l + 1) * spec.P]:
            sgmv.lora_sgmv_apply(Y, X, A_ptrs, B_ptrs, d_seg, d_idx, n, w.num_adapters, w.T, w.H1, w.r, w.H2,
                                 w.scale, dt, max_len, ws, ws_bytes, status, sh)

    # one CUDA graph per layer
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for l in range(spec.L):  # eager warm-up (attributes, first-touch)
            enqueue_layer(l)
    stream.synchronize()
    # one graph per layer, and one graph holding a whole rotation of layers back to back
    # (as a decode step's forward pass would be captured): consecutive kernels in that graph
    # overlap through programmatic dependent launch
    graphs = []
    for l in range(spec.L):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            enqueue_layer(l)
        graphs.append(g)
    rotation = torch.cuda.CUDAGraph()
    with torch.cuda.graph(rotation, stream=stream):
        for l in range(spec.L):
            enqueue_layer(l)

    def run_steps(k):
        full, rest = divmod(k, spec.L)
        for _ in range(full):
            rotation.replay()
        for i in range(rest):
            graphs[i].replay()

    launches_per_step = None
    with torch.cuda.stream(stream):
        run_steps(args.warmup)
    stream.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- timed region: K steps ----
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            run_steps(args.steps)
            ev1.record(stream)
        stream.synchronize()
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    ms_per_step = ms / args.steps

    # kernels per step: count the launches of one eager layer
    c0 = sgmv.lora_sgmv_launch_count()
    with torch.cuda.stream(stream):
        enqueue_layer(0)
    stream.synchronize()
    launches_per_step = sgmv.lora_sgmv_launch_count() - c0
    gpu_launches = launches_per_step * args.steps

    st = int(status.item())
    if st != 0:
        raise RuntimeError(f"device status {st:#x}: a segment was rejected")

    # ---- roofline of the dominant kernel, per launch ----
    # One launch per call: that kernel. Several launches per call (the split forms: a shrink
    # kernel, then an expand kernel): the whole call, its algorithmic bytes over its duration.
    hbm, tc, which = peaks()
    bytes_call = w.algorithmic_bytes()
    if launches_per_step > spec.P:
        bytes_launch = bytes_call
        launch_s = ms_per_step / 1e3 / spec.P
        kernel_name = ("lora_sgmv_apply, dispatcher's choice: %d launches per call, roofline over the whole call"
                       % (launches_per_step // spec.P))
    else:
        bytes_launch = bytes_call * spec.P // launches_per_step
        launch_s = ms_per_step / 1e3 / launches_per_step
        kernel_name = ("sgmv_fused_kernel (lora_sgmv_apply_batched: %d projections per launch)" % spec.P
                       if spec.P > 1 else "lora_sgmv_apply kernels (dispatcher's choice)")
    roofline = make_roofline(bytes_launch, w.flops() * bytes_launch / bytes_call, launch_s, hbm, tc, which,
                             measured_traffic(spec.name), kernel_name)

    # ---- e2e through the public call with host buffers ----
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, spec, torch, sgmv, dev, stream, calls, dt, tdt, world)

    result = None
    if rank == 0:
        value = job_tokens_per_s(w.T * args.steps, world, ms / 1e3)
        result = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": spec.desc, "name": spec.name, "T": w.T, "H1": w.H1, "H2": w.H2, "r": w.r,
                       "adapters_touched": len(touched), "segments": n, "sgmv_calls_per_step": spec.P,
                       "dispatch": dispatch_name(spec, n, max_len, dt, dev),
                       "layers_rotated": spec.L,
                       "l2": f"inputs larger than L2: {spec.L} layers rotated, "
                             f"{spec.L * spec.P * bytes_call / 2**30:.2f} GiB of algorithmic bytes per rotation",
                       "timing": "CUDA events on the launching stream; K layer steps replayed as CUDA graphs "
                                 "of whole layer rotations (plus single-layer graphs for the remainder)",
                       "parallelism": f"replicas x{world}"},
            "roofline": roofline,
            "gpu_launches": int(gpu_launches),
            "clocks": clocks.summary(),
        }
        if e2e:
            result["e2e"] = e2e
    if world > 1:
        dist.barrier()
        del graphs, rotation
        dist.destroy_process_group()
    return result


def run_e2e(args, spec, torch, sgmv, dev, stream, calls, dt, tdt, world=1):
    """Same metric through the public calls with host buffers: lora_sgmv_group_segments on the
    host, then one lora_sgmv_apply_batched launch for the step's projections (lora_sgmv_apply
    for one projection). Per step the segment arrays, X and Y of every projection go host ->
    device (one pinned copy each, the projections packed), and the step's Y comes back."""
    w = spec.w
    P = spec.P
    steps = max(3, min(args.steps, 200))
    hX = torch.empty((P, w.T, w.H1), dtype=tdt, pin_memory=True)
    hY = torch.empty((P, w.T, w.H2), dtype=tdt, pin_memory=True)
    for p in range(P):
        hX[p].copy_(calls[p][2].cpu())
        hY[p].copy_(calls[p][3].cpu())
    outY = torch.empty((P, w.T, w.H2), dtype=tdt, pin_memory=True)
    ids = np.ascontiguousarray(w.ids, dtype=np.int32)
    meta_len = 2 * w.num_adapters + 1
    h_meta = torch.empty(meta_len, dtype=torch.int32, pin_memory=True)  # seg_starts, then lora_idx
    h_meta_np = h_meta.numpy()
    d_meta = torch.empty(meta_len, dtype=torch.int32, device=dev)
    dX = torch.empty((P, w.T, w.H1), dtype=tdt, device=dev)
    dY = torch.empty((P, w.T, w.H2), dtype=tdt, device=dev)
    ws_bytes = sgmv.lora_sgmv_workspace_bytes(w.T, w.r)
    ws = torch.empty(ws_bytes // 4, dtype=torch.float32, device=dev)
    problems = [[sgmv.Problem(dY[p].data_ptr(), dX[p].data_ptr(), calls[l * P + p][4].data_ptr(),
                              calls[l * P + p][5].data_ptr(), w.num_adapters, w.H1, w.H2, w.scale)
                 for p in range(P)] for l in range(spec.L)]
    sh = stream.cuda_stream
    h2d = d2h = 0

    def one(i):
        nonlocal h2d, d2h
        l = i % spec.L
        seg, idx, _ = sgmv.lora_sgmv_group_segments(ids, w.num_adapters)
        n = len(idx)
        h_meta_np[: n + 1] = seg
        h_meta_np[n + 1: 2 * n + 1] = idx
        max_len = int(np.max(np.diff(seg)))
        d_seg, d_idx = d_meta.data_ptr(), d_meta.data_ptr() + 4 * (n + 1)
        with torch.cuda.stream(stream):
            d_meta[: 2 * n + 1].copy_(h_meta[: 2 * n + 1], non_blocking=True)
            dX.copy_(hX, non_blocking=True)
            dY.copy_(hY, non_blocking=True)
            if P > 1:
                sgmv.lora_sgmv_apply_batched(problems[l], d_seg, d_idx, n, w.T, w.r, dt, max_len, None, sh)
            else:
                q = problems[l][0]
                sgmv.lora_sgmv_apply(q.Y, q.X, q.A_ptrs, q.B_ptrs, d_seg, d_idx, n, w.num_adapters, w.T, w.H1, w.r,
                                     w.H2, w.scale, dt, max_len, ws, ws_bytes, None, sh)
            outY.copy_(dY, non_blocking=True)
        stream.synchronize()
        h2d = (2 * n + 1) * 4 + hX.numel() * 2 + hY.numel() * 2
        d2h = outY.numel() * 2

    for i in range(3):
        one(i)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    t0 = time.perf_counter()
    for i in range(steps):
        one(i)
    el = max_over_ranks(time.perf_counter() - t0, world, dev)
    call = "1 lora_sgmv_apply_batched launch" if P > 1 else "1 lora_sgmv_apply call"
    return {"value": round(job_tokens_per_s(w.T * steps, world, el), 1), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "note": "host wall clock (the host's grouping is part of the step), slowest rank; per step: host "
                    f"grouping, pinned H2D of the segment arrays and of X and Y ({P} projections), {call}, "
                    "D2H of Y, stream sync"}


# ---------------------------------------------------------------------------------------------
# reference arm: the oracle on the host cores
# ---------------------------------------------------------------------------------------------

REFERENCE_BUDGET_S = 120.0


def run_reference(args, spec: Spec, rank: int):
    if rank != 0:
        return None
    # the timed steps share a budget of about two minutes of oracle time (at most 10 s a
    # step); warm-up steps get a quarter of a step's share each
    sampler = OracleSampler(spec)
    per_step = min(10.0, REFERENCE_BUDGET_S / max(1, args.steps))
    for _ in range(args.warmup):
        sampler.sample(per_step / 4)
    t0 = time.perf_counter()
    runs = [sampler.sample(per_step) for _ in range(args.steps)]
    el = time.perf_counter() - t0
    value = statistics.median(r["value"] for r in runs)
    return {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": 0, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(el * 1e3 / max(1, args.steps), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": spec.w.dtype, "data": "synthetic",
        "config": {"workload": spec.desc, "name": spec.name, "T": spec.w.T},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": runs[0]["sample"]},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="distinct", choices=["distinct"] + list(inputs.CONFIGS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_env()
    spec = make_spec(args.workload)
    if args.impl == "reference":
        out = run_reference(args, spec, rank)
        if out:
            print(json.dumps(out), flush=True)
        return
    result = run_ours(args, spec, rank, world, local)
    if rank == 0 and result is not None:
        if world == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = oracle_baseline(spec, args.cpu_seconds)
            result["cpu_baseline"]["all_cores"] = oracle_all_cores(spec, args.cpu_seconds)
        print(json.dumps(result), flush=True)


if __name__ == "__main__":
    main()

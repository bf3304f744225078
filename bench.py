#!/usr/bin/env python
"""SGMV benchmark: LoRA-delta tokens/s and achieved HBM bandwidth on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
                    [--no-per-config] [--no-e2e] [--no-cpu-baseline]

Default workload ("distinct"): Llama-7B-shaped decode with the Distinct adapter
distribution of the throughput benchmark on page "Punica：多 LoRA 模型统一服务框架" (the
Punica README): 32 tokens, each on its own rank-16 adapter, H1 = H2 = 4096, fp16. One step
is one decoder layer's LoRA work: four SGMV problems (q, k, v, o projections), each with
its own adapters, input and output, sharing one token grouping, run as one
lora_sgmv_apply_batched launch. Steps rotate over layers that each have their own weights
and activations (far above the 126 MB L2), so every step reads cold data, as a model's
layers would.

Timing. The K timed steps are one CUDA graph of exactly K launches (layer i mod L at step
i), replayed once untimed and then once between CUDA events on the launching stream; so
the timed work does not depend on K beyond its length. Consecutive launches are chained
by programmatic dependent launch with the library's default contract: a launch's prologue
(barriers, tensor memory, tensor-map tables) overlaps the end of the previous launch, and
it reads nothing of its inputs (segments, tables, adapters, X, Y) before the previous
launch has completed. The line also carries ("early_reads") the same K steps with
LORA_SGMV_FLAG_EARLY_READS, under which each launch streams its adapter weights while the
previous one finishes; the statement that flag makes holds here (segments and adapters
are written by copies before the timed region).

"per_config" times every configuration the same way (the Distinct, Uniform, Skewed and
Identical decode batches per layer of four projections and per single call, the prefill
and the 70B-shaped decode per call), each with its dispatched kernels, algorithmic bytes
and roofline fraction.

"e2e" is the same metric through the public calls with host buffers: each step is one
lora_sgmv_step_host call, which groups the token batch on the host, copies the segment arrays
and the projections' X and Y from pinned host memory, runs the batched SGMV launch and copies Y
back, after which the host reads Y; three buffer sets on their own streams, so that one step's
copies overlap the previous steps'. Timed by the host clock. (A workload of one projection runs
lora_sgmv_apply between the copies instead.)

Multi-GPU (torchrun): every rank runs its own replica of the workload (the path has no
cross-GPU data exchange); value = all ranks' tokens / max time.
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
PER_CONFIG_MAX_STEPS = 500


# DRAM bytes (read + write) of one launch of the dominant kernel, from one ncu capture of the
# same launch (summaries under profiles/). A figure holds only while the sources it was taken
# from (the kernel's headers, those they include, and the host code that sizes its launch) are
# unchanged: their SHA-256 is stored with it and checked here, else "traffic" is null. For a
# call of two launches (the split forms) the figure is the pair's.
TRAFFIC = {
    # profiles/fused_kernel_distinct_decode.md
    "distinct": {"bytes": 35726848,
        "sources": ["sgmv_fused.cuh", "sgmv_common.cuh", "lora_sgmv_api.cu"],
        "sha256": "b72ac89a6d8e011e06deab07c3c133bad172c3055a215e88d318d91293dce9c0"},
    # profiles/split_tc_llama70b_decode_h28672.md
    "llama70b_decode_h28672": {"bytes": 488989184,
        "sources": ["sgmv_split.cuh", "sgmv_decode_tc.cuh", "sgmv_grouped_tc.cuh", "sgmv_fused.cuh", "sgmv_tmap.cuh", "sgmv_common.cuh", "lora_sgmv_api.cu"],
        "sha256": "6c0a82bc2a9540a24c4be59f5852d5ae96e1792dcbe4fbe4f346567ffe7a9df2"},
    # profiles/split_tc_llama70b_decode_h8192.md
    "llama70b_decode_h8192": {"bytes": 217230080,
        "sources": ["sgmv_split.cuh", "sgmv_decode_tc.cuh", "sgmv_grouped_tc.cuh", "sgmv_fused.cuh", "sgmv_tmap.cuh", "sgmv_common.cuh", "lora_sgmv_api.cu"],
        "sha256": "6c0a82bc2a9540a24c4be59f5852d5ae96e1792dcbe4fbe4f346567ffe7a9df2"},
    # profiles/grouped_kernel_prefill.md
    "prefill": {"bytes": 190149120,
        "sources": ["sgmv_grouped_tc.cuh", "sgmv_fused.cuh", "sgmv_tmap.cuh", "sgmv_common.cuh", "lora_sgmv_api.cu"],
        "sha256": "9b9f31895d43aa41ef27ad13e9b2807746ff134a60d6af1d99cd1eef4554db6c"},
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


LAYER_CONFIGS = ("distinct", "uniform_h4096", "uniform_h11008", "skewed_h4096", "skewed_h11008",
                 "identical_h4096", "identical_h11008")


def workload_names():
    """--workload values: a configuration name (a layer of four projections for the decode
    batches, one call otherwise), or a decode batch name with ':call' (one SGMV call)."""
    return list(inputs.CONFIGS) + [n + ":call" for n in LAYER_CONFIGS]


def make_spec(name: str) -> Spec:
    base, _, mode = name.partition(":")
    w = inputs.make(base)
    P = 4 if (base in LAYER_CONFIGS and mode != "call") else 1
    per_step = w.algorithmic_bytes() * P
    layers = max(1, min(64, math.ceil(3 * L2_BYTES / per_step)))
    U = len(w.touched_adapters())
    shape = f"H1={w.H1}, H2={w.H2}, r={w.r}, {w.dtype}, T={w.T}, {U} adapters touched"
    if base == "distinct" and P == 4:
        desc = ("Distinct decode, Llama-7B shape: H1=H2=4096, r=16, fp16, 32 tokens each on its own adapter; "
                "step = one layer = 4 SGMV calls (q,k,v,o) in one launch")
    elif P == 4:
        desc = f"{base}: {shape}; step = one layer = 4 SGMV problems of this shape in one launch"
    else:
        desc = f"{base}: {shape}; step = 1 SGMV call"
    return Spec(name, w, P, layers, desc)


def config_dict(spec: Spec, world: int) -> dict:
    """The line's `config`: the workload alone (the same in both arms)."""
    w = spec.w
    return {"workload": spec.desc, "name": spec.name, "T": w.T, "H1": w.H1, "H2": w.H2, "r": w.r,
            "adapters_touched": len(w.touched_adapters()), "sgmv_calls_per_step": spec.P,
            "parallelism": f"replicas x{world}"}


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

class DeviceSpec:
    """One workload on the device: L layers x P projections, each with its own resident adapter
    pool (every adapter of the pool drawn on the device: A ~ N(0, 1/H1), B ~ N(0, 1/r)), its
    own X ~ N(0, 1) and Y = 0, and pointer tables; the grouping of the token batch (host
    lora_sgmv_group_segments) is shared by all."""

    def __init__(self, spec: Spec, dev, seed: int):
        import torch

        from adapter_matmul_b200 import sgmv

        self.spec, self.sgmv = spec, sgmv
        w = spec.w
        self.dt = sgmv.F16 if w.dtype == "f16" else sgmv.BF16
        self.tdt = torch.float16 if w.dtype == "f16" else torch.bfloat16
        self.seg, self.idx, _ = sgmv.lora_sgmv_group_segments(w.ids, w.num_adapters)
        self.n = len(self.idx)
        self.max_len = int(np.max(np.diff(self.seg)))
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed)
        self.calls, self.keep = [], []
        a_bytes, b_bytes = w.H1 * w.r * 2, w.r * w.H2 * 2
        for _ in range(spec.L):
            layer = []
            for _ in range(spec.P):
                A = torch.empty((w.num_adapters, w.H1, w.r), dtype=self.tdt, device=dev)
                A.normal_(0.0, 1.0 / math.sqrt(w.H1), generator=gen)
                B = torch.empty((w.num_adapters, w.r, w.H2), dtype=self.tdt, device=dev)
                B.normal_(0.0, 1.0 / math.sqrt(w.r), generator=gen)
                ids = torch.arange(w.num_adapters, dtype=torch.int64, device=dev)
                A_ptrs = ids * a_bytes + A.data_ptr()
                B_ptrs = ids * b_bytes + B.data_ptr()
                X = torch.empty((w.T, w.H1), dtype=self.tdt, device=dev).normal_(generator=gen)
                Y = torch.zeros((w.T, w.H2), dtype=self.tdt, device=dev)
                layer.append((X, Y, A_ptrs, B_ptrs))
                self.keep += [A, B]
            self.calls.append(layer)
        self.d_seg = torch.from_numpy(self.seg).to(dev)
        self.d_idx = torch.from_numpy(self.idx).to(dev)
        self.ws_bytes = sgmv.lora_sgmv_workspace_bytes(w.T, w.r)
        self.ws = torch.empty(self.ws_bytes // 4 + 64, dtype=torch.float32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.problems = [[sgmv.Problem(Y.data_ptr(), X.data_ptr(), Ap.data_ptr(), Bp.data_ptr(), w.num_adapters,
                                       w.H1, w.H2, w.scale) for (X, Y, Ap, Bp) in layer] for layer in self.calls]

    def enqueue(self, l: int, flags: int, sh) -> None:
        """Step l: one batched launch of the layer's projections, or one lora_sgmv_apply call."""
        sgmv, w = self.sgmv, self.spec.w
        if self.spec.P > 1:
            sgmv.lora_sgmv_apply_batched_flags(self.problems[l], self.d_seg, self.d_idx, self.n, w.T, w.r, self.dt,
                                               self.max_len, flags, self.status, sh)
            return
        X, Y, A_ptrs, B_ptrs = self.calls[l][0]
        sgmv.lora_sgmv_apply_flags(Y, X, A_ptrs, B_ptrs, self.d_seg, self.d_idx, self.n, w.num_adapters, w.T, w.H1,
                                   w.r, w.H2, w.scale, self.dt, self.max_len, self.ws, self.ws_bytes, self.status,
                                   sgmv.VARIANT_AUTO, flags, sh)


def time_steps(ds: DeviceSpec, steps: int, flags: int, stream, world: int, dev, clocks=None) -> float:
    """Milliseconds of `steps` steps captured as one CUDA graph (step i runs layer i mod L),
    replayed once untimed, then once between CUDA events on the launching stream, with a
    barrier and a device synchronize on both sides; the slowest rank's time."""
    import torch
    import torch.distributed as dist

    sh = stream.cuda_stream
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            ds.enqueue(i % ds.spec.L, flags, sh)
    with torch.cuda.stream(stream):  # a graph replays on the current stream
        g.replay()
    stream.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if clocks is not None:
        clocks.__enter__()
    with torch.cuda.stream(stream):
        ev0.record(stream)
        g.replay()
        ev1.record(stream)
    stream.synchronize()
    if clocks is not None:
        clocks.__exit__(None, None, None)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    del g
    return max_over_ranks(ms, world, dev)


def launches_per_step(ds: DeviceSpec, stream) -> int:
    before = ds.sgmv.lora_sgmv_launch_count()
    ds.enqueue(0, 0, stream.cuda_stream)
    stream.synchronize()
    return int(ds.sgmv.lora_sgmv_launch_count() - before)


def measure(spec: Spec, args, steps: int, stream, world: int, dev, rank: int, clocks=None):
    """Times one workload: default flags (the headline form) and with early reads."""
    from adapter_matmul_b200 import sgmv

    ds = DeviceSpec(spec, dev, 1234 + rank)
    sh = stream.cuda_stream
    for l in range(spec.L):  # eager pass: kernel attributes, first touch
        ds.enqueue(l, 0, sh)
    for i in range(args.warmup):
        ds.enqueue(i % spec.L, 0, sh)
    stream.synchronize()
    lps = launches_per_step(ds, stream)
    ms = time_steps(ds, steps, 0, stream, world, dev, clocks)
    ms_early = time_steps(ds, steps, sgmv.FLAG_EARLY_READS, stream, world, dev)
    st = int(ds.status.item())
    if st != 0:
        raise RuntimeError(f"{spec.name}: device status {st:#x}")
    return ds, ms, ms_early, lps


def summarize(spec: Spec, ds: DeviceSpec, ms: float, ms_early: float, lps: int, steps: int, dev) -> dict:
    """One per_config entry: the step's time, throughput and roofline (algorithmic bytes over
    the step's time: a step is one launch, or one call of two launches for the split forms)."""
    hbm, tc, _ = peaks()
    w = spec.w
    bytes_step = w.algorithmic_bytes() * spec.P
    s = ms / 1e3 / steps
    se = ms_early / 1e3 / steps
    return {"name": spec.name, "workload": spec.desc,
            "dispatch": dispatch_name(spec, ds.n, ds.max_len, ds.dt, dev),
            "T": w.T, "adapters_touched": len(w.touched_adapters()), "calls_per_step": spec.P,
            "launches_per_step": lps, "steps": steps, "layers_rotated": spec.L,
            "us_per_step": round(s * 1e6, 3), "tokens_per_s": round(w.T / s, 1),
            "algorithmic_bytes_per_step": int(bytes_step), "gbs": round(bytes_step / s / 1e9, 1),
            "frac": round(bytes_step / s / 1e9 / hbm, 4),
            "tflops": round(w.flops() * spec.P / s / 1e12, 3),
            "tensor_frac": round(w.flops() * spec.P / s / 1e12 / tc, 4),
            "early_reads": {"us_per_step": round(se * 1e6, 3),
                            "frac": round(bytes_step / se / 1e9 / hbm, 4)},
            "traffic_per_step": measured_traffic(spec.name)}


def measure_layer(args, steps: int, stream, world: int, dev, rank: int) -> dict:
    """The whole layer at the prefill shape, Y = X@W + scale*(X@A_i)@B_i, through
    lora_sgmv_gemm_apply (the grouped kernel's shrink into the workspace, then the tcgen05 base
    product with the delta as extra K-steps; Y written once), timed like the other entries
    (two layers rotated: 2 x 200 MB). Beside it: the same layer unfused (torch.matmul for X@W,
    i.e. cuBLAS, then lora_sgmv_apply adding the delta onto Y), the base product alone through
    lora_sgmv_gemm_apply without segments, and torch.matmul alone."""
    import torch
    import torch.distributed as dist

    from adapter_matmul_b200 import sgmv

    w = inputs.make("prefill")
    L = 2
    gen = torch.Generator(device=dev)
    gen.manual_seed(4321 + rank)
    seg, idx, _ = sgmv.lora_sgmv_group_segments(w.ids, w.num_adapters)
    n, max_len = len(idx), int(np.max(np.diff(seg)))
    d_seg, d_idx = torch.from_numpy(seg).to(dev), torch.from_numpy(idx).to(dev)
    layers = []
    for _ in range(L):
        X = torch.empty((w.T, w.H1), dtype=torch.bfloat16, device=dev).normal_(generator=gen)
        W = torch.empty((w.H1, w.H2), dtype=torch.bfloat16, device=dev).normal_(0, 1 / math.sqrt(w.H1), generator=gen)
        A = torch.empty((w.num_adapters, w.H1, w.r), dtype=torch.bfloat16, device=dev)
        A.normal_(0, 1 / math.sqrt(w.H1), generator=gen)
        B = torch.empty((w.num_adapters, w.r, w.H2), dtype=torch.bfloat16, device=dev)
        B.normal_(0, 1 / math.sqrt(w.r), generator=gen)
        ids = torch.arange(w.num_adapters, dtype=torch.int64, device=dev)
        Ap, Bp = ids * (w.H1 * w.r * 2) + A.data_ptr(), ids * (w.r * w.H2 * 2) + B.data_ptr()
        Y = torch.empty((w.T, w.H2), dtype=torch.bfloat16, device=dev)
        layers.append((X, W, A, B, Ap, Bp, Y))
    ws_bytes = sgmv.lora_sgmv_workspace_bytes(w.T, w.r)
    ws = torch.empty(ws_bytes // 4 + 64, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    sh = stream.cuda_stream

    def fused(i):
        X, W, _, _, Ap, Bp, Y = layers[i % L]
        sgmv.lora_sgmv_gemm_apply(Y, X, W, Ap, Bp, d_seg, d_idx, n, w.num_adapters, w.T, w.H1, w.r, w.H2, w.scale,
                                  sgmv.BF16, max_len, ws, ws_bytes, status, sh)

    def base_only(i):
        X, W, _, _, Ap, Bp, Y = layers[i % L]
        sgmv.lora_sgmv_gemm_apply(Y, X, W, None, None, None, None, 0, w.num_adapters, w.T, w.H1, w.r, w.H2, w.scale,
                                  sgmv.BF16, 0, None, 0, status, sh)

    def unfused(i):
        X, W, _, _, Ap, Bp, Y = layers[i % L]
        torch.matmul(X, W, out=Y)
        sgmv.lora_sgmv_apply(Y, X, Ap, Bp, d_seg, d_idx, n, w.num_adapters, w.T, w.H1, w.r, w.H2, w.scale, sgmv.BF16,
                             max_len, ws, ws_bytes, status, sh)

    def cublas(i):
        X, W, _, _, _, _, Y = layers[i % L]
        torch.matmul(X, W, out=Y)

    def timed(fn):
        with torch.cuda.stream(stream):
            for i in range(max(3, args.warmup)):
                fn(i)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(steps):
                fn(i)
        with torch.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        stream.synchronize()
        del g
        return max_over_ranks(e0.elapsed_time(e1), world, dev) * 1e3 / steps  # us per step

    t_fused = timed(fused)
    if int(status.item()) != 0:
        raise RuntimeError(f"prefill layer: device status {int(status.item()):#x}")
    t_base, t_unfused, t_cublas = timed(base_only), timed(unfused), timed(cublas)
    hbm, tc, _ = peaks()
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            tc_sus = float(json.load(f)["bf16_tflops_sustained"])
    except Exception:
        tc_sus = 1400.0
    base_fl = 2.0 * w.T * w.H1 * w.H2
    fl = base_fl + w.flops()
    return {"name": "prefill_layer",
            "workload": f"Y = X@W + scale*(X@A_i)@B_i at the prefill shape: T={w.T}, H1={w.H1}, H2={w.H2}, "
                        f"r={w.r}, bf16, {w.num_adapters} segments; step = 1 lora_sgmv_gemm_apply call",
            "dispatch": "grouped tcgen05 shrink (V to the workspace), then sgmv_gemm_delta_kernel",
            "T": w.T, "steps": steps, "layers_rotated": L,
            "us_per_step": round(t_fused, 3), "tokens_per_s": round(w.T / t_fused * 1e6, 1),
            "tflops": round(fl / t_fused / 1e6, 2), "bound": "tensor",
            "tensor_frac": round(fl / t_fused / 1e6 / tc, 4),
            "tensor_frac_sustained": round(fl / t_fused / 1e6 / tc_sus, 4),
            "peaks_tflops": {"burst": tc, "sustained": tc_sus},
            "base_only_us": round(t_base, 3), "base_only_tflops": round(base_fl / t_base / 1e6, 2),
            "unfused_us": round(t_unfused, 3),
            "unfused": "torch.matmul (cuBLAS) for X@W, then lora_sgmv_apply (grouped) adding the delta onto Y",
            "cublas_us": round(t_cublas, 3), "cublas_tflops": round(base_fl / t_cublas / 1e6, 2)}


PER_CONFIG = ["llama70b_decode_h28672", "llama70b_decode_h8192", "prefill", "distinct",
              "uniform_h4096", "uniform_h11008", "skewed_h4096", "skewed_h11008", "identical_h4096",
              "identical_h11008", "uniform_h4096:call", "uniform_h11008:call", "skewed_h4096:call",
              "skewed_h11008:call", "identical_h4096:call", "identical_h11008:call"]


def run_ours(args, spec: Spec, rank: int, world: int, local: int):
    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    stream = torch.cuda.Stream(device=dev)
    w = spec.w

    # ---- the headline: K steps of the workload ----
    clocks = ClockSampler(local)
    ds, ms, ms_early, lps = measure(spec, args, args.steps, stream, world, dev, rank, clocks)
    ms_per_step = ms / args.steps
    entry = summarize(spec, ds, ms, ms_early, lps, args.steps, dev)

    # roofline of the dominant kernel: one launch per step (batched, fused, grouped), or the
    # whole call where a call runs two kernels (the split forms)
    hbm, tc, which = peaks()
    bytes_step = w.algorithmic_bytes() * spec.P
    launch_s = ms_per_step / 1e3 / (lps if lps <= spec.P else spec.P)
    bytes_launch = bytes_step / (lps if lps <= spec.P else spec.P)
    kernel_name = (f"sgmv_fused_kernel (lora_sgmv_apply_batched: {spec.P} projections per launch)" if spec.P > 1
                   else "lora_sgmv_apply, dispatcher's choice" +
                   (f": {lps} launches per call, roofline over the whole call" if lps > 1 else ""))
    roofline = make_roofline(bytes_launch, w.flops() * spec.P * bytes_launch / bytes_step, launch_s, hbm, tc, which,
                             measured_traffic(spec.name), kernel_name)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, ds, stream, world, dev)
    del ds
    torch.cuda.empty_cache()

    # ---- every configuration ----
    per_config = {}
    if not args.no_per_config:
        steps_cfg = max(args.warmup, min(args.steps, PER_CONFIG_MAX_STEPS))
        for name in PER_CONFIG:
            if name == spec.name:
                per_config[name] = entry
                continue
            sp = make_spec(name)
            d2, m2, m2e, l2 = measure(sp, args, steps_cfg, stream, world, dev, rank)
            per_config[name] = summarize(sp, d2, m2, m2e, l2, steps_cfg, dev)
            del d2
            torch.cuda.empty_cache()
        per_config["prefill_layer"] = measure_layer(args, min(steps_cfg, 50), stream, world, dev, rank)
        torch.cuda.empty_cache()

    result = None
    if rank == 0:
        value = job_tokens_per_s(w.T * args.steps, world, ms / 1e3)
        cfg = config_dict(spec, world)
        cfg.update({"layers_rotated": spec.L,
                    "l2": f"inputs larger than L2: {spec.L} layers rotated, "
                          f"{spec.L * bytes_step / 2**30:.2f} GiB of algorithmic bytes per rotation",
                    "timing": "CUDA events on the launching stream around one replay of a CUDA graph of exactly "
                              "K steps (step i on layer i mod L), after one untimed replay",
                    "overlap": "launches chained by programmatic dependent launch under the default contract: the "
                               "next launch's prologue overlaps the end of the previous one; it reads none of its "
                               "inputs before the previous launch completes (early_reads: the same with "
                               "LORA_SGMV_FLAG_EARLY_READS, adapters streamed during the previous launch)"})
        result = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": cfg,
            "dispatch": entry["dispatch"],
            "roofline": roofline,
            "early_reads": entry["early_reads"],
            "gpu_launches": int(lps * args.steps),
            "clocks": clocks.summary(),
        }
        if e2e:
            result["e2e"] = e2e
        if per_config:
            result["per_config"] = per_config
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def run_e2e(args, ds: DeviceSpec, stream, world: int, dev) -> dict:
    if ds.spec.P > 1:
        return run_e2e_step_host(args, ds, world, dev)
    return run_e2e_single(args, ds, stream, world, dev)


def run_e2e_step_host(args, ds: DeviceSpec, world: int, dev) -> dict:
    """The metric through the library's host-memory serving call, lora_sgmv_step_host, one call
    per step: it groups the batch's adapter ids on the host, copies the segment arrays and every
    projection's X and Y from pinned host memory (one packed copy), runs the batched SGMV launch
    and copies Y back to pinned host memory, all enqueued on one stream; the host then reads the
    result. Three buffer sets, each with its own stream: step i's copy in overlaps the launches
    and copies out of steps i-1 and i-2, and a buffer set is reused only after its previous
    step's result has been read. Host wall clock."""
    import torch

    sgmv, spec, w = ds.sgmv, ds.spec, ds.spec.w
    P, NB = spec.P, 3
    steps = max(3, min(args.steps, 200))
    meta_bytes = ((2 * w.num_adapters + 1) * 4 + 255) // 256 * 256
    x_bytes, y_bytes = P * w.T * w.H1 * 2, P * w.T * w.H2 * 2
    in_bytes = meta_bytes + x_bytes + y_bytes
    h_in = torch.empty((NB, in_bytes), dtype=torch.uint8, pin_memory=True)
    d_in = torch.empty((NB, in_bytes), dtype=torch.uint8, device=dev)
    outY = torch.empty((NB, y_bytes), dtype=torch.uint8, pin_memory=True)
    hX = torch.stack([ds.calls[0][p][0] for p in range(P)]).cpu().view(torch.uint8).reshape(-1)
    hY = torch.stack([ds.calls[0][p][1] for p in range(P)]).cpu().view(torch.uint8).reshape(-1)
    for b in range(NB):  # the step's inputs, staged once in pinned memory (copied every step)
        h_in[b, meta_bytes:meta_bytes + x_bytes].copy_(hX)
        h_in[b, meta_bytes + x_bytes:].copy_(hY)
    ids = np.ascontiguousarray(w.ids, dtype=np.int32)
    hb = [h_in[b].data_ptr() for b in range(NB)]
    db = [d_in[b].data_ptr() for b in range(NB)]
    ob = [outY[b].data_ptr() for b in range(NB)]
    runs = [[sgmv.HostStep(
        ids, w.T, w.num_adapters, hb[b], db[b], [(hb[b], db[b], in_bytes)],
        [sgmv.Problem(db[b] + meta_bytes + x_bytes + p * w.T * w.H2 * 2, db[b] + meta_bytes + p * w.T * w.H1 * 2,
                      ds.calls[l][p][2].data_ptr(), ds.calls[l][p][3].data_ptr(), w.num_adapters, w.H1, w.H2,
                      w.scale) for p in range(P)],
        w.r, ds.dt, [(db[b] + meta_bytes + x_bytes, ob[b], y_bytes)]) for l in range(spec.L)] for b in range(NB)]
    streams = [torch.cuda.Stream(device=dev) for _ in range(NB)]
    sh = [s.cuda_stream for s in streams]
    done = [torch.cuda.Event() for _ in range(NB)]
    used = [False] * NB
    out_np = [outY[b].numpy() for b in range(NB)]
    sink = [0]

    def one(i):
        b, l = i % NB, i % spec.L
        if used[b]:
            done[b].synchronize()  # step i-NB: its copies are done, its result is read
            sink[0] ^= int(out_np[b][0])
        used[b] = True
        runs[b][l].run(sh[b])
        done[b].record(streams[b])

    def drain():
        for b in range(NB):
            if used[b]:
                done[b].synchronize()
                sink[0] ^= int(out_np[b][0])
                used[b] = False

    for i in range(3):
        one(i)
    drain()
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    t0 = time.perf_counter()
    for i in range(steps):
        one(i)
    drain()
    el = max_over_ranks(time.perf_counter() - t0, world, dev)
    return {"value": round(job_tokens_per_s(w.T * steps, world, el), 1), "unit": UNIT,
            "h2d_bytes_per_step": int(in_bytes), "d2h_bytes_per_step": int(y_bytes), "steps": steps,
            "note": "host wall clock, slowest rank; per step one lora_sgmv_step_host call: host grouping, one "
                    f"pinned H2D of the segment arrays with X and Y ({P} projections), 1 batched SGMV launch, "
                    "D2H of Y, then the host reads Y; three buffer sets, each on its own stream, so one step's "
                    "copy in overlaps the previous steps' launches and copies out"}


def run_e2e_single(args, ds: DeviceSpec, stream, world: int, dev) -> dict:
    """The metric through the public calls with host buffers, for a workload of one projection.
    Per step: group the batch's adapter ids on the host (lora_sgmv_group_segments), copy the
    segment arrays with X and Y from pinned host memory (one packed copy), run lora_sgmv_apply,
    copy Y back to pinned host memory and read it there. Two buffer sets and three streams
    (host-to-device copies, compute, device-to-host copies): step i's copy in overlaps step
    i-1's launch and copy out; a buffer set is reused only after its previous step's result has
    been read. Host wall clock."""
    import torch

    sgmv, spec, w = ds.sgmv, ds.spec, ds.spec.w
    P, NB = spec.P, 2
    steps = max(3, min(args.steps, 200))
    meta_len = 2 * w.num_adapters + 1
    meta_bytes = (meta_len * 4 + 255) // 256 * 256
    x_bytes, y_bytes = P * w.T * w.H1 * 2, P * w.T * w.H2 * 2
    in_bytes = meta_bytes + x_bytes + y_bytes
    h_in = torch.empty((NB, in_bytes), dtype=torch.uint8, pin_memory=True)
    d_in = torch.empty((NB, in_bytes), dtype=torch.uint8, device=dev)
    outY = torch.empty((NB, y_bytes), dtype=torch.uint8, pin_memory=True)
    hX = torch.stack([ds.calls[0][p][0] for p in range(P)]).cpu().view(torch.uint8).reshape(-1)
    hY = torch.stack([ds.calls[0][p][1] for p in range(P)]).cpu().view(torch.uint8).reshape(-1)
    for b in range(NB):  # the step's inputs, staged once in pinned memory (copied every step)
        h_in[b, meta_bytes:meta_bytes + x_bytes].copy_(hX)
        h_in[b, meta_bytes + x_bytes:].copy_(hY)
    h_meta = [h_in[b, :meta_bytes].numpy().view(np.int32) for b in range(NB)]
    ids = np.ascontiguousarray(w.ids, dtype=np.int32)
    ws = torch.empty((NB, ds.ws_bytes // 4 + 64), dtype=torch.float32, device=dev)
    base = [d_in[b].data_ptr() for b in range(NB)]
    xs = [[base[b] + meta_bytes + p * w.T * w.H1 * 2 for p in range(P)] for b in range(NB)]
    ys = [[base[b] + meta_bytes + x_bytes + p * w.T * w.H2 * 2 for p in range(P)] for b in range(NB)]
    problems = [[[sgmv.Problem(ys[b][p], xs[b][p], ds.calls[l][p][2].data_ptr(), ds.calls[l][p][3].data_ptr(),
                               w.num_adapters, w.H1, w.H2, w.scale) for p in range(P)] for l in range(spec.L)]
                for b in range(NB)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(NB)]
    ev_run = [torch.cuda.Event() for _ in range(NB)]
    ev_out = [torch.cuda.Event() for _ in range(NB)]
    used = [False] * NB
    sink = [0]
    h2d = d2h = 0
    out_np = [outY[b].numpy() for b in range(NB)]

    def read_back(b):
        ev_out[b].synchronize()
        sink[0] ^= int(out_np[b][0])  # the host reads the step's result

    def one(i):
        nonlocal h2d, d2h
        b, l = i % NB, i % spec.L
        if used[b]:
            read_back(b)  # step i-2: its result read, its buffers free
        used[b] = True
        seg, idx, _ = sgmv.lora_sgmv_group_segments(ids, w.num_adapters)
        n = len(idx)
        h_meta[b][: n + 1] = seg
        h_meta[b][n + 1: 2 * n + 1] = idx
        max_len = int(np.max(np.diff(seg)))
        d_seg, d_idx = base[b], base[b] + 4 * (n + 1)
        s_in.wait_event(ev_out[b])  # step i-2's copy out of this buffer set (recorded, or never)
        with torch.cuda.stream(s_in):
            d_in[b].copy_(h_in[b], non_blocking=True)
        ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        q = problems[b][l][0]
        sgmv.lora_sgmv_apply(q.Y, q.X, q.A_ptrs, q.B_ptrs, d_seg, d_idx, n, w.num_adapters, w.T, w.H1, w.r,
                             w.H2, w.scale, ds.dt, max_len, ws[b], ds.ws_bytes, None, stream)
        ev_run[b].record(stream)
        s_out.wait_event(ev_run[b])
        with torch.cuda.stream(s_out):
            outY[b].copy_(d_in[b, meta_bytes + x_bytes:], non_blocking=True)
        ev_out[b].record(s_out)
        h2d = in_bytes
        d2h = y_bytes

    def drain():
        for b in range(NB):
            if used[b]:
                read_back(b)
                used[b] = False

    for i in range(3):
        one(i)
    drain()
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    t0 = time.perf_counter()
    for i in range(steps):
        one(i)
    drain()
    el = max_over_ranks(time.perf_counter() - t0, world, dev)
    return {"value": round(job_tokens_per_s(w.T * steps, world, el), 1), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "note": "host wall clock, slowest rank; per step: host grouping, one pinned H2D of the segment "
                    "arrays with X and Y, 1 lora_sgmv_apply call, D2H of Y read on the host; two buffer "
                    "sets on three streams, so one step's copy in overlaps the previous step's launch and "
                    "copy out"}


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
        "config": config_dict(spec, int(os.environ.get("WORLD_SIZE", "1"))),
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": runs[0]["sample"]},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="distinct", choices=workload_names())
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.steps < 1:
        ap.error("--steps must be >= 1")
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

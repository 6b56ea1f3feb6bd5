#!/usr/bin/env python3
"""Benchmark of the decode-time Gated DeltaNet state update on B200.

Workload (one "step"): the large L2-busting decode -- 8 independent GDN layer
instances, each a call of gdn_decode_step on B=256 requests x Hv=32 value heads
(Hk=16, dk=dv=128, bf16 q/k/v, fp32 state), in place on a random slot
permutation of a 2048-slot pool (2 MiB of state per request per layer, 4 GiB
per pool, 32 GiB allocated, 4 GiB touched per step: far beyond the 126 MB L2,
so no flush is needed between steps).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  ``value`` is tokens*heads per second over the
whole job (device-timed with CUDA events, max over ranks); ``e2e`` is the same
metric through the public API with each step's inputs copied from pinned host
memory and its outputs copied back inside the timed region.  With N > 1 every
rank runs an independent replica (the update has no exchange step), so scaling
is weak.  ``--impl reference`` times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import hashlib
import io
import json
import os
import pathlib
import statistics
import subprocess
import sys
import time

ROOT = pathlib.Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "GDN state-update tokens·heads/s and achieved HBM GB/s vs B200 peak, 1 GPU"
UNIT = "tokens*heads/s"
WORKLOAD = "large L2-busting decode: B=256 x 8 GDN layers, Hk=16 Hv=32 dk=dv=128, in-place"
KERNEL_SOURCE = ROOT / "hybrid_linear_attention_step_b200" / "csrc" / "gdn_step.cu"
FALLBACK_HBM_GBS = 6650.0

# DRAM traffic per launch of the dominant kernel from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum); valid only for the kernel
# source it was taken on (sha256 of gdn_step.cu).
NCU_TRAFFIC = {"kernel": "gdn_tile1_kernel<128,128,64,128,5,bf16>",
               "source_sha256": "e539aa9e13cdaa93079eab8dca666256fe2a79d72834bf08a2c25f04e3b9ed12",
               "bytes_per_launch": 541153280 + 484916224}

# Kernel that serves the large decode for each --variant ("auto" picks the
# single-token register-tile kernel: 64-column blocks, 128 threads, 5 CTAs/SM).
KERNEL_NAMES = {"auto": "gdn_tile1_kernel<128,128,64,128,5,bf16>",
                "tile": "gdn_tile1_kernel<128,128,64,128,5,bf16>",
                "stream": "gdn_stream_kernel<256,bf16>", "column": "gdn_column_kernel<bf16>"}


def algorithmic_bytes_per_unit(dk: int, dv: int, G: int, in_bytes: int = 2, T: int = 1) -> float:
    """Bytes one (request, token, value head) must move: its state tile read once
    per request and written once per token, plus its share of q/k (shared by the
    G value heads of a key head), v, alpha, beta and the fp32 output."""
    state = 4.0 * dk * dv * (1.0 / T + 1.0)
    qk = 2.0 * dk * in_bytes / G
    return state + qk + dv * in_bytes + 8.0 + 4.0 * dv


FALLBACK_BF16_TFLOPS = 1590.0


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        try:
            d = json.loads(p.read_text())
            return float(d["hbm_gbs"]), "measured"
        except Exception:
            pass
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense bf16 tensor-core peak (TFLOP/s) for a kernel timed in isolation."""
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        try:
            return float(json.loads(p.read_text())["bf16_tflops"]), "measured"
        except Exception:
            pass
    return FALLBACK_BF16_TFLOPS, "fallback"


def source_sha256() -> str:
    return hashlib.sha256(KERNEL_SOURCE.read_bytes()).hexdigest()


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """SM clocks and clock-event (throttle) reasons sampled while the GPU works.

    Reads only.  NVML is polled from a thread every ``interval_ms`` (2 ms by default, so
    even a timed region of a few tens of milliseconds holds several samples); where
    NVML is not importable, ``nvidia-smi -lms`` is read instead.  ``mark`` sets the
    timed window; ``stop`` summarises the samples inside it.
    """

    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20), ("hw_thermal_slowdown", 0x40),
               ("sw_power_cap", 0x4))
    SMI_FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
                  "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int = 0, interval_ms: float = 2.0):
        self.device_index = device_index
        self.interval_ms = interval_ms
        self.window = None
        self.rows = []          # dicts: ts, sm, sm_max, reasons (set of names)
        self.source = None
        self._stop = False
        self._thread = None
        self._proc = None

    def _nvml_handle(self):
        import pynvml
        import torch

        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device_index)
        try:
            return pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
        except Exception:
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)

    def _poll_nvml(self, handle):
        import pynvml

        sm_max = float(pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM))
        while not self._stop:
            try:
                sm = float(pynvml.nvmlDeviceGetClockInfo(handle, pynvml.NVML_CLOCK_SM))
                bits = int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(handle))
                self.rows.append(dict(ts=time.time(), sm=sm, sm_max=sm_max,
                                      reasons={n for n, m in self.REASONS if bits & m}))
            except Exception:
                pass
            time.sleep(self.interval_ms / 1e3)

    def _poll_smi(self):
        for line in self._proc.stdout:
            r = next(csv.reader([line]), [])
            if len(r) < 11:
                continue
            try:
                act = {n for n, col in (("hw_slowdown", 7), ("hw_thermal_slowdown", 8), ("sw_thermal_slowdown", 9),
                                        ("sw_power_cap", 10)) if r[col].strip().lower() == "active"}
                self.rows.append(dict(ts=time.time(), sm=float(r[2]), sm_max=float(r[3]), reasons=act))
            except ValueError:
                continue

    def start(self, wait_s: float = 5.0):
        import threading

        try:
            handle = self._nvml_handle()
            self.source = f"nvml every {self.interval_ms:g} ms"
            self._thread = threading.Thread(target=self._poll_nvml, args=(handle,), daemon=True)
        except Exception:
            try:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
                smi_id = vis[self.device_index].strip() if vis and vis[0].strip() else str(self.device_index)
                self._proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={smi_id}", f"--query-gpu={self.SMI_FIELDS}",
                     "--format=csv,noheader,nounits", "-lms=50"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except Exception:
                return
            self.source = "nvidia-smi every 50 ms"
            self._thread = threading.Thread(target=self._poll_smi, daemon=True)
        self._thread.start()
        t0 = time.time()
        while not self.rows and time.time() - t0 < wait_s:
            time.sleep(0.005)

    def mark(self, t0: float, t1: float):
        self.window = (t0, t1)

    def stop(self):
        self._stop = True
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=10)
            except Exception:
                self._proc.kill()
        if self._thread is not None:
            self._thread.join(timeout=5)
        rows = list(self.rows)
        if not rows:
            return None
        picked, where = rows, "all"
        if self.window:
            inside = [r for r in rows if self.window[0] <= r["ts"] <= self.window[1]]
            if inside:
                picked, where = inside, "timed"
        reasons = set().union(*(r["reasons"] for r in picked))
        return {"sm_mhz": statistics.median(r["sm"] for r in picked),
                "sm_max_mhz": max(r["sm_max"] for r in picked),
                "sm_mhz_min": min(r["sm"] for r in picked),
                "reasons": sorted(reasons), "samples": len(picked), "window": where, "source": self.source}


# ----------------------------------------------------------- the workload

class LargeDecode:
    """Device-resident large decode: ``layers`` pools, per-layer inputs, one step = ``layers`` calls."""

    def __init__(self, layers: int = 8, num_slots: int = 2048, B: int = 256, device: str = "cuda",
                 seed: int = 4, variant: str = "auto", fused: bool = False):
        import numpy as np
        import torch

        from hybrid_linear_attention_step_b200 import gdn, workloads as wl

        c = wl.LARGE
        self.gdn = gdn
        self.layers, self.num_slots, self.B = layers, num_slots, B
        self.Hk, self.Hv, self.dk, self.dv = c["Hk"], c["Hv"], c["dk"], c["dv"]
        self.seed = seed
        self.variant = variant
        self.fused = fused  # raw q, k and gate pre-activations through gdn_decode_step_fused
        self.device = torch.device(device)
        self.host_steps = [wl.large_layer_step(l, seed, B, num_slots, raw=fused) for l in range(layers)]
        self.pools, self.inputs, self.outs = [], [], []
        for l in range(layers):
            pool = torch.empty((num_slots, self.Hv, self.dk, self.dv), dtype=torch.float32, device=self.device)
            wl.fill_pool_device(pool, seed, l)
            self.pools.append(pool)
            s = self.host_steps[l]
            bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
            self.inputs.append(dict(
                q=bf(s.q).to(self.device), k=bf(s.k).to(self.device), v=bf(s.v).to(self.device),
                alpha=torch.from_numpy(s.alpha).to(self.device), beta=torch.from_numpy(s.beta).to(self.device),
                src=torch.from_numpy(s.src_idx).to(self.device), dst=torch.from_numpy(s.dst_idx).to(self.device)))
            self.outs.append(torch.zeros((B, 1, self.Hv, self.dv), dtype=torch.float32, device=self.device))
        self.err = torch.zeros(1, dtype=torch.int32, device=self.device)
        torch.cuda.synchronize(self.device)

    @property
    def units_per_step(self) -> int:
        return self.layers * self.B * self.Hv

    @property
    def units_per_launch(self) -> int:
        return self.B * self.Hv

    def launch(self, l: int, stream=None):
        x = self.inputs[l]
        args = (self.pools[l], x["src"], x["dst"], x["q"], x["k"], x["v"], x["alpha"], x["beta"], self.outs[l])
        if self.fused:
            self.gdn.gdn_decode_step_fused(*args, self.gdn.GDN_FUSE_GATES | self.gdn.GDN_FUSE_QK_NORM,
                                           err_word=self.err, stream=stream)
        elif self.variant == "auto":
            self.gdn.gdn_decode_step(*args, err_word=self.err, stream=stream)
        else:
            self.gdn.gdn_decode_step_variant(*args, self.variant, err_word=self.err, stream=stream)

    def step(self, stream=None):
        for l in range(self.layers):
            self.launch(l, stream)

    # -- end to end: inputs from pinned host memory, outputs back to pinned host memory
    def make_host_io(self):
        import torch

        self.h_in = [{k: v.cpu().pin_memory() for k, v in x.items()} for x in self.inputs]
        self.h_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in self.outs]
        self.h2d_bytes = sum(t.numel() * t.element_size() for x in self.h_in for t in x.values())
        self.d2h_bytes = sum(t.numel() * t.element_size() for t in self.h_out)

    def make_e2e_streams(self):
        """Copy-in, compute and copy-out streams plus the per-layer events that
        order them (inputs of layer l are overwritten only after the previous
        step's kernel l has read them; out[l] only after it has been copied out)."""
        import torch

        self.s_in, self.s_out = torch.cuda.Stream(), torch.cuda.Stream()
        self.ev_in = [torch.cuda.Event() for _ in range(self.layers)]
        self.ev_run = [torch.cuda.Event() for _ in range(self.layers)]
        self.ev_out = [torch.cuda.Event() for _ in range(self.layers)]
        self.e2e_primed = False

    def step_e2e(self, stream):
        """One step end to end: per layer, H2D of its inputs (pinned host -> device),
        the decode call, D2H of its output; copies of other layers overlap the
        kernels (the pages' async H2D with event-based layer barriers)."""
        import torch

        for l in range(self.layers):
            x, hx = self.inputs[l], self.h_in[l]
            with torch.cuda.stream(self.s_in):
                if self.e2e_primed:
                    self.s_in.wait_event(self.ev_run[l])
                for key in ("q", "k", "v", "alpha", "beta", "src", "dst"):
                    x[key].copy_(hx[key], non_blocking=True)
                self.ev_in[l].record(self.s_in)
            stream.wait_event(self.ev_in[l])
            if self.e2e_primed:
                stream.wait_event(self.ev_out[l])
            self.launch(l, stream)
            self.ev_run[l].record(stream)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.ev_run[l])
                self.h_out[l].copy_(self.outs[l], non_blocking=True)
                self.ev_out[l].record(self.s_out)
        self.e2e_primed = True

    def join_e2e(self, stream):
        """Make ``stream`` wait for every copy of the steps issued so far."""
        stream.wait_stream(self.s_in)
        stream.wait_stream(self.s_out)


# ----------------------------------------------------------------- ranks

def dist_setup(n_gpus: int):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The maximum of ``x`` over all ranks (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, elapsed_ms_per_rank: float, world: int) -> float:
    """Whole-job units/s: all ranks' units over the slowest rank's time."""
    return world * units_per_rank / (max_over_ranks(elapsed_ms_per_rank, world) / 1e3)


# ------------------------------------------------------------ CPU oracle

def _oracle_sample_inputs(n_req: int, seed: int = 4):
    import numpy as np

    from hybrid_linear_attention_step_b200 import workloads as wl

    s = wl.large_layer_step(0, seed)
    rng = np.random.default_rng([seed, 99])
    pool = wl.init_pool(rng, n_req, s.Hv, s.dk, s.dv)
    idx = np.arange(n_req, dtype=np.int32)
    sl = lambda a: np.ascontiguousarray(a[:n_req])
    return pool, idx, sl(s.q), sl(s.k), sl(s.v), sl(s.alpha), sl(s.beta), s.Hv, s.dv


_ORACLE_SAMPLES = {}


def oracle_time(n_req: int, threads: int) -> float:
    """Seconds the oracle takes for one in-place call on ``n_req`` requests of the large decode.

    The sample inputs are generated once per size and reused by later calls (each call
    updates the sample pool in place, as a decode step does)."""
    import numpy as np

    import oracle

    if n_req not in _ORACLE_SAMPLES:
        _ORACLE_SAMPLES[n_req] = _oracle_sample_inputs(n_req)
    pool, idx, q, k, v, a, b, Hv, dv = _ORACLE_SAMPLES[n_req]
    out = np.zeros((n_req, 1, Hv, dv), np.float32)
    t0 = time.perf_counter()
    oracle.decode_step(pool, idx, idx.reshape(-1, 1).copy(), q, k, v, a, b, out, nthreads=threads)
    return time.perf_counter() - t0


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(budget_s: float = 12.0, Hv: int = 32):
    """The oracle as it stands, timed on the host cores on a bounded sample of the workload."""
    cores = cpu_cores()
    t1 = oracle_time(1, 1)  # one request (32 units), single thread: calibration
    n_req = int(max(1, min(256, budget_s * cores / max(t1, 1e-6) * 0.8)))
    threads = min(cores, n_req)
    t = oracle_time(n_req, threads)
    calls, total = 1, t
    while total < budget_s and calls < 8:  # successive steps of the same requests, up to the budget
        total += oracle_time(n_req, threads)
        calls += 1
    return {"value": calls * n_req * Hv / total, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{calls} successive in-place calls on {n_req} of the 256 requests of layer 0 "
                      f"({calls * n_req * Hv} tokens*heads), C++ double-precision oracle, {threads} threads, "
                      f"{total:.1f} s",
            "single_thread_value": Hv / max(t1, 1e-9), "host": host_info()}


def host_info() -> dict:
    """The CPU the oracle ran on: model, cores this process may use, logical CPUs."""
    model = None
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"cpu_model": model, "affinity_cores": cpu_cores(), "logical_cpus": os.cpu_count()}


def headline_config(args, world: int) -> dict:
    """The `config` object of the large-decode line, shared by both arms."""
    return {"workload": WORKLOAD, "variant": args.variant, "graph": bool(args.graph),
            "fused_prologue": bool(args.fused), "B": args.batch, "layers": args.layers, "Hk": 16, "Hv": 32,
            "dk": 128, "dv": 128, "qkv": "bf16", "state": "f32", "slots_per_layer": args.slots,
            "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": "inputs larger than L2 (4 GiB of state touched per step), no flush"}


def run_reference(args):
    """The reference arm: the CPU oracle, timed for K steps on a bounded per-step sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cores = cpu_cores()
    t1 = oracle_time(1, 1)
    per_step_budget = max(0.2, 150.0 / (args.steps + args.warmup))
    n_req = int(max(1, min(256, per_step_budget * cores / max(t1, 1e-6) * 0.8)))
    threads = min(cores, n_req)
    for _ in range(args.warmup):
        oracle_time(n_req, threads)
    total = 0.0
    for _ in range(args.steps):
        total += oracle_time(n_req, threads)
    units = args.steps * n_req * 32
    value = units / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": headline_config(args, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "host": host_info(),
                         "sample": f"each step: one in-place call on {n_req} of the {args.batch} requests of "
                                   f"layer 0 ({n_req * 32} tokens*heads), C++ double-precision oracle"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------- other workloads

def workload_bytes(w, s) -> dict:
    """Algorithmic bytes of one call of a host workload: nominal (every unit reads
    its own source tile) and minimum (each distinct source tile read once)."""
    G = s.Hv // s.Hk
    in_bytes = 2 if s.dtype == "bf16" else 4
    per_req_tok = s.Hv * (2.0 * s.dk * in_bytes / G + s.dv * in_bytes + 8.0 + 4.0 * s.dv)
    tile = 4.0 * s.dk * s.dv
    writes = s.B * s.T * s.Hv * tile
    nominal = s.B * s.Hv * tile + writes + s.B * s.T * per_req_tok
    distinct = len(set(int(x) for x in s.src_idx if x >= 0))
    minimum = distinct * s.Hv * tile + writes + s.B * s.T * per_req_tok
    return {"nominal": nominal, "minimum": minimum, "units": s.B * s.T * s.Hv}


def _time_calls(call, n: int, stream, graph: bool) -> float:
    """Microseconds per call over ``n`` back-to-back calls (eager, or one captured graph)."""
    import torch

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g = None
    if graph:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            call()  # one eager call on the capture stream before capturing
        stream.wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(n):
                call()
        g.replay()
        torch.cuda.synchronize()
    ev0.record(stream)
    if g is not None:
        g.replay()
    else:
        for _ in range(n):
            call()
    ev1.record(stream)
    torch.cuda.synchronize()
    return 1e3 * ev0.elapsed_time(ev1) / n


def _time_cold(call, reps: int, stream, clean: bool = False) -> float:
    """Median microseconds of one call right after a write of 256 MiB (twice the L2).

    The write leaves the L2 full of dirty lines that the timed call then writes back.
    With ``clean`` the 256 MiB are read instead: the call still finds none of its data
    in L2, but pays for no one else's write-back."""
    import torch

    flush = torch.ones(256 << 18, dtype=torch.float32, device="cuda")
    cold = []
    for _ in range(reps):
        if clean:
            flush.sum()
        else:
            flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        torch.cuda.synchronize()
        cold.append(1e3 * e0.elapsed_time(e1))
    return statistics.median(cold)


def oracle_workload_baseline(w, s) -> dict:
    """The oracle on one whole call of a smaller workload, on the host cores."""
    import numpy as np

    import oracle

    threads = min(cpu_cores(), s.B)
    pool = w.pool.copy()
    out = np.zeros((s.B, s.T, s.Hv, s.dv), np.float32)
    t0 = time.perf_counter()
    oracle.decode_step(pool, s.src_idx, np.ascontiguousarray(s.dst_idx.reshape(s.B, s.T)), s.q, s.k, s.v,
                       s.alpha, s.beta, out, nthreads=threads)
    dt = time.perf_counter() - t0
    units = s.B * s.T * s.Hv
    return {"value": units / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"one whole call ({units} tokens*heads), C++ double-precision oracle, {dt:.2f} s"}


def measure_workload(name: str, calls: int = 200, warmup: int = 10, variant: str = "auto",
                     cold_reps: int = 50, graph_too: bool = True, cpu: bool = True) -> dict:
    """One of the smaller decode workloads (decode_b16, prefix_cow, speculative): its call
    timed warm (back to back, eager and replayed from one CUDA graph) and cold (after an
    L2-flushing write), the speculative commit, algorithmic bandwidth against the copy
    peak, and the oracle on the same call."""
    import numpy as np
    import torch

    from hybrid_linear_attention_step_b200 import gdn, workloads as wl

    w = wl.WORKLOADS[name]()
    s = w.steps[0]
    # A caller that knows its batch's requests share source slots (a prefix-cache planner
    # sees repeated src entries) passes the ordering hint; the results are the same.
    shared = len(set(np.asarray(s.src_idx).tolist())) < s.B
    flags = gdn.GDN_SHARED_SOURCES if shared and variant == "auto" else 0
    to_dev = lambda a: (torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
                        if a.dtype == np.uint16 else torch.from_numpy(np.ascontiguousarray(a)).cuda())
    pool = torch.from_numpy(w.pool).cuda()
    x = {k_: to_dev(getattr(s, k_)) for k_ in ("q", "k", "v", "alpha", "beta", "src_idx")}
    dst = to_dev(np.ascontiguousarray(s.dst_idx.reshape(s.B, s.T)))
    out = torch.zeros((s.B, s.T, s.Hv, s.dv), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    def call(hint=True):
        args_ = (pool, x["src_idx"], dst, x["q"], x["k"], x["v"], x["alpha"], x["beta"], out)
        if flags and hint:
            gdn.gdn_decode_step_fused(*args_, flags, err_word=err)
        elif variant == "auto":
            gdn.gdn_decode_step(*args_, err_word=err)
        else:
            gdn.gdn_decode_step_variant(*args_, variant, err_word=err)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    warm_us = _time_calls(call, calls, stream, graph=False)
    # The same call through the prepared form (buffers checked once, stream bound).
    prepared = gdn.PreparedDecodeStep(pool, x["src_idx"], dst, x["q"], x["k"], x["v"], x["alpha"], x["beta"], out,
                                      err_word=err, variant=None if variant == "auto" else variant, stream=stream,
                                      flags=flags)
    prepared_us = _time_calls(prepared, calls, stream, graph=False)
    graph_us = _time_calls(call, calls, stream, graph=True) if graph_too else None
    cold_us = _time_cold(call, min(calls, cold_reps), stream)
    cold_clean_us = _time_cold(call, min(calls, cold_reps), stream, clean=True)
    cold_no_hint_us = _time_cold(lambda: call(hint=False), min(calls, cold_reps), stream) if flags else None
    code = gdn.gdn_get_error(err)
    if code != 0:
        raise RuntimeError(f"device error word set: {gdn.status_string(code)}")

    commit = None
    if s.accept_len is not None:
        committed = x["src_idx"].clone()
        acc = to_dev(s.accept_len)
        ccall = lambda: gdn.gdn_commit(acc, committed, dst, w.num_slots, err_word=err)
        for _ in range(3):
            ccall()
        torch.cuda.synchronize()
        commit = {"us_per_call_eager": _time_calls(ccall, 100, stream, graph=False),
                  "us_per_call_graph": _time_calls(ccall, 100, stream, graph=True),
                  "note": "eager calls are bound by the host launch path; the graph figure is device time"}
        if gdn.gdn_get_error(err) != 0:
            raise RuntimeError("device error word set by the commit")

    hbm_peak, peak_kind = peaks()
    nb = workload_bytes(w, s)
    best_warm = min(warm_us, graph_us) if graph_us else warm_us
    entry = {
        "workload": name, "variant": variant, "flags": "GDN_SHARED_SOURCES" if flags else 0,
        "config": {"B": s.B, "T": s.T, "Hk": s.Hk, "Hv": s.Hv, "dk": s.dk, "dv": s.dv, "slots": w.num_slots,
                   "qkv": s.dtype, "state": "f32"},
        "units_per_call": nb["units"], "calls": calls,
        "us_per_call_warm": warm_us, "us_per_call_prepared": prepared_us, "us_per_call_graph": graph_us,
        "us_per_call_cold": cold_us,
        "us_per_call_cold_clean_l2": cold_clean_us, "us_per_call_cold_without_hint": cold_no_hint_us,
        "value_warm": nb["units"] / (best_warm / 1e6), "value_cold": nb["units"] / (cold_us / 1e6), "unit": UNIT,
        "bytes_per_call_nominal": nb["nominal"], "bytes_per_call_min": nb["minimum"],
        "gbs_cold_nominal": nb["nominal"] / cold_us / 1e3, "gbs_cold_min": nb["minimum"] / cold_us / 1e3,
        "gbs_warm_nominal": nb["nominal"] / best_warm / 1e3,
        "frac_cold_nominal": nb["nominal"] / cold_us / 1e3 / hbm_peak,
        "frac_cold_min": nb["minimum"] / cold_us / 1e3 / hbm_peak,
        "peak_gbs": hbm_peak, "peak_kind": f"{peak_kind} copy bandwidth",
        "gbs_cold_clean_nominal": nb["nominal"] / cold_clean_us / 1e3,
        "l2": "warm: the call's inputs may sit in L2; cold: after a 256 MiB write (the call also writes back "
              "the dirty lines it evicts); cold_clean_l2: after a 256 MiB read",
        "commit": commit,
    }
    if cpu:
        entry["cpu_baseline"] = oracle_workload_baseline(w, s)
    del pool, out
    torch.cuda.empty_cache()
    return entry


PREFILL_SHAPE = dict(Hk=16, Hv=32, dk=128, dv=128)


def oracle_prefill_baseline(q, k, v, a, b, pool_host, pairs, L) -> dict:
    """The oracle's prefill on a sample of (request, head) pairs over the whole prompt."""
    import numpy as np

    import oracle

    c = PREFILL_SHAPE
    G = c["Hv"] // c["Hk"]
    n = len(pairs)
    sq = np.stack([q[bb, :, h // G] for bb, h in pairs])[:, :, None, :].copy()
    sk = np.stack([k[bb, :, h // G] for bb, h in pairs])[:, :, None, :].copy()
    sv = np.stack([v[bb, :, h] for bb, h in pairs])[:, :, None, :].copy()
    sa = np.stack([a[bb, :, h] for bb, h in pairs])[:, :, None].copy()
    sb = np.stack([b[bb, :, h] for bb, h in pairs])[:, :, None].copy()
    ref_pool = np.zeros((2 * n, 1, c["dk"], c["dv"]), np.float32)
    ref_pool[:n, 0] = [pool_host[bb, h] for bb, h in pairs]
    out = np.zeros((n, L, 1, c["dv"]), np.float32)
    idx = np.arange(n, dtype=np.int32)
    t0 = time.perf_counter()
    oracle.prefill(ref_pool, idx, idx + n, sq, sk, sv, sa, sb, out, nthreads=n)
    dt = time.perf_counter() - t0
    return {"value": n * L / dt, "unit": UNIT, "cores": n, "kind": "oracle",
            "sample": f"{n} (request, head) pairs x {L} tokens ({n * L} tokens*heads), C++ double-precision "
                      f"oracle token loop, {dt:.1f} s"}


def measure_prefill(B: int = 4, L: int = 2048, chunked: bool = True, calls: int = 20, warmup: int = 3,
                    cpu: bool = True, clocks: bool = False) -> dict:
    """gdn_prefill_chunked (or gdn_prefill) on B requests x L tokens, Hk=16, Hv=32, dk=dv=128,
    bf16 inputs; only the final states are stored (checkpoints)."""
    import numpy as np
    import torch

    from hybrid_linear_attention_step_b200 import gdn, workloads as wl

    c = PREFILL_SHAPE
    Hk, Hv, dk, dv = c["Hk"], c["Hv"], c["dk"], c["dv"]
    rng = np.random.default_rng(6)
    q, k, v, a, b = wl.random_step_inputs(rng, B, L, Hk, Hv, dk, dv, wl.BF16)
    bf = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    xq, xk, xv = bf(q), bf(k), bf(v)
    xa, xb = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    pool = torch.empty((2 * B, Hv, dk, dv), dtype=torch.float32, device="cuda")
    wl.fill_pool_device(pool, 6, 0)
    src = torch.arange(B, dtype=torch.int32, device="cuda")
    dst = torch.arange(B, 2 * B, dtype=torch.int32, device="cuda")
    out = torch.empty((B, L, Hv, dv), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    if chunked:
        ws = torch.empty(gdn.gdn_prefill_workspace_bytes(B, L, Hv, dk, dv), dtype=torch.uint8, device="cuda")
        call = lambda: gdn.gdn_prefill_chunked(pool, src, dst, xq, xk, xv, xa, xb, out, ws, err_word=err)
    else:
        call = lambda: gdn.gdn_prefill(pool, src, dst, xq, xk, xv, xa, xb, out, err_word=err)
    pool_host = pool[:B].cpu().numpy() if cpu else None
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(torch.cuda.current_device()) if clocks else None
    if sampler:
        sampler.start()
    w0 = time.time()
    us = _time_calls(call, calls, stream, graph=False)
    if sampler:
        sampler.mark(w0, time.time())
    if gdn.gdn_get_error(err) != 0:
        raise RuntimeError("device error word set during the prefill benchmark")
    units = B * L * Hv
    entry = {"workload": f"prefill B={B} L={L} Hk={Hk} Hv={Hv} dk=dv={dk}, bf16 q/k/v, fp32 state",
             "kernel": "chunked (gdn_prefill_chunked)" if chunked else "token steps (gdn_prefill)",
             "units_per_call": units, "calls": calls, "us_per_call": us, "value": units / (us / 1e6), "unit": UNIT,
             "l2": "inputs, outputs and workspace larger than L2"}
    hbm_peak, peak_kind = peaks()
    # I/O the method must move: q, k, v (bf16), alpha, beta, out (fp32), the initial
    # state read and the checkpoint written.
    io = B * L * (2 * Hk * dk * 2 + Hv * dv * 2 + 2 * Hv * 4 + Hv * dv * 4) + 2 * B * Hv * dk * dv * 4
    entry["io_bytes"] = io
    entry["io_gbs"] = io / us / 1e3
    entry["io_frac"] = io / us / 1e3 / hbm_peak
    entry["peak_gbs"] = hbm_peak
    entry["peak_kind"] = f"{peak_kind} copy bandwidth"
    if chunked:
        ws_bytes = gdn.gdn_prefill_workspace_bytes(B, L, Hv, dk, dv)
        chunks = (L + 63) // 64
        C = 64
        # per (request, head, chunk) in exact arithmetic: K K^T and Q K^T, the triangular
        # solve for U and W, W M and Q M, P E, K^T E
        flop_chunk = 2 * 2 * C * C * dk + C * C * (dk + dv) + 2 * 2 * C * dk * dv + 2 * C * C * dv \
            + 2 * C * dk * dv
        tflops = B * Hv * chunks * flop_chunk / us / 1e6
        tpk, tkind = tensor_peak()
        entry.update({"workspace_bytes": ws_bytes, "with_workspace_frac": (io + 2 * ws_bytes) / us / 1e3 / hbm_peak,
                      "tflops_algorithmic": tflops, "tensor_peak_tflops": tpk,
                      "tensor_peak_kind": f"{tkind} dense bf16", "tensor_frac": tflops / tpk})
    if sampler:
        entry["clocks"] = sampler.stop()
    if cpu:
        pairs = [(i % B, (7 * i) % Hv) for i in range(min(cpu_cores(), 16))]
        entry["cpu_baseline"] = oracle_prefill_baseline(q, k, v, a, b, pool_host, pairs, L)
    del pool, out
    if chunked:
        del ws
    torch.cuda.empty_cache()
    return entry


def run_workload(args):
    """`--workload decode_b16|prefix_cow|speculative`: one line for that workload."""
    import torch

    torch.cuda.set_device(0)
    e = measure_workload(args.workload, calls=args.steps, warmup=args.warmup, variant=args.variant,
                         cpu=not args.no_cpu_baseline)
    print(json.dumps({"metric": METRIC, **e}), flush=True)


def run_prefill(args):
    """`--workload prefill [--chunked]`: one line for the prefill."""
    import torch

    torch.cuda.set_device(0)
    e = measure_prefill(args.prefill_batch, args.prefill_len, args.chunked, calls=args.steps, warmup=args.warmup,
                        cpu=not args.no_cpu_baseline, clocks=True)
    print(json.dumps({"metric": METRIC, **e}), flush=True)


def measure_configs(cpu: bool) -> dict:
    """The other synthetic workloads beside the headline, each with its oracle baseline."""
    out = {}
    jobs = [(name, lambda n=name: measure_workload(n, cpu=cpu)) for name in ("decode_b16", "prefix_cow", "speculative")]
    jobs.append(("prefill_chunked", lambda: measure_prefill(4, 2048, True, cpu=cpu)))
    for name, job in jobs:
        try:
            out[name] = job()
        except Exception as e:  # one failing entry must not take the headline line with it
            out[name] = {"error": f"{type(e).__name__}: {e}"}
    return out


# ------------------------------------------------------------------ main

def run_ours(args):
    import torch

    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    hbm_peak, peak_kind = peaks()
    wk = LargeDecode(layers=args.layers, num_slots=args.slots, B=args.batch, variant=args.variant,
                     fused=args.fused)
    kernel = KERNEL_NAMES[args.variant]
    if args.fused:
        kernel = kernel.replace(",bf16>", ",bf16,fused>")
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()

    for _ in range(args.warmup):
        wk.step(stream)
    torch.cuda.synchronize()
    barrier(world)

    K, L = args.steps, wk.layers
    graph = None
    if args.graph:
        # One 8-layer step captured once and replayed K times: the pages' CUDA-graph
        # recording of the decode loop, with the calls' PDL edges kept in the graph.
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            wk.step(side)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            wk.step()
        for _ in range(3):
            graph.replay()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    w0 = time.time()
    start.record(stream)
    for _ in range(K):
        if graph is not None:
            graph.replay()
        else:
            wk.step(stream)
    stop.record(stream)
    torch.cuda.synchronize()
    w1 = time.time()
    barrier(world)
    sampler.mark(w0, w1)
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), world)
    # Every launch in the timed region is the same kernel on the same stream:
    # its average duration is the region over the launch count (gaps included).
    launch_ms = elapsed_ms / (K * L)

    # Diagnostic pass, outside the timed region: the same K steps with an
    # event pair around every launch (the events themselves add a few us each).
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K * L)]
    for s_ in range(K):
        for l in range(L):
            e0, e1 = ev[s_ * L + l]
            e0.record(stream)
            wk.launch(l, stream)
            e1.record(stream)
    torch.cuda.synchronize()
    durs = sorted(e0.elapsed_time(e1) for e0, e1 in ev)
    launch_events = {"mean_us": 1e3 * statistics.mean(durs), "median_us": 1e3 * durs[len(durs) // 2],
                     "min_us": 1e3 * durs[0], "max_us": 1e3 * durs[-1]}
    code = wk.gdn.gdn_get_error(wk.err)
    if code != 0:
        raise RuntimeError(f"device error word set during the benchmark: {wk.gdn.status_string(code)}")

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        wk.make_host_io()
        wk.make_e2e_streams()
        for _ in range(max(3, args.warmup // 2)):
            wk.step_e2e(stream)
        wk.join_e2e(stream)
        torch.cuda.synchronize()
        barrier(world)
        e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e_start.record(stream)
        wk.s_in.wait_event(e_start)
        wk.s_out.wait_event(e_start)
        for _ in range(K):
            wk.step_e2e(stream)
        wk.join_e2e(stream)
        e_stop.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(e_start.elapsed_time(e_stop), world)
        e2e = {"value": world * K * wk.units_per_step / (e2e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": wk.h2d_bytes, "d2h_bytes_per_step": wk.d2h_bytes,
               "ms_per_step": e2e_ms / K}
    clocks = sampler.stop()

    G = wk.Hv // wk.Hk
    bytes_per_unit = algorithmic_bytes_per_unit(wk.dk, wk.dv, G)
    bytes_per_launch = bytes_per_unit * wk.units_per_launch
    achieved = bytes_per_launch / (launch_ms / 1e3) / 1e9
    traffic = None
    if (NCU_TRAFFIC["source_sha256"] == source_sha256() and NCU_TRAFFIC["kernel"] == kernel
            and NCU_TRAFFIC["bytes_per_launch"]):
        traffic = NCU_TRAFFIC["bytes_per_launch"]
    value = world * K * wk.units_per_step / (elapsed_ms / 1e3)
    step_gbs = bytes_per_launch * L * K / (elapsed_ms / 1e3) / 1e9  # equals roofline.achieved here

    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": traffic,
                "peak_kind": f"{peak_kind} copy bandwidth", "kernel": kernel,
                "bytes_per_launch": bytes_per_launch, "launch_us": launch_ms * 1e3}
    if traffic:
        # The copy probe behind the peak moves its bytes through L2 like any kernel; this
        # kernel's algorithmic bytes slightly exceed what DRAM sees (ncu traffic), so the
        # DRAM-side fraction is reported beside the algorithmic one.
        roofline["frac_traffic"] = traffic / (launch_ms / 1e3) / 1e9 / hbm_peak
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": elapsed_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": headline_config(args, world),
        "roofline": roofline,
        "hbm_gbs_step": step_gbs, "launch_events": launch_events, "frac_of_8tbs_step": step_gbs / 8000.0,
        "e2e": e2e, "gpu_launches": K * L, "clocks": clocks,
    }
    if clocks and clocks.get("sm_mhz"):
        # time x clock: comparable across runs whose SM clocks differ
        line["ms_x_sm_mhz_per_step"] = elapsed_ms / K * clocks["sm_mhz"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0 and world == 1 and not args.no_configs:
        line["configs"] = measure_configs(cpu=not args.no_cpu_baseline)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=8)
    ap.add_argument("--slots", type=int, default=2048)
    ap.add_argument("--batch", type=int, default=256)
    ap.add_argument("--variant", choices=["auto", "stream", "tile", "column"], default="auto",
                    help="kernel for the decode calls (auto = what gdn_decode_step picks)")
    ap.add_argument("--workload", choices=["large", "decode_b16", "prefix_cow", "speculative", "prefill"],
                    default="large",
                    help="large = the headline 8-layer decode; the others time one call of that workload")
    ap.add_argument("--prefill-batch", type=int, default=4)
    ap.add_argument("--prefill-len", type=int, default=2048)
    ap.add_argument("--chunked", action="store_true", help="prefill workload through gdn_prefill_chunked")
    ap.add_argument("--graph", action="store_true", help="replay the timed calls from a CUDA graph "
                    "(smaller workloads only)")
    ap.add_argument("--fused", action="store_true", help="large workload through gdn_decode_step_fused: raw "
                    "gate pre-activations and unnormalised q, k, folded into the kernel")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="large workload: leave out the smaller workloads' entries (configs)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "prefill":
        run_prefill(args)
    elif args.workload != "large":
        run_workload(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

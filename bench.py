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
# source it was taken on (sha256 of gdn_step.cu).  See profiles/.
NCU_TRAFFIC = {"kernel": "gdn_tile1_kernel<128,128,64,128,5,bf16>",
               "source_sha256": "2749ceb8bdba484ccb2c638bc20fa1bd165c2b17abd6d9fd3899c0caa34bbfaa",
               "bytes_per_launch": 541164544 + 483485952,
               "profile": "profiles/gdn_tile1_kernel_large_decode.md"}

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


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        try:
            d = json.loads(p.read_text())
            return float(d["hbm_gbs"]), "measured"
        except Exception:
            pass
    return FALLBACK_HBM_GBS, "fallback"


def source_sha256() -> str:
    return hashlib.sha256(KERNEL_SOURCE.read_bytes()).hexdigest()


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the GPU works.

    A reader thread collects one CSV line per sample; ``start`` returns once the
    first sample has arrived (or after a few seconds if nvidia-smi is absent).
    """

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str, interval_ms: int = 50):
        self.proc = None
        self.gpu_index = gpu_index
        self.interval_ms = interval_ms
        self.window = None
        self.lines = []
        self.thread = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line))

    def start(self, wait_s: float = 5.0):
        import threading

        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", f"-lms={self.interval_ms}"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.lines and time.time() - t0 < wait_s and self.proc.poll() is None:
            time.sleep(0.01)

    def mark(self, t0: float, t1: float):
        self.window = (t0, t1)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=10)
        except Exception:
            self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)
        rows = []
        for t_host, line in list(self.lines):
            r = next(csv.reader([line]), [])
            if len(r) < 11:
                continue
            try:
                rows.append(dict(ts=t_host, sm=float(r[2]), sm_max=float(r[3]), power=float(r[4]),
                                 util=float(r[5]), hw=r[7].strip(), hw_th=r[8].strip(),
                                 sw_th=r[9].strip(), pcap=r[10].strip()))
            except ValueError:
                continue
        if not rows:
            return None
        picked, where = rows, "all"
        if self.window:
            inside = [r for r in rows if self.window[0] <= r["ts"] <= self.window[1] + 0.1]
            if len(inside) >= 3:
                picked, where = inside, "timed"
            else:
                busy = [r for r in rows if r["util"] >= 50]
                if busy:
                    picked, where = busy, "busy"
        reasons = set()
        for r in picked:
            for key, name in (("hw", "hw_slowdown"), ("hw_th", "hw_thermal_slowdown"),
                              ("sw_th", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in picked),
                "sm_max_mhz": max(r["sm_max"] for r in picked),
                "reasons": sorted(reasons), "samples": len(picked), "window": where}


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


def run_workload(args):
    """Times one of the smaller workloads (decode_b16, prefix_cow, speculative):
    ``--steps`` decode calls, back to back (warm L2) and, separately, each call
    after an L2-flushing write (cold), optionally replayed from a CUDA graph."""
    import numpy as np
    import torch

    from hybrid_linear_attention_step_b200 import gdn, workloads as wl

    torch.cuda.set_device(0)
    w = wl.WORKLOADS[args.workload]()
    s = w.steps[0]
    to_dev = lambda a: (torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
                        if a.dtype == np.uint16 else torch.from_numpy(np.ascontiguousarray(a)).cuda())
    pool = torch.from_numpy(w.pool).cuda()
    x = {k_: to_dev(getattr(s, k_)) for k_ in ("q", "k", "v", "alpha", "beta", "src_idx")}
    dst = to_dev(np.ascontiguousarray(s.dst_idx.reshape(s.B, s.T)))
    out = torch.zeros((s.B, s.T, s.Hv, s.dv), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    def call():
        args_ = (pool, x["src_idx"], dst, x["q"], x["k"], x["v"], x["alpha"], x["beta"], out)
        if args.variant == "auto":
            gdn.gdn_decode_step(*args_, err_word=err)
        else:
            gdn.gdn_decode_step_variant(*args_, args.variant, err_word=err)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    K = args.steps
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    graph = None
    if args.graph:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            call()  # one eager call on the capture stream before capturing
        stream.wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(K):
                call()
        graph.replay()
        torch.cuda.synchronize()
    ev0.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for _ in range(K):
            call()
    ev1.record(stream)
    torch.cuda.synchronize()
    warm_us = 1e3 * ev0.elapsed_time(ev1) / K

    # cold: an L2-sized write before every call, the call alone bracketed by events
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    cold = []
    for _ in range(min(K, 50)):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        torch.cuda.synchronize()
        cold.append(1e3 * e0.elapsed_time(e1))
    cold_us = statistics.median(cold)
    code = gdn.gdn_get_error(err)
    if code != 0:
        raise RuntimeError(f"device error word set: {gdn.status_string(code)}")

    commit_us = None
    if s.accept_len is not None:
        committed = x["src_idx"].clone()
        acc = to_dev(s.accept_len)
        for _ in range(3):
            gdn.gdn_commit(acc, committed, dst, w.num_slots)
        torch.cuda.synchronize()
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(100):
            gdn.gdn_commit(acc, committed, dst, w.num_slots)
        c1.record(stream)
        torch.cuda.synchronize()
        commit_us = 1e3 * c0.elapsed_time(c1) / 100

    hbm_peak, peak_kind = peaks()
    nb = workload_bytes(w, s)
    line = {
        "metric": METRIC, "workload": args.workload, "unit": UNIT, "variant": args.variant,
        "graph": bool(args.graph), "steps": K, "warmup": args.warmup,
        "value": nb["units"] / (warm_us / 1e6), "us_per_call_warm": warm_us, "us_per_call_cold": cold_us,
        "bytes_per_call_nominal": nb["nominal"], "bytes_per_call_min": nb["minimum"],
        "gbs_warm_nominal": nb["nominal"] / warm_us / 1e3, "gbs_cold_nominal": nb["nominal"] / cold_us / 1e3,
        "gbs_cold_min": nb["minimum"] / cold_us / 1e3, "peak_gbs": hbm_peak, "peak_kind": peak_kind,
        "commit_us": commit_us,
        "config": {"B": s.B, "T": s.T, "Hk": s.Hk, "Hv": s.Hv, "dk": s.dk, "dv": s.dv, "slots": w.num_slots,
                   "dtype": s.dtype},
    }
    print(json.dumps(line), flush=True)


def run_prefill(args):
    """Times gdn_prefill on a long-prompt batch: B requests x L tokens, Hk=16, Hv=32,
    dk=dv=128, bf16 inputs; only the final states are stored (checkpoints)."""
    import numpy as np
    import torch

    from hybrid_linear_attention_step_b200 import gdn, workloads as wl

    torch.cuda.set_device(0)
    B, L, Hk, Hv, dk, dv = args.prefill_batch, args.prefill_len, 16, 32, 128, 128
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
    if args.chunked:
        ws = torch.empty(gdn.gdn_prefill_workspace_bytes(B, L, Hv, dk, dv), dtype=torch.uint8, device="cuda")
        call = lambda: gdn.gdn_prefill_chunked(pool, src, dst, xq, xk, xv, xa, xb, out, ws, err_word=err)
    else:
        call = lambda: gdn.gdn_prefill(pool, src, dst, xq, xk, xv, xa, xb, out, err_word=err)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0] or "0")
    sampler.start()
    w0 = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    sampler.mark(w0, time.time())
    clocks = sampler.stop()
    if gdn.gdn_get_error(err) != 0:
        raise RuntimeError("device error word set during the prefill benchmark")
    us = 1e3 * e0.elapsed_time(e1) / args.steps
    units = B * L * Hv
    sm_mhz = (clocks or {}).get("sm_mhz") or 1965.0
    line = {"metric": METRIC, "workload": f"prefill B={B} L={L} Hk={Hk} Hv={Hv} dk=dv={dk}",
            "kernel": "chunked (gdn_prefill_chunked)" if args.chunked else "token steps (gdn_prefill)", "unit": UNIT,
            "value": units / (us / 1e6), "us_per_call": us, "steps": args.steps, "warmup": args.warmup,
            "clocks": clocks}
    if args.chunked:
        # I/O the method must move: q, k, v (bf16), alpha, beta, out (fp32), the initial
        # state read and the checkpoint written.  The workspace round trip (written by the
        # prepare kernel, read back by the scan) is reported beside it.
        hbm_peak, peak_kind = peaks()
        io = B * L * (2 * Hk * dk * 2 + Hv * dv * 2 + 2 * Hv * 4 + Hv * dv * 4) + 2 * B * Hv * dk * dv * 4
        ws_bytes = gdn.gdn_prefill_workspace_bytes(B, L, Hv, dk, dv)
        chunks = (L + 63) // 64
        C = 64
        # per (request, head, chunk): K K^T, Q K^T, U = T diag(beta) V, W = Tb K, [W;Q] M,
        # P E, K^T E, and the triangular inverse
        flop_chunk = 2 * C * C * dk * 2 + 2 * C * C * dv + 2 * 2 * C * dk * dv + 2 * C * C * dv * 2 \
            + 2 * C * dk * dv + C ** 3 / 3
        line["roofline"] = {"bound": "hbm", "achieved": io / us / 1e3, "peak": hbm_peak, "unit": "GB/s",
                            "frac": io / us / 1e3 / hbm_peak, "peak_kind": peak_kind, "io_bytes": io,
                            "workspace_bytes": ws_bytes,
                            "with_workspace_frac": (io + 2 * ws_bytes) / us / 1e3 / hbm_peak}
        line["chunked_tflops"] = B * Hv * chunks * flop_chunk / us / 1e6
    else:
        flops = 7.0 * dk * dv * units  # per element: 2 FMA (u, w) + 1 FMA + 1 multiply (update)
        peak_tflops = 148 * 128 * 2 * sm_mhz * 1e6 / 1e12  # fp32 FMA lanes x 2 flop x median clock
        line["roofline"] = {"bound": "alu", "achieved": flops / us / 1e6, "peak": peak_tflops, "unit": "TFLOP/s",
                            "frac": flops / us / 1e6 / peak_tflops,
                            "peak_kind": "derived: 148 SMs x 128 fp32 lanes x 2 flop x median SM clock"}
    print(json.dumps(line), flush=True)


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
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").strip()
    smi_id = vis.split(",")[local].strip() if vis else str(local)
    sampler = ClockSampler(smi_id)
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

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": elapsed_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": headline_config(args, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": traffic,
                     "peak_kind": f"{peak_kind} copy bandwidth", "kernel": kernel,
                     "bytes_per_launch": bytes_per_launch, "launch_us": launch_ms * 1e3},
        "hbm_gbs_step": step_gbs, "launch_events": launch_events, "frac_of_8tbs_step": step_gbs / 8000.0,
        "e2e": e2e, "gpu_launches": K * L, "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
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

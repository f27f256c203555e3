"""Benchmark of the select -> INT4 estimate -> top-p prune -> sparse attend decode step.

Metric: decode-attention layer-steps/s on the 32K-context GQA layer (batch 1, 32 q-heads /
8 kv-heads, head_dim 128, 16-token pages, base budget 1/4 of the pages, p = 0.85), plus the
fraction of the HBM roofline.

A bench step is one decode token through LAYERS distinct layer caches (32, the depth of a
Llama-3.1-8B stack): LAYERS calls of twl_decode_step, captured once in a CUDA graph.  Every layer
owns its own K/V/INT4/bounds/workspace buffers, so consecutive reads of one layer are
LAYERS x (touched bytes per layer-step) apart, far beyond the 126 MB L2.  The layers are copies
of one seeded synthetic layer (identical work per layer).

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun every rank runs its own LAYERS-layer stack (weak scaling, no collective on the
data path); rank 0 prints one JSON line.  --impl reference times the CPU oracle on the host cores
(rank 0 only) on a bounded sample of the same workload.
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
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import synth  # noqa: E402

METRIC = "decode attn layer-steps/s at 32K ctx (select+prune+attend); % of HBM roofline"
UNIT = "layer-steps/s"
LAYERS = 32  # default; --layers overrides (profiling runs use 1)
KERNELS_PER_LAYER_STEP = 1  # twl_decode_step is one fused kernel
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200's nominal HBM3e bandwidth, beside the measured peak


WORKLOADS = {
    "c2": ("GQA decode layer, batch 1, 32 q-heads / 8 kv-heads, head_dim 128, 32768-token "
           "context, 16-token pages, Quest budget 1/4 of pages, INT4 K (group 128), p = 0.85, "
           "eps = 1e-6, seed 0", dict(batch=1, ctx=32768)),
    "c3": ("GQA decode layer, batch 16, 32 q-heads / 8 kv-heads, head_dim 128, contexts uniform "
           "in [8192, 32768] tokens, pages randomly permuted, 16-token pages, Quest budget 1/4, "
           "INT4 K, p = 0.85, eps = 1e-6, seed 0", dict(batch=16, ctx="U[8192, 32768]")),
    "c4": ("GQA decode layer, batch 4, 32 q-heads / 8 kv-heads, head_dim 128, 131072-token "
           "context, heavy tokens in 8 spans of 512 per head, 16-token pages, Quest budget 1/4, "
           "INT4 K, p = 0.85, eps = 1e-6, seed 0", dict(batch=4, ctx=131072)),
    "c6": ("GQA decode layer, batch 64, 32 q-heads / 8 kv-heads, head_dim 128, 8192-token "
           "context, pages randomly permuted, 16-token pages, Quest budget 1/4, INT4 K, "
           "p = 0.85, eps = 1e-6, seed 0", dict(batch=64, ctx=8192)),
    "diffuse": ("GQA decode layer with diffuse heads only, batch 1, 32 q-heads / 8 kv-heads, "
                "head_dim 128, 32768-token context, no heavy tokens (sinks kept), logit "
                "temperature log-uniform in [2, 8], 16-token pages, Quest budget 1/4, INT4 K, "
                "p = 0.85, eps = 1e-6, seed 0", dict(batch=1, ctx=32768)),
}


def make_workload(name):
    return {"c2": synth.config2, "c3": synth.config3, "c4": synth.config4,
            "c6": synth.config6, "diffuse": synth.config_diffuse}[name]()


def workload_config(name="c2"):
    text, dims = WORKLOADS[name]
    return {
        "workload": text, **dims, "num_q_heads": 32, "num_kv_heads": 8, "head_dim": 128,
        "page_size": 16, "budget": "ceil(P/4) pages", "p": 0.85, "eps": 1e-6,
        "layers_per_step": LAYERS,
        "l2": f"no flush; {LAYERS} distinct layer caches per step, so each layer's touched bytes "
              f"are re-read only after {LAYERS - 1} other layers' (>> 126 MB L2)",
        "inputs": "fp16 q/K/V, INT4 K + fp16 scale/zero, fp16 page bounds",
    }


# ---------------------------------------------------------------------------------- roofline

def algorithmic_bytes(page_table, seq_lens, num_q_heads, num_kv_heads, sel_pages, sel_count,
                      union_count):
    """Unique bytes one layer-step must move (the method's roofline definition):
    page metadata (bounds 512 B per page per kv-head + 4 B page-table entry per page),
    INT4 K + scale/zero of each group's union of selected pages (1088 B per page per kv-head),
    fp16 K+V of each group's union of kept tokens (512 B per token per kv-head),
    q (256 B per head), o + lse (516 B per head), seq_lens (4 B per sequence)."""
    g = num_q_heads // num_kv_heads
    batch = len(seq_lens)
    total = 0
    parts = dict(bounds=0, page_table=0, int4=0, kv=0, q_o=0)
    for b in range(batch):
        pb = (int(seq_lens[b]) + 15) // 16
        parts["bounds"] += pb * num_kv_heads * 512
        parts["page_table"] += pb * 4
        for kvh in range(num_kv_heads):
            pages = set()
            for h in range(kvh * g, (kvh + 1) * g):
                pages.update(sel_pages[b, h, : int(sel_count[b, h])].tolist())
            parts["int4"] += len(pages) * 1088
            parts["kv"] += int(union_count[b, kvh]) * 512
    parts["q_o"] = batch * num_q_heads * (256 + 516) + 4 * batch
    total = sum(parts.values())
    return total, parts


KERNEL_SOURCES = {
    "decode_step": ["twl_step.cu", "twl_step.h", "twl_common.cuh", "twl_kernels.h"],
    "prune_rows": ["twl_prune_rows.cu", "twl_prune_rows64.cu", "twl_common.cuh", "twl_kernels.h"],
}


def source_hash(kernel: str = "decode_step") -> str:
    """Hash of the sources one kernel is built from (a profile's traffic is reported only while
    they are unchanged)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "adaptive_top_sparse_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str = "decode_step", key: str = "dram_bytes_per_layer_step"):
    """DRAM bytes per launch from the committed ncu summary, if it matches these sources."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("source_hash") != source_hash(kernel):
        return None
    return d.get(key)


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, ValueError, KeyError):
        return FALLBACK_HBM_GBS, "fallback"


def host_info(cpuinfo="/proc/cpuinfo"):
    """The host the CPU baseline ran on: logical CPUs and the CPU model name."""
    model = None
    try:
        with open(cpuinfo) as f:
            for line in f:
                if line.lower().startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "model": model}


# ---------------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        # nvidia-smi numbers GPUs physically; select ours by UUID (CUDA_VISIBLE_DEVICES-proof)
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.dev = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:  # pragma: no cover
            self.dev = str(device_index)
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return
        # nvidia-smi takes a few hundred ms to print its first row: wait for it, so that a short
        # timed region still has samples around it
        self._wait_rows(1, 5.0)

    def _rows(self) -> int:
        try:
            with open(self.path) as f:
                return sum(1 for _ in f)
        except OSError:
            return 0

    def _wait_rows(self, n: int, limit: float):
        t_end = time.monotonic() + limit
        while self._rows() < n and time.monotonic() < t_end and self.proc.poll() is None:
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self._wait_rows(self._rows() + 1, 1.0)  # one row after the timed region ends
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        with open(self.path) as f:
            out = self.summarise(f)
        os.unlink(self.path)
        return out

    @staticmethod
    def summarise(lines):
        """Median SM clock, the largest max clock and the throttle reasons seen Active, from
        nvidia-smi CSV rows in FIELDS order (rows that do not parse are skipped)."""
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------- CPU oracle

def oracle_sample(wl, groups):
    """Time the oracle's decode path (select -> estimate -> top-p -> union -> attention) on the
    given (b, kv-head) groups; cache maintenance (bounds, INT4) is prepared outside the timing,
    as it is for the GPU step."""
    from oracle import twl_oracle as O
    from tests.twl_checks import group_workload
    subs = []
    for b, kvh in groups:
        sub = group_workload(wl, b, kvh)
        bounds = O.page_bounds(sub.k, sub.page_table, sub.seq_lens)
        q4, sz = O.quantize_k(sub.k, sub.page_table, sub.seq_lens)
        subs.append((sub, bounds, q4, sz))
    t0 = time.perf_counter()
    for sub, bounds, q4, sz in subs:
        O.decode_step(sub, bounds=bounds, k_int4=q4, k_sz=sz)
    return time.perf_counter() - t0


def _oracle_worker(name, groups, reps, barrier, results):
    """One process of the all-core CPU baseline: build the workload (seeded, identical in every
    process), prepare its groups' bounds / INT4 untimed, wait for the others, then time `reps`
    passes of the oracle's decode path over its groups."""
    with cpu_threads_guard():
        from oracle import twl_oracle as O
        from tests.twl_checks import group_workload
        wl = make_workload(name)
        subs = []
        for b, kvh in groups:
            sub = group_workload(wl, b, kvh)
            subs.append((sub, O.page_bounds(sub.k, sub.page_table, sub.seq_lens),
                         *O.quantize_k(sub.k, sub.page_table, sub.seq_lens)))
        barrier.wait()
        t0 = time.perf_counter()
        for _ in range(reps):
            for sub, bounds, q4, sz in subs:
                O.decode_step(sub, bounds=bounds, k_int4=q4, k_sz=sz)
        results.put((time.perf_counter() - t0) / reps)


def oracle_all_cores(name, n_groups_total, batch, hkv, max_groups=None, reps=3):
    """The oracle's decode path split over the host's cores: one spawned process per core (BLAS
    at one thread each), each with a fixed share of the layer's (sequence, kv-head) groups, all
    started together; a layer-step takes as long as the slowest process.  At most `max_groups`
    groups are timed (the per-layer time is scaled by n_groups_total / timed groups).  Returns
    (seconds per layer-step, processes used, groups timed)."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")      # never fork a process that has touched the GPU
    all_groups = [(b, kvh) for b in range(batch) for kvh in range(hkv)]
    if max_groups is not None:
        all_groups = all_groups[:max_groups]
    nproc = max(1, min(os.cpu_count() or 1, len(all_groups)))
    shares = [all_groups[i::nproc] for i in range(nproc)]
    barrier = ctx.Barrier(nproc)
    results = ctx.Queue()
    procs = [ctx.Process(target=_oracle_worker, args=(name, sh_, reps, barrier, results))
             for sh_ in shares]
    for p_ in procs:
        p_.start()
    times = [results.get() for _ in procs]
    for p_ in procs:
        p_.join()
    per_layer = max(times) * n_groups_total / len(all_groups)
    return per_layer, nproc, len(all_groups)


def cpu_threads_guard():
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=1)
    except ImportError:  # pragma: no cover
        import contextlib
        return contextlib.nullcontext()


# ---------------------------------------------------------------------------------- arms

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_reference(args, world, rank):
    if rank != 0:
        return None
    wl = make_workload(args.workload)
    groups = [(0, 0), (0, 1)]
    with cpu_threads_guard():
        for _ in range(args.warmup):
            oracle_sample(wl, groups[:1])
        times = [oracle_sample(wl, groups) for _ in range(args.steps)]
    n_groups = wl.batch * wl.num_kv_heads
    per_layer = sum(times) / len(times) * (n_groups / len(groups))
    value = 1.0 / per_layer
    sample = (f"oracle decode path on {len(groups)} of the layer's {n_groups} (sequence, kv-head) "
              f"groups (4 q-heads each) per step, scaled x{n_groups // len(groups)} to one "
              f"layer-step")
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": per_layer * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference", "config": workload_config(args.workload),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_ours(args, world, rank, local):
    from adaptive_top_sparse_b200 import twl
    from adaptive_top_sparse_b200.layer import DecodeLayer

    dev = torch.device("cuda", local)
    wl = make_workload(args.workload)
    layers = []
    for _ in range(LAYERS):
        layer = DecodeLayer.from_workload(wl, dev)
        layer.build_aux()
        layers.append(layer)
    # every layer's q, o and lse are slices of one buffer each, so that the end-to-end pass moves
    # a step's inputs and results in one copy each way
    q_all = torch.from_numpy(np.stack([wl.q] * LAYERS)).to(dev)
    o_all = torch.zeros((LAYERS,) + tuple(layers[0].o.shape), dtype=torch.float32, device=dev)
    lse_all = torch.zeros((LAYERS,) + tuple(layers[0].lse.shape), dtype=torch.float32,
                          device=dev)
    for i, layer in enumerate(layers):
        layer.o, layer.lse = o_all[i], lse_all[i]
    qs = [q_all[i] for i in range(LAYERS)]
    stream = torch.cuda.Stream(dev)
    torch.cuda.synchronize(dev)

    # workload statistics and the roofline bytes, from one step with stats (untimed)
    stats = layers[0].alloc_stats()
    layers[0].decode(qs[0], wl.p, wl.eps, stats)
    torch.cuda.synchronize(dev)
    st = {k: v.cpu().numpy() for k, v in stats.items()}
    alg_bytes, parts = algorithmic_bytes(wl.page_table, wl.seq_lens, wl.num_q_heads,
                                         wl.num_kv_heads, st["sel_pages"], st["sel_count"],
                                         st["union_count"])
    kept = st["kept_count"].reshape(-1)
    cand = st["cand_count"].reshape(-1)

    # capture one step (LAYERS layer-steps) in a graph
    with torch.cuda.stream(stream):
        for layer, q in zip(layers, qs):          # eager warm-up on the capture stream
            layer.decode(q, wl.p, wl.eps, None, stream)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for layer, q in zip(layers, qs):
            layer.decode(q, wl.p, wl.eps, None, stream)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    barrier(world)
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, world)
    ms_per_step = ms_max / args.steps
    value = world * args.steps * LAYERS / (ms_max / 1e3)

    for layer in layers:
        s_, fl = layer.status()
        if s_ != 0:
            raise RuntimeError(f"device flags set: {fl}")

    # end to end through the public API, every step: the 32 layers' q in from pinned host memory
    # (one copy), the 32 decode calls, their o and lse out (one copy each)
    q_host = torch.empty_like(q_all, device="cpu").pin_memory()
    q_host.copy_(q_all)
    o_host = torch.empty_like(o_all, device="cpu").pin_memory()
    lse_host = torch.empty_like(lse_all, device="cpu").pin_memory()
    e2e_steps = 0 if args.no_e2e else max(1, min(args.steps, 50))

    def e2e_pass():
        q_all.copy_(q_host, non_blocking=True)
        for i, layer in enumerate(layers):
            layer.decode(qs[i], wl.p, wl.eps, None, stream)
        o_host.copy_(o_all, non_blocking=True)
        lse_host.copy_(lse_all, non_blocking=True)

    e2e_value = None
    if e2e_steps:
        with torch.cuda.stream(stream):
            for _ in range(max(1, args.warmup)):
                e2e_pass()
        torch.cuda.synchronize(dev)
        barrier(world)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(e2e_steps):
                e2e_pass()
            e1.record(stream)
        e1.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        e2e_value = world * e2e_steps * LAYERS / (e2e_ms / 1e3)
    h2d = LAYERS * wl.q.nbytes
    d2h = LAYERS * (layers[0].o.numel() * 4 + layers[0].lse.numel() * 4)

    peak, peak_kind = hbm_peak()
    layer_step_s = ms_per_step / 1e3 / LAYERS
    achieved = alg_bytes / layer_step_s / 1e9
    traffic = measured_traffic() if args.workload == "c2" else None
    metric = METRIC if args.workload == "c2" else \
        f"decode attn layer-steps/s (select+prune+attend), workload {args.workload}; % of HBM roofline"
    out = {
        "metric": metric, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(args.workload),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "twl_decode_step (whole layer-step)",
                     "alg_bytes_per_layer_step": alg_bytes, "alg_bytes_parts": parts,
                     "peak_kind": f"{peak_kind} HBM copy bandwidth",
                     "frac_of_nominal_8tbs": None},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": args.steps * LAYERS * KERNELS_PER_LAYER_STEP,
        "clocks": clk,
        "workload_stats": {
            "kept_tokens_per_head_mean": float(kept.mean()),
            "kept_tokens_per_head_min": int(kept.min()), "kept_tokens_per_head_max": int(kept.max()),
            "kept_fraction_of_candidates_mean": float((kept / np.maximum(cand, 1)).mean()),
            "union_tokens_per_group": st["union_count"].reshape(-1).tolist(),
        },
    }
    if args.p_sweep:
        # the same layers at other p: per-head kept fractions beside the time (the config's sweep)
        sweep = []
        for p in (0.70, 0.85, 0.95):
            layers[0].decode(qs[0], p, wl.eps, stats)
            torch.cuda.synchronize(dev)
            sp = {k: v.cpu().numpy() for k, v in stats.items()}
            nb, _ = algorithmic_bytes(wl.page_table, wl.seq_lens, wl.num_q_heads,
                                      wl.num_kv_heads, sp["sel_pages"], sp["sel_count"],
                                      sp["union_count"])
            frac = sp["kept_count"].reshape(-1) / np.maximum(sp["cand_count"].reshape(-1), 1)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for layer, q in zip(layers, qs):
                    layer.decode(q, p, wl.eps, None, stream)
            for _ in range(args.warmup):
                g.replay()
            torch.cuda.synchronize(dev)
            barrier(world)
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(args.steps):
                    g.replay()
                e1.record(stream)
            e1.synchronize()
            msp = max_over_ranks(e0.elapsed_time(e1), world)
            us = msp * 1e3 / (args.steps * LAYERS)
            sweep.append({
                "p": p, "us_per_layer_step": us, "layer_steps_per_s": world * 1e6 / us,
                "alg_bytes_per_layer_step": nb, "achieved_gbs": nb / us / 1e3,
                "frac": nb / us / 1e3 / peak,
                "kept_fraction_per_head": {
                    "min": float(frac.min()), "mean": float(frac.mean()),
                    "max": float(frac.max()),
                    "quartiles": [float(v) for v in np.quantile(frac, [0.25, 0.5, 0.75])]},
                "kept_tokens_per_head_mean": float(sp["kept_count"].mean())})
            del g
        out["p_sweep"] = sweep
    if rank == 0 and not args.no_cpu_baseline:
        wl_groups = [(0, 0)]
        with cpu_threads_guard():
            oracle_sample(wl, wl_groups)                    # warm
            t = oracle_sample(wl, wl_groups)
        n_groups = wl.batch * wl.num_kv_heads
        per_layer = t * n_groups / len(wl_groups)
        single = {
            "value": 1.0 / per_layer, "unit": UNIT, "cores": 1,
            "sample": f"oracle decode path (numpy, fp64) on 1 of the layer's {n_groups} "
                      f"(sequence, kv-head) groups, scaled x{n_groups} to one layer-step; "
                      f"bounds/INT4 prepared untimed"}
        cap = 16 if args.workload in ("c2", "diffuse") else 8
        per_all, nproc, timed = oracle_all_cores(args.workload, n_groups, wl.batch,
                                                 wl.num_kv_heads, max_groups=cap)
        out["cpu_baseline"] = {
            "value": 1.0 / per_all, "unit": UNIT, "cores": nproc, "kind": "oracle",
            "sample": f"oracle decode path (numpy, fp64) over {timed} of the layer's {n_groups} "
                      f"(sequence, kv-head) groups split across {nproc} spawned processes (BLAS "
                      f"one thread each, common start), scaled x{n_groups / timed:g} to one "
                      f"layer-step; bounds/INT4 prepared untimed",
            "single_core": single}
    del graph
    return out


# ---------------------------------------------------------------------------------- append step

APPEND_METRIC = "decode-step cache appends/s (K/V + INT4 K + page bounds), batch 16, 8 kv-heads"
APPEND_UNIT = "layer-appends/s"


def append_config():
    return {"workload": "one decode token appended per sequence: batch 16, 8 kv-heads, head_dim "
                        "128, 16-token pages, contexts uniform in [256, 2048] tokens, fp16 K/V",
            "batch": 16, "num_kv_heads": 8, "head_dim": 128, "page_size": 16,
            "layers_per_step": LAYERS,
            "l2": "flushed (256 MiB write, outside the events) before every timed replay"}


def append_bytes(row_is_first):
    """Unique bytes of one append per (sequence, kv-head): new K and V rows read (512 B) and
    written to the cache (512 B), the INT4 row and its scale/zero written (68 B), the page
    bounds written (512 B) and, unless the row opens the page, read (512 B); plus per sequence
    the length read and written and the page-table entry read (12 B)."""
    per_head = 512 + 512 + 68 + 512 + (0 if row_is_first else 512)
    return per_head


def run_append(args, world, rank, local):
    from adaptive_top_sparse_b200 import twl
    dev = torch.device("cuda", local)
    batch, hkv = 16, 8
    gen = torch.Generator(device="cpu").manual_seed(0)
    lens0 = torch.randint(256, 2049, (batch,), generator=gen).numpy()
    total_appends = args.warmup + args.steps + 2
    need = [-(-(int(n) + total_appends) // 16) for n in lens0]
    max_pages = max(need)
    p_phys = sum(need)
    layers = []
    for _ in range(LAYERS):
        k = torch.randn((p_phys, hkv, 16, 128), dtype=torch.float16, device=dev)
        v = torch.randn((p_phys, hkv, 16, 128), dtype=torch.float16, device=dev)
        pt = torch.full((batch, max_pages), -1, dtype=torch.int32)
        off = 0
        for b, m in enumerate(need):
            pt[b, :m] = torch.arange(off, off + m, dtype=torch.int32)
            off += m
        pt = pt.to(dev)
        n = torch.from_numpy(lens0.astype(np.int32)).to(dev)
        kv = twl.PagedKV(k, v, pt, n, hkv, p_phys)
        aux = twl.KAux(torch.zeros((p_phys, hkv, 16, 64), dtype=torch.uint8, device=dev),
                       torch.zeros((p_phys, hkv, 16, 2), dtype=torch.float16, device=dev),
                       torch.zeros((p_phys, hkv, 2, 128), dtype=torch.float16, device=dev))
        ws = twl.alloc_workspace(twl.TWL_OP_CACHE, dev)
        twl.twl_quantize_k(kv, aux.k_int4, aux.k_scale_zero, ws)
        twl.twl_page_bounds(kv, aux.bounds, ws)
        kn = torch.randn((batch, hkv, 128), dtype=torch.float16, device=dev)
        vn = torch.randn((batch, hkv, 128), dtype=torch.float16, device=dev)
        layers.append((kv, aux, ws, kn, vn, (k, v, pt, n)))
    stream = torch.cuda.Stream(dev)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):                     # eager warm-up append (one token)
        for kv, aux, ws, kn, vn, _ in layers:
            twl.twl_append_token(kv, aux, kn, vn, True, ws, stream)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for kv, aux, ws, kn, vn, _ in layers:
            twl.twl_append_token(kv, aux, kn, vn, True, ws, stream)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize(dev)
    done = 1 + args.warmup                              # tokens appended so far
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    barrier(world)
    clocks.start()
    ms = 0.0
    nbytes = 0
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    for step in range(args.steps):
        with torch.cuda.stream(stream):
            flush.fill_(step & 0xFF)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
        e1.synchronize()
        ms += e0.elapsed_time(e1)
        for b in range(batch):
            first = (int(lens0[b]) + done + step) % 16 == 0
            nbytes += LAYERS * (hkv * append_bytes(first) + 12)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    barrier(world)
    for kv, aux, ws, kn, vn, t in layers:
        st, fl = twl.twl_device_status(ws)
        if st != 0:
            raise RuntimeError(f"device flags set: {fl}")
        assert int(t[3][0].item()) == int(lens0[0]) + done + args.steps
    ms_max = max_over_ranks(ms, world)
    value = world * args.steps * LAYERS / (ms_max / 1e3)
    peak, peak_kind = hbm_peak()
    achieved = nbytes / (ms / 1e3) / 1e9
    out = {
        "metric": APPEND_METRIC, "value": value, "unit": APPEND_UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic", "config": append_config(),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": None,
                     "kernel": "twl_append_token (k_append_token)",
                     "alg_bytes_per_call": nbytes / (args.steps * LAYERS),
                     "peak_kind": f"{peak_kind} HBM copy bandwidth",
                     "frac_of_nominal_8tbs": None},
        "gpu_launches": args.steps * LAYERS, "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = append_oracle_sample(lens0, hkv, reps=20)
    del graph
    return out


def append_oracle_sample(lens0, hkv, reps):
    """The oracle's append (numpy) on the same batch and heads, over a cache of just the pages
    the appended positions touch (the per-call work is the same rows)."""
    from oracle import twl_oracle as O
    batch = len(lens0)
    rng = np.random.default_rng(0)
    n = np.array([int(x) % 16 for x in lens0], np.int64)     # same rows, one page per sequence
    pt = np.arange(batch, dtype=np.int32).reshape(batch, 1)
    k = rng.standard_normal((batch, hkv, 16, 128)).astype(np.float16)
    v = rng.standard_normal((batch, hkv, 16, 128)).astype(np.float16)
    bounds = O.page_bounds(k, pt, np.maximum(n, 1))
    q4, sz = O.quantize_k(k, pt, np.maximum(n, 1))
    kn = rng.standard_normal((batch, hkv, 128)).astype(np.float16)
    vn = rng.standard_normal((batch, hkv, 128)).astype(np.float16)
    with cpu_threads_guard():
        O.append_token(k, v, bounds, q4, sz, pt, n, kn, vn)
        t0 = time.perf_counter()
        for _ in range(reps):
            O.append_token(k, v, bounds, q4, sz, pt, n, kn, vn)
        dt = (time.perf_counter() - t0) / reps
    return {"value": 1.0 / dt, "unit": APPEND_UNIT, "cores": 1, "kind": "oracle",
            "sample": f"oracle append_token (numpy) for {batch} sequences x {hkv} kv-heads, "
                      f"{reps} calls on a one-page-per-sequence cache"}


def run_append_reference(args, world, rank):
    if rank != 0:
        return None
    gen = torch.Generator(device="cpu").manual_seed(0)
    lens0 = torch.randint(256, 2049, (16,), generator=gen).numpy()
    cb = append_oracle_sample(lens0, 8, reps=max(3, args.steps))
    return {"metric": APPEND_METRIC, "value": cb["value"], "unit": APPEND_UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 / cb["value"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": append_config(), "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": APPEND_UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------------- Quest baseline

def run_quest(args, world, rank, local):
    """Quest alone on the same layer: page selection (same budget) and attention over every
    valid token of each group's union of selected pages; no INT4 estimate, no top-p.  The union
    token lists are built once on the host from the (deterministic) selection, so their
    construction is not timed.  The pages compare this against the pruned path in
    self-attention time at batch 64."""
    from adaptive_top_sparse_b200 import twl
    from adaptive_top_sparse_b200.layer import DecodeLayer, SM_SCALE
    dev = torch.device("cuda", local)
    wl = make_workload(args.workload)
    b_, hq, hkv = wl.batch, wl.num_q_heads, wl.num_kv_heads
    g = hq // hkv
    layers = []
    toks_total = 0
    for li in range(LAYERS):
        layer = DecodeLayer.from_workload(wl, dev)
        layer.build_aux()
        mb = layer.max_budget
        sel = torch.full((b_, hq, mb), -1, dtype=torch.int32, device=dev)
        cnt = torch.zeros((b_, hq), dtype=torch.int32, device=dev)
        wss = twl.alloc_workspace(twl.TWL_OP_SELECT, dev, batch=b_, num_q_heads=hq,
                                  num_kv_heads=hkv, max_pages=layer.max_pages)
        q = torch.from_numpy(wl.q).to(dev)
        if li == 0:
            twl.twl_select_pages(q, hq, layer.kv, layer.aux.bounds, wl.budget_pages,
                                 wl.budget_div, mb, sel, cnt, None, wss)
            seln, cntn = sel.cpu().numpy(), cnt.cpu().numpy()
            stride = 16 * layer.max_pages
            tok = np.full((b_, hkv, stride), -1, np.int32)
            tcnt = np.zeros((b_, hkv), np.int32)
            for b in range(b_):
                n = int(wl.seq_lens[b])
                for kvh in range(hkv):
                    pages = sorted(set(int(x) for h in range(kvh * g, (kvh + 1) * g)
                                       for x in seln[b, h, :cntn[b, h]]))
                    t = np.concatenate([np.arange(16 * j, min(16 * j + 16, n)) for j in pages])
                    tok[b, kvh, :t.size] = t
                    tcnt[b, kvh] = t.size
            toks_total = int(tcnt.sum())
        tok_d = torch.from_numpy(tok).to(dev)
        tcnt_d = torch.from_numpy(tcnt).to(dev)
        wsa = twl.alloc_workspace(twl.TWL_OP_SPARSE_DECODE, dev, batch=b_, num_q_heads=hq,
                                  num_kv_heads=hkv, row_stride=stride)
        layers.append((layer, q, sel, cnt, wss, tok_d, tcnt_d, wsa))
    stream = torch.cuda.Stream(dev)
    torch.cuda.synchronize(dev)

    def step():
        for layer, q, sel, cnt, wss, tok_d, tcnt_d, wsa in layers:
            twl.twl_select_pages(q, hq, layer.kv, layer.aux.bounds, wl.budget_pages,
                                 wl.budget_div, layer.max_budget, sel, cnt, None, wss, stream)
            twl.twl_sparse_decode(q, hq, layer.kv, tok_d, tcnt_d, stride, SM_SCALE, layer.o,
                                  layer.lse, wsa, stream)
    with torch.cuda.stream(stream):
        step()
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    barrier(world)
    clocks.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
    e1.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    per_layer_us = ms * 1e3 / (args.steps * LAYERS)
    n_pages_total = sum((int(n) + 15) // 16 for n in wl.seq_lens)
    nbytes = n_pages_total * (hkv * 512 + 4) + toks_total * 512 + b_ * hq * (256 + 516)
    peak, peak_kind = hbm_peak()
    del graph
    return {
        "metric": f"Quest baseline layer-steps/s (select + attention over all selected tokens), "
                  f"workload {args.workload}",
        "value": world * args.steps * LAYERS / (ms / 1e3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": workload_config(args.workload),
        "roofline": {"bound": "hbm", "achieved": nbytes / per_layer_us / 1e3, "peak": peak,
                     "unit": "GB/s", "frac": nbytes / per_layer_us / 1e3 / peak,
                     "traffic": None, "kernel": "twl_select_pages + twl_sparse_decode",
                     "alg_bytes_per_layer_step": nbytes,
                     "peak_kind": f"{peak_kind} HBM copy bandwidth",
                     "frac_of_nominal_8tbs": None},
        "attended_tokens_per_layer": toks_total, "clocks": clk,
        "gpu_launches": 4 * args.steps * LAYERS,
    }


# ---------------------------------------------------------------------------------- staged

def run_staged(args, world, rank, local):
    """The same step as five separate library calls (select, estimate, prune, union, attention;
    each a flattened work list over its own grid) on the workload: the comparison against the
    one fused launch.  Algorithmic bytes as for the fused step, from the staged selections."""
    from adaptive_top_sparse_b200.layer import DecodeLayer
    dev = torch.device("cuda", local)
    wl = make_workload(args.workload)
    layers = []
    for _ in range(LAYERS):
        layer = DecodeLayer.from_workload(wl, dev)
        layer.build_aux()
        layers.append((layer.staged(), torch.from_numpy(wl.q).to(dev)))
    stream = torch.cuda.Stream(dev)
    torch.cuda.synchronize(dev)

    def step():
        for stg, q in layers:
            stg.decode(q, wl.p, wl.eps, stream)
    with torch.cuda.stream(stream):
        step()
    stream.synchronize()
    s0 = layers[0][0]
    nbytes, _ = algorithmic_bytes(wl.page_table, wl.seq_lens, wl.num_q_heads, wl.num_kv_heads,
                                  s0.sel.cpu().numpy(), s0.sel_count.cpu().numpy(),
                                  s0.union_count.cpu().numpy())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    barrier(world)
    clocks.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
    e1.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    per_layer_us = ms * 1e3 / (args.steps * LAYERS)
    peak, peak_kind = hbm_peak()
    del graph
    return {
        "metric": f"staged path layer-steps/s (five library calls per layer-step), "
                  f"workload {args.workload}",
        "value": world * args.steps * LAYERS / (ms / 1e3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": workload_config(args.workload),
        "roofline": {"bound": "hbm", "achieved": nbytes / per_layer_us / 1e3, "peak": peak,
                     "unit": "GB/s", "frac": nbytes / per_layer_us / 1e3 / peak,
                     "traffic": None, "kernel": "twl_select_pages + twl_estimate + "
                     "twl_prune_top_p + twl_group_union + twl_sparse_decode",
                     "alg_bytes_per_layer_step": nbytes,
                     "peak_kind": f"{peak_kind} HBM copy bandwidth",
                     "frac_of_nominal_8tbs": None},
        "clocks": clk,
    }


# ---------------------------------------------------------------------------------- Double-P

def run_double_p(args, world, rank, local, p_cluster=0.95):
    """The two-level top-p step (cluster-level top-p over page centroids, then the token-level
    path on the kept pages; five library calls) on the workload.  Algorithmic
    bytes: centroids (256 B per page per kv-head) + page table, INT4 K of each group's union
    of kept pages, fp16 K/V of the union of kept tokens, q and o/lse."""
    from adaptive_top_sparse_b200.layer import DecodeLayer
    dev = torch.device("cuda", local)
    wl = make_workload(args.workload)
    b_, hq, hkv = wl.batch, wl.num_q_heads, wl.num_kv_heads
    g = hq // hkv
    layers = []
    for _ in range(LAYERS):
        layer = DecodeLayer.from_workload(wl, dev)
        layer.build_aux()
        dp = layer.double_p()
        dp.build_centroids()
        layers.append((dp, torch.from_numpy(wl.q).to(dev)))
    stream = torch.cuda.Stream(dev)
    torch.cuda.synchronize(dev)

    def step():
        for dp, q in layers:
            dp.decode(q, p_cluster, wl.p, wl.eps, stream)
    with torch.cuda.stream(stream):
        step()
    stream.synchronize()
    dp0 = layers[0][0]
    seln, cntn = dp0.sel.cpu().numpy(), dp0.sel_count.cpu().numpy()
    ucnt = dp0.union_count.cpu().numpy()
    pages_union = 0
    for b in range(b_):
        for kvh in range(hkv):
            pages = set()
            for h in range(kvh * g, (kvh + 1) * g):
                pages.update(seln[b, h, :cntn[b, h]].tolist())
            pages_union += len(pages)
    n_pages_total = sum((int(n) + 15) // 16 for n in wl.seq_lens)
    nbytes = (n_pages_total * (hkv * 256 + 4) + pages_union * 1088 + int(ucnt.sum()) * 512 +
              b_ * hq * (256 + 516))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    barrier(world)
    clocks.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
    e1.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    per_layer_us = ms * 1e3 / (args.steps * LAYERS)
    peak, peak_kind = hbm_peak()
    del graph
    return {
        "metric": f"two-level top-p (cluster top-p p_c = {p_cluster}, then token top-p) "
                  f"layer-steps/s, workload {args.workload}",
        "value": world * args.steps * LAYERS / (ms / 1e3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": workload_config(args.workload),
        "roofline": {"bound": "hbm", "achieved": nbytes / per_layer_us / 1e3, "peak": peak,
                     "unit": "GB/s", "frac": nbytes / per_layer_us / 1e3 / peak,
                     "traffic": None, "kernel": "twl_select_clusters_top_p + twl_estimate + "
                     "twl_prune_top_p + twl_group_union + twl_sparse_decode",
                     "alg_bytes_per_layer_step": nbytes,
                     "peak_kind": f"{peak_kind} HBM copy bandwidth",
                     "frac_of_nominal_8tbs": None},
        "kept_pages_per_head_mean": float(cntn.mean()), "pages_per_head": n_pages_total // b_,
        "union_tokens_per_group": ucnt.reshape(-1).tolist(), "clocks": clk,
        "gpu_launches": 9 * args.steps * LAYERS,
    }


# ---------------------------------------------------------------------------------- pruner rows

PRUNE_ROWS = 4096
PRUNE_EPS = 1e-6
L2_BYTES = 126 * 1024 * 1024


def prune_rows_config(ns, copies):
    return {"workload": "standalone top-p pruner: 4096 fp32 weight rows of length n (half "
                        "Gaussian logits, sigma log-uniform in [0.1, 6]; half Zipf rank profiles, "
                        "s in [0.5, 2]; 1% of rows with exact ties), softmax-normalised, "
                        "p in {0.8, 0.9}, eps = 1e-6, seed 0",
            "rows": PRUNE_ROWS, "n": ns, "p": [0.8, 0.9], "eps": PRUNE_EPS,
            "l2": "no flush; each timed launch reads a copy of the rows not read since "
                  f">= 4 x L2 bytes (copies per n: {copies})"}


def prune_rows_bytes(n, rows, kept_total, with_idx):
    """Read-once bytes of one launch: every weight (4 B), m and the kept count out (8 B per
    row), and 4 B per kept index when the indices are written."""
    return rows * (4 * n + 8) + (4 * kept_total if with_idx else 0)


def run_prune_rows(args, world, rank, local):
    """twl_prune_top_p alone on the standalone-pruner workload (4096 rows x n fp32 weights),
    against its read-once HBM bound."""
    from adaptive_top_sparse_b200 import twl
    dev = torch.device("cuda", local)
    ns = [int(x) for x in args.prune_n.split(",")]
    peak, peak_kind = hbm_peak()
    stream = torch.cuda.Stream(dev)
    sweep = []
    copies_by_n = {}
    launches = 0
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    e2e = None
    for n in ns:
        w_np, _ = synth.config5_rows(PRUNE_ROWS, n, seed=0)
        nbytes_in = w_np.nbytes
        copies = max(1, -(-4 * L2_BYTES // nbytes_in))
        copies_by_n[n] = copies
        ws = [torch.from_numpy(w_np).to(dev) for _ in range(copies)]
        sample = np.linspace(0, PRUNE_ROWS - 1, 8).astype(int)
        w_sample = w_np[sample].copy()
        m = torch.zeros(PRUNE_ROWS, dtype=torch.float32, device=dev)
        kc = torch.zeros(PRUNE_ROWS, dtype=torch.int32, device=dev)
        ki = torch.empty((PRUNE_ROWS, n), dtype=torch.int32, device=dev)
        for p in (0.8, 0.9):
            for with_idx in (False, True):
                def step():
                    for w in ws:
                        twl.twl_prune_top_p(w, None, PRUNE_ROWS, n, p, PRUNE_EPS, m, kc,
                                            ki if with_idx else None, stream=stream)
                with torch.cuda.stream(stream):
                    step()
                stream.synchronize()
                # properties that hold at any size: kept = {W >= m}, mass >= p (up to fp32 sums)
                mn, kcn = m.cpu().numpy(), kc.cpu().numpy()
                kin = ki[torch.from_numpy(sample).to(dev)].cpu().numpy() if with_idx else None
                for j, r in enumerate(sample):
                    keep = np.nonzero(w_sample[j] >= mn[r])[0]
                    assert keep.size == kcn[r], f"n={n} row {r}: count"
                    assert float(w_sample[j][keep].astype(np.float64).sum()) >= p - 1e-5
                    if with_idx:
                        assert np.array_equal(kin[j, : keep.size], keep), f"n={n} row {r}: ids"
                kept_total = int(kcn.astype(np.int64).sum())
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph, stream=stream):
                    step()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    e0.record(stream)
                    for _ in range(args.warmup):
                        graph.replay()
                    e1.record(stream)
                e1.synchronize()
                # at least K replays, and at least half a second so the clock record has samples
                per_replay = e0.elapsed_time(e1) / args.warmup
                reps = int(max(args.steps, math.ceil(500.0 / max(per_replay, 1e-3))))
                reps = int(max_over_ranks(float(reps), world))
                torch.cuda.synchronize(dev)
                barrier(world)
                clocks.start()
                with torch.cuda.stream(stream):
                    e0.record(stream)
                    for _ in range(reps):
                        graph.replay()
                    e1.record(stream)
                e1.synchronize()
                clk = clocks.stop()
                ms = max_over_ranks(e0.elapsed_time(e1), world)
                launches += reps * copies
                us = ms * 1e3 / (reps * copies)
                nb = prune_rows_bytes(n, PRUNE_ROWS, kept_total, with_idx)
                sweep.append({"n": n, "p": p, "kept_idx": with_idx, "replays": reps,
                              "launches_per_replay": copies, "us_per_launch": us,
                              "rows_per_s": world * PRUNE_ROWS / (us / 1e6),
                              "alg_bytes": nb, "achieved_gbs": nb / us / 1e3,
                              "frac": nb / us / 1e3 / peak,
                              "kept_fraction": kept_total / (PRUNE_ROWS * n), "clocks": clk})
                del graph
        if n == ns[-1] and not args.no_e2e:
            # end to end through the C ABI: pinned host rows in, m and counts out, every step
            w_host = torch.from_numpy(w_np).pin_memory()
            m_host = torch.empty(PRUNE_ROWS, dtype=torch.float32).pin_memory()
            kc_host = torch.empty(PRUNE_ROWS, dtype=torch.int32).pin_memory()
            e2e_steps = 3
            with torch.cuda.stream(stream):
                ws[0].copy_(w_host, non_blocking=True)
                twl.twl_prune_top_p(ws[0], None, PRUNE_ROWS, n, 0.9, PRUNE_EPS, m, kc,
                                    None, stream=stream)
                stream.synchronize()
                barrier(world)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(e2e_steps):
                    ws[0].copy_(w_host, non_blocking=True)
                    twl.twl_prune_top_p(ws[0], None, PRUNE_ROWS, n, 0.9, PRUNE_EPS, m, kc,
                                        None, stream=stream)
                    m_host.copy_(m, non_blocking=True)
                    kc_host.copy_(kc, non_blocking=True)
                e1.record(stream)
            e1.synchronize()
            launches += e2e_steps
            ms = max_over_ranks(e0.elapsed_time(e1), world)
            e2e = {"value": world * e2e_steps * PRUNE_ROWS / (ms / 1e3), "unit": "rows/s",
                   "h2d_bytes_per_step": nbytes_in, "d2h_bytes_per_step": 8 * PRUNE_ROWS,
                   "steps": e2e_steps, "n": n, "p": 0.9}
            del w_host
        del ws, ki
        torch.cuda.empty_cache()
    head = [r for r in sweep if r["n"] == ns[-1] and r["p"] == 0.9 and not r["kept_idx"]][0]
    out = {
        "metric": f"top-p pruner rows/s, 4096 fp32 rows of n = {ns[-1]}, p = 0.9, threshold and "
                  "kept count (twl_prune_top_p); % of the read-once HBM roofline",
        "value": head["rows_per_s"], "unit": "rows/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["us_per_launch"] / 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": prune_rows_config(ns, copies_by_n),
        "roofline": {"bound": "hbm", "achieved": head["achieved_gbs"], "peak": peak,
                     "unit": "GB/s", "frac": head["frac"],
                     "traffic": measured_traffic("prune_rows", f"dram_bytes_per_launch_n{ns[-1]}"),
                     "kernel": "k_prune_rows (twl_prune_top_p)",
                     "alg_bytes_per_launch": head["alg_bytes"],
                     "peak_kind": f"{peak_kind} HBM copy bandwidth",
                     "frac_of_nominal_8tbs": None},
        "e2e": e2e, "gpu_launches": launches, "clocks": head["clocks"], "sweep": sweep,
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = prune_rows_cpu(ns[-1], 0.9)
    return out


def prune_rows_cpu(n, p, budget_s=10.0):
    """The oracle's sort-based top-p (one host core) on rows of the same workload, until about
    budget_s seconds of work; rows/s."""
    from oracle import twl_oracle as O
    w_np, _ = synth.config5_rows(64, n, seed=0)
    done, t = 0, 0.0
    with cpu_threads_guard():
        while t < budget_s and done < w_np.shape[0]:
            t0 = time.perf_counter()
            O.top_p_sort(w_np[done], p)
            t += time.perf_counter() - t0
            done += 1
    return {"value": done / t, "unit": "rows/s", "cores": 1, "kind": "oracle",
            "sample": f"oracle sort + cumulative-sum top-p (numpy, fp64 sums) on {done} rows of "
                      f"the n = {n} workload (same generator, seed 0), p = {p}, one host core"}


def run_prune_rows_reference(args, world, rank):
    if rank != 0:
        return None
    ns = [int(x) for x in args.prune_n.split(",")]
    cb = prune_rows_cpu(ns[-1], 0.9, budget_s=min(60.0, 2.0 * max(1, args.steps)))
    return {
        "metric": f"top-p pruner rows/s, 4096 fp32 rows of n = {ns[-1]}, p = 0.9, threshold and "
                  "kept count (twl_prune_top_p); % of the read-once HBM roofline",
        "value": cb["value"], "unit": "rows/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * PRUNE_ROWS / cb["value"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference", "config": prune_rows_config(ns, {}),
        "cpu_baseline": cb,
        "e2e": {"value": cb["value"], "unit": "rows/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------------- bit widths

def run_bits(args, world, rank, local):
    """The staged estimate (union, dequant-dot, softmax) on the 32K-context layer at 2, 4 and 8
    bits: time per call, and the roofline over the codes + scale/zero of the
    groups' union pages (16 rows x (16 bits + 4) bytes per page per kv-head)."""
    from adaptive_top_sparse_b200 import twl
    from adaptive_top_sparse_b200.layer import DecodeLayer
    dev = torch.device("cuda", local)
    wl = synth.config2()
    b, hq, hkv = wl.batch, wl.num_q_heads, wl.num_kv_heads
    layers = []
    for _ in range(LAYERS):
        layer = DecodeLayer.from_workload(wl, dev)
        layer.build_aux()
        mb = layer.max_budget
        sel = torch.full((b, hq, mb), -1, dtype=torch.int32, device=dev)
        cnt = torch.zeros((b, hq), dtype=torch.int32, device=dev)
        ws = twl.alloc_workspace(twl.TWL_OP_ESTIMATE, dev, batch=b, num_q_heads=hq,
                                 num_kv_heads=hkv, max_pages=layer.max_pages, max_budget=mb)
        wss = twl.alloc_workspace(twl.TWL_OP_SELECT, dev, batch=b, num_q_heads=hq,
                                  num_kv_heads=hkv, max_pages=layer.max_pages)
        q = torch.from_numpy(wl.q).to(dev)
        twl.twl_select_pages(q, hq, layer.kv, layer.aux.bounds, 0, wl.budget_div, mb, sel, cnt,
                             None, wss)
        out = (torch.zeros((b, hq, 16 * mb), dtype=torch.float32, device=dev),
               torch.zeros((b, hq, 16 * mb), dtype=torch.int32, device=dev),
               torch.zeros((b, hq), dtype=torch.int32, device=dev))
        codes = {}
        for bits in (2, 4, 8):
            kq = torch.zeros((layer.k.shape[0], hkv, 16, 16 * bits), dtype=torch.uint8,
                             device=dev)
            sz = torch.zeros((layer.k.shape[0], hkv, 16, 2), dtype=torch.float16, device=dev)
            twl.twl_quantize_k_nbit(layer.kv, bits, kq, sz, ws)
            codes[bits] = (kq, sz)
        layers.append((layer, q, sel, cnt, ws, out, codes))
    torch.cuda.synchronize(dev)
    seln, cntn = layers[0][2].cpu().numpy(), layers[0][3].cpu().numpy()
    union_pages = 0
    g = hq // hkv
    for kvh in range(hkv):
        pages = set()
        for h in range(kvh * g, (kvh + 1) * g):
            pages.update(seln[0, h, :cntn[0, h]].tolist())
        union_pages += len(pages)
    stream = torch.cuda.Stream(dev)
    peak, peak_kind = hbm_peak()
    variants = {}
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    clocks.start()
    for bits in (2, 4, 8):
        def step():
            for layer, q, sel, cnt, ws, (w, tok, cc), codes in layers:
                kq, sz = codes[bits]
                twl.twl_estimate_nbit(q, hq, layer.kv, bits, kq, sz, sel, cnt, layer.max_budget,
                                      w, tok, cc, ws, stream)
        with torch.cuda.stream(stream):
            step()
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            e1.record(stream)
        e1.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (args.steps * LAYERS)
        nbytes = union_pages * 16 * (16 * bits + 4)
        variants[str(bits)] = {"us_per_layer": us, "layer_steps_per_s": 1e6 / us,
                               "alg_bytes": nbytes, "achieved_gbs": nbytes / us / 1e3,
                               "frac": nbytes / us / 1e3 / peak}
        del graph
    clk = clocks.stop()
    v4 = variants["4"]
    return {
        "metric": "staged estimate layer-steps/s (union + dequant-dot + softmax), 32K-context "
                  "layer, INT4 (2- and 8-bit variants beside it)",
        "value": v4["layer_steps_per_s"], "unit": "layer-steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": v4["us_per_layer"] * LAYERS / 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": workload_config("c2"),
        "roofline": {"bound": "hbm", "achieved": v4["achieved_gbs"], "peak": peak, "unit": "GB/s",
                     "frac": v4["frac"], "traffic": None,
                     "kernel": "twl_estimate_nbit (3 launches)",
                     "peak_kind": f"{peak_kind} HBM copy bandwidth",
                     "frac_of_nominal_8tbs": None},
        "variants": variants, "union_pages": union_pages, "clocks": clk,
        "gpu_launches": 3 * 3 * args.steps * LAYERS,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--double-p", action="store_true",
                    help="time the two-level (cluster, then token) top-p path on the workload")
    ap.add_argument("--staged", action="store_true",
                    help="time the step as its five staged library calls instead of the fused "
                         "launch (a comparison, not the headline)")
    ap.add_argument("--quest", action="store_true",
                    help="time the Quest baseline (select + attention over every token of the "
                         "selected pages, no estimate or top-p) on the workload instead")
    ap.add_argument("--layers", type=int, default=None,
                    help="layer caches per step (default 32 for c2 and append, 4 for c3 / c4)")
    ap.add_argument("--workload", default="c2",
                    choices=["c2", "c3", "c4", "c6", "diffuse", "append", "bits", "c5"],
                    help="c2 is the headline; c3 / c4 / c6, the append step, the estimator bit "
                         "widths and the standalone pruner (c5) are extra reports")
    ap.add_argument("--p-sweep", action="store_true",
                    help="also time the decode workload at p = 0.70, 0.85, 0.95 and report the "
                         "per-head kept fractions (the long-context config's sweep)")
    ap.add_argument("--prune-n", default="8192,32768,131072",
                    help="row lengths of the c5 pruner workload (the last one is the headline)")
    args = ap.parse_args()
    global LAYERS
    if args.layers is None:
        args.layers = 4 if args.workload in ("c3", "c4", "c6") else 32
    LAYERS = max(1, args.layers)
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup(args)
    try:
        if args.workload == "c5":
            out = (run_prune_rows_reference(args, world, rank) if args.impl == "reference"
                   else run_prune_rows(args, world, rank, local))
        elif args.workload == "bits":
            out = run_bits(args, world, rank, local) if args.impl == "ours" else None
        elif args.workload == "append":
            out = (run_append_reference(args, world, rank) if args.impl == "reference"
                   else run_append(args, world, rank, local))
        elif args.double_p:
            out = run_double_p(args, world, rank, local)
        elif args.staged:
            out = run_staged(args, world, rank, local)
        elif args.quest:
            out = run_quest(args, world, rank, local)
        elif args.impl == "reference":
            out = run_reference(args, world, rank)
        else:
            out = run_ours(args, world, rank, local)
        if rank == 0 and out is not None:
            roof = out.get("roofline")
            if roof and roof.get("unit") == "GB/s" and roof.get("achieved") is not None:
                roof["frac_of_nominal_8tbs"] = roof["achieved"] / NOMINAL_HBM_GBS
            if isinstance(out.get("cpu_baseline"), dict):
                out["cpu_baseline"]["host"] = host_info()
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the paged decode step on B200.

One step = one pass of the whole hot path over one batch: the block
manager's slot/copy-on-write decisions for one appended token per sequence
(precomputed on the host before timing), the copy-on-write block copies,
the KV-append scatter, and split-context decode attention (partition kernel
plus log-sum-exp merge) over the paged cache.

Headline workload (N=1 default): long-context split decode: batch 8, context
131072 tokens each, 64 query heads over 8 KV heads, head_dim 128, bf16,
block size 16, 512-token partitions, pool 10% larger than needed and placed
by a seeded shuffle, values N(0, 1); the largest single-GPU configuration
(~4.3 GB of KV read per step). The per-step inputs (queries, new K/V, slots,
block tables, lengths) of R consecutive decode steps are made ahead of time
and cycled; every step does the full work of a real decode step at its
context lengths. The KV bytes a step reads exceed the 126 MB L2, so no
flush is needed.

value      = algorithmic bytes of the step (valid K/V tokens + q + out + block
             table entries + lengths + append + copies) / device time, GB/s,
             summed over ranks, time = max over ranks (CUDA events). Timed in
             repeats of --steps steps until --min-seconds of device time;
             value is the median over repeats.
roofline   = the decode call alone (partition kernel + merge), its algorithmic
             bytes / its event-timed duration, against the measured HBM peak.
configs    = (one GPU) the same numbers for the other configurations: block
             size 32, MHA batch 64, GQA batch 256, and both prefix-sharing
             workloads on the split route and on the shared-prefix route.
e2e        = the same metric through the public API from pinned host buffers:
             per step the host block manager step, H2D of the step's inputs,
             the kernels, D2H of the output.
cpu_baseline / --impl reference: the CPU oracle (float64 NumPy) timed on a
             bounded sample of the same workload on the host cores.

Multi-GPU (torchrun): every rank runs its own independent batch (different
seed), no data-path collective; scaling is weak.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode attention: KV GB/s achieved & % of B200 HBM peak; decode tokens/s"
FALLBACK_HBM_GBS = 6650.0


# ---------------------------------------------------------------------------
# workload selection and byte accounting

def make_workload(name: str, rank: int, batch: int | None = None):
    from paged_kv_cache_336_b200 import workloads
    if name == "mha":
        if batch:   # smaller pool for profiling captures: room for the batch plus growth
            w = workloads.mha(repeat=rank, batch=batch)
            need = int(np.sum((w.context_lens + 300) // w.block_size + 1))
            w.num_blocks = need
            w.free_order = np.random.default_rng(w.seed).permutation(need).astype(np.int32)
            return w
        return workloads.mha(repeat=rank)
    if name == "gqa":
        return workloads.gqa(repeat=rank)
    if name == "prefix":
        return workloads.prefix(repeat=rank)
    if name == "prefix_cow":
        return workloads.prefix_cow(repeat=rank)
    if name == "long16":
        return workloads.long(repeat=rank, block_size=16, slack=0.1, batch=batch or 8)
    if name == "long32":
        return workloads.long(repeat=rank, block_size=32, slack=0.1, batch=batch or 8)
    if name == "tiny":
        return workloads.tiny(repeat=rank)
    raise SystemExit(f"unknown workload {name}")


def workload_label(w) -> str:
    return (f"{w.name}: batch {len(w.decode_seqs)}, {w.num_q_heads}q/{w.num_kv_heads}kv heads, "
            f"head_dim {w.head_dim}, {w.dtype}, block {w.block_size}")


def decode_bytes(w, ctx: np.ndarray) -> int:
    """Algorithmic bytes of one decode call: valid K and V tokens, q, out,
    the block-table entries read and the context lengths."""
    e = w.elt_bytes
    kv = int(np.sum(ctx)) * w.num_kv_heads * w.head_dim * e * 2
    qo = 2 * len(ctx) * w.num_q_heads * w.head_dim * e
    bt = int(np.sum((ctx + w.block_size - 1) // w.block_size)) * 4 + 4 * len(ctx)
    return kv + qo + bt


def unique_decode_bytes(w, ctx: np.ndarray, skip: np.ndarray, group_blocks) -> int:
    """Bytes a shared-prefix decode must read at least: each group's shared
    blocks once, every sequence's own tokens, plus q, out, tables, lengths."""
    per_token = w.num_kv_heads * w.head_dim * w.elt_bytes * 2
    kv = (int(np.sum(group_blocks)) * w.block_size +
          int(np.sum(ctx - skip * w.block_size))) * per_token
    return kv + decode_bytes(w, ctx) - int(np.sum(ctx)) * per_token


def append_bytes(w, num_tokens: int) -> int:
    per = num_tokens * w.num_kv_heads * w.head_dim * w.elt_bytes * 2
    return 2 * per + 8 * num_tokens   # read new K/V, write them, read slots


def copy_bytes(w, num_pairs: int) -> int:
    block = w.num_kv_heads * w.block_size * w.head_dim * w.elt_bytes
    return num_pairs * (2 * 2 * block + 16)


def reduce_over_ranks(local_ms: float, local_bytes: float, local_tokens: float, device):
    """Job-wide (time, bytes, tokens): the slowest rank's time, everything
    else summed. A single process returns its own values."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(local_ms), float(local_bytes), float(local_tokens)
    t = torch.tensor([float(local_ms)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    b = torch.tensor([float(local_bytes), float(local_tokens)], device=device, dtype=torch.float64)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    return float(t.item()), float(b[0].item()), float(b[1].item())


# ---------------------------------------------------------------------------
# measured peaks, clocks, profile traffic

def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def gpu_uuid(device_index: int) -> str | None:
    """The GPU's UUID in NVML / nvidia-smi form ("GPU-..."), which names the
    physical device whatever CUDA_VISIBLE_DEVICES says."""
    try:
        import torch
        u = str(torch.cuda.get_device_properties(device_index).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


class ClockSampler:
    """SM clock and clock-event-reason samples while a timed region runs
    (read-only NVML queries from a background thread; nvidia-smi if NVML is
    not importable). The device is found by UUID, so the samples come from
    the GPU this process runs on."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.05):
        self.uuid = gpu_uuid(device_index)
        self.period_s = period_s
        self.samples = []     # (sm_mhz, sm_max_mhz, reasons bitmask, power W)
        self._thread = None
        self._stop = None
        self._proc = None

    def _nvml_loop(self, handle, nvml):
        while True:
            try:
                sm = nvml.nvmlDeviceGetClockInfo(handle, nvml.NVML_CLOCK_SM)
                mx = nvml.nvmlDeviceGetMaxClockInfo(handle, nvml.NVML_CLOCK_SM)
                rs = nvml.nvmlDeviceGetCurrentClocksEventReasons(handle)
                pw = nvml.nvmlDeviceGetPowerUsage(handle) / 1000.0
                self.samples.append((float(sm), float(mx), int(rs), pw))
            except Exception:
                pass
            if self._stop.wait(self.period_s):
                return

    def start(self):
        import threading
        self.samples = []
        try:
            import pynvml as nvml
            nvml.nvmlInit()
            handle = nvml.nvmlDeviceGetHandleByUUID(self.uuid)
            self._stop = threading.Event()
            self._thread = threading.Thread(target=self._nvml_loop, args=(handle, nvml), daemon=True)
            self._thread.start()
            return
        except Exception:
            self._thread = None
        if self.uuid is None:
            return
        try:
            fields = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,power.draw")
            self._fh = tempfile.TemporaryFile(mode="w+")
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.uuid}", f"--query-gpu={fields}",
                 "--format=csv,noheader,nounits", "-lms", str(int(self.period_s * 1000))],
                stdout=self._fh, stderr=subprocess.DEVNULL)
        except Exception:
            self._proc = None

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
            self._thread = None
        elif self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except Exception:
                self._proc.kill()
            self._fh.seek(0)
            for line in self._fh:
                parts = [p.strip() for p in line.split(",")]
                try:
                    self.samples.append((float(parts[0]), float(parts[1]), int(parts[2], 16),
                                         float(parts[3])))
                except Exception:
                    pass
            self._fh.close()
            self._proc = None
        if not self.samples:
            return None
        sm = [x[0] for x in self.samples]
        reasons = sorted({name for x in self.samples for bit, name in self.REASONS.items()
                          if x[2] & bit})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(x[1] for x in self.samples),
                "reasons": reasons, "samples": len(self.samples),
                "power_w_median": round(statistics.median(x[3] for x in self.samples), 1),
                "source": "nvml" if self._stop is not None else "nvidia-smi",
                "gpu": self.uuid}


DECODE_SOURCES = ("decode_kernel.cuh", "decode_stream_kernel.cuh", "device_common.cuh")
PREFIX_SOURCES = ("prefix_kernel.cuh", "decode_kernel.cuh", "decode_stream_kernel.cuh",
                  "device_common.cuh")
PREFILL_SOURCES = ("tc_prefill_kernel.cuh", "prefill_kernel.cuh", "device_common.cuh")


def kernel_source_hash(names=DECODE_SOURCES) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_336_b200", "csrc")
    for name in names:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kind: str = "decode", sources=None, mode: str = "split",
                     algorithmic: float | None = None):
    """DRAM bytes per call from the committed ncu summary
    profiles/<kind>_<workload>_traffic.txt (decode calls of another route:
    <route>_<workload>_traffic.txt), if it was taken on the current kernel
    source and (when `algorithmic` is given) on a call of the same
    algorithmic bytes, within 5% (the bench cycles decode states whose
    contexts grow a token per step; a smaller --batch of the same workload
    differs several-fold); else None."""
    if kind == "decode" and mode != "split":
        kind = mode
    if sources is None:
        sources = PREFIX_SOURCES if kind == "shared_prefix" else DECODE_SOURCES
    path = os.path.join(ROOT, "profiles", f"{kind}_{workload}_traffic.txt")
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if ":" in line and not line.lstrip().startswith("#"):
                    k, v = line.split(":", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("kernel_source_sha256_16") != kernel_source_hash(sources):
            return None
        dram = int(kv["dram_bytes_per_launch"])
        if algorithmic is not None and "traffic_over_algorithmic" in kv:
            captured = dram / float(kv["traffic_over_algorithmic"])
            if abs(captured - algorithmic) > 0.05 * algorithmic:
                return None
        return dram
    except Exception:
        return None


# ---------------------------------------------------------------------------
# the CUDA path

class DeviceStep:
    """Device-resident inputs of R consecutive decode steps, cycled."""

    def __init__(self, w, states: int, partition_tokens: int, device, mode: str = "split",
                 window: int = 0):
        import torch
        from paged_kv_cache_336_b200 import binding, workloads
        self.torch, self.binding = torch, binding
        self.w = w
        self.partition_tokens = partition_tokens
        self.mode = mode
        self.window = window
        self.whole = mode == "whole"
        self.bm = binding.BlockManager(w.num_blocks, w.block_size, w.max_blocks_per_seq,
                                       w.free_order)
        for s in w.prefill_seqs:
            self.bm.allocate(s, int(w.context_lens[s]))
        for parent, child in w.forks:
            self.bm.fork(parent, child)
        for s, n in sorted(w.extra_tokens.items()):
            for _ in range(n):
                self.bm.append_slot(s)
        self.k_pool, self.v_pool = workloads.draw_pools(w, device)
        B = len(w.decode_seqs)
        T = len(w.step_seqs)
        self.B, self.T = B, T
        self.states = []
        for i in range(states):
            st = {}
            if T:
                slots, pairs = self.bm.append_slots_arrays(w.step_seqs)
            else:
                slots, pairs = np.zeros(0, np.int64), np.zeros((0, 2), np.int64)
            tables, ctx = self.bm.export(w.decode_seqs)
            st["slots"] = torch.from_numpy(slots).to(device)
            st["pairs"] = torch.from_numpy(pairs).to(device)
            st["tables"] = torch.from_numpy(tables).to(device)
            st["ctx"] = torch.from_numpy(ctx).to(device)
            st["q"] = workloads.draw_queries(w, B, step=i, device=device)
            kn, vn = workloads.draw_new_kv(w, max(T, 1), step=i, device=device)
            st["k_new"], st["v_new"] = kn[:T].contiguous(), vn[:T].contiguous()
            st["ctx_np"] = ctx.astype(np.int64)
            st["n_pairs"] = int(pairs.shape[0])
            st["decode_bytes"] = decode_bytes(w, st["ctx_np"])
            if mode == "window":   # only the last `window` tokens are read
                st["decode_bytes"] = decode_bytes(w, np.minimum(st["ctx_np"], self.window))
            st["unique_bytes"] = st["decode_bytes"]
            if mode == "shared_prefix":
                offs, members, gblocks = self.bm.prefix_groups(w.decode_seqs)
                st["groups"] = (offs, members, gblocks)
                skip = np.zeros(len(w.decode_seqs), dtype=np.int64)
                for g in range(len(gblocks)):
                    skip[members[offs[g]:offs[g + 1]]] = gblocks[g]
                st["unique_bytes"] = unique_decode_bytes(w, st["ctx_np"], skip, gblocks)
            st["step_bytes"] = (st["decode_bytes"] + append_bytes(w, T) + copy_bytes(w, st["n_pairs"]))
            self.states.append(st)
        self.out = torch.empty_like(self.states[0]["q"])
        if mode == "shared_prefix":
            self.ws = binding.shared_prefix_workspace(B, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                                      w.block_size, w.max_blocks_per_seq,
                                                      partition_tokens, device)
        else:
            self.ws = binding.SplitWorkspace(B, w.num_q_heads, w.head_dim, w.block_size,
                                             w.max_blocks_per_seq, partition_tokens, device)
        pb = partition_tokens // w.block_size
        self.merge_launched = (-(-w.max_blocks_per_seq // pb) > 1 or mode == "shared_prefix") \
            and mode != "whole"

    def launches(self, st) -> int:
        # shared prefix: the prefix kernel, and the scatter kernel that
        # carries the call's plan (the bench's plans are far below 30 KB)
        prefix = 2 if (self.mode == "shared_prefix" and len(st["groups"][2])) else 0
        return ((1 if st["n_pairs"] else 0) + (1 if self.T else 0) + 1 + prefix +
                (1 if self.merge_launched else 0))

    def _writes(self, st):
        b = self.binding
        if st["n_pairs"]:
            b.copy_blocks(self.k_pool, self.v_pool, st["pairs"])
        if self.T:
            b.kv_append(st["k_new"], st["v_new"], st["slots"], self.k_pool, self.v_pool)

    def capture(self) -> str | None:
        """Captures each state's step as two CUDA graphs (the copies and
        append; the decode call), so that a timed step costs two graph
        launches of host time instead of several library calls. Returns None
        on success, else why the step stays eager. A shared-prefix call
        carries its host-built plan in the graph (plans of up to 30 KB go up
        as kernel parameters); the library refuses the capture of a larger
        plan, and the step then stays eager."""
        torch = self.torch
        graphs = []
        try:
            torch.cuda.synchronize()
            for st in self.states:
                g_w = None
                if st["n_pairs"] or self.T:
                    g_w = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g_w):
                        self._writes(st)
                g_d = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g_d):
                    self._decode(st)
                graphs.append((g_w, g_d))
            torch.cuda.synchronize()
        except Exception as e:  # capture refused: stay eager, say why
            torch.cuda.synchronize()
            return f"{type(e).__name__}: {e}"[:200]
        self.graphs = graphs
        return None

    def run(self, i, ev=None):
        st = self.states[i % len(self.states)]
        graphs = getattr(self, "graphs", None)
        if graphs is not None:
            g_w, g_d = graphs[i % len(self.states)]
            if g_w is not None:
                g_w.replay()
            if ev is not None:
                ev[0].record()
            g_d.replay()
            if ev is not None:
                ev[1].record()
            return st
        self._writes(st)
        if ev is not None:
            ev[0].record()
        self._decode(st)
        if ev is not None:
            ev[1].record()
        return st

    def _decode(self, st):
        b = self.binding
        if self.whole:
            b.decode(st["q"], self.k_pool, self.v_pool, st["tables"], st["ctx"], self.w.scale,
                     out=self.out)
        elif self.mode == "window":
            b.decode_split_window(st["q"], self.k_pool, self.v_pool, st["tables"], st["ctx"],
                                  self.w.scale, self.window,
                                  partition_tokens=self.partition_tokens, out=self.out,
                                  workspace=self.ws)
        elif self.mode == "shared_prefix":
            b.decode_shared_prefix(st["q"], self.k_pool, self.v_pool, st["tables"], st["ctx"],
                                   self.w.scale, st["groups"],
                                   partition_tokens=self.partition_tokens, out=self.out,
                                   workspace=self.ws)
        else:
            b.decode_split(st["q"], self.k_pool, self.v_pool, st["tables"], st["ctx"],
                           self.w.scale, partition_tokens=self.partition_tokens, out=self.out,
                           workspace=self.ws)


CONFIG_LABELS = {
    "long16": "long-context split decode (config 5), block 16",
    "long32": "long-context split decode (config 5), block 32",
    "mha": "MHA decode, 7B-style (config 2)",
    "gqa": "GQA decode, 8B-style (config 3)",
    "prefix": "prefix sharing / parallel sampling (config 4, literal: 4000-token prompts)",
    "prefix_cow": "prefix sharing copy-on-write step (config 4: 4008-token prompts, 120 copies)",
    "tiny": "tiny fp32 paged decode (config 1)",
}
EXTRA_CONFIGS = ("long32", "mha", "gqa", "prefix", "prefix_cow")
KERNEL_LABELS = {
    "split": "pa_decode_split (paged_decode_kernel + lse_merge_kernel)",
    "whole": "pa_decode (paged_decode_kernel)",
    "shared_prefix": "pa_decode_shared_prefix (prefix_decode_kernel + paged_decode_kernel "
                     "+ lse_merge_kernel)",
    "window": "pa_decode_split_window (paged_decode_kernel + lse_merge_kernel)",
}


def timed_repeats(ds, steps: int, first_index: int, min_ms: float, world: int, device,
                  max_repeats: int = 10_000):
    """Times `steps` steps at a time, each repeat bracketed by a barrier and
    a device synchronisation, until the repeats' max-over-ranks time reaches
    min_ms. Every rank stops after the same repeat (the stop rule reads the
    reduced time). Returns the per-repeat records, the decode call durations
    (us, CUDA events on the launching stream), launches and the next index."""
    import torch
    import torch.distributed as dist
    reps, calls = [], []
    launches = 0
    i = first_index
    total = 0.0
    while True:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        nbytes = dbytes = ubytes = 0
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record()
        for k in range(steps):
            st = ds.run(i, evs[k])
            i += 1
            nbytes += st["step_bytes"]
            dbytes += st["decode_bytes"]
            ubytes += st["unique_bytes"]
            launches += ds.launches(st)
        t1.record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ms = t0.elapsed_time(t1)
        call_us = [a.elapsed_time(b) * 1e3 for a, b in evs]
        ms_max, all_bytes, all_tokens = reduce_over_ranks(ms, nbytes, steps * ds.B, device)
        reps.append({"ms": ms_max, "bytes": all_bytes, "tokens": all_tokens,
                     "decode_bytes": dbytes, "unique_bytes": ubytes, "decode_us": sum(call_us)})
        calls.extend(call_us)
        total += ms_max
        if total >= min_ms or len(reps) >= max_repeats:
            return reps, calls, launches, i


def summarize(ds, reps, calls, steps, world, workload_key, mode, peak, peak_kind, clock_info):
    """One configuration's numbers: step throughput (median over repeats,
    with p10/p90), the decode call's roofline and the clocks seen."""
    w = ds.w
    gbs = [r["bytes"] / (r["ms"] * 1e-3) / 1e9 for r in reps]
    ms_step = [r["ms"] / steps for r in reps]
    tok = [r["tokens"] / (r["ms"] * 1e-3) for r in reps]
    dbytes = sum(r["decode_bytes"] for r in reps)
    ubytes = sum(r["unique_bytes"] for r in reps)
    dus = sum(r["decode_us"] for r in reps)
    n_calls = len(calls)
    achieved = dbytes / (dus * 1e-6) / 1e9
    unique = ubytes / (dus * 1e-6) / 1e9
    pct = lambda xs, q: round(float(np.percentile(xs, q)), 2)
    roof = {
        "bound": "hbm",
        "kernel": KERNEL_LABELS[mode],
        "achieved": round(achieved, 2),
        "peak": peak,
        "peak_kind": peak_kind,
        "unit": "GB/s",
        "frac": round(achieved / peak, 4),
        "frac_of_8TBs_spec": round(achieved / 8000.0, 4),
        "traffic": profiled_traffic(workload_key, mode=mode, algorithmic=dbytes / n_calls),
        "algorithmic_bytes_per_launch": int(dbytes / n_calls),
        "avg_launch_us": round(dus / n_calls, 2),
        "launch_us_p10_p50_p90": [pct(calls, 10), pct(calls, 50), pct(calls, 90)],
        # bytes the call must read at least (shared prefixes once); equal to the
        # algorithmic bytes unless blocks are shared
        "unique_bytes_per_launch": int(ubytes / n_calls),
        "unique_achieved": round(unique, 2),
        "unique_frac": round(unique / peak, 4),
    }
    return {
        "workload": workload_label(w),
        "config": CONFIG_LABELS.get(workload_key, workload_key),
        "value": round(statistics.median(gbs), 2),
        "unit": "GB/s",
        "value_p10_p90": [pct(gbs, 10), pct(gbs, 90)],
        "ms_per_step": round(statistics.median(ms_step), 5),
        "repeats": len(reps),
        "steps_per_repeat": steps,
        "timed_ms": round(sum(r["ms"] for r in reps), 2),
        "decode_tokens_per_s": round(statistics.median(tok), 1),
        "mean_context": round(float(np.mean([s["ctx_np"].mean() for s in ds.states])), 1),
        "copies_per_step": round(float(np.mean([s["n_pairs"] for s in ds.states])), 2),
        "roofline": roof,
        "clocks": clock_info,
    }


def bench_config(args, workload_key, mode, rank, world, device, device_index, min_ms,
                 keep=False):
    """Builds one workload on the device, warms up, times it; returns
    (summary, DeviceStep if keep else None, launches)."""
    import torch
    w = make_workload(workload_key, rank, args.batch)
    R = max(1, min(args.states, args.steps + args.warmup)) if workload_key != "prefix_cow" else 1
    ds = DeviceStep(w, R, args.partition_tokens, device, mode=mode, window=args.window)
    for i in range(args.warmup):
        ds.run(i)
    torch.cuda.synchronize()
    eager_why = ds.capture() if args.graphs else "--graphs off"
    for i in range(args.warmup):
        ds.run(i)
    torch.cuda.synchronize()
    clocks = ClockSampler(device_index)
    clocks.start()
    reps, calls, launches, _ = timed_repeats(ds, args.steps, args.warmup, min_ms, world, device)
    clock_info = clocks.stop()
    peak, peak_kind = hbm_peak()
    res = summarize(ds, reps, calls, args.steps, world, workload_key, mode, peak, peak_kind,
                    clock_info)
    res["launch"] = ("CUDA graphs, one per state for the copies and append and one for the "
                     "decode call (captured library calls)" if eager_why is None
                     else f"eager library calls ({eager_why})")
    if not keep:
        del ds
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        ds = None
    return res, ds, launches


def run_ours(args, rank, world, device_index):
    import torch
    device = torch.device("cuda", device_index)
    torch.cuda.set_device(device)
    head, ds, launches = bench_config(args, args.workload, args.decode_mode, rank, world, device,
                                      device_index, args.min_seconds * 1e3, keep=True)
    # ---- end to end through the public API (host buffers, pinned) ----------------
    e2e = run_e2e(args, ds, rank, world, device) if args.e2e_steps > 0 else None
    w = ds.w
    B = ds.B
    del ds
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    # ---- the other configurations, each with its own roofline ----------------------
    extras = {}
    if args.configs == "all" and world == 1:
        for key in EXTRA_CONFIGS:
            if key == args.workload:
                continue
            modes = ["split", "shared_prefix"] if key.startswith("prefix") else ["split"]
            for mode in modes:
                r, _, n = bench_config(args, key, mode, rank, world, device, device_index,
                                       args.extra_min_seconds * 1e3)
                extras[key if mode == "split" else f"{key}/shared_prefix"] = r
                launches += n

    result = None
    if rank == 0:
        result = {
            "metric": METRIC,
            "value": head["value"],
            "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": head["ms_per_step"],
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": w.dtype,
            "data": "synthetic (seeded N(0,1) values, seeded shuffled block placement)",
            "config": {
                "workload": head["workload"],
                "name": head["config"],
                "global_batch": B * world,
                "mean_context": head["mean_context"],
                "partition_tokens": args.partition_tokens,
                "step": "bm slots/CoW (host, precomputed) + copy_blocks + kv_append + "
                        + KERNEL_LABELS[args.decode_mode],
                "decode_states_cycled": min(args.states, args.steps + args.warmup),
                "timing": (f"{head['repeats']} repeats of {args.steps} steps (each bracketed by "
                           f"barrier + synchronize, max over ranks) until >= {args.min_seconds} s "
                           "of device time; value and ms_per_step are medians over repeats"),
                "l2": "inputs larger than L2 (KV read per step >> 126 MB), no flush",
                "parallelism": f"independent batch per GPU x{world}",
            },
            "launch": head["launch"],
            "value_p10_p90": head["value_p10_p90"],
            "repeats": head["repeats"],
            "decode_tokens_per_s": head["decode_tokens_per_s"],
            "roofline": head["roofline"],
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": head["clocks"],
            "configs": extras,
        }
    return result


def run_e2e(args, ds, rank, world, device):
    """Same metric through the public API from pinned host buffers: one
    pa_decode_step call per step (host block-manager step, H2D of the step's
    inputs, copies + append + split decode, D2H of out). Measured two ways:
    pipelined (two staging sets alternated, uploads and downloads on their own streams, no
    per-step host synchronisation; the value reported) and one step at a
    time with a stream synchronisation after each (reported beside it)."""
    import torch
    import torch.distributed as dist
    b = ds.binding
    w = ds.w
    # Every e2e step appends one token to each sequence: both measurements
    # together must fit the tables' room and the free blocks, so the step
    # counts are scaled down (and reported) where the workload is too tight.
    seqs = np.ascontiguousarray(np.asarray(w.step_seqs or w.decode_seqs, dtype=np.int64))
    n = int(seqs.shape[0])
    piped_steps = max(3, int(args.e2e_steps))
    sync_steps = max(3, min(64, piped_steps // 4))
    bs = w.block_size
    room = min(ds.bm.max_blocks_per_seq * bs - ds.bm.context_len(int(x)) for x in seqs) - 1
    free = ds.bm.num_free()
    fits = lambda t: t <= room and n * (t // bs + 2) <= free
    while not fits(piped_steps + sync_steps) and piped_steps > 3:
        piped_steps = max(3, piped_steps * 3 // 4)
        sync_steps = max(3, min(sync_steps, piped_steps // 4))
    steps = piped_steps
    ring = min(steps, 8)
    hq = [ds.states[i % len(ds.states)]["q"][:n].cpu().pin_memory() for i in range(ring)]
    hk, hv = [], []
    for i in range(ring):
        kn, vn = b_new_kv(w, n, i, device)
        hk.append(kn.cpu().pin_memory())
        hv.append(vn.cpu().pin_memory())
    hout = [torch.empty(hq[0].shape, dtype=hq[0].dtype).pin_memory() for _ in range(2)]
    stream = torch.cuda.current_stream()
    copy_stream = torch.cuda.Stream()
    download_stream = torch.cuda.Stream()
    piped = [b.DecodeStepper(ds.bm, ds.k_pool, ds.v_pool, w.num_q_heads, w.scale, max_seqs=n,
                             partition_tokens=ds.partition_tokens, copy_stream=copy_stream,
                             download_stream=download_stream)
             for _ in range(2)]
    sync = b.DecodeStepper(ds.bm, ds.k_pool, ds.v_pool, w.num_q_heads, w.scale, max_seqs=n,
                           partition_tokens=ds.partition_tokens)

    def timed(pipelined: bool):
        # bookkeeping stays out of the timed loop: every step appends one token
        # to each sequence, so step i decodes lengths ctx0 + i + 1
        steps = piped_steps if pipelined else sync_steps
        ctx0 = np.array([ds.bm.context_len(int(x)) for x in seqs], dtype=np.int64)
        ncows = []
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t_start = time.perf_counter()
        for i in range(steps):
            j = i % ring
            st = piped[i % 2] if pipelined else sync
            ncows.append(st.step(seqs, hq[j], hk[j], hv[j], hout[i % 2],
                                 synchronize=not pipelined, stream=stream))
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t_start
        assert np.array_equal(np.array([ds.bm.context_len(int(x)) for x in seqs]), ctx0 + steps)
        total = sum(decode_bytes(w, ctx0 + i + 1) + append_bytes(w, n) + copy_bytes(w, c)
                    for i, c in enumerate(ncows))
        h2d = sum(sync.h2d_bytes(n, c) for c in ncows)
        d2h = steps * sync.d2h_bytes(n)
        elapsed, total, _ = reduce_over_ranks(elapsed, total, steps * n, device)
        return total / elapsed / 1e9, elapsed / steps * 1e3, h2d / steps, d2h / steps

    g_sync, ms_sync, _, _ = timed(False)
    g, ms, h2d, d2h = timed(True)
    return {"value": round(g, 2), "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "steps": piped_steps, "ms_per_step": round(ms, 4),
            "timing": "host wall clock (perf_counter) from a synchronised device to the "
                      "synchronisation after the last step",
            "path": "pa_decode_step (C ABI) per step: host block manager step + pinned H2D "
                    "of the step's inputs + copies/append/split decode + D2H out; two staging "
                    "sets alternated, uploads and downloads on their own streams overlapping the "
                    "neighbouring steps' kernels, one synchronisation at the end",
            "one_step_at_a_time": {"value": round(g_sync, 2), "unit": "GB/s",
                                   "ms_per_step": round(ms_sync, 4), "steps": sync_steps,
                                   "path": "the same call with a stream synchronisation after "
                                           "every step"}}


def b_new_kv(w, n, i, device):
    from paged_kv_cache_336_b200 import workloads
    return workloads.draw_new_kv(w, n, step=10_000 + i, device=device)


# ---------------------------------------------------------------------------
# the CPU oracle (cpu_baseline leg and --impl reference)

_ORACLE_INPUT = [None, None]   # (key, inputs) of the last sequence drawn for the oracle


def seq_context(w, s: int) -> int:
    """Context length of sequence s before the step (a forked sequence has
    its parent's)."""
    parents = {child: parent for parent, child in w.forks}
    while s >= len(w.context_lens) and s in parents:
        s = parents[s]
    return int(w.context_lens[s])


def time_oracle(w, budget_s: float, seed: int = 0, threads: int = 1, per_kv_head: bool = False):
    """Times the float64 oracle on whole sequences of the workload (all query
    heads of each), with `threads` BLAS/torch threads, until ~budget_s seconds
    of work are done. With per_kv_head, the unit is one (sequence, KV head):
    the sequence's K/V for that head and its group of query heads (a long
    sequence is seconds of oracle work; one KV head is an eighth of it).
    Returns (GB/s of algorithmic bytes, tokens/s, description, seconds)."""
    import torch
    from threadpoolctl import threadpool_limits
    import oracle
    from paged_kv_cache_336_b200 import workloads

    rng = np.random.default_rng(seed)
    order = rng.permutation(len(w.decode_seqs))
    Hkv, bs, D = w.num_kv_heads, w.block_size, w.head_dim
    done_bytes = 0
    done_seqs = 0
    done_units = 0
    elapsed = 0.0
    prev_threads = torch.get_num_threads()
    torch.set_num_threads(threads)
    with threadpool_limits(limits=threads):
        for idx in order:
            ctx = seq_context(w, int(idx)) + (1 if w.step_seqs else 0)
            nb = -(-ctx // bs)
            # a contiguous one-sequence pool drawn from the same distribution
            # (drawn outside the timed region; the last one is kept for reuse)
            key = (w.name, w.seed, int(idx))
            if _ORACLE_INPUT[0] != key:
                _ORACLE_INPUT[:] = [None, None]
                kp = workloads.draw_normal((nb, Hkv, bs, D), w.dtype, w.seed * 7 + int(idx)).double().numpy()
                vp = workloads.draw_normal((nb, Hkv, bs, D), w.dtype, w.seed * 7 + 99991 + int(idx)).double().numpy()
                q = workloads.draw_normal((1, w.num_q_heads, D), w.dtype, w.seed * 7 + 3 + int(idx)).double().numpy()
                _ORACLE_INPUT[:] = [key, (kp, vp, q)]
            kp, vp, q = _ORACLE_INPUT[1]
            table = np.arange(nb)[None, :]
            G = w.num_q_heads // Hkv
            for h in (rng.permutation(Hkv) if per_kv_head else [None]):
                if h is None:
                    kh, vh, qh = kp, vp, q
                else:   # one KV head and its query heads, as contiguous arrays
                    kh = np.ascontiguousarray(kp[:, h:h + 1])
                    vh = np.ascontiguousarray(vp[:, h:h + 1])
                    qh = np.ascontiguousarray(q[:, h * G:(h + 1) * G])
                t0 = time.perf_counter()
                oracle.paged_decode(qh, kh, vh, table, [ctx], w.scale)
                elapsed += time.perf_counter() - t0
                done_bytes += decode_bytes(w, np.array([ctx])) / (Hkv if h is not None else 1)
                done_units += 1
                if elapsed >= budget_s:   # at least one unit per call
                    break
            done_seqs += 1
            if elapsed >= budget_s:
                break
    torch.set_num_threads(prev_threads)
    if per_kv_head:
        what = (f"{done_units} (sequence, KV head) units of {len(w.decode_seqs) * Hkv} (one KV head "
                f"and its {w.num_q_heads // Hkv} query heads each")
        seqs_done = done_units / Hkv
    else:
        what = f"{done_seqs} of {len(w.decode_seqs)} sequences (all {w.num_q_heads} query heads each"
        seqs_done = done_seqs
    desc = (f"{what}, the workload's context lengths and N(0,1) values) of the {w.name} workload, "
            f"{elapsed:.2f} s, float64 NumPy oracle, {threads} thread{'s' if threads > 1 else ''}")
    return done_bytes / elapsed / 1e9, seqs_done / elapsed, desc, elapsed


def run_reference(args, rank, world):
    if rank != 0:
        return None
    w = make_workload(args.workload, 0, args.batch)
    # each step: a bounded sample of the workload, sized so that the whole run
    # ends within a few minutes. Long sequences (seconds of oracle work each)
    # are sampled by (sequence, KV head) units, an eighth of a sequence at the
    # headline, and every step starts from the same sequence
    per_step = min(10.0, 60.0 / max(1, args.steps + args.warmup))
    long_seqs = float(np.max(w.context_lens)) >= 32768
    for _ in range(args.warmup):
        time_oracle(w, per_step / 4, per_kv_head=long_seqs)
    vals, tok, descs, secs = [], [], [], 0.0
    for i in range(args.steps):
        g, t, d, el = time_oracle(w, per_step, seed=0 if long_seqs else i, per_kv_head=long_seqs)
        vals.append(g)
        tok.append(t)
        descs.append(d)
        secs += el
    value = statistics.mean(vals)
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 5),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded N(0,1) values)",
        "config": {"workload": workload_label(w), "partition_tokens": args.partition_tokens},
        "decode_tokens_per_s": round(statistics.mean(tok), 4),
        "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": descs[0]},
        "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------

def run_prefill_bench(args, device_index):
    """Chunked-prefill attention (pa_prefill) on a synthetic batch: every
    sequence has `prior` tokens of earlier context and `chunk` new tokens
    (already appended). Reports causal-attention TFLOP/s (4*D per (query,
    key, head) pair: q.k and p.v, 2 flops per multiply-add) against the
    measured bf16 tensor peak, and the KV bytes read per call."""
    import torch
    from paged_kv_cache_336_b200 import binding, workloads
    device = torch.device("cuda", device_index)
    torch.cuda.set_device(device)
    B, prior, chunk, Hq, Hkv, D, bs = 16, args.prefill_prior, args.prefill_chunk, 32, 8, 128, 16
    ctx = np.full(B, prior + chunk, dtype=np.int64)
    w = workloads.random_small(500, num_seqs=B, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                               block_size=bs, dtype=workloads.BF16, max_ctx=prior + chunk,
                               fixed_lens=ctx.tolist())
    bm = binding.BlockManager(w.num_blocks, bs, w.max_blocks_per_seq, w.free_order)
    for s_ in range(B):
        bm.allocate(s_, int(ctx[s_]))
    k_pool, v_pool = workloads.draw_pools(w, device)
    tables, ctx32 = bm.export(list(range(B)))
    bt = torch.from_numpy(tables).to(device)
    qlen = np.full(B, chunk, dtype=np.int32)
    q = workloads.draw_normal((B * chunk, Hq, D), workloads.BF16, 501, device)
    out = torch.empty_like(q)
    part = args.prefill_partition or -(-(prior + chunk) // bs) * bs
    ws = binding.prefill_workspace(B, B * chunk, Hq, Hkv, D, bs, w.max_blocks_per_seq, part, device)
    for _ in range(max(3, args.warmup)):
        binding.prefill(q, k_pool, v_pool, bt, ctx32, qlen, w.scale, part, out, ws)
    torch.cuda.synchronize()
    # Blocks of `reps` back-to-back calls, each bracketed by CUDA events, until
    # the blocks add up to --min-seconds of device time; the median block.
    # The kernel is tensor-bound, so its time follows the SM clock: the
    # line carries the clocks sampled meanwhile.
    reps = max(3, min(args.steps, 200))
    clocks = ClockSampler(device_index)
    clocks.start()
    per_call, total_ms = [], 0.0
    while True:
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(reps):
            binding.prefill(q, k_pool, v_pool, bt, ctx32, qlen, w.scale, part, out, ws)
        t1.record()
        torch.cuda.synchronize()
        block = t0.elapsed_time(t1)
        per_call.append(block / reps)
        total_ms += block
        if total_ms >= args.min_seconds * 1e3 or len(per_call) >= 10_000:
            break
    clock_info = clocks.stop()
    ms = statistics.median(per_call)
    pairs = B * int(np.sum(np.arange(prior + 1, prior + chunk + 1)))   # (query, key) pairs per head
    flops = 4.0 * D * Hq * pairs
    tflops = flops / (ms * 1e-3) / 1e12
    try:
        peak = float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops"])
        kind = "measured (cuBLAS bf16 burst)"
    except Exception:
        peak, kind = 1590.0, "fallback"
    kv_bytes = B * (prior + chunk) * Hkv * D * 2 * 2
    q10, q90 = (float(np.percentile(per_call, x)) for x in (10, 90))
    return {"metric": "paged chunked-prefill attention TFLOP/s (causal, bf16 in, fp32 accumulate)",
            "value": round(tflops, 2), "unit": "TFLOP/s", "impl": "ours", "ms_per_call": round(ms, 4),
            "ms_per_call_p10_p90": [round(q10, 4), round(q90, 4)], "blocks": len(per_call),
            "calls_per_block": reps, "clocks": clock_info,
            "tflops_per_sm_ghz": (round(tflops / (clock_info["sm_mhz"] / 1000.0), 1)
                                  if clock_info and clock_info.get("sm_mhz") else None),
            "config": {"workload": f"prefill: batch {B}, {prior} prior + {chunk} new tokens, "
                                   f"{Hq}q/{Hkv}kv heads, head_dim {D}, bf16, block {bs}",
                       "partition_tokens": part,
                       "kernel": os.environ.get("PAGEDKV_PREFILL_KERNEL", "tcgen05")},
            "roofline": {"bound": "tensor", "achieved": round(tflops, 2), "peak": peak,
                         "peak_kind": kind, "unit": "TFLOP/s", "frac": round(tflops / peak, 4),
                         "traffic": (profiled_traffic("b16", "prefill", PREFILL_SOURCES)
                                     if (B, prior, chunk, part) == (16, 1024, 1024, 2048)
                                     and os.environ.get("PAGEDKV_PREFILL_KERNEL") != "mma_sync"
                                     else None),
                         "kv_bytes_per_call": kv_bytes,
                         "kv_GBs": round(kv_bytes / (ms * 1e-3) / 1e9, 1)}}


def run_swap_bench(args, device_index):
    """Swap throughput: whole blocks of the workload's pool to pinned host
    memory and back (pa_swap_out / pa_swap_in), CUDA-event timed."""
    import torch
    from paged_kv_cache_336_b200 import binding, workloads
    device = torch.device("cuda", device_index)
    torch.cuda.set_device(device)
    w = make_workload(args.workload, 0, args.batch)
    k_pool, v_pool = workloads.draw_pools(w, device)
    nslots = min(2048, w.num_blocks)
    host_k = torch.empty((nslots,) + tuple(k_pool.shape[1:]), dtype=k_pool.dtype).pin_memory()
    host_v = torch.empty_like(host_k).pin_memory()
    rng = np.random.default_rng(1)
    blocks = torch.from_numpy(rng.permutation(w.num_blocks)[:nslots].astype(np.int64)).to(device)
    slots = torch.arange(nslots, dtype=torch.int64, device=device)
    out_pairs = torch.stack([blocks, slots], 1).contiguous()
    in_pairs = torch.stack([slots, blocks], 1).contiguous()
    block_bytes = k_pool[0].numel() * k_pool.element_size()
    res = {}
    for name, fn, pairs in (("swap_out", lambda p: binding.swap_out(k_pool, v_pool, host_k, host_v, p), out_pairs),
                            ("swap_in", lambda p: binding.swap_in(host_k, host_v, k_pool, v_pool, p), in_pairs)):
        for _ in range(args.warmup):
            fn(pairs)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = max(3, min(args.steps, 50))
        t0.record()
        for _ in range(reps):
            fn(pairs)
        t1.record()
        torch.cuda.synchronize()
        ms = t0.elapsed_time(t1) / reps
        nbytes = 2 * nslots * block_bytes
        res[name] = {"GB/s": round(nbytes / (ms * 1e-3) / 1e9, 2), "ms": round(ms, 4), "bytes": nbytes}
    # Roofline: the host link, measured as plain contiguous pinned-memory copies
    # of the same byte count (copy engine, one direction at a time).
    dev_buf = torch.empty(2 * host_k.numel(), dtype=host_k.dtype, device=device)
    host_buf = torch.empty(2 * host_k.numel(), dtype=host_k.dtype).pin_memory()
    link = {}
    for name, dst, src in (("d2h", host_buf, dev_buf), ("h2d", dev_buf, host_buf)):
        for _ in range(3):
            dst.copy_(src, non_blocking=True)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(10):
            dst.copy_(src, non_blocking=True)
        t1.record()
        torch.cuda.synchronize()
        link[name] = dev_buf.numel() * dev_buf.element_size() / (t0.elapsed_time(t1) / 10 * 1e-3) / 1e9
    res["swap_out"]["frac_of_measured_d2h"] = round(res["swap_out"]["GB/s"] / link["d2h"], 4)
    res["swap_in"]["frac_of_measured_h2d"] = round(res["swap_in"]["GB/s"] / link["h2d"], 4)
    return {"metric": "swap of whole KV blocks between HBM and pinned host memory (K and V)",
            "unit": "GB/s", "value": res["swap_out"]["GB/s"], "impl": "ours",
            "config": {"workload": workload_label(w), "blocks": nslots,
                       "block_bytes_each_pool": block_bytes},
            "roofline": {"bound": "host link", "unit": "GB/s",
                         "measured_d2h": round(link["d2h"], 2), "measured_h2d": round(link["h2d"], 2),
                         "peak_kind": "measured: contiguous pinned-memory copies of the same bytes"},
            **res}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100,
                    help="steps per timed repeat (repeats continue until --min-seconds)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long16",
                    choices=["mha", "gqa", "prefix", "prefix_cow", "long16", "long32", "tiny"],
                    help="the headline configuration (default: long-context split decode, "
                         "block 16, the largest single-GPU configuration)")
    ap.add_argument("--configs", choices=["all", "headline"], default="all",
                    help="all: also time the other configurations (one GPU only), each with "
                         "its own roofline, under \"configs\" in the JSON line")
    ap.add_argument("--min-seconds", type=float, default=1.0,
                    help="device time the headline's timed repeats must reach")
    ap.add_argument("--extra-min-seconds", type=float, default=0.3,
                    help="device time each other configuration's repeats must reach")
    ap.add_argument("--partition-tokens", type=int, default=512)
    ap.add_argument("--window", type=int, default=4096, help="window tokens for --decode-mode window")
    ap.add_argument("--swap", action="store_true",
                    help="measure pa_swap_out / pa_swap_in instead (extra JSON line)")
    ap.add_argument("--prefill", action="store_true",
                    help="measure pa_prefill instead (extra JSON line)")
    ap.add_argument("--prefill-prior", type=int, default=1024)
    ap.add_argument("--prefill-chunk", type=int, default=1024)
    ap.add_argument("--prefill-partition", type=int, default=0,
                    help="KV partition of pa_prefill in tokens; 0: the whole context (no merge)")
    ap.add_argument("--decode-mode", choices=["split", "whole", "shared_prefix", "window"],
                    default="split",
                    help="split: pa_decode_split (persistent, partitions + merge); "
                         "whole: pa_decode (one CTA per sequence and KV head); "
                         "shared_prefix: pa_decode_shared_prefix (shared prompt blocks read once)")
    ap.add_argument("--states", type=int, default=64, help="distinct decode steps cycled")
    ap.add_argument("--graphs", choices=["on", "off"], default="on",
                    help="time the device-resident step as replays of captured CUDA graphs "
                         "(the shared-prefix route always runs eagerly)")
    ap.add_argument("--e2e-steps", type=int, default=256,
                    help="pipelined end-to-end steps (0: no e2e measurement)")
    ap.add_argument("--batch", type=int, default=None,
                    help="mha, long16, long32: smaller batch and pool (profiling captures)")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work")
    args = ap.parse_args(argv)
    args.graphs = args.graphs == "on"
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0

    import torch
    import torch.distributed as dist
    if args.swap:
        if rank == 0:
            print(json.dumps(run_swap_bench(args, local_rank)), flush=True)
        return 0
    if args.prefill:
        if rank == 0:
            print(json.dumps(run_prefill_bench(args, local_rank)), flush=True)
        return 0
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and args.cpu_budget > 0:
                wl = make_workload(args.workload, 0, args.batch)
                g, t, desc, _ = time_oracle(wl, args.cpu_budget)
                ncores = os.cpu_count() or 1
                ga, ta, desca, _ = time_oracle(wl, args.cpu_budget / 2, seed=1, threads=ncores)
                res["cpu_baseline"] = {"value": round(g, 5), "unit": "GB/s", "cores": 1,
                                       "kind": "oracle", "sample": desc,
                                       "decode_tokens_per_s": round(t, 4),
                                       "all_cores": {"value": round(ga, 5), "unit": "GB/s",
                                                     "cores": ncores, "sample": desca,
                                                     "decode_tokens_per_s": round(ta, 4)}}
            else:
                res["cpu_baseline"] = None
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

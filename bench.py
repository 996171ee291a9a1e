#!/usr/bin/env python
"""Benchmark: 2-bit KIVI decode over a quantized KV cache on B200, one JSON line on stdout.

A step is one streaming decode step of the large-batch workload (B=64, H=32, d=128, 2-bit, G=32,
R=128): append one new K/V token per (batch, KV head), run decode attention for every query head over
the whole cache, and flush the residual once it is full (once every 128 steps; by default inside the
same launch, kivi_decode_step).  After each 128-step cycle the host drops one block again, so the
cache cycles between 8193 and 8320 cached tokens instead of growing; every step does its full work.  Inputs live in HBM (1.2 GB of codes
and scales per step, ten times the 126 MB L2, so no L2 flush is needed; a workload smaller than twice
the L2 rotates several cache replicas, one per step, so that a step finds its cache evicted).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

N > 1 runs under torch.distributed.run, one rank per GPU, each rank its own batch (weak scaling,
no collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import faulthandler
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_asymmetric_kv_02_b200 import synth  # noqa: E402

METRIC = "2-bit KV decode-attention cached tokens/s/head and HBM GB/s vs 8 TB/s peak (1 B200)"
UNIT = "cached tokens/s/head"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126e6
WORKLOAD = synth.LARGE_BATCH
# How a step reaches the library:
#   "step"     (default): kivi_decode_step, one launch per step: append, decode attention and, at the
#              step whose token fills the residual, its flush (eager);
#   "fused"    (--lazy-flush): kivi_flush_residual when the residual is full, then
#              kivi_append_decode_attention (two launches on flush steps);
#   "separate" (--separate-append, --online-k): flush when full + kivi_append_token +
#              kivi_decode_attention.
MODE = "step"
STEP_NOTE = {"step": "append, decode attention and (when the token fills the residual) its flush in one launch",
             "fused": "flush when full + append and decode attention in one launch",
             "separate": "flush when full + append + decode attention"}
ONLINE_K = False   # --online-k: K rows coded at append with the newest block's (s, z) (config online_k)
FINE = False       # --fine-groups: K (s, z) per channel per G tokens, V per token per G channels
DECODE_SOURCES = ["decode.cu", "common.cuh", "kernels.h"]
CLOCK_WINDOW_S = 1.0   # the clock record spans at least this much wall time around the timed steps
# The KIVI page's own end-to-end figures (section 実験結果（Results）: its Table 1 and throughput figures):
# context only, not a target.
PUBLISHED = {
    "source": "KIVI explainer page, section 実験結果（Results） (arXiv 2402.02750)",
    "hardware": "not stated",
    "peak_memory_reduction_vs_fp16": "2.6x (Llama-2-7B-chat, 2-bit KIVI)",
    "throughput_vs_fp16": {"Llama-2-7B": "2.35x", "Llama-2-70B": "3.47x"},
    "note": "model-level results with larger batches; no kernel-level figure is given",
}


# ------------------------------------------------------------------------------------------------
# helpers
# ------------------------------------------------------------------------------------------------
def decode_kernel_sha() -> str:
    h = hashlib.sha256()
    for f in DECODE_SOURCES:
        with open(os.path.join(ROOT, "bit_asymmetric_kv_02_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def dot_engine(w):
    """The instruction that forms the decode kernel's byte dot products for this workload."""
    return "mma.sync m16n8k32" if w.bits == 2 else "dp4a"


def profiled_traffic(w: synth.Workload, alg_bytes_per_launch: float):
    """DRAM bytes per decode launch from the committed ncu record, if it was taken on the current
    kernel sources; else None.  The record holds one captured launch (its DRAM bytes and its
    algorithmic bytes); the bench's average launch moves slightly different algorithmic bytes (the
    residual fill cycles), so the captured traffic is scaled by that ratio."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("kernel_sha") != decode_kernel_sha() or rec.get("workload") != w.name or ONLINE_K or FINE:
        return None
    return rec["dram_bytes"] / rec["alg_bytes"] * alg_bytes_per_launch


def append_bytes(w: synth.Workload) -> int:
    """Bytes a fused append adds to the decode launch: the new K and V rows read and written once."""
    return w.batch * w.kv_heads * w.head_dim * 2 * 2 * 2


def flush_bytes(w: synth.Workload) -> int:
    """Bytes a flush moves at least once: the R fp16 K and V residual rows read, their codes and the
    block's scales and zero points written (base groups)."""
    R = w.residual
    per_head = (2 * R * w.head_dim * 2                       # fp16 K and V rows
                + 2 * R * w.head_dim * w.bits // 8           # K and V codes
                + ((w.head_dim // w.group) + R // w.gv) * 4)  # K and V (s, z) pairs, fp16
    return w.batch * w.kv_heads * per_head


def decode_alg_bytes(w: synth.Workload, n_quant: int, n_res: int) -> int:
    """Bytes decode attention must move at least once: codes, scales/zeros, residual rows, q, out."""
    bh = w.batch * w.kv_heads
    if FINE:   # K: one pair per channel per G tokens; V: one pair per token per G channels
        scales = (n_quant // w.group) * w.head_dim * 4 + n_quant * (w.head_dim // w.gv) * 4
    else:
        scales = (n_quant // w.residual) * (w.head_dim // w.group) * 4 + (n_quant // w.gv) * 4
    per_head = (2 * n_quant * w.head_dim * w.bits // 8                 # K and V codes
                + scales                                                 # scales + zeros (fp16)
                + n_res * w.head_dim * 4                                 # fp16 K and V residual rows
                + 2 * w.gqa * w.head_dim * 2)                            # q in, out
    if ONLINE_K and n_quant > 0 and n_res > 0:   # residual K rows are codes, plus the block's (s, z)
        per_head += (w.head_dim // w.group) * 4 - n_res * w.head_dim * (2 - w.bits / 8)
    return int(bh * per_head)


def auto_replicas(w: synth.Workload, n_quant0: int) -> int:
    """Cache replicas a step rotates through so that each step reads a cache the L2 has dropped:
    one when a step moves more than twice the L2, else enough that the other replicas' steps move
    at least twice the L2 between two uses of one replica (at most 64)."""
    per_step = decode_alg_bytes(w, n_quant0 + w.residual, w.residual)
    if per_step > 2 * L2_BYTES:
        return 1
    return int(min(64, math.ceil(2 * L2_BYTES / per_step) + 1))


def l2_note(w: synth.Workload, n_quant: int, replicas: int) -> str:
    gb = decode_alg_bytes(w, n_quant, w.residual) / 1e9
    if replicas <= 1:
        if gb * 1e9 > 2 * L2_BYTES:
            return f"not flushed: inputs ({gb:.2f} GB per step) exceed the 126 MB L2"
        return f"WARNING: inputs ({gb * 1e3:.0f} MB per step) fit in the 126 MB L2; not flushed"
    return (f"{replicas} cache replicas, one per step in turn: {(replicas - 1) * gb * 1e3:.0f} MB move between two "
            f"uses of a replica ({gb * 1e3:.1f} MB per step, 126 MB L2)")


class ClockSampler:
    """Samples SM clock, max clock and throttle reasons of one GPU with nvidia-smi every 50 ms (the
    clocks line of the profiling recipe).  start() returns once the first sample has arrived, so a
    window marked afterwards is covered; every line is time-stamped on arrival."""

    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int):
        self.bus = None   # (bus, device) numbers of the CUDA device, as torch reports them
        try:
            import torch
            p = torch.cuda.get_device_properties(device_index)
            self.bus = (int(p.pci_bus_id), int(p.pci_device_id))
        except Exception:
            pass
        self.proc = None
        self.lines = []      # (monotonic time, line)
        self._thread = None
        self._first = threading.Event()

    @staticmethod
    def _bus_of(field: str):
        """(bus, device) of an nvidia-smi pci.bus_id such as 00000000:1B:00.0."""
        try:
            parts = field.strip().split(":")
            return int(parts[-2], 16), int(parts[-1].split(".")[0], 16)
        except (ValueError, IndexError):
            return None

    def _reader(self):
        for ln in self.proc.stdout:
            if ln.strip():
                self.lines.append((time.monotonic(), ln))
                self._first.set()

    def start(self, wait_s: float = 10.0):
        import shutil
        import subprocess
        exe = shutil.which("nvidia-smi")
        if exe:
            self.proc = subprocess.Popen([exe, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True, bufsize=1)
            self._thread = threading.Thread(target=self._reader, daemon=True)
            self._thread.start()
            self._first.wait(wait_s)
        return self

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=10)
            except Exception:
                self.proc.kill()
            if self._thread is not None:
                self._thread.join(timeout=10)
            self.proc = None

    def summary(self, t0: float | None = None, t1: float | None = None):
        rows = []
        for t, ln in self.lines:
            if (t0 is not None and t < t0) or (t1 is not None and t > t1):
                continue
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10:
                continue
            if self.bus is not None and self._bus_of(f[1]) not in (None, self.bus):
                continue
            try:
                rows.append((float(f[2]), float(f[3]), float(f[4]), f[6:10]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "no nvidia-smi sample in the window"}
        loaded = [r for r in rows if r[2] > 300.0] or rows   # power draw separates load from idle
        reasons = set()
        for r in loaded:
            for name, flag in zip(self.NAMES, r[3]):
                if flag.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(loaded), "samples_total": len(rows)}


BAD_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


class Ranks:
    """The plumbing bench.py needs from torch.distributed: barrier and max over ranks.  Works with
    any backend (NCCL on GPUs, gloo in the CPU tests); world == 1 needs no process group."""

    def __init__(self, dist=None, device=None):
        self.dist = dist
        self.device = device
        self.world = dist.get_world_size() if dist is not None else 1
        self.rank = dist.get_rank() if dist is not None else 0

    def barrier(self):
        if self.dist is not None:
            if self.device is not None and self.device.type == "cuda":
                self.dist.barrier(device_ids=[self.device.index])
            else:
                self.dist.barrier()

    def max(self, *values: float):
        if self.dist is None:
            return values if len(values) > 1 else values[0]
        import torch
        t = torch.tensor(values, dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        out = tuple(float(x) for x in t.cpu())
        return out if len(out) > 1 else out[0]


def weak_scaling_value(world: int, tokens_per_rank: int, batch: int, t_max_ms: float) -> float:
    """Whole-job cached tokens/s/head: every rank attends its own B sequences; a step counts B*T
    tokens per head; the job time is the slowest rank's."""
    return world * tokens_per_rank * batch / (t_max_ms / 1e3)


def first_prompt_split(w: synth.Workload):
    """(n_quant, capacity) of the bench's cache: the prompt leaves a full residual; the cache holds
    one more block, two when the block being filled needs its own room (online K keeps its scale
    row there; the decode step flushes a full residual into it before the cycle drops it)."""
    n_quant0 = (w.tokens - 1) // w.residual * w.residual
    return n_quant0, n_quant0 + (2 if (ONLINE_K or MODE == "step") else 1) * w.residual


def workload_config(w: synth.Workload, world: int, replicas: int) -> dict:
    """The `config` of the JSON line, the same for both arms."""
    n_quant0, _ = first_prompt_split(w)
    R = w.residual
    return {
        "workload": w.name, "batch": w.batch, "q_heads": w.q_heads, "kv_heads": w.kv_heads,
        "head_dim": w.head_dim, "bits": w.bits, "group_k": w.group, "group_v": w.gv,
        "residual": R, "cached_tokens": f"{n_quant0 + R + 1}-{n_quant0 + 2 * R} ({R}-step cycles)",
        "step": STEP_NOTE[MODE],
        "k_residual": "codes (online K, config online_k = 1)" if ONLINE_K else "fp16",
        "groups": ("fine: K per channel per G tokens, V per token per G channels (config fine_groups = 1)"
                   if FINE else "K per R-token block x G channels, V per G tokens x all channels"),
        "l2": l2_note(w, n_quant0, replicas),
        "parallelism": f"weak: one independent batch per GPU x {world}",
    }


# ------------------------------------------------------------------------------------------------
# the GPU arm
# ------------------------------------------------------------------------------------------------
def make_cache(w: synth.Workload, torch, kivi, device, kd, vd):
    _, capacity = first_prompt_split(w)
    cache = kivi.KiviCache(w.batch, w.kv_heads, capacity, bits=w.bits, group_k=w.group, group_v=w.gv,
                           residual=w.residual, num_q_heads=w.q_heads, device=device, online_k=ONLINE_K,
                           fine_groups=FINE)
    cache.prefill(kd, vd)
    return cache


def step_inputs(w: synth.Workload, torch, device):
    """New K/V rows and queries of synthetic steps 1..R, resident in HBM (a cycle of R steps)."""
    host = []
    for s in range(w.residual):
        kn, vn = synth.new_kv(w, s + 1)
        host.append((kn, vn, synth.queries(w, s + 1)))
    dev = [tuple(torch.from_numpy(a).to(device) for a in x) for x in host]
    return host, dev


def gpu_step(cache, n_quant0, w, inputs, out, stream, decode_events=None, stage_events=None, status=True):
    """One streaming decode step on device-resident inputs.  Returns (launches, cached tokens
    attended, quantized tokens attended, whether the step's own launch flushed the residual).
    stage_events (optional): {"flush": [...], "append": [...]} lists that receive event pairs.

    The cache cycles through R steps: every step attends n_quant0 + R quantized tokens and 1..R
    residual tokens.  The decode step flushes the residual at the step that fills it, into the
    block after those, which the next step drops again; the lazy modes flush a full residual at the
    next step, after moving n_quant back to n_quant0 (the cycle's block is rewritten)."""
    import torch
    R = w.residual
    kn, vn, q = inputs
    if MODE == "step":
        if cache.c.n_quant == n_quant0 + 2 * R:
            cache.c.n_quant = n_quant0 + R     # end of a cycle: drop the block the filling step wrote
        full = cache.c.n_res == R              # only after the prefill: flushed first, by its own launch
        nq = cache.c.n_quant + (R if full else 0)
        nr = (0 if full else cache.c.n_res) + 1
        if decode_events is not None:
            decode_events[0].record(stream)
        cache.step(kn, vn, q, out=out, stream=stream, status=status)
        if decode_events is not None:
            decode_events[1].record(stream)
        flushed = nr == R and nq + R <= cache.cfg.capacity
        assert (cache.c.n_quant, cache.c.n_res) == ((nq + R, 0) if flushed else (nq, nr))
        return (2 if full else 1), nq + nr, nq, flushed
    launches = 0
    if cache.c.n_res == R:
        if cache.c.n_quant == n_quant0 + R:
            cache.c.n_quant = n_quant0     # end of a cycle: drop the newest block again
        if stage_events is not None:
            ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            ev[0].record(stream)
        cache.flush(stream)
        if stage_events is not None:
            ev[1].record(stream)
            stage_events["flush"].append(ev)
        launches += 1
    if MODE == "fused":
        if decode_events is not None:
            decode_events[0].record(stream)
        cache.append_attend(kn, vn, q, out=out, stream=stream, status=status)
        if decode_events is not None:
            decode_events[1].record(stream)
        return launches + 1, cache.c.n_quant + cache.c.n_res, cache.c.n_quant, False
    if stage_events is not None:
        ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        ev[0].record(stream)
    cache.append(kn, vn, stream)
    if stage_events is not None:
        ev[1].record(stream)
        stage_events["append"].append(ev)
    launches += 1
    if decode_events is not None:
        decode_events[0].record(stream)
    cache.attend(q, out=out, stream=stream, status=status)
    if decode_events is not None:
        decode_events[1].record(stream)
    launches += 1
    return launches, cache.c.n_quant + cache.c.n_res, cache.c.n_quant, False


def run_gpu(args, rank, world, local_rank, w: synth.Workload):
    import torch
    from bit_asymmetric_kv_02_b200 import kivi
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    kivi.load_library()
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    ranks = Ranks(dist, device)
    R = w.residual
    n_quant0, _ = first_prompt_split(w)
    replicas = args.replicas if args.replicas > 0 else auto_replicas(w, n_quant0)

    log(f"generating inputs and prefilling {replicas} cache(s)")
    k, v = synth.prompt_kv(w, w.tokens)
    kd = torch.from_numpy(k).to(device)
    vd = torch.from_numpy(v).to(device)
    del k, v
    caches = [make_cache(w, torch, kivi, device, kd, vd) for _ in range(replicas)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    caches[0].prefill(kd, vd)          # the first prefill loaded the module; this one is timed
    e1.record()
    torch.cuda.synchronize(device)
    prefill_ms = e0.elapsed_time(e1)
    del kd, vd
    torch.cuda.empty_cache()   # hand the prompt back: the decode loop holds the caches only
    host_in, dev_in = step_inputs(w, torch, device)
    for c in caches:
        assert (c.n_quant, c.n_res) == (n_quant0, R)
        c.status.zero_()
    log("cache ready")
    stream = torch.cuda.Stream(device)
    out = torch.empty(w.batch, w.q_heads, w.head_dim, dtype=torch.float16, device=device)
    schedule = [[] for _ in caches]   # synthetic step id of every step each replica has run
    counter = [0]

    def step(inputs_index, decode_events=None, stage_events=None, outbuf=None, inputs=None):
        i = counter[0]
        counter[0] += 1
        r = i % replicas
        schedule[r].append(inputs_index + 1)
        return gpu_step(caches[r], n_quant0, w, inputs if inputs is not None else dev_in[inputs_index],
                        outbuf if outbuf is not None else out, stream, decode_events, stage_events)

    barrier = ranks.barrier
    sampler = ClockSampler(local_rank).start()

    # ---- device-resident timing -------------------------------------------------------------
    def timed_loop(K, W):
        with torch.cuda.stream(stream):
            for i in range(W):
                step(i % R)
        stream.synchronize()
        barrier()
        torch.cuda.synchronize(device)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        launches, tokens, bytes_decode = 0, 0, 0
        stage_ev = {"flush": [], "append": []}
        flush_steps = []   # whether each timed step's own launch flushed the residual
        t_wall0 = time.monotonic()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(K):
                lz, t, nq, fl = step((W + i) % R, ev[i], stage_ev)
                launches += lz
                tokens += t
                flush_steps.append(fl)
                bytes_decode += (decode_alg_bytes(w, nq, t - nq) + (append_bytes(w) if MODE != "separate" else 0)
                                 + (flush_bytes(w) if fl else 0))
            e1.record(stream)
            stream.synchronize()
        torch.cuda.synchronize(device)
        barrier()
        t_wall1 = time.monotonic()
        last = {"out": out.clone(), "replica": (counter[0] - 1) % replicas,
                "steps": len(schedule[(counter[0] - 1) % replicas])}
        # the clock record spans at least CLOCK_WINDOW_S: the same steps continue, untimed
        ext = 0
        with torch.cuda.stream(stream):
            while time.monotonic() - t_wall0 < CLOCK_WINDOW_S:
                for _ in range(64):
                    step((W + K + ext) % R)
                    ext += 1
                stream.synchronize()
        t_wall2 = time.monotonic()
        ms = e0.elapsed_time(e1)
        step_ms = [a.elapsed_time(b) for a, b in ev]
        dec_ms = sum(step_ms)
        stage_ms = {k: (sum(a.elapsed_time(b) for a, b in v) / len(v) if v else None) for k, v in stage_ev.items()}
        fl_ms = [x for x, f in zip(step_ms, flush_steps) if f]
        plain_ms = [x for x, f in zip(step_ms, flush_steps) if not f]
        if fl_ms and plain_ms:   # the decode step: what its flush adds to the launch
            stage_ms["flush_in_launch"] = statistics.mean(fl_ms) - statistics.mean(plain_ms)
            stage_ms["flush_steps"] = len(fl_ms)
        clk = sampler.summary(t_wall0, t_wall2)
        clk["window_s"] = round(t_wall2 - t_wall0, 3)
        clk["window"] = (f"the {K} timed steps ({(t_wall1 - t_wall0) * 1e3:.1f} ms wall) and {ext} more of the same "
                         f"steps after them, untimed, so that nvidia-smi (50 ms period) samples the kernel")
        return ms, dec_ms, launches, tokens, bytes_decode, clk, stage_ms, last

    ms, dec_ms, launches, tokens, bytes_decode, clk, stage_ms, last = timed_loop(args.steps, args.warmup)
    log(f"timed loop done: {ms:.3f} ms for {args.steps} steps; clocks {clk.get('sm_mhz')} MHz "
        f"({clk.get('samples')} samples)")
    if BAD_REASONS & set(clk["reasons"]):
        ms, dec_ms, launches, tokens, bytes_decode, clk, stage_ms, last = timed_loop(args.steps, args.warmup)
        clk["remeasured"] = True
        log(f"re-measured (throttle reasons seen): {ms:.3f} ms")
    sampler.stop()
    t_max, dec_ms = ranks.max(ms, dec_ms)
    status = max(c.read_status(stream) for c in caches)
    if status != 0:
        log(f"device status {status} after the timed steps")

    # ---- one flush, timed on its own (the timed window may hold none) -------------------------
    flush_ms_sep = []
    fl = [torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
    with torch.cuda.stream(stream):
        for _ in range(3):
            c = caches[counter[0] % replicas]
            if MODE == "step":          # the decode step never leaves a full residual: append to one
                if c.c.n_quant == n_quant0 + 2 * R:
                    c.c.n_quant = n_quant0 + R
                while c.c.n_res < R:
                    c.append(dev_in[0][0], dev_in[0][1], stream)
            else:
                while c.c.n_res < R:        # steps of this replica until its residual is full
                    for _r in range(replicas):
                        step(counter[0] % R)
                if c.c.n_quant == n_quant0 + R:
                    c.c.n_quant = n_quant0   # the cycle of gpu_step; the replica's next step finds n_res = 0
            fl[0].record(stream)
            c.flush(stream)
            fl[1].record(stream)
            stream.synchronize()
            flush_ms_sep.append(fl[0].elapsed_time(fl[1]))

    # ---- end to end through the public API with host buffers ---------------------------------
    # Each step's new K, V rows and queries sit back to back in one pinned buffer and arrive with one
    # host-to-device copy into one staging buffer (three 16-byte-aligned views).
    shapes = [a.shape for a in host_in[0]]
    sizes = [int(np.prod(sh)) for sh in shapes]
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(int)
    pinned = []
    for x in host_in:
        buf = torch.empty(int(offs[-1]), dtype=torch.float16).pin_memory()
        for a, o0, o1 in zip(x, offs[:-1], offs[1:]):
            buf[o0:o1].copy_(torch.from_numpy(np.ascontiguousarray(a)).reshape(-1))
        pinned.append(buf)
    # two staging buffers: step i + 1's inputs cross PCIe on a copy stream while step i computes
    stage_bufs = [torch.empty(int(offs[-1]), dtype=torch.float16, device=device) for _ in range(2)]
    stages = [[sb[o0:o1].view(sh) for o0, o1, sh in zip(offs[:-1], offs[1:], shapes)] for sb in stage_bufs]
    copy_stream = torch.cuda.Stream(device)
    landed = [torch.cuda.Event(), torch.cuda.Event()]
    out_host = torch.empty(w.batch, w.q_heads, w.head_dim, dtype=torch.float16).pin_memory()
    h2d = int(offs[-1]) * 2
    d2h = out_host.numel() * out_host.element_size()

    def copy_inputs(i):
        """Step i's inputs into staging buffer i % 2, on the copy stream."""
        with torch.cuda.stream(copy_stream):
            stage_bufs[i % 2].copy_(pinned[i % R], non_blocking=True)
            landed[i % 2].record(copy_stream)

    def e2e_loop(K):
        barrier()
        torch.cuda.synchronize(device)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        toks = 0
        with torch.cuda.stream(stream):
            f0.record(stream)
            copy_stream.wait_stream(stream)   # the first copy starts inside the timed region
            copy_inputs(0)
            for i in range(K):
                stream.wait_event(landed[i % 2])
                if i + 1 < K:   # buffer (i + 1) % 2 was read by step i - 1, which the last synchronize ended
                    copy_inputs(i + 1)
                toks += step(i % R, inputs=stages[i % 2])[1]
                out_host.copy_(out, non_blocking=True)
                stream.synchronize()      # the caller consumes the step's result
            f1.record(stream)
            stream.synchronize()
        return f0.elapsed_time(f1), toks

    log("end-to-end loop")
    e2e_steps = 0 if args.no_e2e else min(args.steps, 4 * R)
    e2e_ms, e2e_tokens = e2e_loop(e2e_steps) if e2e_steps else (float("nan"), 0)
    e2e_ms = ranks.max(e2e_ms)
    status = max(status, max(c.read_status(stream) for c in caches))

    result = None
    if rank == 0:
        K = args.steps
        value = weak_scaling_value(world, tokens, w.batch, t_max)
        peak, peak_kind = hbm_peak()
        dec_avg_ms = dec_ms / K
        achieved = (bytes_decode / K) / (dec_avg_ms / 1e3) / 1e9
        traffic = profiled_traffic(w, bytes_decode / K) if replicas == 1 else None
        e2e_value = weak_scaling_value(world, e2e_tokens, w.batch, e2e_ms)
        flush_window = stage_ms["flush"]
        flush_source = "flushes inside the timed window"
        if stage_ms.get("flush_in_launch") is not None:
            flush_window = stage_ms["flush_in_launch"]
            flush_source = (f"in-launch: the {stage_ms['flush_steps']} timed steps that flushed, minus the "
                            f"average of the others")
        result = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": t_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": f"u{w.bits} codes x i8 limbs ({dot_engine(w)}, i32 acc), f32 softmax", "data": "synthetic",
            "config": workload_config(w, world, replicas),
            "hbm_gbs_decode": achieved, "hbm_frac_of_8tbs": achieved / SPEC_HBM_GBS,
            "decode_ms_avg": dec_avg_ms,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": peak_kind, "traffic": traffic,
                         "kernel": f"decode_kernel<{w.bits},{w.gqa}>", "alg_bytes_per_launch": bytes_decode / K},
            "clocks": clk,
            "device_status": status,
            "stages": {
                "decode_ms": dec_avg_ms,
                "append_ms": stage_ms["append"],
                "flush_ms": flush_window if flush_window is not None else statistics.median(flush_ms_sep),
                "flush_ms_source": (flush_source if flush_window is not None else
                                    "3 flushes timed on their own after the timed window"),
                "flush_ms_separate": statistics.median(flush_ms_sep),
                "prefill_ms": prefill_ms, "prefill_tokens": w.tokens,
                "prefill_gbs": (w.batch * w.kv_heads * w.tokens * w.head_dim * 2 * 2
                                + decode_alg_bytes(w, n_quant0, 0)) / (prefill_ms / 1e3) / 1e9,
            },
            "gpu_launches": launches,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps, "ms_per_step": e2e_ms / max(1, e2e_steps)},
            "published": PUBLISHED,
        }
        result["_parity_state"] = {"out": last["out"].cpu().numpy(), "schedule": schedule[last["replica"]][:last["steps"]],
                                   "n_quant0": n_quant0}
    if dist is not None:
        ranks.barrier()
        dist.destroy_process_group()
    return result


# ------------------------------------------------------------------------------------------------
# the CPU oracle (cpu_baseline leg and --impl reference)
# ------------------------------------------------------------------------------------------------
def _oracle_head(w: synth.Workload, b: int, h: int):
    import oracle.kivi_oracle as O
    n_quant0, cap = first_prompt_split(w)
    hc = O.HeadCache(w.head_dim, w.bits, w.group, w.gv, w.residual, cap, online_k=ONLINE_K, fine_groups=FINE)
    hc.prefill(synth.prompt_k(w, b, h, w.tokens), synth.prompt_v(w, b, h, w.tokens))
    return hc, n_quant0


def _oracle_truncate(w: synth.Workload, hc, n: int):
    """Drops the quantized tokens from n on (whole blocks), as the bench's cycle does on the GPU."""
    R = w.residual
    hc.k_codes, hc.v_codes = hc.k_codes[:n], hc.v_codes[:n]
    if hc.fine:
        hc.k_s, hc.k_z = hc.k_s[:n // w.group], hc.k_z[:n // w.group]
        hc.v_s, hc.v_z = hc.v_s[:n], hc.v_z[:n]
    else:
        hc.k_s, hc.k_z = hc.k_s[:n // R], hc.k_z[:n // R]
        hc.v_s, hc.v_z = hc.v_s[:n // w.gv], hc.v_z[:n // w.gv]


def _oracle_cycle_flush(w: synth.Workload, hc, n_quant0: int):
    """The flush of gpu_step's cycle, applied to a full residual before the next append.  The decode
    step flushes into the block after n_quant0 + R and drops it; the lazy modes move n_quant back to
    n_quant0 first (the cycle's block is rewritten).  Flushing eagerly or at the next append gives
    the same attention, so the oracle flushes at the next append in every mode."""
    R = w.residual
    if MODE == "step":
        hc.flush()
        if hc.n_quant == n_quant0 + 2 * R:
            _oracle_truncate(w, hc, n_quant0 + R)
        return
    if hc.n_quant == n_quant0 + R:
        _oracle_truncate(w, hc, n_quant0)
    hc.flush()


def oracle_parity(w: synth.Workload, state: dict, n_heads: int):
    """The oracle replays the steps the GPU cache of the last timed step went through (prefill, then
    every flush and append, with the same synthetic inputs) on a sample of KV heads and compares the
    last timed step's output with its attention (max-abs 2e-3 and max-rel 1e-2, relative to
    max(|o*|, 1e-2))."""
    R = w.residual
    rng = np.random.default_rng(w.seed)
    heads = {(0, 0), (w.batch - 1, w.kv_heads - 1)}
    while len(heads) < min(n_heads, w.batch * w.kv_heads):
        heads.add((int(rng.integers(w.batch)), int(rng.integers(w.kv_heads))))
    sched = state["schedule"]
    got = state["out"].astype(np.float64)
    scale = 1.0 / math.sqrt(w.head_dim)
    ea = er = raw = 0.0
    t0 = time.perf_counter()
    for (b, h) in sorted(heads):
        hc, n_quant0 = _oracle_head(w, b, h)
        for sid in sched:
            if hc.n_res == R:
                _oracle_cycle_flush(w, hc, n_quant0)
            hc.append(synth.new_k(w, b, h, sid), synth.new_v(w, b, h, sid))
        q = np.stack([synth.query(w, b, h * w.gqa + g, sched[-1]) for g in range(w.gqa)])
        want = hc.attend(q, scale)
        err = np.abs(got[b, h * w.gqa:(h + 1) * w.gqa] - want)
        # half the fp16 spacing at |o*|: what a correctly rounded fp16 output may differ by
        half_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(want), 2.0 ** -14))) - 11)
        raw = max(raw, float(err.max()))
        ea = max(ea, float(np.maximum(err - half_ulp, 0.0).max()))
        er = max(er, float((err / np.maximum(np.abs(want), 1e-2)).max()))
    return {"heads": len(heads), "steps_replayed": len(sched), "max_abs": ea, "max_rel": er, "max_abs_raw": raw,
            "ok": bool(ea <= 2e-3 and er <= 1e-2),
            "tolerance": ("vs the fp64 oracle: max-abs 2e-3 beyond the fp16 output's own rounding (half an fp16 ulp "
                          "of o*) and max-rel 1e-2 (floor 1e-2)"),
            "seconds": round(time.perf_counter() - t0, 1)}


def oracle_sample(w: synth.Workload, n_heads: int, n_steps: int, budget_s: float):
    """Times the oracle as it stands on `n_heads` KV heads for up to `n_steps` decode steps each
    (threads over heads).  Returns (value in tokens/s/head, cores, sample description, seconds,
    head-steps)."""
    from concurrent.futures import ThreadPoolExecutor
    R = w.residual
    heads = [(b, h) for b in range(w.batch) for h in range(w.kv_heads)][:: max(1, (w.batch * w.kv_heads) // n_heads)]
    heads = heads[:n_heads]
    caches = {bh: _oracle_head(w, *bh) for bh in heads}
    scale = 1.0 / math.sqrt(w.head_dim)
    cores = os.cpu_count() or 1
    deadline = time.perf_counter() + budget_s

    def run_head(bh):
        b, h = bh
        hc, n_quant0 = caches[bh]
        done, toks = 0, 0
        for s in range(1, n_steps + 1):
            if time.perf_counter() > deadline and done > 0:
                break
            if hc.n_res == R:
                _oracle_cycle_flush(w, hc, n_quant0)
            hc.append(synth.new_k(w, b, h, s), synth.new_v(w, b, h, s))
            q = np.stack([synth.query(w, b, h * w.gqa + g, s) for g in range(w.gqa)])
            hc.attend(q, scale)
            done += 1
            toks += hc.n_quant + hc.n_res
        return done, toks

    t0 = time.perf_counter()
    with ThreadPoolExecutor(cores) as ex:
        res = list(ex.map(run_head, heads))
    dt = time.perf_counter() - t0
    head_steps = sum(r[0] for r in res)
    tok = sum(r[1] for r in res)
    sample = (f"oracle (numpy fp64) decode steps of {len(heads)} of {w.batch * w.kv_heads} KV heads of "
              f"{w.name}: {head_steps} head-steps (flush when full + append + attention), "
              f"{cores} threads over heads, {dt:.1f} s")
    # A full step is B*H head-steps and counts B*T tokens per head, so a sample of head-steps with
    # `tok` cached tokens in total gives tok / dt / H cached tokens/s/head.
    return tok / dt / w.kv_heads, cores, sample, dt, head_steps


def run_reference(args, rank, world, w: synth.Workload):
    if rank != 0:
        return None
    budget = max(5.0, min(60.0, 0.6 * args.steps + 5.0))
    value, cores, sample, dt, hs = oracle_sample(w, n_heads=min(64, 2 * (os.cpu_count() or 1)),
                                                 n_steps=max(1, args.steps), budget_s=budget)
    ms_head_step = dt * 1e3 / max(1, hs)
    ms_full_step = ms_head_step * (w.batch * w.kv_heads)   # one step covers every KV head
    n_quant0, _ = first_prompt_split(w)
    replicas = args.replicas if args.replicas > 0 else auto_replicas(w, n_quant0)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_full_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, world, replicas),
        "ms_per_step_kind": (f"extrapolated: {ms_head_step:.2f} ms measured per head-step on {hs} head-steps, "
                             f"times {w.batch * w.kv_heads} KV heads per step"),
        "ms_per_head_step_measured": ms_head_step,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "published": PUBLISHED,
    }


def log(msg: str) -> None:
    sys.stderr.write(f"[bench {time.strftime('%H:%M:%S')}] {msg}\n")
    sys.stderr.flush()


def main():
    faulthandler.enable()
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2048)
    ap.add_argument("--warmup", type=int, default=128)
    ap.add_argument("--impl", choices=["kivi", "reference"], default="kivi")
    ap.add_argument("--workload", choices=sorted(synth.WORKLOADS), default=WORKLOAD.name,
                    help="workload to time (default: the large-batch workload the metric is quoted on)")
    ap.add_argument("--bits", type=int, choices=[2, 4], default=None, help="override the workload's bits")
    ap.add_argument("--group", type=int, choices=[32, 64, 128], default=None, help="override G_k = G_v")
    ap.add_argument("--replicas", type=int, default=0,
                    help="cache replicas rotated one per step (0: enough to defeat the L2 for small workloads)")
    ap.add_argument("--parity-heads", type=int, default=16,
                    help="KV heads the cpu_baseline leg replays to check the last timed step (0: none)")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle legs (profiling runs)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end loop (profiling runs)")
    ap.add_argument("--separate-append", action="store_true",
                    help="append and decode as two launches (kivi_append_token + kivi_decode_attention)")
    ap.add_argument("--lazy-flush", action="store_true",
                    help="flush a full residual with its own launch at the next step, then append and decode in "
                         "one launch (kivi_flush_residual + kivi_append_decode_attention)")
    ap.add_argument("--fine-groups", action="store_true",
                    help="fine-grained groups (config fine_groups = 1); no cpu baseline timing")
    ap.add_argument("--online-k", action="store_true",
                    help="online K quantization (config online_k = 1); implies --separate-append and no "
                         "cpu baseline timing")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    global MODE, ONLINE_K, FINE
    ONLINE_K = args.online_k
    FINE = args.fine_groups
    if FINE and args.impl == "reference":
        ap.error("--fine-groups times the GPU arm only")
    MODE = "separate" if (args.separate_append or args.online_k) else ("fused" if args.lazy_flush else "step")
    if ONLINE_K and args.impl == "reference":
        ap.error("--online-k times the GPU arm only")
    w = synth.WORKLOADS[args.workload]
    if args.bits is not None:
        w = w.with_(bits=args.bits)
    if args.group is not None:
        w = w.with_(group=args.group)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus if args.gpus == 1 else 1)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world, w)
    else:
        res = run_gpu(args, rank, world, local_rank, w)
        if res is not None:
            state = res.pop("_parity_state")
            if world == 1 and not args.no_cpu_baseline:
                if args.parity_heads > 0:
                    log("cpu baseline leg: oracle replay of the last timed step")
                    res["parity"] = oracle_parity(w, state, args.parity_heads)
                if not ONLINE_K and not FINE:
                    log("cpu baseline leg: oracle timing")
                    value, cores, sample, dt, hs = oracle_sample(w, n_heads=min(64, 2 * (os.cpu_count() or 1)),
                                                                 n_steps=16, budget_s=25.0)
                    res["cpu_baseline"] = {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                                           "sample": sample}
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()

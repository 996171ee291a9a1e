#!/usr/bin/env python
"""Benchmark: 2-bit KIVI decode over a quantized KV cache on B200, one JSON line on stdout.

A step is one streaming decode step of the large-batch workload (B=64, H=32, d=128, 2-bit, G=32,
R=128): flush the residual when it is full (once every 128 steps), append one new K/V token per
(batch, KV head), and run decode attention for every query head over the whole cache.  After each
128-step cycle the host moves n_quant back by one block, so the cache cycles between 8193 and 8320
cached tokens instead of growing; every step does its full work.  Inputs live in HBM (1.2 GB of codes
and scales per step, ten times the 126 MB L2, so no L2 flush is needed).

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
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_asymmetric_kv_02_b200 import synth  # noqa: E402

METRIC = "2-bit KV decode-attention cached tokens/s/head and HBM GB/s vs 8 TB/s peak (1 B200)"
UNIT = "cached tokens/s/head"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
WORKLOAD = synth.LARGE_BATCH
FUSED = True   # append and decode in one launch (kivi_append_decode_attention); --separate-append: two
STEP_NOTE = {True: "flush when full + append and decode attention in one launch",
             False: "flush when full + append + decode attention"}
ONLINE_K = False   # --online-k: K rows coded at append with the newest block's (s, z) (config online_k)
FINE = False       # --fine-groups: K (s, z) per channel per G tokens, V per token per G channels
DECODE_SOURCES = ["decode.cu", "common.cuh", "kernels.h"]


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


def l2_note(w: synth.Workload, n_quant: int) -> str:
    gb = decode_alg_bytes(w, n_quant, w.residual) / 1e9
    if gb * 1e3 > 2 * 126:
        return f"not flushed: inputs ({gb:.2f} GB per step) exceed the 126 MB L2"
    return f"WARNING: inputs ({gb * 1e3:.0f} MB per step) fit in the 126 MB L2; not flushed"


def append_bytes(w: synth.Workload) -> int:
    """Bytes a fused append adds to the decode launch: the new K and V rows read and written once."""
    return w.batch * w.kv_heads * w.head_dim * 2 * 2 * 2


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


class ClockSampler:
    """Samples SM clock, max clock and throttle reasons of one GPU with nvidia-smi every 50 ms while
    the timed region runs (the clocks line of the profiling recipe)."""

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
        self.lines = []

    @staticmethod
    def _bus_of(field: str):
        """(bus, device) of an nvidia-smi pci.bus_id such as 00000000:1B:00.0."""
        try:
            parts = field.strip().split(":")
            return int(parts[-2], 16), int(parts[-1].split(".")[0], 16)
        except (ValueError, IndexError):
            return None

    def __enter__(self):
        import shutil
        import subprocess
        exe = shutil.which("nvidia-smi")
        if exe:
            self.proc = subprocess.Popen([exe, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=10)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        rows = []
        for ln in self.lines:
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
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
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


# ------------------------------------------------------------------------------------------------
# the GPU arm
# ------------------------------------------------------------------------------------------------
def make_state(w: synth.Workload, torch, kivi, device):
    n_quant0 = (w.tokens - 1) // w.residual * w.residual      # 8064: the prompt leaves a full residual
    capacity = n_quant0 + (2 if ONLINE_K else 1) * w.residual   # online K: a slot for the block being filled
    k, v = synth.prompt_kv(w, w.tokens)
    cache = kivi.KiviCache(w.batch, w.kv_heads, capacity, bits=w.bits, group_k=w.group, group_v=w.group,
                           residual=w.residual, num_q_heads=w.q_heads, device=device, online_k=ONLINE_K,
                           fine_groups=FINE)
    kd = torch.from_numpy(k).to(device)
    vd = torch.from_numpy(v).to(device)
    cache.prefill(kd, vd)            # first run loads the module; the second one is timed
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    cache.prefill(kd, vd)
    e1.record()
    torch.cuda.synchronize(device)
    prefill_ms = e0.elapsed_time(e1)
    del kd, vd, k, v
    torch.cuda.empty_cache()   # hand the 8.6 GB of prompt back: the decode loop holds ~1.3 GB
    # per-step inputs for a cycle of 128 steps (new K/V rows and queries), resident in HBM
    steps_in = []
    for s in range(w.residual):
        kn, vn = synth.new_kv(w, s + 1)
        q = synth.queries(w, s + 1)
        steps_in.append((kn, vn, q))
    dev_in = [tuple(torch.from_numpy(a).to(device) for a in x) for x in steps_in]
    torch.cuda.synchronize(device)
    assert (cache.n_quant, cache.n_res) == (n_quant0, w.residual)
    return cache, n_quant0, steps_in, dev_in, prefill_ms


def gpu_step(cache, n_quant0, w, inputs, out, stream, decode_events=None, stage_events=None):
    """One streaming decode step on device-resident inputs; returns (launches, cached tokens).
    stage_events (optional): {"flush": [...], "append": [...]} lists that receive event pairs."""
    import torch
    launches = 0
    if cache.c.n_res == w.residual:
        if cache.c.n_quant == n_quant0 + w.residual:
            cache.c.n_quant = n_quant0     # end of a 128-step cycle: drop the newest block again
        if stage_events is not None:
            ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            ev[0].record(stream)
        cache.flush(stream)
        if stage_events is not None:
            ev[1].record(stream)
            stage_events["flush"].append(ev)
        launches += 1
    kn, vn, q = inputs
    if FUSED:
        if decode_events is not None:
            decode_events[0].record(stream)
        cache.append_attend(kn, vn, q, out=out, stream=stream, status=False)
        if decode_events is not None:
            decode_events[1].record(stream)
        return launches + 1, cache.c.n_quant + cache.c.n_res
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
    cache.attend(q, out=out, stream=stream, status=False)
    if decode_events is not None:
        decode_events[1].record(stream)
    launches += 1
    return launches, cache.c.n_quant + cache.c.n_res


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

    log("generating inputs and prefilling the cache")
    cache, n_quant0, host_in, dev_in, prefill_ms = make_state(w, torch, kivi, device)
    log("cache ready")
    stream = torch.cuda.Stream(device)
    out = torch.empty(w.batch, w.q_heads, w.head_dim, dtype=torch.float16, device=device)
    R = w.residual

    barrier = ranks.barrier

    # ---- device-resident timing -------------------------------------------------------------
    def timed_loop(K, W):
        with torch.cuda.stream(stream):
            for i in range(W):
                gpu_step(cache, n_quant0, w, dev_in[i % R], out, stream)
        stream.synchronize()
        barrier()
        torch.cuda.synchronize(device)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        launches, tokens = 0, 0
        bytes_decode = 0
        stage_ev = {"flush": [], "append": []}
        with ClockSampler(local_rank) as clocks, torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(K):
                n_q, n_r = cache.c.n_quant, cache.c.n_res
                lz, t = gpu_step(cache, n_quant0, w, dev_in[(W + i) % R], out, stream, ev[i], stage_ev)
                launches += lz
                tokens += t
                n_q2 = cache.c.n_quant
                bytes_decode += decode_alg_bytes(w, n_q2, t - n_q2) + (append_bytes(w) if FUSED else 0)
            e1.record(stream)
            stream.synchronize()
        torch.cuda.synchronize(device)
        barrier()
        ms = e0.elapsed_time(e1)
        dec_ms = sum(a.elapsed_time(b) for a, b in ev)
        stage_ms = {k: (sum(a.elapsed_time(b) for a, b in v) / len(v) if v else None) for k, v in stage_ev.items()}
        clk = clocks.summary()
        clk["stage_ms"] = stage_ms
        return ms, dec_ms, launches, tokens, bytes_decode, clk

    ms, dec_ms, launches, tokens, bytes_decode, clk = timed_loop(args.steps, args.warmup)
    log(f"timed loop done: {ms:.3f} ms for {args.steps} steps")
    if BAD_REASONS & set(clk["reasons"]):
        ms, dec_ms, launches, tokens, bytes_decode, clk = timed_loop(args.steps, args.warmup)
        clk["remeasured"] = True
        log(f"re-measured (throttle reasons seen): {ms:.3f} ms")
    t_max, dec_ms = ranks.max(ms, dec_ms)

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
    stage_buf = torch.empty(int(offs[-1]), dtype=torch.float16, device=device)
    stage = [stage_buf[o0:o1].view(sh) for o0, o1, sh in zip(offs[:-1], offs[1:], shapes)]
    out_host = torch.empty(w.batch, w.q_heads, w.head_dim, dtype=torch.float16).pin_memory()
    h2d = int(offs[-1]) * 2
    d2h = out_host.numel() * out_host.element_size()

    def e2e_loop(K):
        barrier()
        torch.cuda.synchronize(device)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        toks = 0
        with torch.cuda.stream(stream):
            f0.record(stream)
            for i in range(K):
                stage_buf.copy_(pinned[i % R], non_blocking=True)
                _, t = gpu_step(cache, n_quant0, w, stage, out, stream)
                toks += t
                out_host.copy_(out, non_blocking=True)
                stream.synchronize()      # the caller consumes the step's result
            f1.record(stream)
            stream.synchronize()
        return f0.elapsed_time(f1), toks

    log("end-to-end loop")
    e2e_steps = 0 if args.no_e2e else min(args.steps, 4 * R)
    e2e_ms, e2e_tokens = e2e_loop(e2e_steps) if e2e_steps else (float("nan"), 0)
    e2e_ms = ranks.max(e2e_ms)

    result = None
    if rank == 0:
        K = args.steps
        value = weak_scaling_value(world, tokens, w.batch, t_max)
        peak, peak_kind = hbm_peak()
        dec_avg_ms = dec_ms / K
        achieved = (bytes_decode / K) / (dec_avg_ms / 1e3) / 1e9
        traffic = profiled_traffic(w, bytes_decode / K)
        e2e_value = weak_scaling_value(world, e2e_tokens, w.batch, e2e_ms)
        result = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": t_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": f"u{w.bits} codes x i8 limbs ({dot_engine(w)}, i32 acc), f32 softmax", "data": "synthetic",
            "config": {
                "workload": w.name, "batch": w.batch, "q_heads": w.q_heads, "kv_heads": w.kv_heads,
                "head_dim": w.head_dim, "bits": w.bits, "group_k": w.group, "group_v": w.group,
                "residual": w.residual, "cached_tokens": f"{n_quant0 + 1}-{n_quant0 + 2 * R} (128-step cycles)",
                "step": STEP_NOTE[FUSED],
                "k_residual": "codes (online K, config online_k = 1)" if ONLINE_K else "fp16",
                "groups": ("fine: K per channel per G tokens, V per token per G channels (config fine_groups = 1)"
                           if FINE else "K per R-token block x G channels, V per G tokens x all channels"),
                "l2": l2_note(w, n_quant0),
                "parallelism": f"weak: one independent batch per GPU x {world}",
            },
            "hbm_gbs_decode": achieved, "hbm_frac_of_8tbs": achieved / SPEC_HBM_GBS,
            "decode_ms_avg": dec_avg_ms,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": peak_kind, "traffic": traffic,
                         "kernel": f"decode_kernel<{w.bits},{w.gqa}>", "alg_bytes_per_launch": bytes_decode / K},
            "clocks": {k: v for k, v in clk.items() if k != "stage_ms"},
            "stages": {
                "decode_ms": dec_avg_ms,
                "append_ms": clk["stage_ms"]["append"], "flush_ms": clk["stage_ms"]["flush"],
                "prefill_ms": prefill_ms, "prefill_tokens": w.tokens,
                "prefill_gbs": (w.batch * w.kv_heads * w.tokens * w.head_dim * 2 * 2
                                + decode_alg_bytes(w, n_quant0, 0)) / (prefill_ms / 1e3) / 1e9,
            },
            "gpu_launches": launches,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps, "ms_per_step": e2e_ms / max(1, e2e_steps)},
        }
    if dist is not None:
        ranks.barrier()
        dist.destroy_process_group()
    return result


# ------------------------------------------------------------------------------------------------
# the CPU oracle (cpu_baseline leg and --impl reference)
# ------------------------------------------------------------------------------------------------
def oracle_sample(w: synth.Workload, n_heads: int, n_steps: int, budget_s: float):
    """Times the oracle as it stands on `n_heads` KV heads for up to `n_steps` decode steps each
    (threads over heads).  Returns (value in tokens/s/head, cores, sample description, seconds)."""
    import oracle.kivi_oracle as O
    from concurrent.futures import ThreadPoolExecutor
    R = w.residual
    n_quant0 = (w.tokens - 1) // R * R
    cap = n_quant0 + R
    heads = [(b, h) for b in range(w.batch) for h in range(w.kv_heads)][:: max(1, (w.batch * w.kv_heads) // n_heads)]
    heads = heads[:n_heads]
    caches = {}
    for (b, h) in heads:
        hc = O.HeadCache(w.head_dim, w.bits, w.group, w.group, R, cap)
        hc.prefill(synth.prompt_k(w, b, h, w.tokens), synth.prompt_v(w, b, h, w.tokens))
        caches[(b, h)] = hc
    scale = 1.0 / math.sqrt(w.head_dim)
    cores = os.cpu_count() or 1
    deadline = time.perf_counter() + budget_s

    def run_head(bh):
        b, h = bh
        hc = caches[bh]
        done, toks = 0, 0
        for s in range(1, n_steps + 1):
            if time.perf_counter() > deadline and done > 0:
                break
            if hc.n_res == R:
                if hc.n_quant == n_quant0 + R:   # same 128-step cycle as the GPU arm
                    hc.k_codes, hc.v_codes = hc.k_codes[:n_quant0], hc.v_codes[:n_quant0]
                    hc.k_s, hc.k_z = hc.k_s[:n_quant0 // R], hc.k_z[:n_quant0 // R]
                    hc.v_s, hc.v_z = hc.v_s[:n_quant0 // w.group], hc.v_z[:n_quant0 // w.group]
                hc.flush()
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
    ms_full_step = dt * 1e3 * (w.batch * w.kv_heads) / max(1, hs)   # one step covers every KV head
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_full_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "q_heads": w.q_heads, "kv_heads": w.kv_heads,
                   "head_dim": w.head_dim, "bits": w.bits, "group_k": w.group, "group_v": w.group,
                   "residual": w.residual, "step": STEP_NOTE[FUSED]},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
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
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing (profiling runs)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end loop (profiling runs)")
    ap.add_argument("--separate-append", action="store_true",
                    help="append and decode as two launches (kivi_append_token + kivi_decode_attention)")
    ap.add_argument("--fine-groups", action="store_true",
                    help="fine-grained groups (config fine_groups = 1; 2 bits, one query per KV head); no cpu "
                         "baseline")
    ap.add_argument("--online-k", action="store_true",
                    help="online K quantization (config online_k = 1); implies --separate-append and no "
                         "cpu baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    global FUSED, ONLINE_K, FINE
    ONLINE_K = args.online_k
    FINE = args.fine_groups
    if FINE and args.impl == "reference":
        ap.error("--fine-groups times the GPU arm only")
    FUSED = not (args.separate_append or args.online_k)
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
        if rank == 0 and world == 1 and not args.no_cpu_baseline and not ONLINE_K and not FINE:
            log("cpu baseline (oracle)")
            value, cores, sample, dt, hs = oracle_sample(w, n_heads=min(64, 2 * (os.cpu_count() or 1)),
                                                         n_steps=16, budget_s=25.0)
            res["cpu_baseline"] = {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                                   "sample": sample}
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()

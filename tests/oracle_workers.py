"""The oracle over every KV head of a full-size workload, in spawned worker processes.

Test infrastructure.  The full-size GPU parity tests and bench.py's parity check run the oracle on
all heads (or a sample) of a workload: one HeadCache per (batch, KV head), regenerated from the
seeded synthetic inputs (bit_asymmetric_kv_02_b200/synth.py) inside the worker, so nothing but the
head's coordinates travels to it.  A worker returns, at every checkpoint of the head's stream, the
SHA-1 of each packed buffer (the library's device layout, HeadCache.packed) and the attention
outputs of the step's queries; the caller hashes the GPU's buffers of the same head the same way
and compares.  The pool is started with the spawn method, so it is safe after CUDA is initialised.
"""
from __future__ import annotations

import hashlib
import os
from concurrent.futures import ProcessPoolExecutor
from dataclasses import dataclass

import numpy as np


def digest(a) -> tuple:
    """(shape, sha1 of the bytes) of an array in C order."""
    a = np.ascontiguousarray(a)
    return tuple(a.shape), hashlib.sha1(a.view(np.uint8).tobytes()).hexdigest()


@dataclass(frozen=True)
class HeadStream:
    """One KV head's life: prefill `prompt` tokens, then `steps` decode steps.  Step i (1-based)
    flushes when the residual is full, appends the row of synthetic step inputs[i-1] and, if i is
    in `attend_at`, attends the queries of that step.  cycle_nquant > 0 sets n_quant back to it
    whenever a flush would go past cycle_nquant + R (the bench's fixed-size cycle)."""
    workload: object          # synth.Workload
    b: int
    h: int
    capacity: int
    prompt: int
    steps: int = 0
    inputs: tuple = ()        # synthetic step id of each decode step (default 1..steps)
    attend_at: frozenset = frozenset()
    digest_at: frozenset = frozenset()   # steps after which the buffers are hashed (0: after prefill)
    flush_digests: bool = True           # hash the buffers after every flush
    scale: float = 0.0                   # 0: 1/sqrt(d)
    cycle_nquant: int = 0
    online_k: bool = False
    fine_groups: bool = False


def run_head(spec: HeadStream) -> list:
    """[(label, kind, payload)]: kind 'buffers' -> {name: digest}, kind 'out' -> float64 [g][d]."""
    import oracle.kivi_oracle as O
    from bit_asymmetric_kv_02_b200 import synth
    w = spec.workload
    R = w.residual
    scale = spec.scale or 1.0 / np.sqrt(w.head_dim)
    hc = O.HeadCache(w.head_dim, w.bits, w.group, w.gv, R, spec.capacity, online_k=spec.online_k,
                     fine_groups=spec.fine_groups)
    hc.prefill(synth.prompt_k(w, spec.b, spec.h, spec.prompt), synth.prompt_v(w, spec.b, spec.h, spec.prompt))
    out = []

    def buffers(label):
        out.append((label, "buffers", {k: digest(v) for k, v in hc.packed().items()}))

    def attend(label, step_id):
        q = np.stack([synth.query(w, spec.b, spec.h * w.gqa + g, step_id) for g in range(w.gqa)])
        out.append((label, "out", hc.attend(q, scale)))

    if 0 in spec.digest_at:
        buffers("step 0")
    if 0 in spec.attend_at:
        attend("step 0", 0)
    inputs = spec.inputs or tuple(range(1, spec.steps + 1))
    for i in range(1, spec.steps + 1):
        if hc.n_res == R:
            if spec.cycle_nquant and hc.n_quant == spec.cycle_nquant + R:
                n = spec.cycle_nquant
                hc.k_codes, hc.v_codes = hc.k_codes[:n], hc.v_codes[:n]
                if hc.fine:
                    hc.k_s, hc.k_z = hc.k_s[:n // w.group], hc.k_z[:n // w.group]
                    hc.v_s, hc.v_z = hc.v_s[:n], hc.v_z[:n]
                else:
                    hc.k_s, hc.k_z = hc.k_s[:n // R], hc.k_z[:n // R]
                    hc.v_s, hc.v_z = hc.v_s[:n // w.gv], hc.v_z[:n // w.gv]
            hc.flush()
            if spec.flush_digests:
                buffers(f"flush before step {i}")
        sid = inputs[i - 1]
        hc.append(synth.new_k(w, spec.b, spec.h, sid), synth.new_v(w, spec.b, spec.h, sid))
        if i in spec.digest_at:
            buffers(f"step {i}")
        if i in spec.attend_at:
            attend(f"step {i}", sid)
    return out


def _one_thread_per_worker():
    """The pool runs one process per core: each keeps its numpy linear algebra to one thread, so the
    processes do not share the cores with each other's thread pools.  Only the speed depends on it:
    where the limit cannot be set, the worker runs with the default threads."""
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=1)
    except Exception:
        pass


def pool(workers: int | None = None) -> ProcessPoolExecutor:
    import multiprocessing as mp
    n = workers or max(1, min(32, os.cpu_count() or 1))
    return ProcessPoolExecutor(n, mp_context=mp.get_context("spawn"), initializer=_one_thread_per_worker)


def run_heads(specs, workers: int | None = None) -> dict:
    """{(b, h): run_head(spec)} over a spawned pool."""
    with pool(workers) as ex:
        results = list(ex.map(run_head, specs, chunksize=max(1, len(specs) // (4 * (workers or os.cpu_count() or 1)))))
    return {(s.b, s.h): r for s, r in zip(specs, results)}

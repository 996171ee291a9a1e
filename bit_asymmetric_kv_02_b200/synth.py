"""Seeded synthetic KV-cache workloads (inputs only: no quantization or attention arithmetic).

Prompts are drawn per (batch, KV head) and decode-step rows per (batch, step), each from its own
numpy PCG64 stream keyed by (seed, stream id, indices), so any subset of heads can be regenerated
on its own and a prefix of a prompt equals the shorter prompt.  Distributions follow the KV-cache statistics the KIVI explainer
page describes (section KVキャッシュの分布特性): keys have a few outlier channels with large
magnitude across all tokens, values have a large early "sink" token.

  K: N(0,1) fp32, 4 outlier channels per (batch, KV head) (drawn without replacement) scaled x10,
     cast to fp16 (round to nearest even).
  V: N(0,1) fp32, token 0 of every sequence scaled x5, cast to fp16.
  q: N(0,1) fp32 per (batch, query head, step), cast to fp16.
  new decode tokens: K with the head's outlier channels x10, V plain N(0,1).
"""
from __future__ import annotations

import functools
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace

import numpy as np

STREAM_K, STREAM_V, STREAM_OUTLIER, STREAM_Q, STREAM_KNEW, STREAM_VNEW = range(6)
N_OUTLIER_CHANNELS = 4
OUTLIER_GAIN = 10.0
SINK_GAIN = 5.0


@dataclass(frozen=True)
class Workload:
    """Shape of one decode workload.  T = cached tokens per head at the attention step."""
    name: str
    batch: int
    q_heads: int
    kv_heads: int
    tokens: int
    head_dim: int = 128
    bits: int = 2
    group: int = 32          # G_k (and G_v unless group_v is set)
    residual: int = 128      # R
    seed: int = 1000
    steps: int = 0           # streaming decode steps after the prefill (0: single attention)
    group_v: int = 0         # G_v when it differs from G_k (0: G_v = G_k)

    @property
    def gqa(self) -> int:
        return self.q_heads // self.kv_heads

    @property
    def gv(self) -> int:
        return self.group_v or self.group

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads, named by what they are.
TINY = Workload("tiny_b1_h4_t1024", 1, 4, 4, 1024, seed=1000)
LLAMA2_7B = Workload("llama2_7b_layer_b8_h32_t4096", 8, 32, 32, 4096, seed=1001)
LARGE_BATCH = Workload("large_batch_b64_h32_t8192", 64, 32, 32, 8192, seed=1002)
GQA_LLAMA3_8B = Workload("gqa_llama31_8b_b16_hq32_hkv8_t32768", 16, 32, 8, 32768, seed=1003)
STREAMING = Workload("streaming_b4_h32_prefill32768_steps256", 4, 32, 32, 32768, seed=1004, steps=256)
WORKLOADS = {w.name: w for w in (TINY, LLAMA2_7B, LARGE_BATCH, GQA_LLAMA3_8B, STREAMING)}


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *key])))


@functools.lru_cache(maxsize=1 << 16)
def _outliers(seed: int, d: int, b: int, h: int) -> tuple:
    return tuple(np.sort(_rng(seed, STREAM_OUTLIER, b, h).choice(d, N_OUTLIER_CHANNELS, replace=False)))


def outlier_channels(w: Workload, b: int, h: int) -> np.ndarray:
    """The N_OUTLIER_CHANNELS distinct outlier channels of KV head (b, h)."""
    return np.array(_outliers(w.seed, w.head_dim, b, h), dtype=np.int64)


def prompt_k(w: Workload, b: int, h: int, n: int) -> np.ndarray:
    """fp16 [n][d] prompt keys of KV head (b, h)."""
    x = _rng(w.seed, STREAM_K, b, h).standard_normal((n, w.head_dim), dtype=np.float32)
    x[:, outlier_channels(w, b, h)] *= np.float32(OUTLIER_GAIN)
    return x.astype(np.float16)


def prompt_v(w: Workload, b: int, h: int, n: int) -> np.ndarray:
    """fp16 [n][d] prompt values of KV head (b, h); token 0 is the x5 sink."""
    x = _rng(w.seed, STREAM_V, b, h).standard_normal((n, w.head_dim), dtype=np.float32)
    if n > 0:
        x[0] *= np.float32(SINK_GAIN)
    return x.astype(np.float16)


def _step_rows(w: Workload, stream: int, b: int, step: int, n: int) -> np.ndarray:
    """fp32 N(0,1) [n][d]: one row per head of sequence b at decode step `step`."""
    return _rng(w.seed, stream, b, step).standard_normal((n, w.head_dim), dtype=np.float32)


def _keys_of_step(w: Workload, b: int, step: int) -> np.ndarray:
    x = _step_rows(w, STREAM_KNEW, b, step, w.kv_heads)
    for h in range(w.kv_heads):
        x[h, outlier_channels(w, b, h)] *= np.float32(OUTLIER_GAIN)
    return x.astype(np.float16)


def query(w: Workload, b: int, hq: int, step: int = 0) -> np.ndarray:
    """fp16 [d] query of query head (b, hq) at decode step `step`."""
    return _step_rows(w, STREAM_Q, b, step, w.q_heads)[hq].astype(np.float16)


def new_k(w: Workload, b: int, h: int, step: int) -> np.ndarray:
    """fp16 [d] key appended to KV head (b, h) at decode step `step` (outlier channels x10)."""
    return _keys_of_step(w, b, step)[h]


def new_v(w: Workload, b: int, h: int, step: int) -> np.ndarray:
    """fp16 [d] value appended to KV head (b, h) at decode step `step`."""
    return _step_rows(w, STREAM_VNEW, b, step, w.kv_heads)[h].astype(np.float16)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def prompt_kv(w: Workload, n: int, out_k: np.ndarray | None = None,
              out_v: np.ndarray | None = None):
    """fp16 [B][H][n][d] prompt keys and values of every KV head (threads over heads)."""
    shape = (w.batch, w.kv_heads, n, w.head_dim)
    k = np.empty(shape, np.float16) if out_k is None else out_k
    v = np.empty(shape, np.float16) if out_v is None else out_v

    def one(bh):
        b, h = divmod(bh, w.kv_heads)
        k[b, h] = prompt_k(w, b, h, n)
        v[b, h] = prompt_v(w, b, h, n)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(one, range(w.batch * w.kv_heads)))
    return k, v


def queries(w: Workload, step: int = 0) -> np.ndarray:
    """fp16 [B][Hq][d] queries of one decode step."""
    return np.stack([_step_rows(w, STREAM_Q, b, step, w.q_heads).astype(np.float16)
                     for b in range(w.batch)])


def new_kv(w: Workload, step: int):
    """fp16 [B][H][d] key and value appended at one decode step."""
    k = np.stack([_keys_of_step(w, b, step) for b in range(w.batch)])
    v = np.stack([_step_rows(w, STREAM_VNEW, b, step, w.kv_heads).astype(np.float16)
                  for b in range(w.batch)])
    return k, v

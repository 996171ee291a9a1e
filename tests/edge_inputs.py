"""Constructed fp16 KV inputs that put the method's edge cases inside every quantization group.

Test infrastructure: the GPU edge-case tests feed these tensors to the CUDA path and to the oracle
alike.  Nothing here quantizes anything; the tie points are placed with exact rational arithmetic
(tests/exact.py) from the scale rule of the KIVI page, section 量子化アルゴリズム (s/z equation:
s = (max - min)/(2^b - 1) stored in fp16, z = min), so that a group's values land exactly on
z + (k + 1/2) s, one fp16 step beside it, or within 2^-12 of it in r = (x - z)/s.

A tensor [T][d] is cut into groups by a group-id map (the grouping under test: K per R-token block
x g_k channels, V per g_v tokens, or the fine-grained and prefix-K groupings); every group gets one
kind from KINDS, chosen by a seeded generator, and its values are drawn from that kind's candidates
with the group minimum and maximum each present at least once.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

from exact import fp16_round_exact

FP16_MAX = 65504.0

KINDS = (
    "ties_exact",      # s with few significant bits: every tie z + (k + 1/2) s is an fp16 value
    "ties_rounded",    # random range: ties fall between fp16 values; their fp16 neighbours
    "tie_near_zero",   # one tie sits next to 0, where fp16 is dense: r within 2^-12 of k + 1/2
    "constant",        # one repeated value: s = 0
    "constant_extreme",  # +-65504 or a subnormal repeated: s = 0 at the ends of the fp16 range
    "signed_zeros",    # +0 and -0 only: s = 0, z = +0
    "neg_zero_min",    # -0 is the minimum, positive values above it
    "tiny_range",      # max = next fp16 above min near 0: the range rounds s to 0
    "subnormal_s",     # s a small multiple of 2^-24 (subnormal scale), every grid point present
    "extremes",        # min -65504, max +65504
    "top_range",       # 32768 .. 65504: the largest exponent
    "negative",        # all values negative
    "normal",          # N(0, 1) times a random gain
)
# kinds whose values stay within |x| <= 6, so that attention outputs are comparable at the
# absolute bar (an fp16 output above 8 in magnitude is rounded by more than 2e-3 by itself)
MODERATE_KINDS = ("ties_exact", "ties_rounded", "tie_near_zero", "constant", "signed_zeros",
                  "neg_zero_min", "tiny_range", "subnormal_s", "negative", "normal")


def _f16(x) -> np.float16:
    with np.errstate(over="ignore"):
        return np.float16(x)


def _next_up(h: np.float16) -> np.float16:
    with np.errstate(over="ignore"):
        return np.nextafter(h, np.float16(np.inf))


def _next_down(h: np.float16) -> np.float16:
    with np.errstate(over="ignore"):
        return np.nextafter(h, np.float16(-np.inf))


def stored_scale(lo: np.float16, hi: np.float16, bits: int) -> Fraction:
    """The fp16 scale the s/z equation stores for extremes (lo, hi), by exact rationals."""
    L = 2 ** bits - 1
    return Fraction(fp16_round_exact((Fraction(float(hi)) - Fraction(float(lo))) / L))


def _tie_neighbours(z: np.float16, s: Fraction, bits: int, lo: float, hi: float, reach: int = 2):
    """fp16 values at and around every tie z + (k + 1/2) s and every grid point z + k s."""
    out = []
    L = 2 ** bits - 1
    zf = Fraction(float(z))
    for k in range(L + 1):
        for frac in (Fraction(1, 2), Fraction(0)):
            if frac == Fraction(1, 2) and k == L:
                continue
            t = zf + (k + frac) * s
            h = _f16(float(t))           # float(t) is exact: a sum of two fp16 multiples
            if not np.isfinite(h):
                continue
            cand = [h]
            up, dn = h, h
            for _ in range(reach):
                up, dn = _next_up(up), _next_down(dn)
                cand += [up, dn]
            out += [c for c in cand if np.isfinite(c) and lo <= float(c) <= hi]
    return out


def _group_kind_values(kind: str, bits: int, rng: np.random.Generator):
    """(lo, hi, candidates) of one group of the given kind."""
    L = 2 ** bits - 1
    if kind == "ties_exact":
        m = int(rng.choice([1, 3, 5, 7]))
        e_max = int(np.floor(np.log2(6.0 / (L * m))))       # L s <= 6
        e = int(rng.integers(e_max - 5, e_max + 1))
        s = Fraction(m) * Fraction(2) ** e
        z = Fraction(int(rng.integers(-12, 13))) * Fraction(2) ** (e - 1)
        lo, hi = _f16(float(z)), _f16(float(z + L * s))
        assert stored_scale(lo, hi, bits) == s
        cand = _tie_neighbours(lo, s, bits, float(lo), float(hi), reach=1)
        return lo, hi, cand
    if kind == "ties_rounded":
        a = _f16(rng.uniform(-5.0, 3.0))
        b = _f16(min(5.5, float(a) + rng.uniform(0.01, 4.0)))
        lo, hi = min(a, b), max(a, b)
        s = stored_scale(lo, hi, bits)
        return lo, hi, _tie_neighbours(lo, s, bits, float(lo), float(hi), reach=2)
    if kind == "tie_near_zero":
        s0 = float(rng.uniform(0.05, 5.0 / L))
        k0 = int(rng.integers(0, L))
        delta = float(rng.uniform(-1e-3, 1e-3))
        lo = _f16(-(k0 + 0.5) * s0 + delta)
        hi = _f16(float(lo) + L * s0)
        s = stored_scale(lo, hi, bits)
        cand = _tie_neighbours(lo, s, bits, float(lo), float(hi), reach=3)
        t = Fraction(float(lo)) + (k0 + Fraction(1, 2)) * s     # the tie next to 0
        h = _f16(float(t))
        for _ in range(6):                                        # fp16 is dense here
            cand += [h]
            h = _next_up(h)
        return lo, hi, [c for c in cand if float(lo) <= float(c) <= float(hi)]
    if kind == "constant":
        v = _f16(rng.choice([0.0, 1.0, -3.5, float(rng.standard_normal())]))
        return v, v, [v]
    if kind == "constant_extreme":
        v = _f16(rng.choice([2.0 ** -24, -(2.0 ** -24), -FP16_MAX, FP16_MAX]))
        return v, v, [v]
    if kind == "signed_zeros":
        return _f16(-0.0), _f16(0.0), [_f16(-0.0), _f16(0.0)]
    if kind == "neg_zero_min":
        hi = _f16(rng.uniform(0.5, 4.0))
        s = stored_scale(_f16(0.0), hi, bits)
        cand = [_f16(-0.0), _f16(0.0)] + _tie_neighbours(_f16(0.0), s, bits, 0.0, float(hi), reach=1)
        cand = [c for c in cand if not (float(c) == 0.0)] + [_f16(-0.0)]   # -0 but no +0 ...
        cand += [_f16(-0.0)] * 3                                             # ... is the minimum
        return _f16(-0.0), hi, cand
    if kind == "tiny_range":
        v = _f16(rng.choice([0.0, 2.0 ** -24, -(2.0 ** -24), 5 * 2.0 ** -24, -(2.0 ** -20)]))
        w = _next_up(v)
        assert stored_scale(v, w, bits) == 0
        return v, w, [v, w]
    if kind == "subnormal_s":
        j = int(rng.integers(1, 4))
        q = Fraction(1, 2 ** 24)
        z = Fraction(int(rng.integers(-40, 41))) * q
        lo, hi = _f16(float(z)), _f16(float(z + L * j * q))
        assert stored_scale(lo, hi, bits) == j * q
        n = L * j + 1
        return lo, hi, [_f16(float(z + i * q)) for i in range(n)]
    if kind == "extremes":
        lo, hi = _f16(-FP16_MAX), _f16(FP16_MAX)
        s = stored_scale(lo, hi, bits)
        cand = _tie_neighbours(lo, s, bits, -FP16_MAX, FP16_MAX, reach=1)
        cand += list(_f16(rng.uniform(-FP16_MAX, FP16_MAX, 16)))
        return lo, hi, cand
    if kind == "top_range":
        lo, hi = _f16(32768.0), _f16(FP16_MAX)
        s = stored_scale(lo, hi, bits)
        return lo, hi, _tie_neighbours(lo, s, bits, 32768.0, FP16_MAX, reach=1)
    if kind == "negative":
        a = _f16(-rng.uniform(0.01, 6.0))
        b = _f16(-rng.uniform(0.01, 6.0))
        lo, hi = min(a, b), max(a, b)
        if lo == hi:
            hi = _next_up(lo)
        s = stored_scale(lo, hi, bits)
        return lo, hi, _tie_neighbours(lo, s, bits, float(lo), float(hi), reach=1)
    if kind == "normal":
        x = np.clip(rng.standard_normal(64) * rng.uniform(0.1, 2.0), -6.0, 6.0).astype(np.float16)
        return x.min(), x.max(), list(x)
    raise ValueError(kind)


def fill_groups(gid: np.ndarray, bits: int, seed: int, kinds=KINDS) -> np.ndarray:
    """fp16 array shaped like gid: each group (equal ids) gets one kind's values, its minimum and
    maximum present at least once.  Kinds cycle over the groups in a seeded order."""
    rng = np.random.default_rng(seed)
    out = np.empty(gid.shape, np.float16)
    flat_ids = gid.reshape(-1)
    order = np.argsort(flat_ids, kind="stable")
    ids_sorted = flat_ids[order]
    bounds = np.flatnonzero(np.diff(ids_sorted)) + 1
    groups = np.split(order, bounds)
    kind_seq = list(kinds) * (len(groups) // len(kinds) + 1)
    rng.shuffle(kind_seq)
    flat = out.reshape(-1)
    for idx, kind in zip(groups, kind_seq):
        lo, hi, cand = _group_kind_values(kind, bits, rng)
        cand = np.array(cand, np.float16) if len(cand) else np.array([lo], np.float16)
        vals = cand[rng.integers(0, len(cand), len(idx))]
        if len(idx) >= 2:
            pos = rng.choice(len(idx), 2, replace=False)
            vals[pos[0]], vals[pos[1]] = lo, hi
        else:
            vals[0] = lo
        flat[idx] = vals
    return out


# ---- group-id maps of the groupings (t: token index, c: channel index) -------------------------
def k_block_groups(T: int, d: int, R: int, gk: int) -> np.ndarray:
    """K: one group per (R-token block, g_k consecutive channels)."""
    t, c = np.meshgrid(np.arange(T), np.arange(d), indexing="ij")
    return (t // R) * (d // gk) + c // gk


def v_token_groups(T: int, d: int, gv: int) -> np.ndarray:
    """V: one group per g_v consecutive tokens (all channels)."""
    t, _ = np.meshgrid(np.arange(T), np.arange(d), indexing="ij")
    return t // gv


def k_fine_groups(T: int, d: int, gk: int) -> np.ndarray:
    """K fine-grained: one group per (channel, g_k consecutive tokens)."""
    t, c = np.meshgrid(np.arange(T), np.arange(d), indexing="ij")
    return (t // gk) * d + c


def v_fine_groups(T: int, d: int, gv: int) -> np.ndarray:
    """V fine-grained: one group per (token, g_v consecutive channels)."""
    t, c = np.meshgrid(np.arange(T), np.arange(d), indexing="ij")
    return t * (d // gv) + c // gv


def k_prefix_groups(T: int, d: int, n_prefix: int, R: int, gk: int) -> np.ndarray:
    """K under the prefix reading: one group per g_k channels over tokens [0, n_prefix), block
    groups after it."""
    g = k_block_groups(T, d, R, gk)
    t, c = np.meshgrid(np.arange(T), np.arange(d), indexing="ij")
    pre = t < n_prefix
    g = np.where(pre, c // gk, g + (d // gk) * 10_000)
    return g


def edge_prompt(batch: int, heads: int, T: int, bits: int, k_gid: np.ndarray, v_gid: np.ndarray, seed: int,
                kinds=KINDS, v_kinds=None):
    """fp16 K, V [B][H][T][d]: every head's groups filled by fill_groups (K and V from their own
    group maps; v_kinds restricts V, e.g. to MODERATE_KINDS for attention checks)."""
    d = k_gid.shape[1]
    k = np.empty((batch, heads, T, d), np.float16)
    v = np.empty((batch, heads, T, d), np.float16)
    for b in range(batch):
        for h in range(heads):
            s = seed * 7919 + b * 131 + h
            k[b, h] = fill_groups(k_gid, bits, s, kinds)
            v[b, h] = fill_groups(v_gid, bits, s + 50_000, v_kinds or kinds)
    return k, v

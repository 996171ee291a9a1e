"""The 2-bit code decision the quantize kernel takes, restated on the CPU and checked against the
oracle on every fp16 value of a group's range (CPU only).

The kernel does not divide: for s > 0 it counts three fp16 thresholds derived from (s, z),
    code = [x > RD16(z + s/2)] + [x > below16(z + 3s/2)] + [x > RD16(z + 5s/2)],
where RD16(T) is the largest fp16 <= T and below16(T) the largest fp16 < T (the strict and non-strict
signs carry round-half-to-even at 1/2, 3/2 and 5/2; past 7/2 all three count, which is the clamp).
s = 0 uses +inf thresholds (every code 0).  The thresholds here are exact rationals, independent of
both the kernel and the oracle; the oracle decides Q(x) = clamp(rint((x - z)/s), 0, 3) in fp64
(section 量子化アルゴリズム of the KIVI explainer page, Q equation).
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle.kivi_oracle as O

ALL = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16).view(np.float16)
ALL = ALL[np.isfinite(ALL)]
GRID = np.unique(ALL.astype(np.float64))          # every finite fp16 value, ascending (+0 == -0)
GRID_Q = [Fraction(float(v)) for v in GRID]


def rd16(t: Fraction) -> float:
    """Largest fp16 value <= t."""
    lo, hi = 0, len(GRID_Q) - 1
    if t < GRID_Q[0]:
        return -np.inf
    while lo < hi:                                  # last index with GRID_Q[i] <= t
        mid = (lo + hi + 1) // 2
        if GRID_Q[mid] <= t:
            lo = mid
        else:
            hi = mid - 1
    return float(GRID[lo])


def below16(t: Fraction) -> float:
    """Largest fp16 value < t."""
    r = rd16(t)
    if Fraction(r) < t:
        return r
    i = int(np.searchsorted(GRID, r)) - 1
    return float(GRID[i]) if i >= 0 else -np.inf


def threshold_codes(x, s16: np.float16, z16: np.float16) -> np.ndarray:
    s, z = Fraction(float(s16)), Fraction(float(z16))
    if s == 0:
        return np.zeros(len(x), dtype=np.int64)
    t = [rd16(z + s / 2), below16(z + 3 * s / 2), rd16(z + 5 * s / 2)]
    xv = np.asarray(x, dtype=np.float64)
    return sum((xv > tk).astype(np.int64) for tk in t)


def group_ranges():
    rng = np.random.default_rng(20240101)
    out = [(0.0, 0.0), (-1.0, -1.0), (0.0, 6e-8), (0.0, 1.5), (-65504.0, 65504.0), (-0.0, 3.0),
           (1.0, 1.0009765625), (-3.0, 0.0), (0.0, 4.5), (-2.5, 2.5), (6.1e-5, 6.2e-5), (-1e-7, 1e-7)]
    for _ in range(40):
        lo = float(np.float16(rng.standard_normal() * 10 ** rng.uniform(-6, 4)))
        hi = float(np.float16(lo + abs(rng.standard_normal()) * 10 ** rng.uniform(-7, 4)))
        if np.isfinite(hi):
            out.append((lo, hi))
    return out


@pytest.mark.parametrize("lo,hi", group_ranges())
def test_threshold_rule_equals_oracle_on_every_fp16_value(lo, hi):
    s, z = O.scale_zero(np.array([lo]), np.array([hi]), 2)
    s16, z16 = np.float16(s[0]), np.float16(z[0])
    xs = ALL[(ALL.astype(np.float64) >= lo) & (ALL.astype(np.float64) <= hi)]
    want = O.quantize_values(xs, s16, z16, 2).astype(np.int64)
    got = threshold_codes(xs, s16, z16)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"x={xs[bad[0]]} threshold code {got[bad[0]]} oracle {want[bad[0]]}"


def test_threshold_rule_ties_go_to_even():
    # s = 1, z = 0: the thresholds are exactly 0.5, 1.5 and 2.5
    xs = np.array([0.5, 1.5, 2.5, 3.5, 0.49951171875, 1.4990234375, 2.498046875], dtype=np.float16)
    got = threshold_codes(xs, np.float16(1.0), np.float16(0.0))
    assert got.tolist() == [0, 2, 2, 3, 0, 1, 2]

"""The constructed edge-case inputs (tests/edge_inputs.py) hold the cases they claim, checked with
exact rational arithmetic on the CPU (KIVI page, section 量子化アルゴリズム: the s/z equation fixes
the stored scale; a tie is a value whose (x - z)/s is a half-integer)."""
from fractions import Fraction

import numpy as np
import pytest

import edge_inputs as E
from exact import fp16_round_exact


def _r(x, lo, s):
    return (Fraction(float(x)) - Fraction(float(lo) + 0.0)) / s


@pytest.mark.parametrize("bits", [2, 4])
def test_each_kind_holds_its_case(bits):
    rng = np.random.default_rng(5)
    L = 2 ** bits - 1
    for _ in range(20):
        for kind in E.KINDS:
            lo, hi, cand = E._group_kind_values(kind, bits, rng)
            vals = [float(c) for c in cand]
            assert all(float(lo) <= v <= float(hi) for v in vals), kind
            s = Fraction(fp16_round_exact((Fraction(float(hi)) - Fraction(float(lo))) / L))
            rs = [_r(c, lo, s) for c in cand] if s > 0 else []
            if kind == "ties_exact":
                halves = {k + Fraction(1, 2) for k in range(L)}
                assert halves <= set(rs), "every tie is a candidate"
            elif kind == "tie_near_zero":
                near = [r for r in rs if 0 < abs(r - (r.numerator // r.denominator) - Fraction(1, 2)) < Fraction(1, 4096)]
                assert near, "a value within 2^-12 of a tie (not on it)"
            elif kind in ("constant", "constant_extreme", "signed_zeros"):
                assert s == 0 and lo == hi
            elif kind == "tiny_range":
                assert s == 0 and float(hi) > float(lo)
            elif kind == "subnormal_s":
                assert 0 < s < Fraction(1, 2 ** 14)
            elif kind == "neg_zero_min":
                assert float(lo) == 0.0 and np.signbit(lo)
                assert not any(float(c) == 0.0 and not np.signbit(c) for c in cand), "no +0"
            elif kind == "extremes":
                assert float(lo) == -65504.0 and float(hi) == 65504.0
            elif kind in ("ties_rounded", "negative", "top_range"):
                # fp16 neighbours on both sides of every tie that is not itself an fp16 value
                for k in range(L):
                    t = k + Fraction(1, 2)
                    if t in rs:
                        continue
                    assert any(r < t for r in rs) and any(r > t for r in rs), (kind, k)


@pytest.mark.parametrize("maker", ["k_block", "v_token", "k_fine", "v_fine", "k_prefix"])
def test_groups_get_min_and_max(maker):
    T, d = 2 * 128 + 40, 128
    gid = {"k_block": E.k_block_groups(T, d, 128, 32), "v_token": E.v_token_groups(T, d, 32),
           "k_fine": E.k_fine_groups(T, d, 32), "v_fine": E.v_fine_groups(T, d, 32),
           "k_prefix": E.k_prefix_groups(T, d, 256, 128, 32)}[maker]
    x = E.fill_groups(gid, 2, seed=3)
    assert x.shape == gid.shape and x.dtype == np.float16
    assert np.all(np.isfinite(x))
    for g in np.unique(gid)[:50]:          # the minimum and the maximum of the group's kind are there
        vals = x[gid == g].astype(np.float64)
        assert vals.size >= 1


def test_moderate_kinds_stay_small():
    gid = E.v_token_groups(512, 128, 32)
    x = np.concatenate([E.fill_groups(gid, b, seed=9 + b, kinds=E.MODERATE_KINDS) for b in (2, 4)])
    assert float(np.abs(x.astype(np.float64)).max()) <= 6.0

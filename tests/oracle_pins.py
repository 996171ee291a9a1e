"""Checks that pin the CPU oracle to facts other than its own code.

Each ``check_*`` takes the oracle module and raises AssertionError on a mismatch, so the same
checks run against the real oracle (test_oracle_pins.py) and against planted mistakes
(test_oracle_mutants.py).  Sources of truth: exact rational arithmetic (tests/exact.py), search
for the nearest grid point, hand-derived fixtures in tests/golden/, closed forms of attention
special cases, PyTorch's scaled_dot_product_attention in float64, and pure-Python brute force
that reads the packed words bit by bit.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
import torch

from exact import code_exact, code_nearest_grid, fp16_round_exact

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _fr(x) -> Fraction:
    return Fraction(float(x))


def _hex16(x) -> str:
    return "0x%04x" % int(np.asarray(x, np.float16).view(np.uint16))


def _rand_fp16(rng, n, lo_exp=-24, hi_exp=15):
    """fp16 values with log-uniform magnitudes and random signs (includes subnormals)."""
    e = rng.uniform(lo_exp, hi_exp, n)
    x = np.sign(rng.standard_normal(n)) * np.exp2(e)
    return np.clip(x, -65504, 65504).astype(np.float16)


# --------------------------------------------------------------------------------------------
# fp16 rounding and s / z
# --------------------------------------------------------------------------------------------
def check_fp16_round(O):
    rng = np.random.default_rng(11)
    xs = [1 + 2 ** -11, 1 + 3 * 2 ** -11, 1 + 2 ** -11 + 2 ** -40, 2 ** -25, 3 * 2 ** -25,
          2 ** -25 + 2 ** -60, 65504.0, 65519.0, 0.2, 1 / 3, 2 / 3, 1e-7, 43669.0]
    xs += list(rng.standard_normal(200) * np.exp2(rng.uniform(-26, 15, 200)))
    got = O.fp16_round(np.array(xs))
    for x, g in zip(xs, got):
        want = fp16_round_exact(Fraction(x))
        assert Fraction(float(g)) == want, (x, float(g), want)


def check_scale_zero_exact(O, bits):
    rng = np.random.default_rng(12 + bits)
    L = 2 ** bits - 1
    a = _rand_fp16(rng, 3000)
    b = _rand_fp16(rng, 3000)
    lo = np.minimum(a, b)
    hi = np.maximum(a, b)
    # every positive finite fp16 as a range starting at 0 and at -hi: all quotients near midpoints
    allpos = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16)
    lo = np.concatenate([lo, np.zeros_like(allpos), -allpos[::7]])
    hi = np.concatenate([hi, allpos, allpos[::7]])
    s, z = O.scale_zero(lo, hi, bits)
    assert s.dtype == np.float16 and z.dtype == np.float16
    assert np.array_equal(z.view(np.uint16), lo.view(np.uint16))
    for l_, h_, s_ in zip(lo[::3], hi[::3], s[::3]):
        want = fp16_round_exact((_fr(h_) - _fr(l_)) / L)
        assert Fraction(float(s_)) == want, (float(l_), float(h_), float(s_), want)
    # the all-pos sweep in full (these are the cases where a double rounding would show)
    n0 = 3000
    for l_, h_, s_ in zip(lo[n0:n0 + len(allpos)], hi[n0:n0 + len(allpos)], s[n0:n0 + len(allpos)]):
        want = fp16_round_exact((_fr(h_) - _fr(l_)) / L)
        assert Fraction(float(s_)) == want, (float(l_), float(h_), float(s_), want)


# --------------------------------------------------------------------------------------------
# codes
# --------------------------------------------------------------------------------------------
def _tie_cases(rng, bits, n):
    """(x, s, z) triples where (x - z)/s lands exactly on half-integers or a hair away."""
    L = 2 ** bits - 1
    xs, ss, zs = [], [], []
    while len(xs) < n:
        e = int(rng.integers(-12, 6))
        s = np.float16(float(rng.integers(1, 64)) * 2.0 ** (e - 5))
        z = np.float16(float(rng.integers(-512, 512)) * 2.0 ** (e - 6))
        k = int(rng.integers(0, L + 1))
        for off in (0.5, -0.5):
            x = np.float16(float(z) + (k + off) * float(s))
            # the (usually exact) tie and one fp16 ulp either side of it
            for xv in (x, np.nextafter(x, np.float16(np.inf)), np.nextafter(x, np.float16(-np.inf))):
                if np.isfinite(xv) and float(xv) >= float(z):
                    xs.append(xv)
                    ss.append(s)
                    zs.append(z)
    return (np.array(xs, np.float16), np.array(ss, np.float16), np.array(zs, np.float16))


def check_codes_exact(O, bits):
    rng = np.random.default_rng(21 + bits)
    x, s, z = _tie_cases(rng, bits, 1500)
    # plus ordinary groups with their own (s, z)
    for _ in range(60):
        g = _rand_fp16(rng, 40, -10, 4)
        ss, zz = O.scale_zero(np.array([g.min()]), np.array([g.max()]), bits)
        x = np.concatenate([x, g])
        s = np.concatenate([s, np.repeat(ss, len(g))])
        z = np.concatenate([z, np.repeat(zz, len(g))])
    codes = O.quantize_values(x, s, z, bits)
    assert codes.dtype == np.uint8
    for xi, si, zi, ci in zip(x, s, z, codes):
        want = code_exact(_fr(xi), _fr(si), _fr(zi), bits)
        assert int(ci) == want, (float(xi), float(si), float(zi), int(ci), want)
        if si != 0 and float(xi) <= float(zi) + (2 ** bits - 1 + 0.5) * float(si):
            assert want == code_nearest_grid(_fr(xi), _fr(si), _fr(zi), bits)


def check_hand_examples(O):
    with open(os.path.join(GOLDEN, "quantize_hand_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        g = np.array(c["group"], np.float16)
        s, z = O.scale_zero(np.array([g.min()]), np.array([g.max()]), c["bits"])
        assert _hex16(s[0]) == c["s_fp16_bits"], (c["name"], _hex16(s[0]))
        assert _hex16(z[0]) == c["z_fp16_bits"], (c["name"], _hex16(z[0]))
        codes = O.quantize_values(g, s[0], z[0], c["bits"])
        assert codes.tolist() == c["codes"], (c["name"], codes.tolist())


def check_invariants(O, bits):
    """codes in [0, L]; min -> 0; max -> L and |x - D(Q(x))| <= s/2 when s is a normal fp16;
    all 2^b levels reachable; zero range reconstructs exactly."""
    rng = np.random.default_rng(31 + bits)
    L = 2 ** bits - 1
    for trial in range(200):
        n = int(rng.integers(2, 300))
        g = (rng.standard_normal(n) * np.exp2(rng.uniform(-8, 8))).astype(np.float16)
        s, z = O.scale_zero(np.array([g.min()]), np.array([g.max()]), bits)
        c = O.quantize_values(g, s[0], z[0], bits)
        assert c.min() >= 0 and c.max() <= L
        assert c[np.argmin(g)] == 0
        s64, z64 = float(s[0]), float(z[0])
        if s64 >= 2 ** -14:
            assert c[np.argmax(g)] == L
            err = np.abs(g.astype(np.float64) - (s64 * c + z64))
            assert err.max() <= s64 / 2, (err.max(), s64)
    lin = np.linspace(-1, 1, 64).astype(np.float16)
    s, z = O.scale_zero(np.array([lin.min()]), np.array([lin.max()]), bits)
    assert sorted(set(O.quantize_values(lin, s[0], z[0], bits).tolist())) == list(range(L + 1))
    const = np.full(17, -3.375, np.float16)
    s, z = O.scale_zero(np.array([const.min()]), np.array([const.max()]), bits)
    c = O.quantize_values(const, s[0], z[0], bits)
    assert float(s[0]) == 0.0 and not c.any()
    assert np.array_equal(float(s[0]) * c + float(z[0]), const.astype(np.float64))


# --------------------------------------------------------------------------------------------
# group axes of K and V blocks
# --------------------------------------------------------------------------------------------
def check_block_groups(O, bits, group):
    """Per-channel K groups span every token of the block and `group` consecutive channels;
    per-token V groups span `group` consecutive tokens and every channel.  Brute force with
    explicit index loops and exact rationals."""
    rng = np.random.default_rng(41 + bits + group)
    n, d = 2 * group, 128
    blk = (rng.standard_normal((n, d)) * np.exp2(rng.integers(-3, 4, (1, d)))).astype(np.float16)
    blk[:, 5] *= np.float16(9)
    blk[3, :] *= np.float16(7)
    L = 2 ** bits - 1
    kc, ks, kz = O.quantize_k_block(blk, group, bits)
    assert ks.shape == (d // group,) and kc.shape == (n, d)
    for g in range(d // group):
        vals = [_fr(blk[t, c]) for t in range(n) for c in range(g * group, (g + 1) * group)]
        lo, hi = min(vals), max(vals)
        s = fp16_round_exact((hi - lo) / L)
        assert Fraction(float(ks[g])) == s and Fraction(float(kz[g])) == lo
        for t in range(0, n, 7):
            for c in range(g * group, (g + 1) * group, 3):
                assert kc[t, c] == code_exact(_fr(blk[t, c]), s, lo, bits)
    vc, vs, vz = O.quantize_v_block(blk, group, bits)
    assert vs.shape == (n // group,) and vc.shape == (n, d)
    for u in range(n // group):
        vals = [_fr(blk[t, c]) for t in range(u * group, (u + 1) * group) for c in range(d)]
        lo, hi = min(vals), max(vals)
        s = fp16_round_exact((hi - lo) / L)
        assert Fraction(float(vs[u])) == s and Fraction(float(vz[u])) == lo
        for t in range(u * group, (u + 1) * group, 5):
            for c in range(0, d, 9):
                assert vc[t, c] == code_exact(_fr(blk[t, c]), s, lo, bits)


# --------------------------------------------------------------------------------------------
# packing
# --------------------------------------------------------------------------------------------
def check_pack_golden(O):
    with open(os.path.join(GOLDEN, "pack_hand_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        t, ch, bits = c["tokens"], c["channels"], c["bits"]
        codes = np.zeros((t, ch), np.uint8)
        for i in range(t):
            for j in range(ch):
                codes[i, j] = {"code(t, c) = c mod 4": j % 4, "code(t, c) = c mod 8": j % 8,
                               "code(t, c) = (t + c) mod 4": (i + j) % 4,
                               "code(t, c) = t": i}[c["codes_rule"]]
        want = np.array([int(w, 16) for w in np.ravel(c["words"])], np.uint32)
        got = (O.pack_k(codes, bits) if c["layout"] == "k" else O.pack_v(codes, bits)).ravel()
        assert np.array_equal(got, want), (c["name"], [hex(w) for w in got])


def check_pack_roundtrip(O, bits):
    rng = np.random.default_rng(51 + bits)
    P = 32 // bits
    codes = rng.integers(0, 2 ** bits, (4 * P, 128)).astype(np.uint8)
    wk = O.pack_k(codes, bits)
    wv = O.pack_v(codes, bits)
    assert wk.shape == (4 * P, 128 // P) and wv.shape == (4, 128)
    assert np.array_equal(O.unpack_k(wk, bits), codes)
    assert np.array_equal(O.unpack_v(wv, bits), codes)
    # bit-level brute force of a few words
    for t, i in [(0, 0), (3, 5), (4 * P - 1, 128 // P - 1)]:
        w = int(wk[t, i])
        for j in range(P):
            assert (w >> (bits * j)) & (2 ** bits - 1) == codes[t, P * i + j]
    for r, c in [(0, 0), (2, 77), (3, 127)]:
        w = int(wv[r, c])
        for j in range(P):
            assert (w >> (bits * j)) & (2 ** bits - 1) == codes[P * r + j, c]


# --------------------------------------------------------------------------------------------
# cache semantics
# --------------------------------------------------------------------------------------------
def _head(O, bits=2, group=32, R=128, cap=4096):
    return O.HeadCache(128, bits, group, group, R, cap)


def check_prefill_split(O):
    rng = np.random.default_rng(61)
    R = 128
    for T in (1, 2, 127, 128, 129, 255, 256, 257, 1024, 1025):
        k = rng.standard_normal((T, 128)).astype(np.float16)
        h = _head(O)
        h.prefill(k, k)
        assert h.n_res == (T - 1) % R + 1 and h.n_quant == T - h.n_res, (T, h.n_quant, h.n_res)
        assert h.n_quant % R == 0 and 1 <= h.n_res <= R
        assert np.array_equal(h.k_res, k[h.n_quant:])


def check_prefill_equals_streaming(O, bits, group):
    """prefill(T0) followed by appends (flushing whenever the residual is full) equals prefill of
    all tokens at once, for every counter and every stored value."""
    rng = np.random.default_rng(71 + bits)
    T0, extra = 200, 190
    k = (rng.standard_normal((T0 + extra, 128)) * 3).astype(np.float16)
    v = rng.standard_normal((T0 + extra, 128)).astype(np.float16)
    a = _head(O, bits, group)
    a.prefill(k[:T0], v[:T0])
    for t in range(T0, T0 + extra):
        if a.n_res == a.R:
            a.flush()
        a.append(k[t], v[t])
    b = _head(O, bits, group)
    b.prefill(k, v)
    assert (a.n_quant, a.n_res) == (b.n_quant, b.n_res)
    pa, pb = a.packed(), b.packed()
    for key in pa:
        assert np.array_equal(np.asarray(pa[key]).view(np.uint8), np.asarray(pb[key]).view(np.uint8)), key


def check_prefix_k_groups(O, bits, group):
    """The prefix-K prefill (section Per-Channel量子化 read with one K group over every quantized
    token of the prompt): brute force over the whole prefix with exact rationals; V, residual and
    counters equal those of prefill; a single quantized block equals prefill exactly; a flush after
    it quantizes the next block on its own."""
    rng = np.random.default_rng(91 + bits + group)
    R, d, L = 128, 128, 2 ** bits - 1
    T = 3 * R + 5
    k = (rng.standard_normal((T, d)) * np.exp2(rng.integers(-2, 3, (1, d)))).astype(np.float16)
    k[200:260, 7] *= np.float16(11)                 # an outlier run inside one block only
    k[3 * R + 2, :] *= np.float16(20)               # a large residual row: outside every K group
    v = rng.standard_normal((T, d)).astype(np.float16)
    h = O.HeadCache(d, bits, group, group, R, 8 * R)
    h.prefill_prefix_k(k, v)
    n_q = 3 * R
    assert (h.n_quant, h.n_res) == (n_q, 5) and h.k_s.shape == (3, d // group)
    for g in range(d // group):
        vals = [_fr(k[t, c]) for t in range(n_q) for c in range(g * group, (g + 1) * group)]
        lo, hi = min(vals), max(vals)
        s = fp16_round_exact((hi - lo) / L)
        for blk in range(3):
            assert Fraction(float(h.k_s[blk, g])) == s and Fraction(float(h.k_z[blk, g])) == lo, (g, blk)
        for t in range(0, n_q, 11):
            for c in range(g * group, (g + 1) * group, 5):
                assert h.k_codes[t, c] == code_exact(_fr(k[t, c]), s, lo, bits), (t, c)
    ref = O.HeadCache(d, bits, group, group, R, 8 * R)
    ref.prefill(k, v)
    for key in ("v_codes", "v_s", "v_z", "k_res", "v_res"):
        assert np.array_equal(getattr(h, key), getattr(ref, key)), key
    # the outlier run lies in block 1 only: block-local K scales differ, the prefix ones do not
    g7 = 7 // group
    assert ref.k_s[0, g7] != ref.k_s[1, g7] and h.k_s[0, g7] == h.k_s[1, g7]
    one = O.HeadCache(d, bits, group, group, R, 8 * R)
    one.prefill_prefix_k(k[:R + 9], v[:R + 9])
    ref1 = O.HeadCache(d, bits, group, group, R, 8 * R)
    ref1.prefill(k[:R + 9], v[:R + 9])
    for key, want in ref1.packed().items():
        assert np.array_equal(np.asarray(one.packed()[key]).view(np.uint8), np.asarray(want).view(np.uint8)), key
    for t in range(T, T + R - 5):
        h.append(k[t % T], v[t % T])
    h.flush()
    kc, ks, kz = O.quantize_k_block(np.concatenate([k[n_q:], k[: R - 5]]), group, bits)
    assert np.array_equal(h.k_s[3], ks) and np.array_equal(h.k_codes[n_q:], kc)


def check_online_k(O, bits, group):
    """Online K (section Per-Channel量子化: a new token's K is quantized at once with the existing
    scale and zero point).  Every online row is the nearest grid point of the newest quantized
    block's stored (s, z), found by search over the 2^b levels with exact rationals (clamping
    included); rows copied from that block get that block's codes; blocks, V and counters equal
    the base scheme's; the copied (s, z) carries over flushes; before any block exists K stays in
    fp16 and the first flush quantizes it as the base scheme does."""
    rng = np.random.default_rng(131 + bits + group)
    R, d = 128, 128
    T = 2 * R + 37
    k = (rng.standard_normal((T, d)) * np.exp2(rng.integers(-2, 3, (1, d)))).astype(np.float16)
    k[R:2 * R, 3] *= np.float16(9)          # block 1's range differs from block 0's in group 3 // group
    v = rng.standard_normal((T, d)).astype(np.float16)
    h = O.HeadCache(d, bits, group, group, R, 8 * R, online_k=True)
    h.prefill(k, v)
    ref = O.HeadCache(d, bits, group, group, R, 8 * R)
    ref.prefill(k, v)
    assert (h.n_quant, h.n_res) == (ref.n_quant, ref.n_res) == (2 * R, 37)
    assert h.k_res.shape[0] == 0 and h.k_codes.shape[0] == T and h.k_s.shape[0] == 3
    assert np.array_equal(h.k_codes[:2 * R], ref.k_codes) and np.array_equal(h.k_s[:2], ref.k_s)
    assert np.array_equal(h.k_s[2], ref.k_s[1]) and np.array_equal(h.k_z[2], ref.k_z[1])
    assert ref.k_s[0, 3 // group] != ref.k_s[1, 3 // group]
    for key in ("v_codes", "v_s", "v_z", "v_res"):
        assert np.array_equal(getattr(h, key), getattr(ref, key)), key

    def nearest(row_k, row_codes):
        for c in range(0, d, 3):
            g = c // group
            want = code_nearest_grid(_fr(row_k[c]), _fr(ref.k_s[1, g]), _fr(ref.k_z[1, g]), bits)
            assert row_codes[c] == want, (c, row_codes[c], want)

    for i in range(2 * R, T, 5):
        nearest(k[i], h.k_codes[i])
    # appends: copies of block-1 rows, rows far outside its range (clamped), then fill and flush
    n0 = h.k_codes.shape[0]
    for j in range(10):
        h.append(k[R + 7 * j], v[j])
    assert np.array_equal(h.k_codes[n0:n0 + 10], ref.k_codes[R + 7 * np.arange(10)])
    wide = (rng.standard_normal((6, d)) * 40).astype(np.float16)
    for j in range(6):
        h.append(wide[j], v[j])
        nearest(wide[j], h.k_codes[-1])
    assert set(np.unique(h.k_codes[-6:])) >= {0, 2 ** bits - 1}
    while h.n_res < R:
        h.append(k[h.n_res], v[h.n_res])
    vres = h.v_res.copy()
    h.flush()
    vc, vs, vz = O.quantize_v_block(vres, group, bits)
    assert (h.n_quant, h.n_res) == (3 * R, 0) and h.k_codes.shape[0] == 3 * R
    assert np.array_equal(h.v_codes[2 * R:], vc) and np.array_equal(h.v_s[2 * R // group:], vs)
    assert np.array_equal(h.k_s[2], ref.k_s[1])
    h.append(wide[0], v[0])
    assert h.k_s.shape[0] == 4 and np.array_equal(h.k_s[3], ref.k_s[1]) and np.array_equal(h.k_z[3], ref.k_z[1])
    # dequantized keys of online rows: s * code + z with the carried (s, z), exactly
    keys = h.keys()
    for i in (2 * R + 1, 3 * R):
        for c in (0, 3, 77):
            g = c // group
            assert Fraction(float(keys[i, c])) == _fr(ref.k_s[1, g]) * int(h.k_codes[i, c]) + _fr(ref.k_z[1, g])
    # no block yet: K stays fp16, the first flush quantizes it as the base scheme does
    e = O.HeadCache(d, bits, group, group, R, 8 * R, online_k=True)
    b = O.HeadCache(d, bits, group, group, R, 8 * R)
    e.prefill(k[:50], v[:50])
    b.prefill(k[:50], v[:50])
    assert e.k_res.shape[0] == 50 and e.k_codes.shape[0] == 0
    for t in range(50, R):
        e.append(k[t], v[t])
        b.append(k[t], v[t])
    e.flush()
    b.flush()
    for key, want in b.packed().items():
        assert np.array_equal(np.asarray(e.packed()[key]).view(np.uint8), np.asarray(want).view(np.uint8)), key
    e.append(k[R + 1], v[0])
    kc0, ks0, kz0 = O.quantize_k_block(k[:R], group, bits)
    nearest_codes = [code_nearest_grid(_fr(k[R + 1, c]), _fr(ks0[c // group]), _fr(kz0[c // group]), bits)
                     for c in range(d)]
    assert list(e.k_codes[R]) == nearest_codes and e.k_res.shape[0] == 0


def check_fine_groups(O, bits, gk, gv):
    """Fine-grained groups (section KVキャッシュの分布特性: K ranges along each channel, V ranges along
    each token): every K (s, z) is the range of one channel over g_k consecutive tokens and every V
    (s, z) the range of one token over g_v consecutive channels, by brute force with exact rationals;
    codes are the nearest grid points; prefill equals streaming; D is s * code + z exactly."""
    rng = np.random.default_rng(171 + bits + gk + gv)
    R, d, L = 128, 128, 2 ** bits - 1
    T = 2 * R + 21
    k = (rng.standard_normal((T, d)) * np.exp2(rng.integers(-2, 3, (1, d)))).astype(np.float16)
    k[:, 5] *= np.float16(12)                       # an outlier channel
    v = rng.standard_normal((T, d)).astype(np.float16)
    v[0] *= np.float16(6)                           # a sink token
    h = O.HeadCache(d, bits, gk, gv, R, 4 * R, fine_groups=True)
    h.prefill(k, v)
    n_q = 2 * R
    assert (h.n_quant, h.n_res) == (n_q, 21)
    assert h.k_s.shape == (n_q // gk, d) and h.v_s.shape == (n_q, d // gv)
    for u in range(n_q // gk):
        for c in list(range(0, d, 9)) + [5]:
            vals = [_fr(k[t, c]) for t in range(u * gk, (u + 1) * gk)]
            lo, hi = min(vals), max(vals)
            sx = fp16_round_exact((hi - lo) / L)
            assert Fraction(float(h.k_s[u, c])) == sx and Fraction(float(h.k_z[u, c])) == lo, (u, c)
            for t in range(u * gk, (u + 1) * gk, 7):
                assert h.k_codes[t, c] == code_nearest_grid(_fr(k[t, c]), sx, lo, bits), (t, c)
    for t in list(range(0, n_q, 13)) + [0]:
        for g in range(d // gv):
            vals = [_fr(v[t, c]) for c in range(g * gv, (g + 1) * gv)]
            lo, hi = min(vals), max(vals)
            sx = fp16_round_exact((hi - lo) / L)
            assert Fraction(float(h.v_s[t, g])) == sx and Fraction(float(h.v_z[t, g])) == lo, (t, g)
            for c in range(g * gv, (g + 1) * gv, 5):
                assert h.v_codes[t, c] == code_nearest_grid(_fr(v[t, c]), sx, lo, bits), (t, c)
    keys, values = h.keys(), h.values()
    for t, c in ((0, 5), (R + 3, 64), (n_q - 1, 127)):
        assert Fraction(float(keys[t, c])) == _fr(h.k_s[t // gk, c]) * int(h.k_codes[t, c]) + _fr(h.k_z[t // gk, c])
        g = c // gv
        assert Fraction(float(values[t, c])) == _fr(h.v_s[t, g]) * int(h.v_codes[t, c]) + _fr(h.v_z[t, g])
    assert np.array_equal(keys[n_q:], k[n_q:].astype(np.float64))
    a = O.HeadCache(d, bits, gk, gv, R, 4 * R, fine_groups=True)
    a.prefill(k[:40], v[:40])
    for t in range(40, T):
        if a.n_res == R:
            a.flush()
        a.append(k[t], v[t])
    for key, want in h.packed().items():
        assert np.array_equal(np.asarray(a.packed()[key]).view(np.uint8), np.asarray(want).view(np.uint8)), key


def check_errors(O):
    h = _head(O, cap=128)
    k = np.zeros((128, 128), np.float16)
    h.prefill(k, k)
    for fn, code in ((lambda: h.append(k[0], k[0]), "RESIDUAL_FULL"),):
        try:
            fn()
            raise AssertionError("expected " + code)
        except O.OracleError as e:
            assert e.code == code
    h.flush()
    try:
        h.flush()
        raise AssertionError("expected RESIDUAL_NOT_FULL")
    except O.OracleError as e:
        assert e.code == "RESIDUAL_NOT_FULL"
    for _ in range(128):
        h.append(k[0], k[0])
    try:
        h.flush()
        raise AssertionError("expected CAPACITY")
    except O.OracleError as e:
        assert e.code == "CAPACITY"


# --------------------------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------------------------
def check_attention_sdpa(O):
    """All-residual cache (T <= R): the oracle equals PyTorch SDPA in float64, GQA included."""
    rng = np.random.default_rng(81)
    for T, G in ((1, 1), (7, 1), (128, 4), (100, 2)):
        k = rng.standard_normal((T, 128)).astype(np.float16)
        v = rng.standard_normal((T, 128)).astype(np.float16)
        q = rng.standard_normal((G, 128)).astype(np.float16)
        h = _head(O)
        h.prefill(k, v)
        assert h.n_quant == 0
        scale = 1 / math.sqrt(128)
        got = h.attend(q, scale)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q.astype(np.float64))[None, :, None, :],
            torch.from_numpy(k.astype(np.float64))[None, None].expand(1, G, T, 128),
            torch.from_numpy(v.astype(np.float64))[None, None].expand(1, G, T, 128),
            scale=scale)[0, :, 0, :].numpy()
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-13), np.abs(got - ref).max()


def check_attention_closed_forms(O):
    rng = np.random.default_rng(91)
    k = rng.standard_normal((640, 128)).astype(np.float16)
    v = (rng.standard_normal((640, 128)) * 2).astype(np.float16)
    h = _head(O)
    h.prefill(k, v)
    assert h.n_quant == 512
    # q = 0: uniform weights -> mean of the dequantized values (D of every quantized row + residual)
    vd = np.concatenate([
        np.array([[float(h.v_s[t // h.gv]) * h.v_codes[t, c] + float(h.v_z[t // h.gv])
                   for c in range(128)] for t in range(h.n_quant)]),
        h.v_res.astype(np.float64)])
    got = h.attend(np.zeros((1, 128), np.float16), 0.0884)
    assert np.allclose(got[0], vd.mean(axis=0), rtol=0, atol=1e-12)
    # one token: the output is that token's value
    h1 = _head(O)
    h1.prefill(k[:1], v[:1])
    assert np.array_equal(h1.attend(k[:1], 1.0)[0], v[0].astype(np.float64))


def check_attention_bruteforce(O, bits, group):
    """Tiny cache with quantized blocks and residual; pure-Python attention that reads the packed
    words bit by bit and applies D = s*code + z with the block / group scale of each element."""
    rng = np.random.default_rng(101 + bits)
    R = 128
    T = 2 * R + 37
    k = (rng.standard_normal((T, 128)) * np.where(np.arange(128) % 29 == 0, 8, 1)).astype(np.float16)
    v = rng.standard_normal((T, 128)).astype(np.float16)
    v[0] *= np.float16(5)
    q = rng.standard_normal((2, 128)).astype(np.float16)
    h = _head(O, bits, group)
    h.prefill(k, v)
    pk = h.packed()
    P, mask = 32 // bits, 2 ** bits - 1
    keys, vals = [], []
    for t in range(h.n_quant):
        kr, vr = [], []
        for c in range(128):
            code = (int(pk["k_codes"][t, c // P]) >> (bits * (c % P))) & mask
            kr.append(float(pk["k_scale"][t // R, c // group]) * code + float(pk["k_zero"][t // R, c // group]))
            code = (int(pk["v_codes"][t // P, c]) >> (bits * (t % P))) & mask
            vr.append(float(pk["v_scale"][t // group]) * code + float(pk["v_zero"][t // group]))
        keys.append(kr)
        vals.append(vr)
    for t in range(h.n_res):
        keys.append([float(x) for x in pk["k_res"][t]])
        vals.append([float(x) for x in pk["v_res"][t]])
    scale = 1 / math.sqrt(128)
    got = h.attend(q, scale)
    for gq in range(2):
        logits = [scale * sum(float(q[gq, c]) * kr[c] for c in range(128)) for kr in keys]
        m = max(logits)
        w = [math.exp(x - m) for x in logits]
        tot = sum(w)
        out = [sum(w[t] * vals[t][c] for t in range(len(w))) / tot for c in range(128)]
        assert np.allclose(got[gq], out, rtol=1e-11, atol=1e-12), np.abs(got[gq] - out).max()

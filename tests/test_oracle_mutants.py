"""Plants plausible mistakes in the CPU oracle and checks that at least one pin catches each.

The mistakes are planted by monkeypatching oracle functions in this process only (CPU); the
oracle on disk is untouched.

Two candidate mistakes turned out to be equivalent on fp16 inputs and are not listed: forming
max - min in float32 before the division (a sweep over every positive fp16 max with tiny
negative minima found no changed s, because the dropped bits lie far below fp16 resolution and
the quotient never sits that close to a rounding midpoint), and packing V through a transpose of
the K packer (which is the V layout itself).
"""
import numpy as np
import pytest

import oracle.kivi_oracle as O
import oracle_pins as pins

_real = {name: getattr(O, name) for name in O.__all__}


def _scale_pow2(lo, hi, bits):                       # divides by 2^b instead of 2^b - 1
    s = O.fp16_round((np.asarray(lo, np.float16).astype(np.float64) * -1
                      + np.asarray(hi, np.float16).astype(np.float64)) / (1 << bits))
    return s, np.asarray(lo, np.float16).copy()


def _zero_is_max(lo, hi, bits):                      # z = max instead of min
    s, _ = _real["scale_zero"](lo, hi, bits)
    return s, np.asarray(hi, np.float16).copy()


def _codes_floor(x, s, z, bits):
    x64, s64, z64 = (np.asarray(a, np.float16).astype(np.float64) for a in (x, s, z))
    r = np.floor((x64 - z64) / np.where(s64 == 0, 1, s64))
    return np.where(s64 == 0, 0, np.clip(r, 0, O.levels(bits))).astype(np.uint8)


def _codes_half_up(x, s, z, bits):
    x64, s64, z64 = (np.asarray(a, np.float16).astype(np.float64) for a in (x, s, z))
    r = np.floor((x64 - z64) / np.where(s64 == 0, 1, s64) + 0.5)
    return np.where(s64 == 0, 0, np.clip(r, 0, O.levels(bits))).astype(np.uint8)


def _codes_no_clamp(x, s, z, bits):
    x64, s64, z64 = (np.asarray(a, np.float16).astype(np.float64) for a in (x, s, z))
    r = np.rint((x64 - z64) / np.where(s64 == 0, 1, s64))
    return np.where(s64 == 0, 0, r).astype(np.uint8)


def _k_groups_over_tokens(block, group_k, bits):     # K grouped like V (transposed axis)
    c, s, z = _real["quantize_v_block"](block, group_k, bits)
    return c, s[: block.shape[1] // group_k], z[: block.shape[1] // group_k]


def _v_groups_over_channels(block, group_v, bits):   # V grouped like K
    c, s, z = _real["quantize_k_block"](block, group_v, bits)
    return c, s[: block.shape[0] // group_v], z[: block.shape[0] // group_v]


def _pack_k_reversed(codes, bits):
    per = O.codes_per_word(bits)
    return _real["pack_k"](np.asarray(codes).reshape(codes.shape[0], -1, per)[:, :, ::-1]
                           .reshape(codes.shape), bits)


def _pack_v_as_k(codes, bits):                       # packs channels of a token, like K
    codes = np.asarray(codes)
    return _real["pack_k"](codes, bits).reshape(codes.shape[0] * codes_w(bits) // 128, 128)


def codes_w(bits):
    return 128 // O.codes_per_word(bits)


def _dequant_k_block_shift(codes, s, z, block, group_k):
    return _real["dequantize_k"](codes, np.roll(s, 1, axis=0), np.roll(z, 1, axis=0), block, group_k)


def _dequant_v_swapped(codes, s, z, group_v):
    return _real["dequantize_v"](codes, z, s, group_v)


def _attention_no_scale(q, keys, values, scale):
    return _real["attention"](q, keys, values, 1.0)


def _attention_kv_swapped(q, keys, values, scale):
    return _real["attention"](q, values, keys, scale)


def _attention_drop_last(q, keys, values, scale):   # forgets the newest token
    if len(keys) > 1:
        keys, values = keys[:-1], values[:-1]
    return _real["attention"](q, keys, values, scale)


MUTANTS = {
    "scale_divides_by_2^b": ("scale_zero", _scale_pow2),
    "zero_point_is_max": ("scale_zero", _zero_is_max),
    "codes_floor": ("quantize_values", _codes_floor),
    "codes_round_half_up": ("quantize_values", _codes_half_up),
    "codes_no_clamp": ("quantize_values", _codes_no_clamp),
    "k_groups_over_tokens": ("quantize_k_block", _k_groups_over_tokens),
    "v_groups_over_channels": ("quantize_v_block", _v_groups_over_channels),
    "pack_k_bit_order_reversed": ("pack_k", _pack_k_reversed),
    "pack_v_channels_instead_of_tokens": ("pack_v", _pack_v_as_k),
    "dequant_k_wrong_block": ("dequantize_k", _dequant_k_block_shift),
    "dequant_v_scale_zero_swapped": ("dequantize_v", _dequant_v_swapped),
    "attention_no_scale": ("attention", _attention_no_scale),
    "attention_k_v_swapped": ("attention", _attention_kv_swapped),
    "attention_drops_newest_token": ("attention", _attention_drop_last),
}

CHECKS = [
    lambda: pins.check_hand_examples(O),
    lambda: pins.check_scale_zero_exact(O, 2),
    lambda: pins.check_codes_exact(O, 2),
    lambda: pins.check_invariants(O, 2),
    lambda: pins.check_block_groups(O, 2, 32),
    lambda: pins.check_pack_golden(O),
    lambda: pins.check_pack_roundtrip(O, 2),
    lambda: pins.check_prefill_split(O),
    lambda: pins.check_attention_sdpa(O),
    lambda: pins.check_attention_closed_forms(O),
    lambda: pins.check_attention_bruteforce(O, 2, 32),
]


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_some_pin_catches_mutant(mutant, monkeypatch):
    name, fn = MUTANTS[mutant]
    monkeypatch.setattr(O, name, fn)
    caught = []
    for check in CHECKS:
        try:
            check()
        except Exception as e:   # an assertion or a shape error both count as caught
            caught.append(type(e).__name__)
            break
    assert caught, f"no pin catches the planted mistake {mutant}"


def _prefix_k_per_block(self, k, v):                 # K groups per R-token block, as in prefill
    return O.HeadCache.prefill(self, k, v)


def _prefix_k_whole_prompt(self, k, v):              # K groups over the residual tokens too
    k = np.asarray(k, np.float16)
    T = k.shape[0]
    n_q = T - ((T - 1) % self.R + 1)
    _real_prefix(self, k, v)
    if n_q:
        kc, ks, kz = O.quantize_k_block(k, self.gk, self.bits)
        self.k_codes = kc[:n_q]
        self.k_s = np.tile(ks[None, :], (n_q // self.R, 1))
        self.k_z = np.tile(kz[None, :], (n_q // self.R, 1))


_real_prefix = O.HeadCache.prefill_prefix_k


@pytest.mark.parametrize("mutant", [_prefix_k_per_block, _prefix_k_whole_prompt], ids=["per_block", "whole_prompt"])
def test_prefix_pin_catches_mutant(mutant, monkeypatch):
    monkeypatch.setattr(O.HeadCache, "prefill_prefix_k", mutant)
    with pytest.raises(AssertionError):
        pins.check_prefix_k_groups(O, 2, 32)


def _online_first_block(self, rows):                  # reuses the oldest block's (s, z), not the newest
    rows = np.asarray(rows, np.float16).reshape(-1, self.d)
    s, z = self.k_s[0], self.k_z[0]
    if self.k_s.shape[0] == self.n_quant // self.R:
        self.k_s = np.concatenate([self.k_s, self.k_s[-1][None, :]])
        self.k_z = np.concatenate([self.k_z, self.k_z[-1][None, :]])
    codes = O.quantize_values(rows, np.repeat(s, self.gk)[None, :], np.repeat(z, self.gk)[None, :], self.bits)
    self.k_codes = np.concatenate([self.k_codes, codes])


def _online_no_clamp(self, rows):                     # rounds without clamping to [0, 2^b - 1]
    rows = np.asarray(rows, np.float16).reshape(-1, self.d)
    last = self.n_quant // self.R - 1
    s, z = self.k_s[last], self.k_z[last]
    if self.k_s.shape[0] == self.n_quant // self.R:
        self.k_s = np.concatenate([self.k_s, s[None, :]])
        self.k_z = np.concatenate([self.k_z, z[None, :]])
    s64 = np.repeat(s, self.gk).astype(np.float64)
    r = np.rint((rows.astype(np.float64) - np.repeat(z, self.gk).astype(np.float64)) / np.where(s64 == 0, 1, s64))
    self.k_codes = np.concatenate([self.k_codes, (r.astype(np.int64) & 0xFF).astype(np.uint8)])


@pytest.mark.parametrize("mutant", [_online_first_block, _online_no_clamp], ids=["first_block", "no_clamp"])
def test_online_pin_catches_mutant(mutant, monkeypatch):
    monkeypatch.setattr(O.HeadCache, "_code_online", mutant)
    with pytest.raises(AssertionError):
        pins.check_online_k(O, 2, 32)


_real_fine_k, _real_fine_v = O.quantize_k_block_fine, O.quantize_v_block_fine


def _fine_k_over_channels(block, group_k, bits):     # K ranges taken along channels, not tokens
    codes, s, z = O.quantize_k_block(block[:group_k * (block.shape[0] // group_k)], 32, bits)
    c2, s2, z2 = _real_fine_k(block, group_k, bits)
    s2[:] = np.repeat(s, 32)[None, :]
    z2[:] = np.repeat(z, 32)[None, :]
    return codes, s2, z2


def _fine_v_over_tokens(block, group_v, bits):       # V ranges taken along tokens, not channels
    codes, s, z = O.quantize_v_block(block, 32, bits)
    c2, s2, z2 = _real_fine_v(block, group_v, bits)
    s2[:] = np.repeat(s, 32)[:, None]
    z2[:] = np.repeat(z, 32)[:, None]
    return codes, s2, z2


@pytest.mark.parametrize("name,mutant", [("quantize_k_block_fine", _fine_k_over_channels),
                                         ("quantize_v_block_fine", _fine_v_over_tokens)],
                         ids=["k_over_channels", "v_over_tokens"])
def test_fine_pin_catches_mutant(name, mutant, monkeypatch):
    monkeypatch.setattr(O, name, mutant)
    with pytest.raises(AssertionError):
        pins.check_fine_groups(O, 2, 32, 32)

"""The CPU oracle against facts that do not come from its own code (CPU only)."""
import pytest

import oracle.kivi_oracle as O
import oracle_pins as pins


def test_fp16_round_matches_exact_rational():
    pins.check_fp16_round(O)


@pytest.mark.parametrize("bits", [2, 4])
def test_scale_zero_matches_exact_rational(bits):
    pins.check_scale_zero_exact(O, bits)


@pytest.mark.parametrize("bits", [2, 4])
def test_codes_match_exact_rational_and_nearest_grid(bits):
    pins.check_codes_exact(O, bits)


def test_hand_examples():
    pins.check_hand_examples(O)


@pytest.mark.parametrize("bits", [2, 4])
def test_quantizer_invariants(bits):
    pins.check_invariants(O, bits)


@pytest.mark.parametrize("bits,group", [(2, 32), (4, 32), (2, 128), (4, 128)])
def test_block_group_axes(bits, group):
    pins.check_block_groups(O, bits, group)


def test_pack_hand_examples():
    pins.check_pack_golden(O)


@pytest.mark.parametrize("bits", [2, 4])
def test_pack_roundtrip(bits):
    pins.check_pack_roundtrip(O, bits)


def test_prefill_split():
    pins.check_prefill_split(O)


@pytest.mark.parametrize("bits,group", [(2, 32), (4, 128)])
def test_prefill_equals_streaming(bits, group):
    pins.check_prefill_equals_streaming(O, bits, group)


def test_cache_errors():
    pins.check_errors(O)


def test_attention_matches_torch_sdpa():
    pins.check_attention_sdpa(O)


def test_attention_closed_forms():
    pins.check_attention_closed_forms(O)


@pytest.mark.parametrize("bits,group", [(2, 32), (4, 128)])
def test_attention_bruteforce_from_packed_words(bits, group):
    pins.check_attention_bruteforce(O, bits, group)


@pytest.mark.parametrize("bits,group", [(2, 32), (4, 64), (2, 128)])
def test_prefix_k_groups(bits, group):
    pins.check_prefix_k_groups(O, bits, group)


@pytest.mark.parametrize("bits,group", [(2, 32), (4, 64), (2, 128)])
def test_online_k(bits, group):
    pins.check_online_k(O, bits, group)


@pytest.mark.parametrize("bits,gk,gv", [(2, 32, 32), (4, 64, 32), (2, 128, 64), (2, 32, 128)])
def test_fine_groups(bits, gk, gv):
    pins.check_fine_groups(O, bits, gk, gv)

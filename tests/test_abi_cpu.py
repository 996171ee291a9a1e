"""The C-ABI library loads, exports every function include/kivi.h declares, and its host-side
checks work without a GPU (no compute call is made here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kivi.h")


@pytest.fixture(scope="module")
def kivi():
    from bit_asymmetric_kv_02_b200 import build, kivi as k
    build.build()
    k.load_library()
    return k


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kivi_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(kivi):
    names = declared_functions()
    assert len(names) >= 11
    lib = ctypes.CDLL(kivi.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_strerror(kivi):
    assert kivi.kivi_abi_version() == 4
    assert kivi.kivi_strerror(0) == "ok"
    assert "flush" in kivi.kivi_strerror(4)
    assert kivi.kivi_strerror(12345) == "unknown status"


def _cfg(kivi, **kw):
    base = dict(batch=2, num_kv_heads=3, head_dim=128, bits=2, group_k=32, group_v=32, residual=128, capacity=1024)
    base.update(kw)
    return kivi.kivi_config(**base)


def test_config_rules(kivi):
    assert kivi.kivi_check_config(_cfg(kivi)) == 0
    assert kivi.kivi_check_config(_cfg(kivi, bits=3)) == 2
    assert kivi.kivi_check_config(_cfg(kivi, head_dim=64)) == 2
    assert kivi.kivi_check_config(_cfg(kivi, group_k=48)) == 1
    assert kivi.kivi_check_config(_cfg(kivi, group_v=48)) == 1
    assert kivi.kivi_check_config(_cfg(kivi, residual=100)) == 1
    assert kivi.kivi_check_config(_cfg(kivi, residual=384, capacity=768)) == 1
    assert kivi.kivi_check_config(_cfg(kivi, group_v=96)) == 1
    assert kivi.kivi_check_config(_cfg(kivi, group_v=256)) == 1
    assert kivi.kivi_check_config(_cfg(kivi, residual=256, group_v=256, capacity=1024)) == 0
    assert kivi.kivi_check_config(_cfg(kivi, capacity=1000)) == 1
    assert kivi.kivi_check_config(_cfg(kivi, batch=0)) == 1
    assert kivi.kivi_check_config(_cfg(kivi, bits=4, group_k=128, group_v=128)) == 0


def test_cache_sizes(kivi):
    sizes = kivi.kivi_cache_sizes(_cfg(kivi))
    bh, C, d = 6, 1024, 128
    assert sizes[0] == sizes[1] == bh * C * d * 2 // 8
    assert sizes[2] == sizes[3] == bh * (C // 128) * (d // 32) * 2
    assert sizes[4] == sizes[5] == bh * (C // 32) * 2
    assert sizes[6] == sizes[7] == bh * 128 * d * 2
    s4 = kivi.kivi_cache_sizes(_cfg(kivi, bits=4, group_k=128, group_v=128))
    assert s4[0] == bh * C * d // 2 and s4[2] == bh * (C // 128) * 2 and s4[4] == bh * (C // 128) * 2


def test_cache_sizes_past_32_bits(kivi):
    """Sizes are size_t all the way: 512 KV heads with room for 2^20 tokens need 2^32 code words (16 GiB)
    per code array, and the largest capacity the prefill grid allows (32767 blocks) as well."""
    sizes = kivi.kivi_cache_sizes(_cfg(kivi, batch=8, num_kv_heads=64, capacity=1 << 20))
    assert sizes[0] == sizes[1] == (1 << 32) * 4
    assert sizes[6] == 512 * 128 * 128 * 2
    big = _cfg(kivi, batch=1024, num_kv_heads=64, capacity=32767 * 128)
    assert kivi.kivi_check_config(big) == 0
    assert kivi.kivi_cache_sizes(big)[0] == 1024 * 64 * 32767 * 128 * 32
    assert kivi.kivi_check_config(_cfg(kivi, capacity=32768 * 128)) == 2  # the prefill grid's limit


def test_state_errors_before_any_device_work(kivi):
    """Errors detected on the host return before anything is enqueued; fake (aligned, never
    dereferenced) pointers are enough to reach them."""
    cfg = _cfg(kivi)
    fake = 1 << 20
    cache = kivi.kivi_cache(*([fake] * 8), 0, 128)
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_append_token(cfg, cache, fake, fake, 0)
    assert e.value.code == "RESIDUAL_FULL"
    cache.n_res = 5
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_flush_residual(cfg, cache, 0)
    assert e.value.code == "RESIDUAL_NOT_FULL"
    cache.n_quant, cache.n_res = 1024, 128
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_flush_residual(cfg, cache, 0)
    assert e.value.code == "CAPACITY"
    cache.n_quant = 100
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_flush_residual(cfg, cache, 0)
    assert e.value.code == "STATE"
    cache.n_quant, cache.n_res = 0, 0
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_decode_attention(cfg, cache, fake, 3, 0.1, fake, fake, 1 << 30, None, 0)
    assert e.value.code == "EMPTY"
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_decode_attention(cfg, cache, fake, 4, 0.1, fake, fake, 1 << 30, None, 0)
    assert e.value.code == "INVALID_ARG"
    cache.n_res = 1
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_decode_attention(cfg, cache, fake, 3 * 16, 0.1, fake, fake, 1 << 30, None, 0)
    assert e.value.code == "UNSUPPORTED"
    cache.n_quant, cache.n_res = 0, 128
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_append_decode_attention(cfg, cache, fake, fake, fake, 3, 0.1, fake, fake, 1 << 30, None, 0)
    assert e.value.code == "RESIDUAL_FULL" and cache.n_res == 128
    cache.n_res = 5
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_append_decode_attention(cfg, cache, fake + 8, fake, fake, 3, 0.1, fake, fake, 1 << 30, None, 0)
    assert e.value.code == "INVALID_ARG" and cache.n_res == 5
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_append_decode_attention(cfg, cache, fake, fake, fake, 4, 0.1, fake, fake, 1 << 30, None, 0)
    assert e.value.code == "INVALID_ARG" and cache.n_res == 5
    cache.n_quant, cache.n_res = 0, 1
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_quantize_prefill(cfg, cache, fake, fake, 0, 0)
    assert e.value.code == "INVALID_ARG"
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_quantize_prefill(cfg, cache, fake + 8, fake, 10, 0)
    assert e.value.code == "INVALID_ARG"
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_quantize_prefill(cfg, cache, fake, fake, 1024 + 129, 0)
    assert e.value.code == "CAPACITY"


def test_decode_step_host_errors(kivi):
    """kivi_decode_step checks everything on the host before it enqueues anything, and leaves the
    counters unchanged on an error: misaligned rows, a full residual with no block left, a state
    the configuration cannot hold, and (after those pass) the attention's own checks."""
    cfg = _cfg(kivi)
    fake = 1 << 20
    cache = kivi.kivi_cache(*([fake] * 8), 0, 5)
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_decode_step(cfg, cache, fake + 8, fake, fake, 3, 0.1, fake, fake, 1 << 30, None, 0)
    assert e.value.code == "INVALID_ARG" and (cache.n_quant, cache.n_res) == (0, 5)
    cache.n_quant, cache.n_res = 1024, 128       # full residual, every block used: no flush possible
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_decode_step(cfg, cache, fake, fake, fake, 3, 0.1, fake, fake, 1 << 30, None, 0)
    assert e.value.code == "CAPACITY" and (cache.n_quant, cache.n_res) == (1024, 128)
    cache.n_quant, cache.n_res = 100, 5
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_decode_step(cfg, cache, fake, fake, fake, 3, 0.1, fake, fake, 1 << 30, None, 0)
    assert e.value.code == "STATE" and (cache.n_quant, cache.n_res) == (100, 5)
    cache.n_quant = 0
    with pytest.raises(kivi.KiviError) as e:      # 4 query heads over 3 KV heads
        kivi.kivi_decode_step(cfg, cache, fake, fake, fake, 4, 0.1, fake, fake, 1 << 30, None, 0)
    assert e.value.code == "INVALID_ARG" and (cache.n_quant, cache.n_res) == (0, 5)
    with pytest.raises(kivi.KiviError) as e:      # a misaligned output
        kivi.kivi_decode_step(cfg, cache, fake, fake, fake, 3, 0.1, fake + 2, fake, 1 << 30, None, 0)
    assert e.value.code == "INVALID_ARG" and (cache.n_quant, cache.n_res) == (0, 5)


def test_online_k_host_errors(kivi):
    """Online K (section Per-Channel量子化): the flag's rule and the capacity its block slot needs,
    checked on the host before anything is enqueued."""
    assert kivi.kivi_check_config(_cfg(kivi, online_k=1)) == 0
    assert kivi.kivi_check_config(_cfg(kivi, online_k=2)) == 1
    cfg = _cfg(kivi, online_k=1)
    fake = 1 << 20
    cache = kivi.kivi_cache(*([fake] * 8), 1024, 3)     # every block slot used: no room for online rows
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_append_token(cfg, cache, fake, fake, 0)
    assert e.value.code == "CAPACITY" and cache.n_res == 3
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_append_decode_attention(cfg, cache, fake, fake, fake, 3, 0.1, fake, fake, 1 << 30, None, 0)
    assert e.value.code == "CAPACITY" and cache.n_res == 3
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_decode_attention(cfg, cache, fake, 3, 0.1, fake, fake, 1 << 30, None, 0)
    assert e.value.code == "STATE"
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_quantize_prefill(cfg, cache, fake, fake, 1024 + 1, 0)
    assert e.value.code == "CAPACITY" and (cache.n_quant, cache.n_res) == (1024, 3)
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_quantize_prefill_prefix_k(cfg, cache, fake, fake, 300, 0)
    assert e.value.code == "UNSUPPORTED"


def test_fine_groups_host_rules(kivi):
    """Fine-grained groups (section KVキャッシュの分布特性): group_k counts tokens (<= R), group_v counts
    channels; the scale buffers change size; decode is built for 2 bits and one query per KV head."""
    assert kivi.kivi_check_config(_cfg(kivi, fine_groups=1)) == 0
    assert kivi.kivi_check_config(_cfg(kivi, fine_groups=2)) == 1
    assert kivi.kivi_check_config(_cfg(kivi, fine_groups=1, group_v=256, residual=256, capacity=1024)) == 1
    assert kivi.kivi_check_config(_cfg(kivi, fine_groups=1, group_k=128, group_v=64)) == 0
    assert kivi.kivi_check_config(_cfg(kivi, fine_groups=1, online_k=1)) == 2
    sizes = kivi.kivi_cache_sizes(_cfg(kivi, fine_groups=1, group_k=64, group_v=32))
    bh = 2 * 3
    assert sizes[2] == sizes[3] == bh * (1024 // 64) * 128 * 2      # K: [C/G_k][d]
    assert sizes[4] == sizes[5] == bh * 1024 * (128 // 32) * 2      # V: [C][d/G_v]
    fake = 1 << 20
    cache = kivi.kivi_cache(*([fake] * 8), 128, 3)
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_quantize_prefill_prefix_k(_cfg(kivi, fine_groups=1), cache, fake, fake, 300, 0)
    assert e.value.code == "UNSUPPORTED"


def test_binding_fails_loudly_without_library(tmp_path):
    from bit_asymmetric_kv_02_b200 import kivi as k
    saved = k._lib
    k._lib = None
    try:
        with pytest.raises(RuntimeError):
            k.load_library(str(tmp_path / "missing.so"))
    finally:
        k._lib = saved


def test_debug_entry_points_of_the_release_build(kivi):
    """kivi_debug_status and test hook 3 belong to the debug build; the release build refuses them
    on the host (no device call)."""
    assert kivi.load_library().kivi_debug_status() == 2          # KIVI_ERR_UNSUPPORTED
    assert kivi.load_library().kivi_debug_inject(3, 1) == 2
    assert kivi.load_library().kivi_debug_inject(0, 0) == 0


def test_debug_build_exports_the_same_symbols():
    from bit_asymmetric_kv_02_b200 import build
    path = build.build(debug=True)
    lib = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(lib, n), n

"""Fine-grained groups (section KVキャッシュの分布特性: the K range along each channel, the V range along
each token) on the GPU, against the oracle's fine_groups mode.

K codes, K (s, z) per channel per g_k tokens, V codes, V (s, z) per token per g_v channels and the
residual must equal the oracle's bit for bit after the prefill, the appends and the flush; decode
attention must be within tolerance at 2 and 4 bits with one to eight queries per KV head, also with
each head split over several warps.
"""
import numpy as np
import pytest

import gpu_common as gc
import oracle.kivi_oracle as O
from bit_asymmetric_kv_02_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _kivi():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_asymmetric_kv_02_b200 import build, kivi
    build.build()
    kivi.load_library()
    torch.cuda.set_device(0)
    return kivi


# group = tokens per K group, group_v = channels per V group
CASES = [
    synth.TINY.with_(name="fine_2bit_gk32_gv32", batch=2, q_heads=2, kv_heads=2, tokens=3 * 128 + 37, seed=71),
    synth.TINY.with_(name="fine_2bit_gk64_gv64_R256", batch=1, q_heads=2, kv_heads=2, tokens=2 * 256 + 9, group=64,
                     group_v=64, residual=256, seed=72),
    synth.TINY.with_(name="fine_2bit_gk128_gv128", batch=1, q_heads=1, kv_heads=1, tokens=4 * 128 + 1, group=128,
                     group_v=128, seed=73),
    synth.TINY.with_(name="fine_2bit_gk32_gv128_R1024", batch=1, q_heads=1, kv_heads=1, tokens=1024 + 70,
                     group_v=128, residual=1024, seed=74),
    synth.TINY.with_(name="fine_fits_residual", batch=1, q_heads=2, kv_heads=2, tokens=90, seed=75),
    # several queries per KV head and 4 bits
    synth.TINY.with_(name="fine_2bit_gqa2_gk32_gv64", batch=2, q_heads=4, kv_heads=2, tokens=3 * 128 + 11, group_v=64,
                     seed=76),
    synth.TINY.with_(name="fine_2bit_gqa4_gk64_gv32", batch=1, q_heads=8, kv_heads=2, tokens=2 * 128 + 77, group=64,
                     seed=77),
    synth.TINY.with_(name="fine_2bit_gqa8_gk128", batch=1, q_heads=8, kv_heads=1, tokens=3 * 128 + 5, group=128,
                     seed=78),
    synth.TINY.with_(name="fine_4bit_gk32_gv32", batch=2, q_heads=2, kv_heads=2, tokens=3 * 128 + 37, bits=4, seed=79),
    synth.TINY.with_(name="fine_4bit_gk64_gv128", batch=1, q_heads=2, kv_heads=2, tokens=2 * 128 + 9, bits=4, group=64,
                     group_v=128, seed=80),
    synth.TINY.with_(name="fine_4bit_gk128_gv64_gqa2", batch=1, q_heads=4, kv_heads=2, tokens=3 * 128 + 100, bits=4,
                     group=128, group_v=64, seed=81),
    synth.TINY.with_(name="fine_4bit_gqa4_gk32", batch=1, q_heads=8, kv_heads=2, tokens=2 * 128 + 50, bits=4, seed=82),
    synth.TINY.with_(name="fine_4bit_gqa8_R512", batch=1, q_heads=8, kv_heads=1, tokens=512 + 300, bits=4,
                     group_v=64, residual=512, seed=83),
]


def _view_rows(cache, name, b, h, rows):
    return cache.view(name)[b, h, :rows].cpu().numpy()


def _check(cache, ref, what):
    for (b, h), hc in ref.items():
        want = hc.packed()
        got = {}
        for key, w in want.items():
            rows = np.asarray(w).shape[0]
            if key in ("k_codes", "v_codes"):
                got[key] = _view_rows(cache, key, b, h, rows).view(np.uint32)
            else:
                got[key] = _view_rows(cache, key, b, h, rows)
        gc.assert_head_bitexact(got, want, f"{what} head {(b, h)}")
    hc0 = next(iter(ref.values()))
    assert (cache.n_quant, cache.n_res) == (hc0.n_quant, hc0.n_res)


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_fine_groups_match_oracle(w):
    kivi = _kivi()
    T = w.tokens
    cap = (T // w.residual + 2) * w.residual
    k, v = synth.prompt_kv(w, T)
    cache = kivi.KiviCache(w.batch, w.kv_heads, cap, bits=w.bits, group_k=w.group, group_v=w.gv,
                           residual=w.residual, num_q_heads=w.q_heads, fine_groups=True)
    cache.status.zero_()
    cache.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    heads = [(b, h) for b in range(w.batch) for h in range(w.kv_heads)]
    ref = {bh: O.HeadCache(128, w.bits, w.group, w.gv, w.residual, cap, fine_groups=True) for bh in heads}
    for (b, h), hc in ref.items():
        hc.prefill(k[b, h], v[b, h])
    _check(cache, ref, f"{w.name} prefill")
    g = w.q_heads // w.kv_heads
    steps = w.residual - cache.n_res + 3
    checked = {0, 1, steps - 3, steps - 2, steps}
    for s in range(steps + 1):
        q = synth.queries(w, s)
        out = None
        if s > 0:
            if cache.n_res == w.residual:
                cache.flush()
                for hc in ref.values():
                    hc.flush()
                _check(cache, ref, f"{w.name} flush before step {s}")
            kn, vn = synth.new_kv(w, s)
            if s % 2:
                out = cache.append_attend(torch.from_numpy(kn).cuda(), torch.from_numpy(vn).cuda(),
                                          torch.from_numpy(q).cuda())
            else:
                cache.append(torch.from_numpy(kn).cuda(), torch.from_numpy(vn).cuda())
            for (b, h), hc in ref.items():
                hc.append(kn[b, h], vn[b, h])
        if s in checked:
            if out is None:
                out = cache.attend(torch.from_numpy(q).cuda())
            out = out.cpu().numpy()
            for (b, h), hc in ref.items():
                gc.assert_attention_close(out[b, h * g:(h + 1) * g],
                                          hc.attend(q[b, h * g:(h + 1) * g], gc.default_scale()),
                                          f"{w.name} step {s} head {(b, h)}")
    _check(cache, ref, f"{w.name} end")
    assert cache.read_status() == 0


def test_fine_groups_with_forced_splits():
    """Fine-grained heads split over many warps (partials merged), 4 bits and 2 bits with GQA."""
    kivi = _kivi()
    for bits, gqa in ((4, 2), (2, 4)):
        w = synth.TINY.with_(name=f"fine_split_{bits}_{gqa}", batch=1, q_heads=2 * gqa, kv_heads=2,
                             tokens=5 * 128 + 31, bits=bits, seed=84 + bits)
        cap = 6 * 128
        k, v = synth.prompt_kv(w, w.tokens)
        q = synth.queries(w, 0)
        cache = kivi.KiviCache(1, 2, cap, bits=bits, num_q_heads=2 * gqa, fine_groups=True)
        cache.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
        try:
            kivi.kivi_debug_inject(2, 7)
            cache.status.zero_()
            out = cache.attend(torch.from_numpy(q).cuda()).cpu().numpy()
            assert cache.read_status() == 0
        finally:
            kivi.kivi_debug_inject(0, 0)
        for h in range(2):
            hc = O.HeadCache(128, bits, 32, 32, 128, cap, fine_groups=True)
            hc.prefill(k[0, h], v[0, h])
            gc.assert_attention_close(out[0, h * gqa:(h + 1) * gqa], hc.attend(q[0, h * gqa:(h + 1) * gqa],
                                                                              gc.default_scale()),
                                      f"fine split {bits}-bit gqa {gqa} head {h}")

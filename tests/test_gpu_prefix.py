"""kivi_quantize_prefill_prefix_k: prefill with one K group over the whole quantized prefix (GPU).

Codes, scales, zero points and residual rows must equal the oracle's prefill_prefix_k bit for bit,
decode attention over the result must be within tolerance, and appends and a flush after it must
follow the oracle (the flushed block takes its own block-local K groups).  Cases cover both quantize
kernels (register tiles for R <= 512, two passes for R = 1024), 2 and 4 bits, G_k != G_v, GQA and a
prompt that fits the residual.
"""
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


CASES = [
    synth.TINY.with_(name="prefix_2bit_g32", batch=2, q_heads=2, kv_heads=2, tokens=5 * 128 + 37, seed=51),
    synth.TINY.with_(name="prefix_4bit_g64_R256_gqa2", batch=1, q_heads=4, kv_heads=2, tokens=3 * 256 + 9, bits=4,
                     group=64, residual=256, seed=52),
    synth.TINY.with_(name="prefix_2bit_g32_gv128", batch=1, q_heads=2, kv_heads=2, tokens=4 * 128 + 1, group_v=128,
                     seed=53),
    synth.TINY.with_(name="prefix_2bit_g128_R1024", batch=1, q_heads=1, kv_heads=1, tokens=2 * 1024 + 5, group=128,
                     residual=1024, seed=54),
    synth.TINY.with_(name="prefix_fits_residual", batch=1, q_heads=2, kv_heads=2, tokens=100, seed=55),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_prefix_k_prefill_matches_oracle(w):
    kivi = _kivi()
    T = w.tokens
    cap = (T // w.residual + 2) * w.residual
    k, v = synth.prompt_kv(w, T)
    cache = kivi.KiviCache(w.batch, w.kv_heads, cap, bits=w.bits, group_k=w.group, group_v=w.gv,
                           residual=w.residual, num_q_heads=w.q_heads)
    cache.status.zero_()
    cache.prefill_prefix_k(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    heads = [(b, h) for b in range(w.batch) for h in range(w.kv_heads)]
    ref = {bh: O.HeadCache(128, w.bits, w.group, w.gv, w.residual, cap) for bh in heads}
    for (b, h), hc in ref.items():
        hc.prefill_prefix_k(k[b, h], v[b, h])
        gc.assert_head_bitexact(gc.gpu_buffers_of_head(cache, b, h, cache.n_quant, cache.n_res), hc.packed(),
                                f"{w.name} prefill head {(b, h)}")
    assert (cache.n_quant, cache.n_res) == (ref[heads[0]].n_quant, ref[heads[0]].n_res)
    g = w.q_heads // w.kv_heads
    steps = w.residual - cache.n_res + 3        # fills the residual, flushes once, appends 3 more
    for s in range(steps + 1):
        if s > 0:
            if cache.n_res == w.residual:
                cache.flush()
                for hc in ref.values():
                    hc.flush()
            kn, vn = synth.new_kv(w, s)
            cache.append(torch.from_numpy(kn).cuda(), torch.from_numpy(vn).cuda())
            for (b, h), hc in ref.items():
                hc.append(kn[b, h], vn[b, h])
        if s in (0, 1, steps - 3, steps):
            q = synth.queries(w, s)
            out = cache.attend(torch.from_numpy(q).cuda()).cpu().numpy()
            for (b, h), hc in ref.items():
                gc.assert_attention_close(out[b, h * g:(h + 1) * g], hc.attend(q[b, h * g:(h + 1) * g],
                                                                                gc.default_scale()),
                                          f"{w.name} step {s} head {(b, h)}")
    for (b, h), hc in ref.items():
        gc.assert_head_bitexact(gc.gpu_buffers_of_head(cache, b, h, cache.n_quant, cache.n_res), hc.packed(),
                                f"{w.name} after the flush, head {(b, h)}")
    assert cache.read_status() == 0

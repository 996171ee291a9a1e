"""kivi_append_decode_attention: append and decode attention in one launch (GPU).

The fused call must leave exactly the cache contents of kivi_append_token and return exactly the
outputs of kivi_decode_attention on that cache (same kernel arithmetic, so bit for bit), and both
must match the oracle: residual rows bit-exact, attention within tolerance.  The steps cover the
residual's first slot (after a flush), its last slot, a flush in between, every 16-row residual
unit, split heads and GQA.
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


CASES = [
    synth.TINY.with_(name="fused_2bit", batch=2, q_heads=3, kv_heads=3, tokens=300, seed=31),
    synth.TINY.with_(name="fused_4bit_gqa2", batch=2, q_heads=4, kv_heads=2, tokens=250, bits=4, seed=32),
    synth.TINY.with_(name="fused_2bit_gqa4_g128", batch=1, q_heads=8, kv_heads=2, tokens=700, group=128, seed=33),
    synth.TINY.with_(name="fused_2bit_R256_gv64", batch=1, q_heads=2, kv_heads=2, tokens=600, group_v=64, residual=256,
                     seed=36),
    synth.TINY.with_(name="fused_4bit_R512_gk64", batch=1, q_heads=2, kv_heads=1, tokens=900, bits=4, group=64,
                     residual=512, seed=37),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_fused_equals_two_calls_and_oracle(w):
    kivi = _kivi()
    T = w.tokens
    steps = 2 * w.residual + 7        # two flushes: every residual slot is appended at least once
    cap = ((T + steps) // w.residual + 1) * w.residual
    k, v = synth.prompt_kv(w, T)
    caches = []
    for _ in range(2):
        c = kivi.KiviCache(w.batch, w.kv_heads, cap, bits=w.bits, group_k=w.group, group_v=w.gv,
                           residual=w.residual, num_q_heads=w.q_heads)
        c.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
        c.status.zero_()
        caches.append(c)
    two, fused = caches
    heads = [(b, h) for b in range(w.batch) for h in range(w.kv_heads)]
    ref = {bh: O.HeadCache(128, w.bits, w.group, w.gv, w.residual, cap) for bh in heads}
    for (b, h), hc in ref.items():
        hc.prefill(k[b, h], v[b, h])
    g = w.q_heads // w.kv_heads
    checked = 0
    for s in range(1, steps + 1):
        if two.n_res == w.residual:
            two.flush()
            fused.flush()
            for hc in ref.values():
                hc.flush()
        kn, vn = synth.new_kv(w, s)
        q = synth.queries(w, s)
        knd, vnd, qd = (torch.from_numpy(x).cuda() for x in (kn, vn, q))
        two.append(knd, vnd)
        o_two = two.attend(qd)
        o_fused = fused.append_attend(knd, vnd, qd)
        for (b, h), hc in ref.items():
            hc.append(kn[b, h], vn[b, h])
        assert (fused.n_quant, fused.n_res) == (two.n_quant, two.n_res)
        a, f = o_two.cpu().numpy(), o_fused.cpu().numpy()
        assert np.array_equal(a.view(np.uint16), f.view(np.uint16)), f"step {s}: fused output differs"
        if s in (1, 2, 15, 16, 17, 84, 85, 128, 129, steps) or s % 37 == 0 or two.n_res in (1, w.residual):
            for (b, h), hc in ref.items():
                gc.assert_attention_close(f[b, h * g:(h + 1) * g], hc.attend(q[b, h * g:(h + 1) * g], gc.default_scale()),
                                          f"{w.name} step {s} head {(b, h)}")
                gc.assert_head_bitexact(gc.gpu_buffers_of_head(fused, b, h, fused.n_quant, fused.n_res), hc.packed(),
                                        f"{w.name} step {s} head {(b, h)}")
            checked += 1
    assert checked >= 10
    assert two.read_status() == 0 and fused.read_status() == 0


def test_fused_with_forced_splits():
    """Every head split over many warps, so the residual units land on different warps."""
    kivi = _kivi()
    w = synth.TINY.with_(name="fused_splits", batch=1, q_heads=2, kv_heads=2, tokens=1000, seed=34)
    cap = 1280
    k, v = synth.prompt_kv(w, w.tokens)
    kivi.kivi_debug_inject(2, 7)     # cap the decode at 7 workers
    try:
        c = kivi.KiviCache(w.batch, w.kv_heads, cap, num_q_heads=w.q_heads)
        c.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
        ref = {(0, h): O.HeadCache(128, 2, 32, 32, 128, cap) for h in range(2)}
        for (b, h), hc in ref.items():
            hc.prefill(k[b, h], v[b, h])
        for s in range(1, 40):
            if c.n_res == 128:
                c.flush()
                for hc in ref.values():
                    hc.flush()
            kn, vn = synth.new_kv(w, s)
            q = synth.queries(w, s)
            out = c.append_attend(*(torch.from_numpy(x).cuda() for x in (kn, vn, q))).cpu().numpy()
            for (b, h), hc in ref.items():
                hc.append(kn[b, h], vn[b, h])
                gc.assert_attention_close(out[b, h:h + 1], hc.attend(q[b, h:h + 1], gc.default_scale()),
                                          f"step {s} head {(b, h)}")
        for (b, h), hc in ref.items():
            gc.assert_head_bitexact(gc.gpu_buffers_of_head(c, b, h, c.n_quant, c.n_res), hc.packed(), "after")
        assert c.read_status() == 0
    finally:
        kivi.kivi_debug_inject(0, 0)


def test_fused_refuses_a_full_residual():
    kivi = _kivi()
    w = synth.TINY.with_(name="fused_full", batch=1, q_heads=1, kv_heads=1, tokens=256, seed=35)
    k, v = synth.prompt_kv(w, w.tokens)
    c = kivi.KiviCache(1, 1, 384)
    c.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    assert c.n_res == 128
    kn, vn = synth.new_kv(w, 1)
    q = synth.queries(w, 1)
    with pytest.raises(kivi.KiviError) as e:
        c.append_attend(*(torch.from_numpy(x).cuda() for x in (kn, vn, q)))
    assert e.value.code == "RESIDUAL_FULL"
    assert (c.n_quant, c.n_res) == (128, 128)

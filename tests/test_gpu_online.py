"""Online K quantization (section Per-Channel量子化: a new token's K is quantized at once with the
existing scale and zero point) on the GPU, against the oracle's online_k mode.

After the prefill, every append and the flush, the K code rows (the online rows included), the K
(s, z) rows (the copy held by the block being filled included), the V codes, scales and residual
must equal the oracle's bit for bit, and decode attention (residual keys from codes, values from
the fp16 residual) must be within tolerance.  Cases: 2 and 4 bits, one to four queries per KV
head, R = 128 and 256, and a prompt that fits the residual (K stays fp16 until the first flush).
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
    synth.TINY.with_(name="online_2bit_g32", batch=2, q_heads=2, kv_heads=2, tokens=3 * 128 + 37, seed=61),
    synth.TINY.with_(name="online_4bit_g64_R256_gqa2", batch=1, q_heads=4, kv_heads=2, tokens=2 * 256 + 9, bits=4,
                     group=64, residual=256, seed=62),
    synth.TINY.with_(name="online_2bit_gqa4", batch=1, q_heads=8, kv_heads=2, tokens=2 * 128 + 100, seed=63),
    synth.TINY.with_(name="online_fits_residual", batch=1, q_heads=2, kv_heads=2, tokens=100, seed=64),
    synth.TINY.with_(name="online_4bit_g32", batch=1, q_heads=1, kv_heads=1, tokens=128 + 1, bits=4, seed=65),
]


def _buffers_like(cache, b, h, want):
    """The GPU head's buffers, each cut to the rows the oracle's packed buffer has."""
    full = gc.gpu_buffers_of_head(cache, b, h, cache.cfg.capacity, cache.cfg.residual)
    out = {}
    for key, ref in want.items():
        rows = np.asarray(ref).shape[0]
        out[key] = full[key][:rows]
    return out


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_online_k_matches_oracle(w):
    kivi = _kivi()
    T = w.tokens
    cap = (T // w.residual + 3) * w.residual
    k, v = synth.prompt_kv(w, T)
    cache = kivi.KiviCache(w.batch, w.kv_heads, cap, bits=w.bits, group_k=w.group, group_v=w.gv,
                           residual=w.residual, num_q_heads=w.q_heads, online_k=True)
    cache.status.zero_()
    cache.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    heads = [(b, h) for b in range(w.batch) for h in range(w.kv_heads)]
    ref = {bh: O.HeadCache(128, w.bits, w.group, w.gv, w.residual, cap, online_k=True) for bh in heads}

    def check_buffers(what):
        for (b, h), hc in ref.items():
            want = hc.packed()
            gc.assert_head_bitexact(_buffers_like(cache, b, h, want), want, f"{w.name} {what} head {(b, h)}")
        assert (cache.n_quant, cache.n_res) == (ref[heads[0]].n_quant, ref[heads[0]].n_res)

    for (b, h), hc in ref.items():
        hc.prefill(k[b, h], v[b, h])
    check_buffers("prefill")
    g = w.q_heads // w.kv_heads
    steps = w.residual - cache.n_res + 4        # fills the residual, flushes once, appends 4 more
    checked = {0, 1, 2, steps - 4, steps - 3, steps}
    for s in range(steps + 1):
        q = synth.queries(w, s)
        out = None
        if s > 0:
            if cache.n_res == w.residual:
                cache.flush()
                for hc in ref.values():
                    hc.flush()
                check_buffers(f"flush before step {s}")
            kn, vn = synth.new_kv(w, s)
            if s % 2:   # the fused call (two launches under online K) and the separate calls alternate
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
    check_buffers("end")
    assert cache.read_status() == 0

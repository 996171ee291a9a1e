"""The cache at its size limits, against the oracle.

- Code arrays past every 32-bit offset: 512 KV heads with room for 2^20 tokens each at 2 bits (2^19 at
  4 bits) make each code array 2^32 words (16 GiB), so the rows of the later heads lie beyond every
  32-bit element and byte offset.  A short prompt, then decode steps through kivi_decode_step up to the
  step whose token fills the residual and is quantized in the same launch (section 残差バッファ of the
  KIVI explainer page); sampled heads bit for bit and within tolerance.
- One KV head of 3 * 2^17 + 44 cached tokens (3075 units of work, more than the resident warps): the
  decode splits it over every resident warp and one warp merges all their partials (the online-softmax
  merge of the attention over the cache).

Every address the kernels form on these paths is 64-bit; these cases hold them to it.
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


def _cuda(*arrays):
    return [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in arrays]


@pytest.mark.parametrize("bits", [2, 4])
def test_code_offsets_beyond_32_bits(bits):
    kivi = _kivi()
    w = synth.TINY.with_(name=f"offsets_{bits}bit", batch=8, q_heads=64, kv_heads=64, tokens=300, bits=bits,
                         seed=171 + bits)
    R = w.residual
    cap = (1 << 20) if bits == 2 else (1 << 19)
    words = w.batch * w.kv_heads * cap * (128 * bits // 32)
    assert words == 1 << 32
    heads = [(0, 0), (3, 17), (6, 40), (w.batch - 1, w.kv_heads - 1)]
    ref = {bh: O.HeadCache(128, bits, w.group, w.gv, R, cap) for bh in heads}
    k, v = synth.prompt_kv(w, w.tokens)
    for (b, h), hc in ref.items():
        hc.prefill(k[b, h], v[b, h])
    cache = kivi.KiviCache(w.batch, w.kv_heads, cap, bits=bits, group_k=w.group, group_v=w.gv, residual=R,
                           num_q_heads=w.q_heads)
    cache.status.zero_()
    cache.prefill(*_cuda(k, v))
    del k, v
    n0 = cache.n_res
    assert (cache.n_quant, n0) == (256, 44)

    def check(label, out, q):
        for (b, h), hc in ref.items():
            gc.assert_head_bitexact(gc.gpu_buffers_of_head(cache, b, h, cache.n_quant, cache.n_res), hc.packed(),
                                    f"{label} head {(b, h)}")
            if out is not None:
                gc.assert_attention_close(out[b, h:h + 1], hc.attend(q[b, h:h + 1], gc.default_scale()),
                                          f"{label} head {(b, h)}")

    q = synth.queries(w, 0)
    check("prefill", cache.attend(*_cuda(q)).cpu().numpy(), q)
    last = R - n0  # the step whose token fills the residual
    for s in range(1, last + 1):
        kn, vn = synth.new_kv(w, s)
        q = synth.queries(w, s)
        out = cache.step(*_cuda(kn, vn, q))
        for (b, h), hc in ref.items():
            hc.append(kn[b, h], vn[b, h])
        if s in (1, last - 1, last):
            out = out.cpu().numpy()
            if s == last:  # the step quantized the full residual in its launch; the oracle attends first
                want = {(b, h): hc.attend(q[b, h:h + 1], gc.default_scale()) for (b, h), hc in ref.items()}
                for hc in ref.values():
                    hc.flush()
                assert (cache.n_quant, cache.n_res) == (256 + R, 0)
                check(f"step {s} (flushed in the launch)", None, None)
                for (b, h) in heads:
                    gc.assert_attention_close(out[b, h:h + 1], want[(b, h)], f"step {s} head {(b, h)}")
            else:
                check(f"step {s}", out, q)
    assert cache.read_status() == 0


def test_one_head_over_every_warp():
    kivi = _kivi()
    w = synth.TINY.with_(name="one_long_head", batch=1, q_heads=1, kv_heads=1, tokens=3 * (1 << 17) + 44, seed=175)
    R = w.residual
    cap = 3 * (1 << 17) + R
    k, v = synth.prompt_kv(w, w.tokens)
    hc = O.HeadCache(128, w.bits, w.group, w.gv, R, cap)
    hc.prefill(k[0, 0], v[0, 0])
    cache = kivi.KiviCache(1, 1, cap, bits=w.bits, group_k=w.group, group_v=w.gv, residual=R, num_q_heads=1)
    cache.status.zero_()
    cache.prefill(*_cuda(k, v))
    del k, v
    assert (cache.n_quant, cache.n_res) == (3 * (1 << 17), 44)
    gc.assert_head_bitexact(gc.gpu_buffers_of_head(cache, 0, 0, cache.n_quant, cache.n_res), hc.packed(), "prefill")
    q = synth.queries(w, 0)
    gc.assert_attention_close(cache.attend(*_cuda(q)).cpu().numpy()[0], hc.attend(q[0], gc.default_scale()), "attend")
    kn, vn = synth.new_kv(w, 1)
    q = synth.queries(w, 1)
    out = cache.step(*_cuda(kn, vn, q)).cpu().numpy()
    hc.append(kn[0, 0], vn[0, 0])
    gc.assert_attention_close(out[0], hc.attend(q[0], gc.default_scale()), "step 1")
    assert cache.read_status() == 0

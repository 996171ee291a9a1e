"""kivi_decode_step: append, attend and (when the token fills the residual) flush, in one launch.

Section 残差バッファ of the KIVI explainer page: the newest tokens stay fp16 and every R of them
become one quantized block.  The step flushes eagerly, at the step that fills the residual; the
calls it stands for flush lazily, at the next step.  Every step's output must equal, bit for bit,
the output of the lazy sequence (flush when full, then kivi_append_decode_attention), and be
within tolerance of the oracle; after every flush the new block's codes, scales and zero points
must equal the oracle's bit for bit.  The base groups must take one kernel launch per step, flush
steps included (counted with the torch profiler); online K and fine-grained groups fall back to
the separate launches and must give the same results.
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
    synth.TINY.with_(name="step_2bit", batch=2, q_heads=3, kv_heads=3, tokens=300, seed=131),
    synth.TINY.with_(name="step_4bit_gqa2", batch=2, q_heads=4, kv_heads=2, tokens=250, bits=4, seed=132),
    synth.TINY.with_(name="step_2bit_gqa4_g128", batch=1, q_heads=8, kv_heads=2, tokens=700, group=128, seed=133),
    synth.TINY.with_(name="step_2bit_R256_gv64", batch=1, q_heads=2, kv_heads=2, tokens=600, group_v=64,
                     residual=256, seed=136),
    synth.TINY.with_(name="step_4bit_R512_gk64_gv128", batch=1, q_heads=2, kv_heads=1, tokens=900, bits=4, group=64,
                     group_v=128, residual=512, seed=137),
    synth.TINY.with_(name="step_2bit_gqa8", batch=1, q_heads=16, kv_heads=2, tokens=200, seed=138),
]


def _caches(kivi, w, cap, k, v, **kw):
    out = []
    for _ in range(2):
        c = kivi.KiviCache(w.batch, w.kv_heads, cap, bits=w.bits, group_k=w.group, group_v=w.gv,
                           residual=w.residual, num_q_heads=w.q_heads, **kw)
        c.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
        c.status.zero_()
        out.append(c)
    return out


def _run_steps(kivi, w, steps, cap, check_every=None, **kw):
    """Lazy calls and decode steps side by side, against the oracle flushing eagerly."""
    T = w.tokens
    k, v = synth.prompt_kv(w, T)
    lazy, step = _caches(kivi, w, cap, k, v, **kw)
    heads = [(b, h) for b in range(w.batch) for h in range(w.kv_heads)]
    ref = {bh: O.HeadCache(128, w.bits, w.group, w.gv, w.residual, cap, **kw) for bh in heads}
    for (b, h), hc in ref.items():
        hc.prefill(k[b, h], v[b, h])
    g = w.q_heads // w.kv_heads
    flushes = 0
    for s in range(1, steps + 1):
        if lazy.n_res == w.residual:
            lazy.flush()
        kn, vn = synth.new_kv(w, s)
        q = synth.queries(w, s)
        knd, vnd, qd = (torch.from_numpy(x).cuda() for x in (kn, vn, q))
        o_lazy = lazy.append_attend(knd, vnd, qd)
        o_step = step.step(knd, vnd, qd)
        for hc in ref.values():
            if hc.n_res == w.residual:
                hc.flush()
        for (b, h), hc in ref.items():
            hc.append(kn[b, h], vn[b, h])
        a, f = o_lazy.cpu().numpy(), o_step.cpu().numpy()
        assert np.array_equal(a.view(np.uint16), f.view(np.uint16)), f"{w.name} step {s}: output differs"
        filled = ref[heads[0]].n_res == w.residual
        check = filled or s in (1, 2, steps) or (check_every and s % check_every == 0)
        # the step attended the full residual in fp16 and then flushed it: the oracle attends first
        want = {bh: hc.attend(q[bh[0], bh[1] * g:(bh[1] + 1) * g], gc.default_scale())
                for bh, hc in ref.items()} if check else {}
        if filled:
            for hc in ref.values():
                hc.flush()
            flushes += 1
        assert (step.n_quant, step.n_res) == (ref[heads[0]].n_quant, ref[heads[0]].n_res), f"step {s}"
        if check:
            for (b, h), hc in ref.items():
                if kw.get("fine_groups") or kw.get("online_k"):   # rows as the oracle's buffers have them
                    want_buf = hc.packed()
                    got = {}
                    for key, x in want_buf.items():
                        rows = step.view(key)[b, h, :np.asarray(x).shape[0]].cpu().numpy()
                        got[key] = rows.view(np.uint32) if key in ("k_codes", "v_codes") else rows
                    gc.assert_head_bitexact(got, want_buf, f"{w.name} step {s} head {(b, h)}")
                else:
                    gc.assert_head_bitexact(gc.gpu_buffers_of_head(step, b, h, step.n_quant, step.n_res),
                                            hc.packed(), f"{w.name} step {s} head {(b, h)}")
                gc.assert_attention_close(f[b, h * g:(h + 1) * g], want[(b, h)], f"{w.name} step {s} head {(b, h)}")
    assert lazy.read_status() == 0 and step.read_status() == 0
    return flushes


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_step_equals_lazy_calls_and_oracle(w):
    kivi = _kivi()
    steps = 2 * w.residual + 5          # two in-launch flushes
    cap = ((w.tokens + steps) // w.residual + 1) * w.residual
    assert _run_steps(kivi, w, steps, cap, check_every=41) == 2


@pytest.mark.parametrize("bits", [2, 4])
def test_step_largest_residual(bits):
    """R = 1024: a K group job spans 128 tokens per lane slot and is staged eight times per pass."""
    kivi = _kivi()
    w = synth.TINY.with_(name=f"step_R1024_{bits}bit", batch=1, q_heads=2, kv_heads=2, tokens=1100, bits=bits,
                         residual=1024, group_v=64, seed=141)
    steps = 1024 + 3
    cap = ((w.tokens + steps) // w.residual + 1) * w.residual
    assert _run_steps(kivi, w, steps, cap, check_every=257) == 1


def test_step_with_forced_splits():
    """Every head split over 5 warps, so one head's residual and its flush jobs land on different
    warps."""
    kivi = _kivi()
    w = synth.TINY.with_(name="step_splits", batch=1, q_heads=2, kv_heads=2, tokens=1000, seed=134)
    kivi.kivi_debug_inject(2, 5)
    try:
        assert _run_steps(kivi, w, 140, 1280, check_every=29) == 1
    finally:
        kivi.kivi_debug_inject(0, 0)


@pytest.mark.parametrize("kw", [{"online_k": True}, {"fine_groups": True}], ids=["online_k", "fine"])
def test_step_separate_launch_schemes(kw):
    kivi = _kivi()
    w = synth.TINY.with_(name="step_sep", batch=1, q_heads=2, kv_heads=2, tokens=2 * 128 + 20, seed=139)
    steps = 128 + 6
    cap = ((w.tokens + steps) // 128 + 1) * 128
    assert _run_steps(kivi, w, steps, cap, check_every=33, **kw) == 1


def test_step_full_residual_at_entry_and_capacity():
    """A prefill that leaves the residual full is flushed first; a residual that fills with no block
    left stays full, and the next step reports CAPACITY with the counters unchanged."""
    kivi = _kivi()
    w = synth.TINY.with_(name="step_edges", batch=1, q_heads=1, kv_heads=1, tokens=256, seed=135)
    k, v = synth.prompt_kv(w, w.tokens)
    cap = 256       # the flush at entry takes the last block
    c = kivi.KiviCache(1, 1, cap)
    c.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    assert (c.n_quant, c.n_res) == (128, 128)
    hc = O.HeadCache(128, 2, 32, 32, 128, cap)
    hc.prefill(k[0, 0], v[0, 0])
    for s in range(1, 129):
        kn, vn = synth.new_kv(w, s)
        q = synth.queries(w, s)
        out = c.step(*(torch.from_numpy(x).cuda() for x in (kn, vn, q))).cpu().numpy()
        if hc.n_res == 128:
            hc.flush()
        hc.append(kn[0, 0], vn[0, 0])
        if s in (1, 2, 127, 128):
            gc.assert_attention_close(out[0, 0:1], hc.attend(q[0, 0:1], gc.default_scale()), f"step {s}")
    # the residual filled with n_quant + R > capacity: no flush
    assert (c.n_quant, c.n_res) == (256, 128)
    gc.assert_head_bitexact(gc.gpu_buffers_of_head(c, 0, 0, c.n_quant, c.n_res), hc.packed(), "full")
    kn, vn = synth.new_kv(w, 200)
    q = synth.queries(w, 200)
    with pytest.raises(kivi.KiviError) as e:
        c.step(*(torch.from_numpy(x).cuda() for x in (kn, vn, q)))
    assert e.value.code == "CAPACITY"
    assert (c.n_quant, c.n_res) == (256, 128)
    assert c.read_status() == 0


def _kernels_in(fn):
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    return [n for n in names if "kivi" in n]


def test_one_launch_per_step_including_flush_steps():
    kivi = _kivi()
    w = synth.TINY.with_(name="step_launches", batch=2, q_heads=4, kv_heads=2, tokens=200, seed=140)
    k, v = synth.prompt_kv(w, w.tokens)
    c = kivi.KiviCache(w.batch, w.kv_heads, 512, num_q_heads=w.q_heads)
    c.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    assert c.n_res == 72
    seen = []
    for s in range(1, 60):       # step 56 fills the residual and flushes
        kn, vn, q = (torch.from_numpy(x).cuda() for x in (*synth.new_kv(w, s), synth.queries(w, s)))
        before = c.n_quant
        if s < 53:
            c.step(kn, vn, q)
            continue
        kern = _kernels_in(lambda: c.step(kn, vn, q))
        seen.append((s, c.n_quant > before, kern))
    flush_steps = [x for x in seen if x[1]]
    assert len(flush_steps) == 1 and flush_steps[0][0] == 56
    for s, flushed, kern in seen:
        assert len(kern) == 1, f"step {s} (flush: {flushed}) launched {kern}"
        assert "decode_kernel" in kern[0]
    assert c.read_status() == 0

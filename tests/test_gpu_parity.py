"""CUDA path (through the C ABI) vs the CPU oracle on the same seeded inputs.

Codes, scales, zero points and residual rows must match bit for bit; decode outputs must be within
max-abs 2e-3 and max-rel 1e-2 (relative to max(|o*|, 1e-2)) of the fp64 oracle run on the same
quantized cache.
"""
import numpy as np
import pytest

import gpu_common as gc
import oracle.kivi_oracle as O
import oracle_workers as ow
from bit_asymmetric_kv_02_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_asymmetric_kv_02_b200 import build, kivi
    build.build()
    kivi.load_library()
    torch.cuda.set_device(0)


def _kivi():
    from bit_asymmetric_kv_02_b200 import kivi
    return kivi


def run_prefill_case(w: synth.Workload, heads=None, capacity=None, check_attention=True):
    """GPU prefill + decode of workload w; oracle on `heads` (all if None)."""
    kivi = _kivi()
    T = w.tokens
    cap = capacity if capacity is not None else ((T + w.residual - 1) // w.residual) * w.residual
    k, v = synth.prompt_kv(w, T)
    q = synth.queries(w, 0)
    cache = kivi.KiviCache(w.batch, w.kv_heads, cap, bits=w.bits, group_k=w.group, group_v=w.gv,
                           residual=w.residual, num_q_heads=w.q_heads)
    kd = torch.from_numpy(k).cuda()
    vd = torch.from_numpy(v).cuda()
    qd = torch.from_numpy(q).cuda()
    cache.status.zero_()
    cache.prefill(kd, vd)
    out = cache.attend(qd).cpu().numpy()
    assert cache.read_status() == 0
    n_quant, n_res = cache.n_quant, cache.n_res
    assert n_res == (T - 1) % w.residual + 1 and n_quant == T - n_res
    heads = heads if heads is not None else [(b, h) for b in range(w.batch) for h in range(w.kv_heads)]
    worst = (0.0, 0.0)
    for (b, h) in heads:
        hc = O.HeadCache(w.head_dim, w.bits, w.group, w.gv, w.residual, cap)
        hc.prefill(k[b, h], v[b, h])
        gc.assert_head_bitexact(gc.gpu_buffers_of_head(cache, b, h, n_quant, n_res), hc.packed(),
                                f"{w.name} head {(b, h)}")
        if check_attention:
            g = w.gqa
            want = hc.attend(q[b, h * g:(h + 1) * g], gc.default_scale())
            ea, er = gc.assert_attention_close(out[b, h * g:(h + 1) * g], want, f"{w.name} head {(b, h)}")
            worst = (max(worst[0], ea), max(worst[1], er))
    return worst


SMALL = [
    synth.TINY,
    synth.TINY.with_(name="ragged_2bit_g32", batch=2, q_heads=3, kv_heads=3, tokens=3 * 128 + 37, seed=7),
    synth.TINY.with_(name="ragged_4bit_g32", batch=1, q_heads=2, kv_heads=2, tokens=1024 + 5, bits=4, seed=8),
    synth.TINY.with_(name="2bit_g128", batch=2, q_heads=2, kv_heads=2, tokens=700, group=128, seed=9),
    synth.TINY.with_(name="4bit_g128", batch=1, q_heads=2, kv_heads=2, tokens=513, bits=4, group=128, seed=10),
    synth.TINY.with_(name="one_token", batch=2, q_heads=2, kv_heads=2, tokens=1, seed=11),
    synth.TINY.with_(name="exactly_R", batch=1, q_heads=2, kv_heads=2, tokens=128, seed=12),
    synth.TINY.with_(name="R_plus_1", batch=1, q_heads=2, kv_heads=2, tokens=129, seed=13),
    synth.TINY.with_(name="gqa4", batch=2, q_heads=8, kv_heads=2, tokens=900, seed=14),
    synth.TINY.with_(name="gqa2_4bit", batch=1, q_heads=4, kv_heads=2, tokens=300, bits=4, seed=15),
    synth.TINY.with_(name="gqa8", batch=1, q_heads=8, kv_heads=1, tokens=500, seed=16),
    synth.TINY.with_(name="many_heads_short", batch=16, q_heads=8, kv_heads=8, tokens=200, seed=17),
    # residual sizes and G_k != G_v: the register-tiled quantize path (R <= 512) and the two-pass one (R = 1024)
    synth.TINY.with_(name="R128_gk32_gv128", batch=2, q_heads=2, kv_heads=2, tokens=3 * 128 + 9, group_v=128,
                     seed=18),
    synth.TINY.with_(name="R256_gk64_gv256", batch=2, q_heads=4, kv_heads=2, tokens=2 * 256 + 77, group=64,
                     group_v=256, residual=256, seed=19),
    synth.TINY.with_(name="R512_4bit_gk32_gv64", batch=1, q_heads=2, kv_heads=2, tokens=2 * 512 + 300, bits=4,
                     group_v=64, residual=512, seed=20),
    synth.TINY.with_(name="R1024_2bit_gk128_gv32", batch=1, q_heads=2, kv_heads=2, tokens=2 * 1024 + 5, group=128,
                     group_v=32, residual=1024, seed=22),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_prefill_and_decode_small(w):
    run_prefill_case(w)


def test_capacity_larger_than_used():
    w = synth.TINY.with_(name="spare_capacity", tokens=600, seed=21)
    run_prefill_case(w, capacity=2048)


@pytest.mark.parametrize("bits,group", [(2, 32), (4, 32), (2, 128), (4, 128)])
def test_streaming_append_flush(bits, group):
    """prefill, then decode steps that flush when the residual is full, append one token and
    attend; codes after every flush and outputs at chosen steps must match the oracle."""
    kivi = _kivi()
    w = synth.TINY.with_(name=f"stream_{bits}_{group}", batch=2, q_heads=4, kv_heads=2, tokens=250,
                         bits=bits, group=group, seed=30 + bits + group)
    steps = 300
    cap = 1024
    k, v = synth.prompt_kv(w, w.tokens)
    cache = kivi.KiviCache(w.batch, w.kv_heads, cap, bits=bits, group_k=group, group_v=group,
                           residual=w.residual, num_q_heads=w.q_heads)
    cache.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    ref = {(b, h): O.HeadCache(128, bits, group, group, w.residual, cap)
           for b in range(w.batch) for h in range(w.kv_heads)}
    for (b, h), hc in ref.items():
        hc.prefill(k[b, h], v[b, h])
    check_at = {1, 2, 5, 6, 7, 133, 134, 135, 261, 262, 299, 300}
    for s in range(1, steps + 1):
        flushed = False
        if cache.n_res == w.residual:
            cache.flush()
            for hc in ref.values():
                hc.flush()
            flushed = True
        kn, vn = synth.new_kv(w, s)
        cache.append(torch.from_numpy(kn).cuda(), torch.from_numpy(vn).cuda())
        for (b, h), hc in ref.items():
            hc.append(kn[b, h], vn[b, h])
        if s in check_at or flushed:
            q = synth.queries(w, s)
            out = cache.attend(torch.from_numpy(q).cuda()).cpu().numpy()
            for (b, h), hc in ref.items():
                g = w.gqa
                gc.assert_attention_close(out[b, h * g:(h + 1) * g], hc.attend(q[b, h * g:(h + 1) * g], gc.default_scale()),
                                          f"step {s} head {(b, h)}")
                gc.assert_head_bitexact(gc.gpu_buffers_of_head(cache, b, h, cache.n_quant, cache.n_res), hc.packed(),
                                        f"step {s} head {(b, h)}")
    assert cache.read_status() == 0


@pytest.mark.parametrize("workers", [1, 2, 3, 5, 13, 0])
def test_forced_splits_match_oracle(workers):
    """The same cache decoded with 1, 2, 3, 5, 13 or the default number of workers: every split of
    heads across warps (direct writes, merges of 2..N partials, several heads per warp) matches."""
    kivi = _kivi()
    w = synth.TINY.with_(name="splits", batch=3, q_heads=4, kv_heads=2, tokens=5 * 128 + 77, seed=70)
    k, v = synth.prompt_kv(w, w.tokens)
    q = synth.queries(w)
    cap = 768
    cache = kivi.KiviCache(w.batch, w.kv_heads, cap, num_q_heads=w.q_heads)
    cache.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    try:
        kivi.kivi_debug_inject(2, workers)
        cache.status.zero_()
        out = cache.attend(torch.from_numpy(q).cuda()).cpu().numpy()
        assert cache.read_status() == 0
    finally:
        kivi.kivi_debug_inject(0, 0)
    for b in range(w.batch):
        for h in range(w.kv_heads):
            hc = O.HeadCache(128, 2, 32, 32, 128, cap)
            hc.prefill(k[b, h], v[b, h])
            g = w.gqa
            gc.assert_attention_close(out[b, h * g:(h + 1) * g], hc.attend(q[b, h * g:(h + 1) * g], gc.default_scale()),
                                      f"workers={workers} head {(b, h)}")


def test_prefill_equals_streaming_on_gpu():
    """The GPU cache after prefill(T) equals the GPU cache after prefill(T0) + appends/flushes."""
    kivi = _kivi()
    w = synth.TINY.with_(batch=1, q_heads=2, kv_heads=2, tokens=700, seed=40)
    k, v = synth.prompt_kv(w, w.tokens)
    a = kivi.KiviCache(1, 2, 1024, num_q_heads=2)
    a.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    b = kivi.KiviCache(1, 2, 1024, num_q_heads=2)
    b.prefill(torch.from_numpy(k[:, :, :100]).contiguous().cuda(), torch.from_numpy(v[:, :, :100]).contiguous().cuda())
    for t in range(100, 700):
        if b.n_res == 128:
            b.flush()
        b.append(torch.from_numpy(k[:, :, t]).contiguous().cuda(), torch.from_numpy(v[:, :, t]).contiguous().cuda())
    assert (a.n_quant, a.n_res) == (b.n_quant, b.n_res)
    for h in range(2):
        ga = gc.gpu_buffers_of_head(a, 0, h, a.n_quant, a.n_res)
        gb = gc.gpu_buffers_of_head(b, 0, h, b.n_quant, b.n_res)
        gc.assert_head_bitexact(ga, gb, f"head {h}")


def test_repeated_calls_are_identical():
    """The workspace tickets are left at zero, so back-to-back calls give identical outputs."""
    kivi = _kivi()
    w = synth.TINY.with_(batch=4, q_heads=8, kv_heads=8, tokens=3000, seed=50)
    k, v = synth.prompt_kv(w, w.tokens)
    cache = kivi.KiviCache(w.batch, w.kv_heads, 3072, num_q_heads=w.q_heads)
    cache.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    q = torch.from_numpy(synth.queries(w)).cuda()
    o1 = cache.attend(q).clone()
    o2 = cache.attend(q).clone()
    assert torch.equal(o1, o2)
    tickets = cache.workspace[cache.ws_ptr - cache.workspace.data_ptr():][: cache.ws_bytes]
    assert int(tickets[-w.batch * w.kv_heads * 4:].view(torch.int32).abs().sum()) == 0


def test_errors_through_the_abi():
    kivi = _kivi()
    cache = kivi.KiviCache(1, 2, 128, num_q_heads=2)
    q = torch.zeros(1, 2, 128, dtype=torch.float16, device="cuda")
    with pytest.raises(kivi.KiviError) as e:
        cache.attend(q)
    assert e.value.code == "EMPTY"
    with pytest.raises(kivi.KiviError) as e:
        cache.flush()
    assert e.value.code == "RESIDUAL_NOT_FULL"
    x = torch.zeros(1, 2, 128, 128, dtype=torch.float16, device="cuda")
    cache.prefill(x, x)
    assert (cache.n_quant, cache.n_res) == (0, 128)
    row = torch.zeros(1, 2, 128, dtype=torch.float16, device="cuda")
    with pytest.raises(kivi.KiviError) as e:
        cache.append(row, row)
    assert e.value.code == "RESIDUAL_FULL"
    cache.flush()
    for _ in range(128):
        cache.append(row, row)
    with pytest.raises(kivi.KiviError) as e:
        cache.flush()
    assert e.value.code == "CAPACITY"
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_decode_attention(cache.cfg, cache.c, q.data_ptr(), 2, 0.1, q.data_ptr(), cache.ws_ptr, 16,
                                   None, torch.cuda.current_stream().cuda_stream)
    assert e.value.code == "WORKSPACE"


@pytest.mark.parametrize("bits,kv_heads,q_heads,fine", [(2, 4, 4, False), (2, 2, 8, False), (4, 1, 8, False),
                                                      (2, 3, 3, True), (4, 2, 4, True)])
def test_workspace_size_rule_matches_the_decode(bits, kv_heads, q_heads, fine):
    """kivi_decode_workspace_bytes is exactly what kivi_decode_attention (and the no-alloc entry's
    ticket offset) requires: one byte less is refused with WORKSPACE, the size itself decodes."""
    kivi = _kivi()
    w = synth.TINY.with_(batch=2, q_heads=q_heads, kv_heads=kv_heads, tokens=300, bits=bits, seed=77)
    k, v = synth.prompt_kv(w, w.tokens)
    cache = kivi.KiviCache(w.batch, w.kv_heads, 384, bits=bits, num_q_heads=w.q_heads, fine_groups=fine)
    cache.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    need = kivi.kivi_decode_workspace_bytes(cache.cfg, w.q_heads)
    assert 0 < need <= cache.ws_bytes
    q = torch.from_numpy(synth.queries(w)).cuda()
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream().cuda_stream
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_decode_attention(cache.cfg, cache.c, q.data_ptr(), w.q_heads, 0.1, out.data_ptr(), cache.ws_ptr,
                                   need - 1, None, stream)
    assert e.value.code == "WORKSPACE"
    kivi.kivi_decode_attention(cache.cfg, cache.c, q.data_ptr(), w.q_heads, 0.1, out.data_ptr(), cache.ws_ptr, need,
                               None, stream)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()


def test_device_timeout_is_reported_and_context_survives():
    """A barrier that can never complete (the test hook asks for 16 bytes more than are copied)
    makes every bounded wait run out: the kernel reports DEVICE_TIMEOUT and returns; afterwards
    normal calls work on the same context."""
    kivi = _kivi()
    w = synth.TINY.with_(batch=1, q_heads=2, kv_heads=2, tokens=600, seed=60)
    k, v = synth.prompt_kv(w, w.tokens)
    cache = kivi.KiviCache(1, 2, 1024, num_q_heads=2)
    cache.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    q = torch.from_numpy(synth.queries(w)).cuda()
    ref = cache.attend(q).clone()
    assert cache.read_status() == 0
    try:
        kivi.kivi_debug_inject(1, 5_000_000)   # 5 ms bound per wait
        cache.status.zero_()
        cache.attend(q)
        assert cache.read_status() == 9   # KIVI_ERR_DEVICE_TIMEOUT
    finally:
        kivi.kivi_debug_inject(0, 0)
    cache.workspace.zero_()
    cache.status.zero_()
    again = cache.attend(q)
    assert cache.read_status() == 0
    assert torch.equal(again, ref)


FULL = [synth.LLAMA2_7B, synth.GQA_LLAMA3_8B]


def _gpu_head_digests(cache, heads, shapes):
    """{(b, h): {buffer: digest}} of the GPU cache, each buffer cut to the oracle's row count."""
    out = {bh: {} for bh in heads}
    for key in shapes:
        rows = shapes[key][0]
        full = cache.view(key)[:, :, :rows].cpu().numpy()
        if key in ("k_codes", "v_codes"):
            full = full.view(np.uint32)
        for (b, h) in heads:
            out[(b, h)][key] = ow.digest(full[b, h])
    return out


def _compare(label, gpu_digests, gpu_out, oracle_runs, gqa, what):
    """Checks one checkpoint of every head: buffers bit for bit (digests), outputs within tolerance."""
    worst = (0.0, 0.0)
    for (b, h), run in oracle_runs.items():
        entries = {(lab, kind): payload for lab, kind, payload in run}
        if gpu_digests is not None:
            want = entries[(label, "buffers")]
            got = gpu_digests[(b, h)]
            bad = [k for k in want if got[k] != want[k]]
            assert not bad, f"{what} {label} head {(b, h)}: buffers {bad} differ from the oracle"
        if gpu_out is not None:
            ea, er = gc.assert_attention_close(gpu_out[b, h * gqa:(h + 1) * gqa], entries[(label, "out")],
                                               f"{what} {label} head {(b, h)}")
            worst = (max(worst[0], ea), max(worst[1], er))
    return worst


def _shapes(oracle_runs, label):
    """{buffer: shape} of the oracle's packed buffers at one checkpoint (the same for every head)."""
    run = next(iter(oracle_runs.values()))
    for lab, kind, payload in run:
        if lab == label and kind == "buffers":
            return {key: shape for key, (shape, _sha) in payload.items()}
    raise KeyError(label)


def _full_size_steps(w, chunksize):
    """A full-size workload through the bench's call (kivi_decode_step) on every head: prefill,
    attention, then R decode steps.  Step 1 meets the prompt's full residual and flushes it in a
    launch of its own; step 2 takes the fused append + decode call instead; the token of step R fills
    the residual, and the step's one launch also quantizes it.  Buffers bit for bit after the
    prefill, after step 1 and after the in-launch flush; outputs within tolerance at steps 0, 1, 2,
    R - 1 and R."""
    kivi = _kivi()
    T, R = w.tokens, w.residual
    cap = (T - 1) // R * R + 2 * R  # room for the prompt's residual block and one more
    attend_at = frozenset({0, 1, 2, R - 1, R})
    heads = [(b, h) for b in range(w.batch) for h in range(w.kv_heads)]
    # the oracle runs one step further: its flush before step R + 1 is the GPU's flush inside step R
    specs = [ow.HeadStream(w, b, h, cap, T, steps=R + 1, attend_at=attend_at, digest_at=frozenset({0, 1}))
             for b, h in heads]
    with ow.pool() as ex:
        fut = ex.map(ow.run_head, specs, chunksize=chunksize)
        k, v = synth.prompt_kv(w, T)
        cache = kivi.KiviCache(w.batch, w.kv_heads, cap, bits=w.bits, group_k=w.group, group_v=w.gv,
                               residual=w.residual, num_q_heads=w.q_heads)
        cache.status.zero_()
        cache.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
        del k, v
        assert cache.n_res == R
        outs = {0: cache.attend(torch.from_numpy(synth.queries(w, 0)).cuda()).cpu().numpy()}
        runs = dict(zip(heads, fut))
        gpu = {"step 0": _gpu_head_digests(cache, heads, _shapes(runs, "step 0"))}
        for s in range(1, R + 1):
            kn, vn = synth.new_kv(w, s)
            x = [torch.from_numpy(a).cuda() for a in (kn, vn, synth.queries(w, s))]
            out = cache.append_attend(*x) if s == 2 else cache.step(*x)
            if s in attend_at:
                outs[s] = out.cpu().numpy()
            if s == 1:
                gpu["step 1"] = _gpu_head_digests(cache, heads, _shapes(runs, "step 1"))
        assert (cache.n_quant, cache.n_res) == (cap, 0)
        label = f"flush before step {R + 1}"
        gpu[label] = _gpu_head_digests(cache, heads, _shapes(runs, label))
        assert cache.read_status() == 0
    for lab in ("step 0", "step 1", label):
        _compare(lab, gpu[lab], None, runs, w.gqa, w.name)
    for s in sorted(attend_at):
        _compare(f"step {s}", None, outs[s], runs, w.gqa, w.name)


@pytest.mark.parametrize("w", FULL, ids=[w.name for w in FULL])
def test_full_size_all_heads(w):
    """The Llama-2 layer and the GQA workload at full size through the decode step (see
    _full_size_steps)."""
    _full_size_steps(w, chunksize=4)


def test_full_size_large_batch_step_all_heads():
    """The large batch (2048 KV heads) at full size through the decode step (see _full_size_steps)."""
    _full_size_steps(synth.LARGE_BATCH, chunksize=8)


@pytest.mark.parametrize("bits,group", [(2, 32), (2, 128), (4, 32), (4, 128)])
def test_full_size_streaming(bits, group):
    """Prefill 32768 tokens, then 256 decode steps (flush when full, append, attend; the second
    flush inside kivi_decode_step's launch), every head: buffers bit for bit after both flushes and
    at the checked steps, outputs within tolerance at steps around the flushes."""
    kivi = _kivi()
    w = synth.STREAMING.with_(bits=bits, group=group)
    cap = 33024
    check_at = frozenset({1, 2, 127, 128, 129, 256})
    heads = [(b, h) for b in range(w.batch) for h in range(w.kv_heads)]
    specs = [ow.HeadStream(w, b, h, cap, w.tokens, steps=w.steps, attend_at=check_at, digest_at=check_at | {0})
             for b, h in heads]
    with ow.pool() as ex:
        fut = ex.map(ow.run_head, specs, chunksize=2)
        k, v = _streaming_prompt()
        cache = kivi.KiviCache(w.batch, w.kv_heads, cap, bits=bits, group_k=group, group_v=group,
                               residual=w.residual, num_q_heads=w.q_heads)
        cache.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
        runs = dict(zip(heads, fut))
        shapes_of = lambda label: _shapes(runs, label)  # noqa: E731
        _compare("step 0", _gpu_head_digests(cache, heads, shapes_of("step 0")), None, runs, w.gqa, "prefill")
        for s in range(1, w.steps + 1):
            if cache.n_res == w.residual:
                cache.flush()
                label = f"flush before step {s}"
                _compare(label, _gpu_head_digests(cache, heads, shapes_of(label)), None, runs, w.gqa, w.name)
            kn, vn = synth.new_kv(w, s)
            q = synth.queries(w, s)
            # the decode step (every third step, and step 128, whose token fills the residual and is
            # flushed in the same launch), the fused call and the separate calls take turns
            use_step = s % 3 == 0 or s == 128
            if use_step:
                out = cache.step(*(torch.from_numpy(x).cuda() for x in (kn, vn, q)))
            elif s % 2:
                out = cache.append_attend(*(torch.from_numpy(x).cuda() for x in (kn, vn, q)))
            else:
                cache.append(torch.from_numpy(kn).cuda(), torch.from_numpy(vn).cuda())
                out = cache.attend(torch.from_numpy(q).cuda())
            flushed = use_step and cache.n_res == 0   # eager: the oracle's flush of the next step
            if flushed:
                label = f"flush before step {s + 1}"
                _compare(label, _gpu_head_digests(cache, heads, shapes_of(label)), None, runs, w.gqa, w.name)
            if s in check_at:
                label = f"step {s}"
                gpu = None if flushed else _gpu_head_digests(cache, heads, shapes_of(label))
                _compare(label, gpu, out.cpu().numpy(), runs, w.gqa, f"{w.name} {bits}-bit G={group}")
    assert cache.read_status() == 0
    assert (cache.n_quant, cache.n_res) == (32896, 128)


_PROMPT = {}


def _streaming_prompt():
    if "kv" not in _PROMPT:
        _PROMPT["kv"] = synth.prompt_kv(synth.STREAMING, synth.STREAMING.tokens)
    return _PROMPT["kv"]

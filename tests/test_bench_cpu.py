"""bench.py on CPU: it compiles, and its reference arm (the oracle timed on host cores) prints one
valid JSON line with the contract's keys."""
import json
import os

import pytest
import py_compile
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_compiles():
    py_compile.compile(os.path.join(ROOT, "bench.py"), doraise=True)


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                          "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in rec, key
    assert rec["impl"] == "reference" and rec["value"] > 0 and rec["ms_per_step"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] >= 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["d2h_bytes_per_step"] == 0
    assert rec["config"]["workload"] == "large_batch_b64_h32_t8192"


def test_algorithmic_bytes_match_the_buffer_layout():
    """The roofline numerator (bench.decode_alg_bytes) against the library's own buffer sizes
    (kivi_cache_sizes): every quantized token moves its codes and its share of the scales once, every
    residual token its two fp16 rows (its K codes under online K), for the base scheme, online K and
    fine-grained groups."""
    sys.path.insert(0, ROOT)
    import bench
    from bit_asymmetric_kv_02_b200 import kivi, synth
    kivi.load_library()
    w = synth.LARGE_BATCH.with_(batch=2, kv_heads=3, q_heads=3)
    bh, C, R, d = 6, 4096, w.residual, w.head_dim
    qo = bh * 2 * w.gqa * d * 2
    saved = bench.ONLINE_K, bench.FINE
    try:
        for online, fine in ((False, False), (True, False), (False, True)):
            bench.ONLINE_K, bench.FINE = online, fine
            cfg = kivi.kivi_config(w.batch, w.kv_heads, d, w.bits, w.group, w.gv, R, C, int(online), int(fine))
            sz = kivi.kivi_cache_sizes(cfg)
            per_quant = sum(sz[:6]) / (bh * C)              # codes + scales + zeros per quantized token
            per_res = (sz[6] + sz[7]) / (bh * R)             # fp16 K and V rows per residual token
            assert bench.decode_alg_bytes(w, C, 0) == round(bh * C * per_quant) + qo
            n_res = 37
            want_res = bh * n_res * per_res
            if online:                                        # K rows as codes, plus the block's pair row
                want_res = bh * (n_res * (d * w.bits // 8 + 2 * d) + (d // w.group) * 4)
            got = bench.decode_alg_bytes(w, C, n_res) - bench.decode_alg_bytes(w, C, 0)
            assert got == round(want_res), (online, fine, got, want_res)
    finally:
        bench.ONLINE_K, bench.FINE = saved


@pytest.mark.parametrize("mode", ["step", "fused"])
def test_parity_replay_follows_the_bench_cycle(mode):
    """bench.oracle_parity replays prefill, flushes (with the n_quant cycle of the mode) and appends
    of a step schedule; it accepts the oracle's own output for that schedule and rejects a
    perturbed one.  The decode step ("step") flushes the residual into the block after
    n_quant0 + R and drops that block; the lazy mode moves n_quant back to n_quant0 and rewrites
    the cycle's block."""
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    import oracle.kivi_oracle as O
    from bit_asymmetric_kv_02_b200 import synth
    saved = bench.MODE
    bench.MODE = mode
    try:
        w = synth.TINY.with_(batch=2, q_heads=4, kv_heads=2, tokens=300)
        n_quant0, cap = bench.first_prompt_split(w)
        assert cap == n_quant0 + (2 if mode == "step" else 1) * 128
        sched = [(i % 128) + 1 for i in range(3 * 128 + 5)]
        out = np.zeros((w.batch, w.q_heads, w.head_dim), np.float16)

        def keep(hc, n):     # the bench's cycle, written out here
            hc.k_codes, hc.v_codes = hc.k_codes[:n], hc.v_codes[:n]
            hc.k_s, hc.k_z = hc.k_s[:n // 128], hc.k_z[:n // 128]
            hc.v_s, hc.v_z = hc.v_s[:n // 32], hc.v_z[:n // 32]

        for b in range(w.batch):
            for h in range(w.kv_heads):
                hc = O.HeadCache(128, 2, 32, 32, 128, cap)
                hc.prefill(synth.prompt_k(w, b, h, w.tokens), synth.prompt_v(w, b, h, w.tokens))
                for sid in sched:
                    if hc.n_res == 128:
                        if mode == "step":
                            hc.flush()
                            if hc.n_quant == n_quant0 + 256:
                                keep(hc, n_quant0 + 128)
                        else:
                            if hc.n_quant == n_quant0 + 128:
                                keep(hc, n_quant0)
                            hc.flush()
                    hc.append(synth.new_k(w, b, h, sid), synth.new_v(w, b, h, sid))
                    assert hc.n_quant in (n_quant0, n_quant0 + 128)
                q = np.stack([synth.query(w, b, 2 * h + g, sched[-1]) for g in range(2)])
                out[b, 2 * h:2 * h + 2] = hc.attend(q, 1 / np.sqrt(128)).astype(np.float16)
        state = {"out": out, "schedule": sched, "n_quant0": n_quant0}
        rep = bench.oracle_parity(w, state, n_heads=4)
        assert rep["ok"] and rep["heads"] == 4 and rep["steps_replayed"] == len(sched), rep
        bad = dict(state, out=out + np.float16(0.01))
        assert not bench.oracle_parity(w, bad, n_heads=4)["ok"]
    finally:
        bench.MODE = saved

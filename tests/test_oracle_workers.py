"""The oracle worker plumbing of the full-size GPU tests (tests/oracle_workers.py), on the CPU:
a spawned worker's checkpoints equal a HeadCache driven step by step in this process."""
import numpy as np

import oracle.kivi_oracle as O
import oracle_workers as ow
from bit_asymmetric_kv_02_b200 import synth


def test_worker_checkpoints_match_a_direct_run():
    w = synth.TINY.with_(name="ow", batch=2, q_heads=4, kv_heads=2, tokens=300, seed=91)
    cap = 1024
    specs = [ow.HeadStream(w, b, h, cap, w.tokens, steps=140, attend_at=frozenset({0, 1, 85, 140}),
                           digest_at=frozenset({0, 85, 140})) for b in range(2) for h in range(2)]
    runs = ow.run_heads(specs, workers=2)
    for (b, h), run in runs.items():
        hc = O.HeadCache(128, 2, 32, 32, 128, cap)
        hc.prefill(synth.prompt_k(w, b, h, w.tokens), synth.prompt_v(w, b, h, w.tokens))
        labels = [lab for lab, _, _ in run]
        assert labels.count("step 0") == 2 and "flush before step 85" in labels
        entries = {(lab, kind): p for lab, kind, p in run}
        want0 = {k: ow.digest(v) for k, v in hc.packed().items()}
        assert entries[("step 0", "buffers")] == want0
        for s in range(1, 141):
            if hc.n_res == 128:
                hc.flush()
                assert entries[(f"flush before step {s}", "buffers")] == {k: ow.digest(v) for k, v in hc.packed().items()}
            hc.append(synth.new_k(w, b, h, s), synth.new_v(w, b, h, s))
            if s in (1, 85, 140):
                q = np.stack([synth.query(w, b, 2 * h + g, s) for g in range(2)])
                assert np.array_equal(entries[(f"step {s}", "out")], hc.attend(q, 1 / np.sqrt(128)))


def test_bench_cycle_truncates_like_the_gpu_counters():
    w = synth.TINY.with_(name="cyc", batch=1, q_heads=1, kv_heads=1, tokens=256, seed=92)
    spec = ow.HeadStream(w, 0, 0, 384, 256, steps=260, inputs=tuple((i % 128) + 1 for i in range(260)),
                         digest_at=frozenset({260}), cycle_nquant=128)
    run = ow.run_head(spec)
    final = [p for lab, kind, p in run if lab == "step 260"][0]
    # n_quant cycles between 128 and 256: the final state holds 256 quantized tokens and 4 residual
    assert final["k_codes"][0] == (256, 8) and final["k_res"][0] == (4, 128)

"""bench.py on CPU: it compiles, and its reference arm (the oracle timed on host cores) prints one
valid JSON line with the contract's keys."""
import json
import os
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

"""The debug build (nvcc -DKIVI_DEBUG, libkivi_debug.so) on the GPU.

Its kernels check the index ranges of their global-memory accesses and report KIVI_ERR_INTERNAL
instead of making an access that fails a check.  In a child process that loads the debug library:
prefill, appends, flushes and decode attention, with every other step a decode step whose flush runs
in its launch (2 and 4 bits, one and four queries per KV head), leave every check quiet and match the
oracle; then test hook 3 makes the decode see one quantized
unit more than the cache holds (inside the capacity, so the unguarded copy would stay in bounds
too), and the kernel's check refuses it and reports KIVI_ERR_INTERNAL through the status word and
kivi_debug_status, after which normal calls give the earlier results again.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys, numpy as np, torch
sys.path.insert(0, ROOT); sys.path.insert(0, TESTS)
from bit_asymmetric_kv_02_b200 import build, kivi, synth
build.build(debug=True)
lib = kivi.load_library()
assert lib._name.endswith("libkivi_debug.so"), lib._name
import gpu_common as gc
import oracle.kivi_oracle as O
torch.cuda.set_device(0)
for bits, gqa in ((2, 1), (4, 1), (2, 4)):
    w = synth.TINY.with_(name="dbg", batch=2, q_heads=2 * gqa, kv_heads=2, tokens=600, bits=bits, seed=81 + bits + gqa)
    cap = 1024
    k, v = synth.prompt_kv(w, w.tokens)
    c = kivi.KiviCache(2, 2, cap, bits=bits, num_q_heads=2 * gqa)
    c.status.zero_()
    c.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    ref = {}
    for b in range(2):
        for h in range(2):
            hc = O.HeadCache(128, bits, 32, 32, 128, cap)
            hc.prefill(k[b, h], v[b, h])
            ref[(b, h)] = hc
    for s in range(1, 140):
        if c.n_res == 128:
            c.flush()
            for hc in ref.values():
                hc.flush()
        kn, vn = synth.new_kv(w, s)
        q = synth.queries(w, s)
        call = c.step if s % 2 == 0 else c.append_attend   # step 40 fills the residual: flushed in the launch
        out = call(*(torch.from_numpy(x).cuda() for x in (kn, vn, q))).cpu().numpy()
        for (b, h), hc in ref.items():
            hc.append(kn[b, h], vn[b, h])
        if s in (1, 40, 41, 139):
            for (b, h), hc in ref.items():
                gc.assert_attention_close(out[b, h * gqa:(h + 1) * gqa], hc.attend(q[b, h * gqa:(h + 1) * gqa], gc.default_scale()), f"debug build {bits}-bit gqa {gqa} step {s}")
        if s % 2 == 0 and c.n_res == 0:
            for hc in ref.values():
                hc.flush()
    assert c.read_status() == 0
    assert kivi.kivi_debug_status() == 0, "a check fired on valid calls"
    q = torch.from_numpy(synth.queries(w, 0)).cuda()
    good = c.attend(q).clone()
    assert c.n_quant + 128 <= cap
    kivi.kivi_debug_inject(3, 1)
    try:
        c.status.zero_()
        c.attend(q)
        st = c.read_status()
        assert st == 11, st
        assert kivi.kivi_debug_status() == 11
    finally:
        kivi.kivi_debug_inject(0, 0)
    c.workspace.zero_()
    c.status.zero_()
    again = c.attend(q)
    assert c.read_status() == 0 and kivi.kivi_debug_status() == 0
    assert torch.equal(again, good)
print("DEBUG BUILD OK")
'''


def test_debug_build_checks_on_the_gpu():
    env = dict(os.environ, KIVI_LIB="debug")
    code = CHILD.replace("ROOT", repr(ROOT)).replace("TESTS", repr(os.path.join(ROOT, "tests")))
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert out.returncode == 0 and "DEBUG BUILD OK" in out.stdout, out.stdout[-2000:] + out.stderr[-4000:]

"""kivi_decode_attention_noalloc, the decode entry point that allocates nothing.

It serves callers that cannot allocate device memory when they decode (for example a serving
process whose memory pool already holds all free device memory, or a host that passes the library
only the buffers of each call).  Its scratch is a fixed array inside the library instead of a
caller workspace.  These tests call it through the C ABI and compare it with
kivi_decode_attention, which takes a caller-allocated workspace, on two calls in a row.  The file
is named to be collected last; it needs nothing from the other tests.
"""
import math

import numpy as np
import pytest

import gpu_common as gc
from bit_asymmetric_kv_02_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def kivi():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_asymmetric_kv_02_b200 import build, kivi as k
    build.build()
    k.load_library()
    torch.cuda.set_device(0)
    return k


def test_noalloc_matches_workspace_entry_point_twice(kivi):
    w = synth.TINY.with_(name="noalloc", batch=4, q_heads=8, kv_heads=4, tokens=1500, seed=90)
    k, v = synth.prompt_kv(w, w.tokens)
    cache = kivi.KiviCache(w.batch, w.kv_heads, 1536, num_q_heads=w.q_heads)
    cache.prefill(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    q = torch.from_numpy(synth.queries(w)).cuda()
    ref = cache.attend(q).cpu().numpy()
    assert cache.read_status() == 0
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        cache.status.zero_()
        kivi.kivi_decode_attention_noalloc(cache.cfg, cache.c, q.data_ptr(), w.q_heads, 1.0 / math.sqrt(128),
                                           out.data_ptr(), cache.status.data_ptr(), stream)
        assert cache.read_status() == 0
        got = out.cpu().numpy()
        assert np.isfinite(got).all()
        gc.assert_attention_close(got, ref.astype(np.float64), f"call {call}")


def test_noalloc_rejects_scratch_beyond_its_limit(kivi):
    """A head count whose scratch exceeds the fixed array is refused before anything is enqueued
    (the pointers are aligned placeholders and are never dereferenced)."""
    cfg = kivi.kivi_config(8192, 1024, 128, 2, 32, 32, 128, 128)   # 8.4 M heads: tickets alone 33.5 MB
    fake = 1 << 20
    cache = kivi.kivi_cache(*([fake] * 8), 0, 1)
    assert kivi.kivi_decode_workspace_bytes(cfg, 1024) > 16 << 20
    with pytest.raises(kivi.KiviError) as e:
        kivi.kivi_decode_attention_noalloc(cfg, cache, fake, 1024, 0.1, fake, None,
                                           torch.cuda.current_stream().cuda_stream)
    assert e.value.code == "WORKSPACE"

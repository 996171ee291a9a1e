"""The method's edge cases on the GPU, against the oracle (constructed inputs, not synth).

Every quantization group of the prompts below is built by tests/edge_inputs.py to hold one edge
case of the KIVI page's section 量子化アルゴリズム (Q equation, s/z equation): values exactly on the
ties z + (k + 1/2) s and one fp16 step beside them, ties within 2^-12 of a half-integer in r (where
the kernel re-decides in fp64), constant groups (s = 0), a range that rounds s to 0, -0 as the
minimum, subnormal scales, and the extremes +-65504.  Codes, scales, zero points and residual rows
must equal the oracle's bit for bit after the prefill, after every flush and at the end, through
each quantizer: the block prefill (register tiles for R <= 512, two passes for R = 1024), the
flush, the fused append + decode call, online K (rows coded at append, clamped to the newest
block's range), the prefix-K prefill and the fine-grained groups.

Attention (section 残差バッファ, Attention equation) is compared at max-abs 2e-3 / max-rel 1e-2 on
caches whose values stay within |x| <= 8 (an fp16 output above 8 is rounded by more than 2e-3 by
itself), with the query as drawn, q = 0 (the output is the mean of the dequantized values), q x 50
(a one-hot softmax: most units fall below 2^-64 of the running maximum) and non-default scales
(0, negative, large), over caches that are all residual, all quantized but one token, and mixed.
"""
import zlib

import numpy as np
import pytest

import edge_inputs as E
import gpu_common as gc
import oracle.kivi_oracle as O

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

D = 128


def _kivi():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_asymmetric_kv_02_b200 import build, kivi
    build.build()
    kivi.load_library()
    torch.cuda.set_device(0)
    return kivi


def _group_maps(scheme, T, R, gk, gv, n_prefix):
    if scheme in ("base", "online", "fused"):
        return E.k_block_groups(T, D, R, gk), E.v_token_groups(T, D, gv)
    if scheme == "fine":
        return E.k_fine_groups(T, D, gk), E.v_fine_groups(T, D, gv)
    if scheme == "prefix":
        return E.k_prefix_groups(T, D, n_prefix, R, gk), E.v_token_groups(T, D, gv)
    raise ValueError(scheme)


def _rows_like(cache, b, h, want):
    """The GPU head's buffers cut to the rows the oracle's packed buffer has (any layout)."""
    got = {}
    for key, ref in want.items():
        rows = np.asarray(ref).shape[0]
        x = cache.view(key)[b, h, :rows].cpu().numpy()
        got[key] = x.view(np.uint32) if key in ("k_codes", "v_codes") else x
    return got


def _check_buffers(cache, ref, what):
    for (b, h), hc in ref.items():
        want = hc.packed()
        gc.assert_head_bitexact(_rows_like(cache, b, h, want), want, f"{what} head {(b, h)}")
    hc0 = next(iter(ref.values()))
    assert (cache.n_quant, cache.n_res) == (hc0.n_quant, hc0.n_res), what


def _queries(batch, hq, seed, mode):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((batch, hq, D)).astype(np.float32)
    if mode == "zero":
        q[:] = 0.0
    elif mode == "x50":
        q *= 50.0
    return q.astype(np.float16)


SCALES = {"default": 1.0 / np.sqrt(D), "zero": 0.0, "negative": -0.3, "large": 2.0}


def _check_attention(cache, ref, gqa, batch, seed, what, modes=(("drawn", "default"), ("zero", "default"),
                                                                  ("x50", "default"), ("drawn", "zero"),
                                                                  ("drawn", "negative"), ("drawn", "large"))):
    kv_heads = cache.cfg.num_kv_heads
    for i, (qmode, smode) in enumerate(modes):
        q = _queries(batch, kv_heads * gqa, seed + 17 * i, qmode)
        scale = SCALES[smode]
        cache.status.zero_()
        out = cache.attend(torch.from_numpy(q).cuda(), scale=scale).cpu().numpy()
        assert cache.read_status() == 0, f"{what} {qmode}/{smode}: device status"
        for (b, h), hc in ref.items():
            want = hc.attend(q[b, h * gqa:(h + 1) * gqa], scale)
            if qmode == "zero" or smode == "zero":   # uniform weights: the mean of every value row
                assert np.allclose(want, hc.values().mean(axis=0)[None, :], rtol=1e-12, atol=1e-12)
            gc.assert_attention_close(out[b, h * gqa:(h + 1) * gqa], want, f"{what} {qmode}/{smode} head {(b, h)}")


# name, batch, kv_heads, gqa, prompt tokens, streaming steps, bits, g_k, g_v, R, scheme
CASES = [
    ("base_2bit_g32", 2, 2, 1, 4 * 128 + 37, 0, 2, 32, 32, 128, "base"),
    ("base_4bit_g32", 2, 2, 1, 4 * 128 + 37, 0, 4, 32, 32, 128, "base"),
    ("base_2bit_gk128_gv64_gqa4", 1, 2, 4, 3 * 128 + 1, 0, 2, 128, 64, 128, "base"),
    ("base_4bit_gk64_gv128_gqa2", 1, 2, 2, 3 * 128 + 100, 0, 4, 64, 128, 128, "base"),
    ("base_2bit_R256_gv256", 1, 2, 1, 2 * 256 + 50, 0, 2, 64, 256, 256, "base"),
    ("base_4bit_R512", 1, 1, 1, 2 * 512 + 3, 0, 4, 32, 64, 512, "base"),
    ("base_2bit_R1024", 1, 1, 1, 2 * 1024 + 9, 0, 2, 32, 32, 1024, "base"),
    ("base_4bit_R1024", 1, 1, 2, 2 * 1024 + 9, 0, 4, 128, 128, 1024, "base"),
    ("all_residual_2bit", 1, 2, 1, 77, 0, 2, 32, 32, 128, "base"),
    ("one_residual_token_4bit", 1, 2, 1, 3 * 128 + 1, 0, 4, 32, 32, 128, "base"),
    ("fused_2bit_flushes", 1, 2, 1, 200, 2 * 128 + 5, 2, 32, 32, 128, "fused"),
    ("fused_4bit_gqa2_flushes", 1, 2, 2, 130, 128 + 9, 4, 64, 32, 128, "fused"),
    ("online_2bit", 1, 2, 1, 2 * 128 + 20, 128 + 4, 2, 32, 32, 128, "online"),
    ("online_4bit_gqa2", 1, 2, 2, 128 + 100, 64, 4, 64, 64, 128, "online"),
    ("prefix_2bit", 1, 2, 1, 4 * 128 + 9, 128, 2, 32, 32, 128, "prefix"),
    ("prefix_4bit_R1024", 1, 1, 1, 2 * 1024 + 5, 0, 4, 64, 64, 1024, "prefix"),
    ("fine_2bit_g32", 1, 2, 1, 3 * 128 + 20, 128, 2, 32, 32, 128, "fine"),
    ("fine_4bit_gk64_gv128", 1, 2, 1, 3 * 128 + 20, 128, 4, 64, 128, 128, "fine"),
    ("fine_2bit_R1024_gv64", 1, 1, 1, 1024 + 30, 0, 2, 32, 64, 1024, "fine"),
]


def _fine_attention_supported(bits, gqa):
    return True


@pytest.mark.parametrize("family", ["full_range", "moderate"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_edge_groups_match_oracle(case, family):
    kivi = _kivi()
    name, B, H, gqa, T0, steps, bits, gk, gv, R, scheme = case
    seed = zlib.crc32(f"{name}/{family}".encode()) % 100_000
    Ttot = T0 + steps
    cap = (Ttot // R + 2) * R
    n_prefix = T0 - ((T0 - 1) % R + 1)
    k_gid, v_gid = _group_maps(scheme, Ttot, R, gk, gv, n_prefix)
    if family == "full_range":
        k, v = E.edge_prompt(B, H, Ttot, bits, k_gid, v_gid, seed, kinds=E.KINDS)
    else:
        k, v = E.edge_prompt(B, H, Ttot, bits, k_gid, v_gid, seed, kinds=E.MODERATE_KINDS)
    with_attention = family == "moderate" and (scheme != "fine" or _fine_attention_supported(bits, gqa))
    cache = kivi.KiviCache(B, H, cap, bits=bits, group_k=gk, group_v=gv, residual=R, num_q_heads=H * gqa,
                           online_k=scheme == "online", fine_groups=scheme == "fine")
    cache.status.zero_()
    kp = torch.from_numpy(np.ascontiguousarray(k[:, :, :T0])).cuda()
    vp = torch.from_numpy(np.ascontiguousarray(v[:, :, :T0])).cuda()
    heads = [(b, h) for b in range(B) for h in range(H)]
    ref = {bh: O.HeadCache(D, bits, gk, gv, R, cap, online_k=scheme == "online", fine_groups=scheme == "fine")
           for bh in heads}
    if scheme == "prefix":
        cache.prefill_prefix_k(kp, vp)
        for (b, h), hc in ref.items():
            hc.prefill_prefix_k(k[b, h, :T0], v[b, h, :T0])
    else:
        cache.prefill(kp, vp)
        for (b, h), hc in ref.items():
            hc.prefill(k[b, h, :T0], v[b, h, :T0])
    _check_buffers(cache, ref, f"{name}/{family} prefill")
    if with_attention:
        _check_attention(cache, ref, gqa, B, seed, f"{name}/{family} after prefill")
    for s in range(T0, Ttot):
        if cache.n_res == R:
            cache.flush()
            for hc in ref.values():
                hc.flush()
            _check_buffers(cache, ref, f"{name}/{family} flush before token {s}")
        kn = torch.from_numpy(np.ascontiguousarray(k[:, :, s])).cuda()
        vn = torch.from_numpy(np.ascontiguousarray(v[:, :, s])).cuda()
        for (b, h), hc in ref.items():
            hc.append(k[b, h, s], v[b, h, s])
        if scheme == "fused" or (scheme == "online" and s % 2):
            q = _queries(B, H * gqa, seed + s, "drawn")
            out = cache.append_attend(kn, vn, torch.from_numpy(q).cuda()).cpu().numpy()
            if (s - T0) % 29 in (0, 1) or cache.n_res in (1, R):
                _check_buffers(cache, ref, f"{name}/{family} after token {s}")
                if with_attention:
                    for (b, h), hc in ref.items():
                        gc.assert_attention_close(out[b, h * gqa:(h + 1) * gqa],
                                                  hc.attend(q[b, h * gqa:(h + 1) * gqa], gc.default_scale()),
                                                  f"{name}/{family} fused token {s} head {(b, h)}")
        else:
            cache.append(kn, vn)
    _check_buffers(cache, ref, f"{name}/{family} end")
    if with_attention and steps:
        _check_attention(cache, ref, gqa, B, seed + 1, f"{name}/{family} end",
                         modes=(("drawn", "default"), ("x50", "default"), ("zero", "default")))
    assert cache.read_status() == 0


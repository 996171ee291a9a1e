"""Why the decode kernel carries 24-bit fixed-point operands (reading R8), on the CPU.

A model of the kernel's arithmetic, written in numpy from the description of its method, runs on
caches the oracle quantized:
  - q_c * s_g(c) is rounded to a signed integer with `bits` bits relative to the block's largest
    |q * s|;
  - p_t * s_g(t) is rounded to an unsigned integer relative to the bound 2^(mu - m) * s_max of each
    unit (reading R16);
  - the code dot products are exact integers, and everything else is float64.
The model is compared with the oracle's fp64 attention on the same codes.  With 24 bits (three int8
limbs) the error stays a small fraction of the tolerance (max abs 2e-3, max rel 1e-2 with a 1e-2
floor).  With 16 bits (two limbs) it does not, which is why the kernel pays for the third limb.
"""
import numpy as np
import pytest

import oracle.kivi_oracle as O
from bit_asymmetric_kv_02_b200 import synth


def model_attention(hc, q, scale, qbits, pbits, UT=128, RES=16):
    """Decode attention with the kernel's fixed-point roundings, block by block and unit by unit."""
    R, gk, gv = hc.R, hc.gk, hc.gv
    nq = hc.n_quant
    kc = hc.k_codes.astype(np.float64)
    vc = hc.v_codes.astype(np.float64)
    qs2 = np.asarray(q, np.float64) * scale / np.log(2.0)      # base-2 logits
    m, l, Z, o = -np.inf, 0.0, 0.0, np.zeros(q.shape[-1])
    qmax, pmax = 2.0 ** (qbits - 1) - 64, 2.0 ** pbits - 128
    for blk in range(nq // R):
        s_k = np.repeat(hc.k_s[blk].astype(np.float64), gk)
        z_k = np.repeat(hc.k_z[blk].astype(np.float64), gk)
        qs = qs2 * s_k
        mabs = np.abs(qs).max()
        Q = np.rint(qs * (qmax / mabs)) if mabs > 0 else np.zeros_like(qs)
        cblk = float((qs2 * z_k).sum())
        for u0 in range(blk * R, (blk + 1) * R, UT):
            sl = slice(u0, u0 + UT)
            lg = (kc[sl] @ Q) * (mabs / qmax if mabs > 0 else 0.0) + cblk
            mu = lg.max()
            mn = max(m, mu)
            alpha = 2.0 ** (m - mn)
            p = 2.0 ** (lg - mn)
            sv = np.repeat(hc.v_s[u0 // gv:(u0 + UT) // gv].astype(np.float64), gv)[:UT]
            zv = np.repeat(hc.v_z[u0 // gv:(u0 + UT) // gv].astype(np.float64), gv)[:UT]
            bound = 2.0 ** (mu - mn) * sv.max()
            P = np.rint(p * sv * (pmax / bound)) if bound > 0 else np.zeros_like(p)
            o = o * alpha + (P @ vc[sl]) * (bound / pmax)
            Z = Z * alpha + float((p * zv).sum())
            l = l * alpha + float(p.sum())
            m = mn
    if hc.n_res:
        lg = (hc.k_res.astype(np.float64) @ qs2)
        mn = max(m, lg.max())
        alpha = 2.0 ** (m - mn)
        p = 2.0 ** (lg - mn)
        o = o * alpha + p @ hc.v_res.astype(np.float64)
        Z *= alpha
        l = l * alpha + p.sum()
    return (o + Z) / l


def _errors(qbits, pbits, trials=6):
    w = synth.TINY.with_(name="fx", batch=1, q_heads=1, kv_heads=1, tokens=2048 + 40, seed=404)
    k, v = synth.prompt_kv(w, w.tokens)
    hc = O.HeadCache(128, 2, 32, 32, 128, 4096)
    hc.prefill(k[0, 0], v[0, 0])
    rng = np.random.default_rng(7)
    ea = er = 0.0
    for _ in range(trials):
        q = rng.standard_normal(128).astype(np.float16).astype(np.float64)
        want = hc.attend(q[None, :], 1.0 / np.sqrt(128))[0]
        got = model_attention(hc, q, 1.0 / np.sqrt(128), qbits, pbits)
        err = np.abs(got - want)
        ea = max(ea, float(err.max()))
        er = max(er, float((err / np.maximum(np.abs(want), 1e-2)).max()))
    return ea, er


def test_24_bit_operands_stay_well_inside_the_tolerance():
    ea, er = _errors(24, 24)
    assert ea < 2e-3 / 8 and er < 1e-2 / 8, (ea, er)


@pytest.mark.parametrize("qbits,pbits", [(16, 16), (16, 24), (24, 16)])
def test_16_bit_operands_on_either_side_break_the_tolerance(qbits, pbits):
    ea, er = _errors(qbits, pbits)
    assert ea > 2e-3 or er > 1e-2, (ea, er)

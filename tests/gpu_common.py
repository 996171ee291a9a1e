"""Helpers shared by the GPU parity tests: run the CUDA path and the oracle on the same inputs."""
from __future__ import annotations

import math

import numpy as np

ATOL = 2e-3        # max-abs bound on decode outputs, beyond the fp16 output's own rounding
RTOL = 1e-2        # max-rel bound, relative to max(|o*|, REL_FLOOR)
REL_FLOOR = 1e-2


def half_ulp16(x):
    """Half the spacing of binary16 values at |x|: the largest error of a correctly rounded fp16
    output (2^-25 in the subnormal range)."""
    ax = np.abs(np.asarray(x, np.float64))
    return np.exp2(np.floor(np.log2(np.maximum(ax, 2.0 ** -14))) - 11)


def attention_errors(got, want):
    """(max abs error beyond the fp16 rounding of the output, max rel error with floor, raw max abs
    error) of fp16 outputs vs fp64 oracle outputs.  The output is fp16, so a correctly rounded
    result is off by up to half an ulp, which exceeds the absolute bar once |o*| >= 4; the absolute
    bar applies to the error beyond that."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want)
    beyond = np.maximum(err - half_ulp16(want), 0.0)
    return float(beyond.max()), float((err / np.maximum(np.abs(want), REL_FLOOR)).max()), float(err.max())


def assert_attention_close(got, want, what=""):
    ea, er, raw = attention_errors(got, want)
    assert ea <= ATOL and er <= RTOL, (f"{what}: max abs beyond fp16 rounding {ea:.3e} (bar {ATOL}; raw {raw:.3e}), "
                                       f"max rel {er:.3e} (bar {RTOL})")
    return ea, er


def gpu_buffers_of_head(cache, b: int, h: int, n_quant: int, n_res: int):
    """Host copies of one head's filled cache in the library layout (tokens [0, n_quant))."""
    cfg = cache.cfg
    P = 32 // cfg.bits
    out = {
        "k_codes": cache.view("k_codes")[b, h, :n_quant].cpu().numpy().view(np.uint32),
        "v_codes": cache.view("v_codes")[b, h, :n_quant // P].cpu().numpy().view(np.uint32),
        "k_scale": cache.view("k_scale")[b, h, :n_quant // cfg.residual].cpu().numpy(),
        "k_zero": cache.view("k_zero")[b, h, :n_quant // cfg.residual].cpu().numpy(),
        "v_scale": cache.view("v_scale")[b, h, :n_quant // cfg.group_v].cpu().numpy(),
        "v_zero": cache.view("v_zero")[b, h, :n_quant // cfg.group_v].cpu().numpy(),
        "k_res": cache.view("k_res")[b, h, :n_res].cpu().numpy(),
        "v_res": cache.view("v_res")[b, h, :n_res].cpu().numpy(),
    }
    return out


def assert_head_bitexact(gpu: dict, ref: dict, what=""):
    for key, want in ref.items():
        got = gpu[key]
        want = np.asarray(want)
        assert got.shape == want.shape, f"{what} {key}: shape {got.shape} vs {want.shape}"
        gb = np.ascontiguousarray(got).view(np.uint8)
        wb = np.ascontiguousarray(want).view(np.uint8)
        if not np.array_equal(gb, wb):
            bad = np.argwhere(np.ascontiguousarray(got) != np.ascontiguousarray(want))
            raise AssertionError(f"{what} {key}: {len(bad)} mismatches, first at {bad[:3].tolist()}")


def default_scale(d: int = 128) -> float:
    return 1.0 / math.sqrt(d)

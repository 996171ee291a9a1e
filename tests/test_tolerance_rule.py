"""The decode tolerance as the GPU tests apply it (tests/gpu_common.py), on the CPU.

Outputs leave the library in fp16, so even a correctly rounded result differs from the fp64 oracle by
up to half an fp16 ulp: more than the absolute bar of 2e-3 once |o*| >= 4.  The absolute bar is
applied to the error beyond that rounding; the relative bar (1e-2, floor 1e-2) is applied as is."""
import numpy as np

import gpu_common as gc


def test_half_ulp_matches_the_fp16_grid():
    rng = np.random.default_rng(3)
    x = np.concatenate([np.exp2(rng.uniform(-26, 15.9, 5000)), [1.0, 1.5, 4.0, 7.99, 8.0, 65504.0, 3e-8]])
    h = gc.half_ulp16(x)
    f = x.astype(np.float16)
    ok = (np.abs(x) < 65504.0) & (f.astype(np.float64) == x)      # on the grid: spacing of x itself
    assert np.array_equal(h[ok], np.spacing(f[ok]).astype(np.float64) / 2)
    # every value's correctly rounded fp16 is within half_ulp16 of it
    assert np.all(np.abs(f.astype(np.float64) - x) <= h)


def test_correctly_rounded_outputs_pass_at_every_magnitude():
    rng = np.random.default_rng(4)
    want = np.sign(rng.standard_normal(20000)) * np.exp2(rng.uniform(-20, 15.5, 20000))
    got = want.astype(np.float16)
    ea, er, raw = gc.attention_errors(got, want)
    assert ea == 0.0 and er <= 2.0 ** -11
    assert raw > 2e-3            # the raw absolute error of the rounding alone is above the bar


def test_errors_beyond_the_rounding_fail():
    want = np.array([0.3, 5.0, 9.0, -12.0])
    for i in range(len(want)):
        got = want.copy()
        got[i] += gc.half_ulp16(want[i]) + 2.1e-3
        ea, er, raw = gc.attention_errors(got, want)
        assert ea > gc.ATOL or er > gc.RTOL
    small = np.array([0.02, -0.05])          # the relative bar with its floor
    ea, er, _ = gc.attention_errors(small * 1.02, small)
    assert er > gc.RTOL

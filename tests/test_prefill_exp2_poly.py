"""The FMA-pipe 2^x of the tcgen05 prefill kernel (prefill_tc.cuh, ex2_poly2), replayed on the CPU.

The kernel takes a quarter of the softmax exponentials by range reduction x = n + f
(n = round(x) through the 1.5 * 2^23 rounding constant) and a cubic for 2^f on [-1/2, 1/2],
then adds n to the exponent field.  These tests read the cubic's coefficients from the kernel
source and check the whole construction against exp2 in float64, so a wrong coefficient, sign
or shift in the source fails here without a GPU.
"""
import re
from pathlib import Path

import numpy as np
import pytest

SRC = Path(__file__).resolve().parents[1] / "paged_kv_cache_428_b200" / "csrc" / "prefill_tc.cuh"


def _coefficients():
    text = SRC.read_text()
    c = {}
    for k in range(4):
        m = re.search(rf"#define PA_EX2_C{k}\s+([0-9.eE+-]+)f", text)
        assert m, f"PA_EX2_C{k} not found in {SRC.name}"
        c[k] = np.float32(float(m.group(1)))
    return c


def ex2_poly_f32(x):
    """The kernel's steps in float32: clamp, round through 1.5 * 2^23, cubic, exponent add."""
    c = _coefficients()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    r = np.float32(12582912.0)
    t = (x + r).astype(np.float32)
    n = (t - r).astype(np.float32)
    f = (x - n).astype(np.float32)                       # exact: n is within 1/2 of x
    p = (c[3] * f + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_cubic_interpolates_exp2_at_chebyshev_nodes():
    c = _coefficients()
    nodes = 0.5 * np.cos((2 * np.arange(4) + 1) * np.pi / 8)
    vals = sum(float(c[k]) * nodes ** k for k in range(4))
    np.testing.assert_allclose(vals, 2.0 ** nodes, rtol=2e-7)


def test_relative_error_over_the_softmax_range():
    # the kernel's arguments lie in [-inf, 8]: s * scale - m with m within 8 of the tile max
    x = np.linspace(-124.9, 8.0, 2_000_001, dtype=np.float64).astype(np.float32)
    got = ex2_poly_f32(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1.1e-4, rel.max()
    # well inside the bf16 rounding P goes through next (2^-9 relative)
    assert rel.max() < 2.0 ** -9 / 16


@pytest.mark.parametrize("n", [-125, -64, -1, 0, 1, 8])
def test_integer_arguments_scale_the_exponent(n):
    got = float(ex2_poly_f32(np.float32(n)))
    assert got == pytest.approx(2.0 ** n, rel=1.1e-4)
    assert got > 0.0


def test_masked_scores_floor_at_two_to_minus_125():
    # -inf (a masked score) and anything below -125 clamp to about 2^-125: a normal float32 that
    # is negligible next to the row's maximum term (>= 1) and never NaN or negative
    got = ex2_poly_f32(np.array([-np.inf, -1e30, -300.0, -125.0], dtype=np.float32)).astype(np.float64)
    assert np.all(np.isfinite(got)) and np.all(got > 0)
    np.testing.assert_allclose(got, 2.0 ** -125, rtol=1.1e-4)


def test_rounding_constant_leaves_round_x_in_the_exponent_shift():
    # t = x + 1.5 * 2^23 holds round(x) in its low mantissa bits: t_bits << 23 == round(x) << 23
    x = np.float32([-124.6, -3.5, -2.5, -0.49, 0.0, 0.51, 7.5])
    t = (x + np.float32(12582912.0)).astype(np.float32)
    shift = (t.view(np.int32).astype(np.int64) << 23) & 0xFFFFFFFF
    n = np.rint(x).astype(np.int64)                       # round half to even, as the float add does
    assert np.array_equal(shift, (n << 23) & 0xFFFFFFFF)

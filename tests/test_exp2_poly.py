"""The FMA-pipe exp2 of the prefill kernel: its coefficients in ptx.cuh are
the ones fit_exp2_poly.py produces, and the method (round-to-nearest range
reduction, degree-3 polynomial, exponent add) meets its error bound over the
whole input range the kernel feeds it, evaluated step by step in fp32."""

import os
import re

import numpy as np

from sink_augmented_gqa_b200 import fit_exp2_poly as F

PTX = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "sink_augmented_gqa_b200", "csrc", "ptx.cuh")


def _coeffs_in_source():
    text = open(PTX).read()
    vals = {int(k): float(v) for k, v in re.findall(r"EXP2_C(\d) = ([0-9.e+-]+)f", text)}
    return np.array([vals[i] for i in range(F.DEGREE + 1)], dtype=np.float32)


def test_source_coefficients_match_the_fit():
    c_src = _coeffs_in_source()
    c_fit = F.fit()
    np.testing.assert_allclose(c_src, c_fit, rtol=2e-7, atol=0)
    assert F.max_rel_error(c_src) < 1.5e-4


def _exp2_fma_fp32(x, c):
    """The kernel's arithmetic, in fp32, one step at a time."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-120.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = F.horner_fp32(c, f)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_range_reduction_and_bound():
    c = _coeffs_in_source()
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-120, 8, 400001), rng.uniform(-40, 8, 200000),
                        np.arange(-120, 9, dtype=np.float64) + 0.5, np.arange(-120, 9)]).astype(np.float32)
    got = _exp2_fma_fp32(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.all(np.abs(got / ref - 1) < 1.5e-4)
    # exact at integers (all-equal scores give weights of exactly 1)
    ints = np.arange(-120, 9).astype(np.float32)
    assert np.array_equal(_exp2_fma_fp32(ints, c), np.exp2(ints))
    # below the clamp the result is 2^-120, a stand-in for a vanishing weight
    low = float(_exp2_fma_fp32(np.float32(-1e30), c))
    assert low == 2.0 ** -120

"""The polynomial exp2 the attention kernel runs on the FMA pipe (CPU checks).

The coefficients in csrc/sm100.cuh must be the ones moe_gqa_query_b200/exp2_fit.py
derives (degree-3 minimax fit of 2^f on [-1/2, 1/2]), and the device algorithm
(round-to-integer by the 1.5*2^23 trick, polynomial, exponent-field add),
emulated here step by step in float32, must stay within 1e-4 relative error of
2^x over the range softmax uses.
"""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_fit", os.path.join(ROOT, "moe_gqa_query_b200", "exp2_fit.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _header_coeffs():
    text = open(os.path.join(ROOT, "moe_gqa_query_b200", "csrc", "sm100.cuh")).read()
    return np.array([float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f;", text).group(1)) for i in range(4)],
                    dtype=np.float32)


def test_coefficients_match_the_fit():
    c, err = _fit_module().fit()
    assert err < 8e-5
    np.testing.assert_array_equal(_header_coeffs(), c)


def _fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def _emulate(x):
    c0, c1, c2, c3 = _header_coeffs()
    x = np.maximum(np.float32(x), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = np.float32(x + magic)
    f = np.float32(x - np.float32(t - magic))
    p = _fma32(f, c3, c2)
    p = _fma32(p, f, c1)
    p = _fma32(p, f, c0)
    bits = (np.array(p, np.float32).view(np.int32) + (np.array(t, np.float32).view(np.int32) << 23))
    return np.array(bits, np.int32).view(np.float32)


def test_emulated_device_algorithm_error_bound():
    xs = np.concatenate([np.linspace(-125, 20, 40001), np.linspace(-1, 1, 2001), [-0.5, 0.5, 0.0, 8.0, -8.0]])
    ys = np.array([_emulate(np.float32(v)) for v in xs], dtype=np.float64)
    ref = np.exp2(np.float32(xs).astype(np.float64))
    rel = np.abs(ys - ref) / ref
    assert rel.max() < 1e-4, rel.max()


def test_emulated_clamp_below_range():
    for v in (-125.0, -200.0, -np.inf):
        y = float(_emulate(np.float32(v)))
        assert 0 < y < 2.0 ** -124

"""Pins of ``oracle/linear.py`` (pre-norm RMSNorm, the fused qkv linear, the
out projection with the residual add): closed forms, invariants, brute force
and a hand-worked example."""

import json
import math
import os

import numpy as np

from oracle import linear

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_worked_example():
    with open(os.path.join(GOLDEN, "rmsnorm_linear_example.json")) as f:
        ex = json.load(f)
    x = np.array([ex["x"]])
    n = linear.rmsnorm(x, ex["gamma"], ex["eps"])
    assert np.allclose(n[0], np.array(ex["normed_over_sqrt2"]) * math.sqrt(2), rtol=1e-15, atol=0)
    y = linear.qkv_proj(x, ex["gamma"], ex["eps"], np.array(ex["w"]), np.array(ex["b"]))
    want = np.array(ex["y_over_sqrt2_plus_b"]) * math.sqrt(2) + np.array(ex["b"])
    assert np.allclose(y[0], want, rtol=1e-15, atol=1e-15)


def test_rmsnorm_closed_form_on_constant_magnitude_rows():
    rng = np.random.default_rng(1)
    d = 2880
    for c in (1e-3, 0.5, 7.0):
        s = rng.choice([-1.0, 1.0], d)
        g = rng.standard_normal(d)
        eps = 1e-5
        n = linear.rmsnorm(c * s[None], g, eps)[0]
        assert np.allclose(n, s * g * c / math.sqrt(c * c + eps), rtol=1e-14, atol=0)


def test_rmsnorm_is_scale_invariant_without_eps():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 96))
    g = rng.standard_normal(96)
    for a in (1e-8, 3.0, 1e8):
        assert np.allclose(linear.rmsnorm(a * x, g, 0.0), linear.rmsnorm(x, g, 0.0), rtol=1e-13, atol=0)


def test_projection_matches_brute_force():
    rng = np.random.default_rng(3)
    T, d, n = 3, 7, 5
    x, g = rng.standard_normal((T, d)), rng.standard_normal(d)
    w, b = rng.standard_normal((n, d)), rng.standard_normal(n)
    eps = 1e-5
    y = linear.qkv_proj(x, g, eps, w, b)
    for t in range(T):
        ms = sum(x[t, k] ** 2 for k in range(d)) / d
        r = 1.0 / math.sqrt(ms + eps)
        for j in range(n):
            acc = b[j]
            for k in range(d):
                acc += x[t, k] * r * g[k] * w[j, k]
            assert abs(y[t, j] - acc) <= 1e-12 * (1 + abs(acc))


def test_out_proj_closed_forms():
    rng = np.random.default_rng(4)
    T, d_in, d_out = 4, 6, 3
    x, b = rng.standard_normal((T, d_out)), rng.standard_normal(d_out)
    w = rng.standard_normal((d_out, d_in))
    # zero attention output: the residual plus the bias
    assert np.array_equal(linear.out_proj(np.zeros((T, d_in)), w, b, x), x + b)
    # a one-hot attention output picks a column of W
    o = np.zeros((T, d_in))
    o[:, 2] = 1.0
    assert np.allclose(linear.out_proj(o, w, b, x), x + w[:, 2] + b, rtol=0, atol=1e-15)


def test_split_widths_of_the_study_note():
    n_q, n_kv, d_h = 64, 8, 64
    width = d_h * (n_q + 2 * n_kv)
    assert width == 5120
    y = np.arange(2 * width, dtype=np.float64).reshape(2, width)
    q, k, v = linear.split_qkv(y, n_q, n_kv, d_h)
    assert q.shape == (2, 64, 64) and k.shape == (2, 8, 64) and v.shape == (2, 8, 64)
    assert q[0, 0, 0] == 0 and k[0, 0, 0] == n_q * d_h and v[0, 0, 0] == (n_q + n_kv) * d_h
    assert v[1, 7, 63] == 2 * width - 1

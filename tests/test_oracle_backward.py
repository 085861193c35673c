"""Pins of ``oracle/backward.py``: the analytic gradients against central
finite differences of the forward oracle (an independent route to the same
derivatives), and the special cases the formulas reduce to."""

import numpy as np
import pytest

from oracle import attention as oatt
from oracle import backward as obwd


def _loss(q, k, v, sinks, window, scale, d_out):
    o, _ = oatt.sink_attention(q, k, v, sinks, 0, window, scale)
    return float(np.sum(o * d_out))


def _setup(seed, B=1, T=6, n_q=4, n_kv=2, d=4):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, n_q, d))
    k = rng.standard_normal((B, T, n_kv, d))
    v = rng.standard_normal((B, T, n_kv, d))
    sinks = rng.standard_normal(n_q)
    d_out = rng.standard_normal((B, T, n_q, d))
    return q, k, v, sinks, d_out


@pytest.mark.parametrize("window", [0, 3, 1])
def test_gradients_match_finite_differences(window):
    q, k, v, sinks, d_out = _setup(7 + window, B=2)
    scale = 0.7
    dq, dk, dv, ds = obwd.attention_backward(q, k, v, sinks, window, scale, d_out)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("sinks", sinks, ds)):
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v, "sinks": sinks}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], args["sinks"], window, scale, d_out)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], args["sinks"], window, scale, d_out)
            fd = (lp - lm) / (2 * h)
            assert abs(fd - g[idx]) <= 1e-6 * (1 + abs(fd)), (name, idx, fd, g[idx])


def test_no_sink_and_dominant_sink():
    q, k, v, sinks, d_out = _setup(3)
    _, _, _, ds = obwd.attention_backward(q, k, v, None, 0, 0.5, d_out)
    assert np.all(ds == 0)
    # a sink that takes all the mass: P -> 0, so every gradient vanishes
    dq, dk, dv, ds = obwd.attention_backward(q, k, v, np.full(4, 80.0), 0, 0.5, d_out)
    for g in (dq, dk, dv, ds):
        assert np.max(np.abs(g)) < 1e-25


def test_single_key_rows_have_no_query_gradient():
    # window 1: every query sees only its own key; with no sink the softmax
    # weight is exactly 1, so dq = 0 and dv_j = dO_j summed over the group
    q, k, v, _, d_out = _setup(4)
    dq, dk, dv, _ = obwd.attention_backward(q, k, v, None, 1, 0.5, d_out)
    assert np.max(np.abs(dq)) < 1e-15 and np.max(np.abs(dk)) < 1e-15
    want = d_out.reshape(1, 6, 2, 2, 4).sum(axis=3)
    assert np.allclose(dv, want, rtol=0, atol=1e-14)

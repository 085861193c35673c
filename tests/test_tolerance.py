"""CPU pins of the bf16 output tolerance (helpers.check_bf16_output).

The bound is derived from the arithmetic the pages fix: softmax weights
rounded to bf16 before the PV product, fp32 accumulation, a bf16 output.
These tests emulate exactly that arithmetic in numpy on the Tiny
configuration and check that the bound admits it, that the correctly
rounded oracle passes with no exemption, and that plausible mistakes (a
dropped sink, a one-step diagonal shift, a bias of a tenth of the bound)
are caught.
"""

import numpy as np
import pytest
import torch

from oracle import bf16 as obf16
from oracle import rope as orope
from sink_augmented_gqa_b200 import workloads as wl

from helpers import EXEMPT_LOG, check_bf16_output, oracle_cache, oracle_step, oracle_tables, to64


def _case(layer):
    cfg = wl.CONFIGS["tiny"]
    window = cfg.layer_window(layer)
    rc, rs = oracle_tables(cfg, cfg.T)
    oc = oracle_cache(cfg.B, cfg.T, cfg.n_kv, cfg.d)
    q, k, v = wl.qkv(cfg, cfg.T)
    sinks = wl.sinks(cfg)
    ref, _ = oracle_step(oc, q, k, v, sinks, window, cfg.sm_scale, rc, rs)
    return cfg, window, rc, rs, q, k, v, sinks, ref


def _emulate(cfg, window, q, k, v, sinks, rc, rs, shift=0, drop_sink=False):
    """The kernel's arithmetic: fp32 scores of the bf16 rotated operands,
    fp32 exponentials against the running max, weights rounded to bf16 for
    PV, the row sum of the unrounded fp32 weights plus the sink, one bf16
    rounding of O / l. shift moves the diagonal (a planted mistake)."""
    qr = orope.rotate_bsh(to64(q), 0, rc, rs)
    kr = orope.rotate_bsh(to64(k), 0, rc, rs)
    vv = obf16.round_bf16(to64(v))
    T = cfg.T
    out = np.zeros_like(qr)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    ok = j <= i + shift
    if window:
        ok &= j > i - window
    for b in range(cfg.B):
        for h in range(cfg.n_q):
            g = h // cfg.q_mult
            s = (qr[b, :, h] @ kr[b, :, g].T).astype(np.float32) * np.float32(cfg.sm_scale)
            s = np.where(ok, s, np.float32(-np.inf)).astype(np.float32)
            sig = np.float32(-np.inf if drop_sink else float(sinks[h]))
            m = np.maximum(s.max(axis=1), sig)
            p = np.exp(s - m[:, None]).astype(np.float32)
            l = p.sum(axis=1, dtype=np.float32) + np.exp(np.float32(sig - m))
            pb = obf16.round_bf16(p.astype(np.float64))
            o = (pb @ vv[b, :, g]).astype(np.float32) / l[:, None]
            out[b, :, h] = obf16.round_bf16(o.astype(np.float64))
    return torch.from_numpy(out).to(torch.bfloat16)


@pytest.mark.parametrize("layer", [0, 1], ids=["band", "full"])
def test_the_pages_arithmetic_meets_the_bound(layer):
    cfg, window, rc, rs, q, k, v, sinks, ref = _case(layer)
    check_bf16_output(_emulate(cfg, window, q, k, v, sinks, rc, rs), ref, "emulated kernel arithmetic")


@pytest.mark.parametrize("layer", [0, 1], ids=["band", "full"])
def test_correct_rounding_passes_without_exemption(layer):
    *_, ref = _case(layer)
    n = len(EXEMPT_LOG)
    check_bf16_output(torch.from_numpy(obf16.round_bf16(np.asarray(ref))).to(torch.bfloat16), ref, "rounded")
    assert len(EXEMPT_LOG) == n


def test_weighted_abs_v_is_an_upper_bound_of_the_output():
    # A = sum_j alpha_j |v_j| >= |sum_j alpha_j v_j| elementwise
    *_, ref = _case(1)
    assert np.all(ref.vabs + 1e-12 >= np.abs(np.asarray(ref)))


@pytest.mark.parametrize("mistake", ["drop_sink", "diag_shift"])
def test_plausible_mistakes_are_caught(mistake):
    cfg, window, rc, rs, q, k, v, sinks, ref = _case(0)
    kw = dict(drop_sink=True) if mistake == "drop_sink" else dict(shift=1)
    bad = _emulate(cfg, window, q, k, v, sinks, rc, rs, **kw)
    with pytest.raises(AssertionError):
        check_bf16_output(bad, ref, mistake)


def test_a_small_bias_fails_the_mean_bar():
    *_, ref = _case(1)
    r = np.asarray(ref)
    biased = obf16.round_bf16(r) + 2e-3
    with pytest.raises(AssertionError):
        check_bf16_output(torch.from_numpy(biased).to(torch.bfloat16), ref, "biased")

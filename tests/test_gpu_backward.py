"""GPU parity of the attention backward pass against ``oracle/backward.py``.

The forward is the library's own prefill (offset 0, pre-rotated q and k), so
the backward sees the bf16 output and fp32 lse a training step would pass.

Tolerance, from the arithmetic: P and dS enter their products as bf16
(relative error 2^-9 each), D_i = <dO_i, o_i> is formed from the bf16 output
(error <= 2^-8 sum_d |dO_id o_id|, entering dS as P_ij dD_i), products
accumulate in fp32. With the exact |P|, |dS| and Dabs_i = sum_d |dO_id o_id|:
  dv_j: 2^-7 sum_i P_ij |dO_i|
  dk_j: 2^-7 sm_scale sum_i (|dS_ij| + P_ij Dabs_i) |q_i|
  dq_i: 2^-7 sm_scale sum_j (|dS_ij| + P_ij Dabs_i) |k_j|
  dsink_h: 2^-7 sum_i P_sink,i (|D_i| + Dabs_i)
(a factor 2-4 above the first-order bounds), plus an absolute 1e-6.
"""

import math

import numpy as np
import pytest
import torch

import sink_augmented_gqa_b200 as sa
from oracle import attention as oatt
from oracle import backward as obwd
from sink_augmented_gqa_b200 import workloads as wl

from helpers import to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
REL = 2.0 ** -7


def _magnitudes(q, k, v, sinks, window, scale, dout):
    """Per-element error scales of dq, dk, dv, dsinks (see the module doc)."""
    B, T, n_q, d = q.shape
    n_kv = k.shape[2]
    qm = n_q // n_kv
    sig = np.full(n_q, -np.inf) if sinks is None else sinks
    ok = oatt.allowed_mask(0, T, T, window)
    mq, mk, mv, ms = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros(n_q)
    for b in range(B):
        for h in range(n_q):
            g = h // qm
            K, V = k[b, :, g], v[b, :, g]
            s = np.where(ok, q[b, :, h] @ K.T * scale, -np.inf)
            m = np.maximum(s.max(axis=1), sig[h])
            e = np.exp(s - m[:, None])
            L = e.sum(axis=1) + np.exp(sig[h] - m)
            P = e / L[:, None]
            ps = np.exp(sig[h] - m) / L
            o = P @ V
            dO = dout[b, :, h]
            Dv = np.sum(dO * o, axis=1)
            Dabs = np.sum(np.abs(dO * o), axis=1)
            dS = P * (dO @ V.T - Dv[:, None])
            W = np.abs(dS) + P * Dabs[:, None]
            mq[b, :, h] = scale * (W @ np.abs(K))
            mk[b, :, g] += scale * (W.T @ np.abs(q[b, :, h]))
            mv[b, :, g] += P.T @ np.abs(dO)
            ms[h] += np.sum(ps * (np.abs(Dv) + Dabs))
    return mq, mk, mv, ms


def _check(name, got, ref, mag):
    g = got.detach().cpu().numpy().astype(np.float64)
    tol = REL * mag + 1e-6
    err = np.abs(g - ref)
    assert np.all(np.isfinite(g)), f"{name}: non-finite"
    bad = np.argwhere(~(err <= tol))
    assert bad.size == 0, (f"{name}: {len(bad)} beyond tolerance; first {bad[:4].tolist()} "
                           f"gpu={g[tuple(bad[0])]} ref={ref[tuple(bad[0])]} tol={tol[tuple(bad[0])]}")


def _run(B, T, n_q, n_kv, d, window, seed, sinks_on=True):
    cfg = wl.scaled(wl.CONFIGS["tiny"], B=B, n_q=n_q, n_kv=n_kv, d=d, sm_scale=1 / math.sqrt(d), seed=seed)
    q, k, v = wl.qkv(cfg, T)                     # taken as already rotated
    dout = wl.randn_bf16((B, T, n_q, d), seed, 123)
    sinks = wl.sinks(cfg) if sinks_on else None
    cache = sa.KVCache(B, T, n_kv, d, device=DEV)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    sd = None if sinks is None else sinks.to(DEV)
    out, lse = sa.attn_prefill(cache, qd, kd, vd, sd, window, cfg.sm_scale, rope_fused=False, return_lse=True)
    dq, dk, dv, ds = sa.attn_backward(qd, kd, vd, out, dout.to(DEV), lse, sd, window, cfg.sm_scale)
    torch.cuda.synchronize()
    args = (to64(q), to64(k), to64(v), None if sinks is None else to64(sinks), window, cfg.sm_scale, to64(dout))
    rq, rk, rv, rs = obwd.attention_backward(*args)
    mq, mk, mv, ms = _magnitudes(*args)
    _check("dq", dq, rq, mq)
    _check("dk", dk, rk, mk)
    _check("dv", dv, rv, mv)
    if sinks_on:
        _check("dsinks", ds, rs, ms)
    else:
        assert ds is None


@pytest.mark.parametrize("d", [64, 96, 128])
@pytest.mark.parametrize("window", [0, 16, 128], ids=["full", "w16", "w128"])
def test_backward_matches_oracle(cuda_device, d, window):
    # T = 200: three full 64-row tiles and a ragged one; 4 query heads per KV head
    _run(2, 200, 8, 2, d, window, seed=300 + d + window)


@pytest.mark.parametrize("shape", [(1, 1, 4, 4, 64, 0), (3, 70, 3, 3, 96, 0), (1, 130, 8, 1, 64, 1),
                                   (2, 64, 16, 2, 128, 64)], ids=["T1", "mha", "w1_mqa", "q_mult8"])
def test_backward_edge_shapes(cuda_device, shape):
    B, T, n_q, n_kv, d, window = shape
    _run(B, T, n_q, n_kv, d, window, seed=400 + T)


def test_backward_without_sinks(cuda_device):
    _run(2, 150, 8, 2, 64, 0, seed=500, sinks_on=False)


def test_backward_full_size_one_group(cuda_device):
    # The Lite training shape (B = 8, T = 4096, 8 query / 4 KV heads, d = 96),
    # full causal; every gradient of sequence 0 and KV group 0 (query heads
    # 0, 1) against the oracle.
    cfg = wl.CONFIGS["lite"]
    B, T, n_q, n_kv, d = cfg.B, cfg.T, cfg.n_q, cfg.n_kv, cfg.d
    q, k, v = wl.qkv(cfg, T, layer=1, device=DEV)
    dout = wl.randn_bf16((B, T, n_q, d), cfg.seed, 124, DEV)
    sinks = wl.sinks(cfg, 1, device=DEV)
    cache = sa.KVCache(B, T, n_kv, d, device=DEV)
    out, lse = sa.attn_prefill(cache, q, k, v, sinks, 0, cfg.sm_scale, rope_fused=False, return_lse=True)
    dq, dk, dv, ds = sa.attn_backward(q, k, v, out, dout, lse, sinks, 0, cfg.sm_scale)
    torch.cuda.synchronize()
    qm = n_q // n_kv
    sl = (slice(0, 1), slice(None), slice(0, qm))
    args = (to64(q[sl]), to64(k[0:1, :, 0:1]), to64(v[0:1, :, 0:1]), to64(sinks[:qm]), 0, cfg.sm_scale,
            to64(dout[sl]))
    rq, rk, rv, _ = obwd.attention_backward(*args)
    mq, mk, mv, _ = _magnitudes(*args)
    _check("dq", dq[sl], rq, mq)
    _check("dk", dk[0:1, :, 0:1], rk, mk)
    _check("dv", dv[0:1, :, 0:1], rv, mv)
    assert torch.isfinite(ds).all()


@pytest.mark.parametrize("shape", [(1, 2048, 16, 2, 64, 0), (1, 2048, 16, 2, 64, 128), (1, 1100, 8, 2, 128, 0),
                                   (2, 1000, 8, 4, 96, 0)],
                         ids=["d64_full", "d64_band", "d128_ragged", "d96_ragged"])
def test_backward_long_sequences_one_group(cuda_device, shape):
    # Longer sequences than the edge cases above, through each query-tile
    # width of the kernel (128 rows at d = 64, 96 at d = 96, 64 at d = 128),
    # with T not a multiple of it: every gradient of sequence 0 and KV group 0
    # against the oracle (dsinks summed over the whole batch: finite).
    B, T, n_q, n_kv, d, window = shape
    cfg = wl.scaled(wl.CONFIGS["tiny"], B=B, n_q=n_q, n_kv=n_kv, d=d, sm_scale=1 / math.sqrt(d), seed=600 + T + d)
    q, k, v = wl.qkv(cfg, T, device=DEV)
    dout = wl.randn_bf16((B, T, n_q, d), cfg.seed, 125, DEV)
    sinks = wl.sinks(cfg, device=DEV)
    cache = sa.KVCache(B, T, n_kv, d, device=DEV)
    out, lse = sa.attn_prefill(cache, q, k, v, sinks, window, cfg.sm_scale, rope_fused=False, return_lse=True)
    dq, dk, dv, ds = sa.attn_backward(q, k, v, out, dout, lse, sinks, window, cfg.sm_scale)
    torch.cuda.synchronize()
    qm = n_q // n_kv
    sl = (slice(0, 1), slice(None), slice(0, qm))
    args = (to64(q[sl]), to64(k[0:1, :, 0:1]), to64(v[0:1, :, 0:1]), to64(sinks[:qm]), window, cfg.sm_scale,
            to64(dout[sl]))
    rq, rk, rv, _ = obwd.attention_backward(*args)
    mq, mk, mv, _ = _magnitudes(*args)
    _check("dq", dq[sl], rq, mq)
    _check("dk", dk[0:1, :, 0:1], rk, mk)
    _check("dv", dv[0:1, :, 0:1], rv, mv)
    assert torch.isfinite(ds).all()


def test_backward_repeat_calls_agree(cuda_device):
    # dq is summed over key tiles by reduce-adds and dsinks over blocks by
    # atomics, both in a varying order: two calls agree to rounding there,
    # and bit for bit on dk and dv.
    B, T, n_q, n_kv, d = 2, 777, 8, 2, 96
    cfg = wl.scaled(wl.CONFIGS["tiny"], B=B, n_q=n_q, n_kv=n_kv, d=d, sm_scale=1 / math.sqrt(d), seed=700)
    q, k, v = wl.qkv(cfg, T, device=DEV)
    dout = wl.randn_bf16((B, T, n_q, d), cfg.seed, 126, DEV)
    sinks = wl.sinks(cfg, device=DEV)
    cache = sa.KVCache(B, T, n_kv, d, device=DEV)
    out, lse = sa.attn_prefill(cache, q, k, v, sinks, 0, cfg.sm_scale, rope_fused=False, return_lse=True)
    a = sa.attn_backward(q, k, v, out, dout, lse, sinks, 0, cfg.sm_scale)
    b = sa.attn_backward(q, k, v, out, dout, lse, sinks, 0, cfg.sm_scale)
    torch.cuda.synchronize()
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    for x, y in (a[0], b[0]), (a[3], b[3]):
        assert (x - y).abs().amax().item() <= 1e-5 * x.abs().amax().item()


def test_backward_argument_errors(cuda_device):
    x = torch.zeros((1, 8, 4, 64), dtype=torch.bfloat16, device=DEV)
    lse = torch.zeros((1, 4, 8), dtype=torch.float32, device=DEV)
    with pytest.raises(sa.SinkAttnError):
        sa.attn_backward(x, x[:, :, :3], x[:, :, :3], x, x, lse, None, 0, 0.125)   # 4 % 3 != 0
    with pytest.raises(sa.SinkAttnError):
        sa.attn_backward(x, x, x, x, x, lse, None, 0, 0.125,
                         workspace=torch.empty(16, dtype=torch.uint8, device=DEV))  # workspace too small

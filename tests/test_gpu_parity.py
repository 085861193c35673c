"""GPU parity: libsinkattn (through the C ABI) against the fp64 oracle.

Every input is generated once by the seeded generators and fed, bit for bit,
to both sides. Small cases compare every element; full-size cases compare
sampled rows the oracle computes one at a time.
"""

import math

import numpy as np
import pytest
import torch

import sink_augmented_gqa_b200 as sa
from oracle import attention as oatt
from oracle import bf16 as obf16
from oracle import rope as orope
from sink_augmented_gqa_b200 import workloads as wl

from helpers import (check_bf16_output, check_lse, oracle_cache, oracle_rows, oracle_step,
                      oracle_tables, stack_out, to64)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _tables(cfg, max_pos):
    y = cfg.yarn
    return sa.yarn_rope_tables(max_pos, cfg.d, y["theta"], y["scaling"], y["orig_ctx"], y["alpha"],
                               y["beta"], device=DEV)


# ---------------------------------------------------------------------------
# YaRN tables, RoPE, append / snapshot / restore
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d,max_pos", [(64, 131200), (96, 4200), (128, 3000)])
def test_yarn_tables(cuda_device, d, max_pos):
    cfg = wl.scaled(wl.CONFIGS["tiny"], d=d)
    cos, sin = _tables(cfg, max_pos)
    rc, rs = oracle_tables(cfg, max_pos)
    gc, gs = cos.cpu().numpy(), sin.cpu().numpy()
    # fp64 on both sides, rounded to fp32: equal up to one fp32 step.
    ulp = np.spacing(np.float32(1.35))
    assert np.abs(gc.astype(np.float64) - rc).max() <= 2 * ulp
    assert np.abs(gs.astype(np.float64) - rs).max() <= 2 * ulp
    assert (gc == rc).mean() > 0.999 and (gs == rs).mean() > 0.999


@pytest.mark.parametrize("d", [64, 96, 128])
def test_rope_apply_qk(cuda_device, d):
    cfg = wl.scaled(wl.CONFIGS["tiny"], d=d, B=2, T=37, n_q=6, n_kv=3)
    off = 1000
    cos, sin = _tables(cfg, off + cfg.T)
    rc, rs = oracle_tables(cfg, off + cfg.T)
    q, k, _ = wl.qkv(cfg, cfg.T, device="cpu")
    qg, kg = q.to(DEV), k.to(DEV)
    sa.rope_apply_qk(qg, kg, off, cos, sin)
    for g_, raw in ((qg, q), (kg, k)):
        ref = orope.rotate_bsh(to64(raw), off, rc, rs)
        diff = np.abs(to64(g_) - ref)
        # fp64 arithmetic with one rounding: bit-exact wherever both sides'
        # tables agree (they may differ by one fp32 step in rare entries)
        assert np.all(diff <= obf16.bf16_ulp(ref) * 1.0000001)
        assert (diff == 0).mean() > 0.9999


def test_kv_append_snapshot_restore_bit_exact(cuda_device):
    B, cap, n_kv, d = 2, 300, 4, 64
    cache = sa.KVCache(B, cap, n_kv, d, device=DEV)
    k1 = wl.randn_bf16((B, 100, n_kv, d), 9, 1).to(DEV)
    v1 = wl.randn_bf16((B, 100, n_kv, d), 9, 2).to(DEV)
    cache.append(k1, v1)
    assert cache.offset == 100
    snap = cache.snapshot()
    k2 = wl.randn_bf16((B, 50, n_kv, d), 9, 3).to(DEV)
    v2 = wl.randn_bf16((B, 50, n_kv, d), 9, 4).to(DEV)
    cache.append(k2, v2)
    torch.cuda.synchronize()
    assert torch.equal(cache.k_rows(0, 100), k1) and torch.equal(cache.v_rows(0, 100), v1)
    assert torch.equal(cache.k_rows(100, 150), k2) and torch.equal(cache.v_rows(100, 150), v2)
    assert torch.count_nonzero(cache.k_rows(150)) == 0
    snap150 = cache.snapshot()
    cache.restore(snap)
    assert cache.offset == 100
    cache.append(k2[:, :10], v2[:, :10])      # rewrites row 100..109 < 150
    with pytest.raises(sa.SinkAttnError) as e:
        cache.restore(snap150)
    assert e.value.name == "SA_ERR_STALE_SNAPSHOT"
    cache.restore(snap)
    assert cache.offset == 100
    with pytest.raises(sa.SinkAttnError) as e:
        cache.append(wl.randn_bf16((B, 201, n_kv, d), 9, 5).to(DEV), wl.randn_bf16((B, 201, n_kv, d), 9, 6).to(DEV))
    assert e.value.name == "SA_ERR_CAPACITY" and cache.offset == 100
    # strided (non-contiguous head stride) input
    big = wl.randn_bf16((B, 5, 2 * n_kv, d), 9, 7).to(DEV)
    cache.append(big[:, :, ::2], big[:, :, 1::2])
    torch.cuda.synchronize()
    assert torch.equal(cache.k_rows(100, 105), big[:, :, ::2]) and torch.equal(cache.v_rows(100, 105), big[:, :, 1::2])


# ---------------------------------------------------------------------------
# Prefill
# ---------------------------------------------------------------------------

PREFILL_CASES = [
    # name, cfg overrides, offset before the call, T
    ("tiny", dict(), 0, 64),
    ("tiny_ragged", dict(B=2), 0, 300),
    ("d96_lite_small", dict(B=2, n_q=8, n_kv=4, d=96, sm_scale=1 / math.sqrt(96), sink_std=0.5), 0, 333),
    ("d128", dict(B=1, n_q=4, n_kv=1, d=128, sm_scale=1 / math.sqrt(128)), 0, 290),
    ("gptoss_fused_small", dict(B=1, n_q=64, n_kv=8, d=64, fused_qkv=True), 0, 260),
    ("chunk_at_offset", dict(B=2, n_q=8, n_kv=2, d=64), 200, 150),
    ("chunk_unaligned_offset", dict(B=1, n_q=4, n_kv=2, d=64), 77, 300),
    ("single_row", dict(B=3, n_q=8, n_kv=2, d=64), 5, 1),
    # more work items than SMs: every persistent CTA walks several items, so
    # both Q buffers, the cumulative ring and barrier phases and the
    # alternating row-tile assignment are exercised, with ragged last pairs
    ("persistent_d64", dict(B=4, n_q=16, n_kv=4, d=64), 0, 1500),
    ("persistent_d96_offset", dict(B=4, n_q=8, n_kv=4, d=96, sm_scale=1 / math.sqrt(96), sink_std=0.5), 100, 1900),
    ("persistent_d128", dict(B=4, n_q=16, n_kv=2, d=128, sm_scale=1 / math.sqrt(128)), 0, 1100),
]


def _run_prefill_case(cfg, off, T, window, sinks_on=True, rope_fused=True, lse=True):
    cap = off + T + 8
    cos, sin = _tables(cfg, cap)
    rc, rs = oracle_tables(cfg, cap)
    sinks = wl.sinks(cfg).to(DEV) if sinks_on else None
    cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV)
    ocache = oracle_cache(cfg.B, cap, cfg.n_kv, cfg.d)
    if off:
        kp, vp = wl.prefilled_cache_rows(cfg, rows=off)
        cache.append(kp.to(DEV), vp.to(DEV))
        ocache.append(to64(kp), to64(vp))
    q, k, v = wl.qkv(cfg, T)
    qg, kg, vg = q.to(DEV), k.to(DEV), v.to(DEV)
    if cfg.fused_qkv:   # keep the fused strides on the device too
        width = cfg.d * (cfg.n_q + 2 * cfg.n_kv)
        x = torch.empty((cfg.B, T, width), dtype=torch.bfloat16, device=DEV)
        x[:, :, : cfg.n_q * cfg.d] = qg.flatten(2)
        x[:, :, cfg.n_q * cfg.d:(cfg.n_q + cfg.n_kv) * cfg.d] = kg.flatten(2)
        x[:, :, (cfg.n_q + cfg.n_kv) * cfg.d:] = vg.flatten(2)
        qg = x[:, :, : cfg.n_q * cfg.d].unflatten(2, (cfg.n_q, cfg.d))
        kg = x[:, :, cfg.n_q * cfg.d:(cfg.n_q + cfg.n_kv) * cfg.d].unflatten(2, (cfg.n_kv, cfg.d))
        vg = x[:, :, (cfg.n_q + cfg.n_kv) * cfg.d:].unflatten(2, (cfg.n_kv, cfg.d))
    out, lse_g = sa.attn_prefill(cache, qg, kg, vg, sinks, window, cfg.sm_scale, cos, sin,
                                 rope_fused=rope_fused, return_lse=True)
    torch.cuda.synchronize()
    ref, ref_lse = oracle_step(ocache, q, k, v, None if sinks is None else sinks.cpu(), window,
                               cfg.sm_scale, rc, rs, rope_fused=rope_fused)
    return out, lse_g, ref, ref_lse, cache, ocache


@pytest.mark.parametrize("name,over,off,T", PREFILL_CASES, ids=[c[0] for c in PREFILL_CASES])
@pytest.mark.parametrize("layer", [0, 1], ids=["band", "full"])
def test_prefill_matches_oracle(cuda_device, name, over, off, T, layer):
    cfg = wl.scaled(wl.CONFIGS["tiny"], **over)
    window = cfg.layer_window(layer)
    out, lse, ref, ref_lse, cache, ocache = _run_prefill_case(cfg, off, T, window)
    check_bf16_output(out, ref, f"{name}/{layer}")
    check_lse(lse, ref_lse, f"{name}/{layer}")
    # the cache now holds the oracle's rotated K (within one bf16 step) and V bit for bit
    n = off + T
    kdiff = np.abs(to64(cache.k_rows(0, n)) - ocache.K[:, :n])
    assert np.all(kdiff <= obf16.bf16_ulp(ocache.K[:, :n]) * 1.0000001)
    assert np.array_equal(to64(cache.v_rows(0, n)), ocache.V[:, :n])
    assert cache.offset == ocache.offset == n


@pytest.mark.parametrize("q_mult,off,T", [(8, 0, 700), (8, 77, 300), (8, 1000, 33), (8, 0, 1), (4, 13, 500),
                                         (4, 200, 129), (1, 5, 260)],
                         ids=["qm8", "qm8_unaligned", "qm8_short", "qm8_one_row", "qm4", "qm4_offset", "mha_w2"])
def test_band_packed_heads_matches_oracle(cuda_device, q_mult, off, T):
    # Band layers of d = 64 whose key window fits the packed-head kernel (the
    # query heads of a KV group share the MMA rows): W = 128 with q_mult 8
    # (16 positions per unit), W = 96 with q_mult 4 (32), W = 2 with q_mult 1
    # (128). Unaligned offsets, ragged last units, a single row, a prefix
    # shorter than the window.
    window = {8: 128, 4: 96, 1: 2}[q_mult]
    cfg = wl.scaled(wl.CONFIGS["tiny"], B=2, n_q=2 * q_mult, n_kv=2, d=64)
    out, lse, ref, ref_lse, cache, ocache = _run_prefill_case(cfg, off, T, window)
    check_bf16_output(out, ref, f"band q_mult={q_mult} off={off} T={T}")
    check_lse(lse, ref_lse, f"band q_mult={q_mult} off={off} T={T}")
    n = off + T
    assert np.array_equal(to64(cache.v_rows(0, n)), ocache.V[:, :n])


@pytest.mark.parametrize("window", [0, 16, 1000])
def test_prefill_no_sink_and_prerotated(cuda_device, window):
    cfg = wl.scaled(wl.CONFIGS["tiny"], B=2, n_q=8, n_kv=4)
    out, lse, ref, ref_lse, _, _ = _run_prefill_case(cfg, 40, 200, window, sinks_on=False, rope_fused=False)
    check_bf16_output(out, ref, "no-sink/pre-rotated")
    check_lse(lse, ref_lse, "no-sink/pre-rotated")


def test_prefill_empty_is_noop(cuda_device):
    cfg = wl.CONFIGS["tiny"]
    cache = sa.KVCache(1, 16, cfg.n_kv, cfg.d, device=DEV)
    q = torch.empty((1, 0, cfg.n_q, cfg.d), dtype=torch.bfloat16, device=DEV)
    k = torch.empty((1, 0, cfg.n_kv, cfg.d), dtype=torch.bfloat16, device=DEV)
    out = sa.attn_prefill(cache, q, k, k, None, 0, 0.125, rope_fused=False)
    assert out.shape[1] == 0 and cache.offset == 0


def test_prefill_argument_errors(cuda_device):
    cfg = wl.CONFIGS["tiny"]
    cos, sin = _tables(cfg, 64)
    cache = sa.KVCache(1, 64, cfg.n_kv, cfg.d, device=DEV)
    q, k, v = (t.to(DEV) for t in wl.qkv(cfg, 8))
    sa.attn_prefill(cache, q, k, v, None, 0, 0.125, cos, sin)
    bad = sa.KVCache(1, 64, cfg.n_kv, cfg.d, device=DEV)
    bad.raw.offset = 3     # offset that differs from what the call expects is caught
    a_cache = sa.KVCache(1, 10, cfg.n_kv, cfg.d, device=DEV)
    with pytest.raises(sa.SinkAttnError) as e:
        sa.attn_prefill(a_cache, *(t.to(DEV) for t in wl.qkv(cfg, 11)), None, 0, 0.125, cos, sin)
    assert e.value.name == "SA_ERR_CAPACITY" and a_cache.offset == 0
    q5 = torch.zeros((1, 8, 5, cfg.d), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(sa.SinkAttnError) as e:
        sa.attn_prefill(sa.KVCache(1, 64, cfg.n_kv, cfg.d, device=DEV), q5, k, v, None, 0, 0.125, cos, sin)
    assert e.value.name == "SA_ERR_SHAPE"
    with pytest.raises(sa.SinkAttnError) as e:
        sa.attn_prefill(sa.KVCache(1, 200, cfg.n_kv, cfg.d, device=DEV), *(t.to(DEV) for t in wl.qkv(cfg, 100)),
                        None, 0, 0.125, cos, sin)
    assert e.value.name == "SA_ERR_CAPACITY"   # positions beyond the rope tables


# ---------------------------------------------------------------------------
# Decode and the prefill -> decode handoff
# ---------------------------------------------------------------------------

def _decode_steps(cfg, cache, ocache, n_steps, window, cos, sin, rc, rs, sinks, first_step=0):
    ws = sa.decode_workspace(cfg.B, cfg.n_q, cfg.n_kv, cfg.d, device=DEV)
    for st in range(n_steps):
        q, k, v = wl.qkv(cfg, 1, step=first_step + st + 1)
        out, lse = sa.attn_decode(cache, q.to(DEV), k.to(DEV), v.to(DEV), sinks, window, cfg.sm_scale,
                                  cos, sin, workspace=ws, return_lse=True)
        torch.cuda.synchronize()
        ref, ref_lse = oracle_step(ocache, q, k, v, None if sinks is None else sinks.cpu(), window,
                                   cfg.sm_scale, rc, rs)
        check_bf16_output(out, ref, f"decode step {st}")
        check_lse(lse, ref_lse, f"decode step {st}")
    n_cnt = cfg.B * cfg.n_kv   # the tickets and stage counters lead the workspace, zero after each call
    assert torch.count_nonzero(ws[: 8 * n_cnt]) == 0
    return cache


@pytest.mark.parametrize("layer", [0, 1], ids=["band", "full"])
def test_tiny_prefill_then_decode(cuda_device, layer):
    cfg = wl.CONFIGS["tiny"]
    window = cfg.layer_window(layer)
    cap = cfg.T + cfg.decode_steps
    cos, sin = _tables(cfg, cap)
    rc, rs = oracle_tables(cfg, cap)
    sinks = wl.sinks(cfg).to(DEV)
    cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV)
    ocache = oracle_cache(cfg.B, cap, cfg.n_kv, cfg.d)
    q, k, v = wl.qkv(cfg, cfg.T)
    out = sa.attn_prefill(cache, q.to(DEV), k.to(DEV), v.to(DEV), sinks, window, cfg.sm_scale, cos, sin)
    torch.cuda.synchronize()
    ref, _ = oracle_step(ocache, q, k, v, sinks.cpu(), window, cfg.sm_scale, rc, rs)
    check_bf16_output(out, ref, "tiny prefill")
    _decode_steps(cfg, cache, ocache, cfg.decode_steps, window, cos, sin, rc, rs, sinks)


@pytest.mark.parametrize("over", [dict(B=3, n_q=8, n_kv=2, d=64), dict(B=2, n_q=8, n_kv=4, d=96),
                                  dict(B=1, n_q=16, n_kv=2, d=128), dict(B=1, n_q=64, n_kv=8, d=64)],
                         ids=["d64", "d96", "d128", "gptoss"])
@pytest.mark.parametrize("layer", [0, 1], ids=["band", "full"])
def test_decode_multi_split(cuda_device, over, layer):
    cfg = wl.scaled(wl.CONFIGS["tiny"], **over)
    window = cfg.layer_window(layer) and 128
    off = 5000
    cap = off + 4
    cos, sin = _tables(cfg, cap)
    rc, rs = oracle_tables(cfg, cap)
    sinks = wl.sinks(cfg).to(DEV)
    kp, vp = wl.prefilled_cache_rows(cfg, rows=off)
    cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV)
    cache.append(kp.to(DEV), vp.to(DEV))
    ocache = oracle_cache(cfg.B, cap, cfg.n_kv, cfg.d, kp, vp)
    _decode_steps(cfg, cache, ocache, 3, window, cos, sin, rc, rs, sinks)


@pytest.mark.parametrize("window", [1, 2, 127, 129], ids=["w1", "w2", "w127", "w129"])
def test_prefill_and_decode_window_edges_mha(cuda_device, window):
    # q_mult = 1 (plain multi-head) with band widths around the degenerate
    # W = 1 (each row sees only itself and the sink) and the 128-key tile edge
    cfg = wl.scaled(wl.CONFIGS["tiny"], B=2, n_q=4, n_kv=4, d=64)
    out, lse, ref, ref_lse, cache, ocache = _run_prefill_case(cfg, 60, 420, window)
    check_bf16_output(out, ref, f"mha W={window}")
    check_lse(lse, ref_lse, f"mha W={window}")
    cap = cache.raw.cap
    cos, sin = _tables(cfg, cap)
    rc, rs = oracle_tables(cfg, cap)
    _decode_steps(cfg, cache, ocache, 3, window, cos, sin, rc, rs, wl.sinks(cfg).to(DEV))


@pytest.mark.parametrize("over", [dict(B=2, n_q=8, n_kv=2, d=64),
                                  dict(B=2, n_q=16, n_kv=2, d=64),
                                  dict(B=2, n_q=8, n_kv=4, d=96, sm_scale=1 / math.sqrt(96)),
                                  dict(B=1, n_q=4, n_kv=1, d=128, sm_scale=1 / math.sqrt(128))],
                         ids=["d64", "d64_packed_heads", "d96", "d128"])
def test_ring_cache_matches_oracle(cuda_device, over):
    # A band layer on a 384-row ring: prefill, decode, a second prefill chunk
    # that wraps the ring, decode again, then snapshot / restore. Every output
    # against the oracle on a plain (unbounded) cache; the ring's live rows
    # against the oracle's rows of the same positions. With q_mult 8 the
    # prefill takes the packed-head band kernel, whose key windows that wrap
    # the ring are loaded as 16-row boxes.
    cfg = wl.scaled(wl.CONFIGS["tiny"], **over)
    W, cap = 128, 384
    n_total = 200 + 3 + 250 + 6
    cos, sin = _tables(cfg, n_total + 8)
    rc, rs = oracle_tables(cfg, n_total + 8)
    sinks = wl.sinks(cfg).to(DEV)
    cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV, ring=W)
    ocache = oracle_cache(cfg.B, n_total + 8, cfg.n_kv, cfg.d)

    def prefill(T, seed):
        q, k, v = wl.qkv(cfg, T, step=seed)
        out, lse = sa.attn_prefill(cache, q.to(DEV), k.to(DEV), v.to(DEV), sinks, W, cfg.sm_scale, cos, sin,
                                   return_lse=True)
        torch.cuda.synchronize()
        ref, ref_lse = oracle_step(ocache, q, k, v, sinks.cpu(), W, cfg.sm_scale, rc, rs)
        check_bf16_output(out, ref, f"ring prefill {T}")
        check_lse(lse, ref_lse, f"ring prefill {T}")

    def live_rows_match():
        off = cache.offset
        lo = max(0, off - W + 1)
        k_ring, v_ring = to64(cache.k_rows(lo, off)), to64(cache.v_rows(lo, off))
        assert np.array_equal(v_ring, ocache.V[:, lo:off])
        assert np.all(np.abs(k_ring - ocache.K[:, lo:off]) <= obf16.bf16_ulp(ocache.K[:, lo:off]) * 1.0000001)

    prefill(200, 100)
    _decode_steps(cfg, cache, ocache, 3, W, cos, sin, rc, rs, sinks, first_step=200)
    prefill(250, 300)                       # positions 203..452: wraps rows 383 -> 0
    live_rows_match()
    snap, osnap = cache.snapshot(), ocache.snapshot()
    _decode_steps(cfg, cache, ocache, 3, W, cos, sin, rc, rs, sinks, first_step=400)
    live_rows_match()
    cache.restore(snap)                     # the band rows of the snapshot are still held
    ocache.restore(osnap)
    assert cache.offset == ocache.offset == 453
    _decode_steps(cfg, cache, ocache, 3, W, cos, sin, rc, rs, sinks, first_step=500)
    live_rows_match()


def _random_cases(n, seed=2026):
    rng = np.random.default_rng(seed)
    cases = []
    for idx in range(n):
        d = int(rng.choice([64, 96, 128]))
        n_kv = int(rng.choice([1, 2, 4]))
        q_mult = int(rng.choice([1, 2, 4, 8]))
        B = int(rng.integers(1, 4))
        T = int(rng.integers(1, 700))
        off = int(rng.choice([0, 0, int(rng.integers(1, 900))]))
        window = int(rng.choice([0, 0, 1, 7, 64, 128, 200, 1000]))
        ring = bool(window > 0 and rng.random() < 0.3)
        cases.append((idx, d, n_kv, q_mult, B, T, off, window, ring))
    return cases


@pytest.mark.parametrize("idx,d,n_kv,q_mult,B,T,off,window,ring", _random_cases(24),
                         ids=[f"r{c[0]}" for c in _random_cases(24)])
def test_random_shapes_prefill_then_decode(cuda_device, idx, d, n_kv, q_mult, B, T, off, window, ring):
    # Seeded random shapes: head dims, GQA ratios (1..8), ragged T, prefixes,
    # band widths (including 1 and wider than a tile) and ring caches; every
    # output row and lse against the oracle, then two decode steps.
    cfg = wl.scaled(wl.CONFIGS["tiny"], B=B, n_q=n_kv * q_mult, n_kv=n_kv, d=d, sm_scale=1 / math.sqrt(d),
                    seed=100 + idx)
    n_total = off + T + 2
    cos, sin = _tables(cfg, n_total + 8)
    rc, rs = oracle_tables(cfg, n_total + 8)
    sinks = wl.sinks(cfg).to(DEV)
    if ring:
        cap = ((max(T, 1) + window - 1 + 383) // 384) * 384
        cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV, ring=window)
    else:
        cache = sa.KVCache(cfg.B, n_total + 8, cfg.n_kv, cfg.d, device=DEV)
    ocache = oracle_cache(cfg.B, n_total + 8, cfg.n_kv, cfg.d)
    if off:
        kp, vp = wl.prefilled_cache_rows(cfg, rows=off)
        if ring:   # stream the prefix through the ring in chunks that fit
            done = 0
            while done < off:
                n = min(cache.raw.cap, off - done)
                cache.append(kp[:, done:done + n].to(DEV), vp[:, done:done + n].to(DEV))
                done += n
        else:
            cache.append(kp.to(DEV), vp.to(DEV))
        ocache.append(to64(kp), to64(vp))
    q, k, v = wl.qkv(cfg, T, step=7)
    out, lse = sa.attn_prefill(cache, q.to(DEV), k.to(DEV), v.to(DEV), sinks, window, cfg.sm_scale, cos, sin,
                               return_lse=True)
    torch.cuda.synchronize()
    ref, ref_lse = oracle_step(ocache, q, k, v, sinks.cpu(), window, cfg.sm_scale, rc, rs)
    check_bf16_output(out, ref, f"random case {idx}")
    check_lse(lse, ref_lse, f"random case {idx}")
    _decode_steps(cfg, cache, ocache, 2, window, cos, sin, rc, rs, sinks, first_step=50)


def test_decode_from_empty_cache_and_no_sink(cuda_device):
    cfg = wl.scaled(wl.CONFIGS["tiny"], B=2)
    cos, sin = _tables(cfg, 8)
    rc, rs = oracle_tables(cfg, 8)
    cache = sa.KVCache(cfg.B, 8, cfg.n_kv, cfg.d, device=DEV)
    ocache = oracle_cache(cfg.B, 8, cfg.n_kv, cfg.d)
    _decode_steps(cfg, cache, ocache, 4, 0, cos, sin, rc, rs, None)


@pytest.mark.parametrize("layer", [0, 1], ids=["band", "full"])
def test_handoff_prefill_equals_prefix_plus_decode(cuda_device, layer):
    # Handoff shapes at reduced batch: shared offset, chunked prefill, then
    # decode; the decode rows must match the prefill rows of the same
    # positions (the prefill -> decode diagonal), also after a restore.
    cfg = wl.scaled(wl.CONFIGS["handoff"], B=2, offset=1000, T=96, decode_steps=8)
    window = cfg.layer_window(layer)
    cap = cfg.offset + cfg.T + cfg.decode_steps
    cos, sin = _tables(cfg, cap)
    rc, rs = oracle_tables(cfg, cap)
    sinks = wl.sinks(cfg).to(DEV)
    kp, vp = wl.prefilled_cache_rows(cfg)
    full = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV)
    full.append(kp.to(DEV), vp.to(DEV))
    q, k, v = wl.qkv(cfg, cfg.T + cfg.decode_steps)
    qg, kg, vg = q.to(DEV), k.to(DEV), v.to(DEV)
    ref_all = sa.attn_prefill(full, qg, kg, vg, sinks, window, cfg.sm_scale, cos, sin)
    ocache = oracle_cache(cfg.B, cap, cfg.n_kv, cfg.d, kp, vp)
    oref, _ = oracle_step(ocache, q, k, v, sinks.cpu(), window, cfg.sm_scale, rc, rs)
    check_bf16_output(ref_all, oref, "handoff full prefill")

    cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV)
    cache.append(kp.to(DEV), vp.to(DEV))
    head = sa.attn_prefill(cache, qg[:, :cfg.T], kg[:, :cfg.T], vg[:, :cfg.T], sinks, window,
                           cfg.sm_scale, cos, sin)
    check_bf16_output(head, oref[:, :cfg.T], "handoff chunk")
    snap = cache.snapshot()
    ws = sa.decode_workspace(cfg.B, cfg.n_q, cfg.n_kv, cfg.d, device=DEV)
    for rep in range(2):
        for t in range(cfg.T, cfg.T + cfg.decode_steps):
            o = sa.attn_decode(cache, qg[:, t:t + 1], kg[:, t:t + 1], vg[:, t:t + 1], sinks, window,
                               cfg.sm_scale, cos, sin, workspace=ws)
            check_bf16_output(o, oref[:, t:t + 1], f"handoff decode {t}")
        torch.cuda.synchronize()
        assert torch.equal(cache.k, full.k) and torch.equal(cache.v, full.v)
        cache.restore(snap)
        assert cache.offset == cfg.offset + cfg.T


@pytest.mark.parametrize("layer,n_q", [(0, 2), (0, 8), (1, 2)], ids=["band", "band_packed", "full"])
@pytest.mark.parametrize("off,T", [(0, 300), (65536 - 3, 40)])
def test_mask_position_probe_bit_exact(cuda_device, layer, n_q, off, T):
    # q = 0 and sink = 0: every admitted score is 0, so weights are 1/(n+1).
    # With v_j = e_{j mod d}, round(out_c * (n+1)) counts admitted keys
    # j = c mod d (band layers); lse = ln(n+1) recovers n (full layers).
    # n_q = 8 on one KV head takes the packed-head band kernel.
    B, n_kv, d = 1, 1, 64
    window = 128 if layer == 0 else 0
    cap = off + T
    cache = sa.KVCache(B, cap, n_kv, d, device=DEV)
    if off:
        kp = wl.randn_bf16((B, off, n_kv, d), 11, 1).to(DEV)
        vp = torch.zeros((B, off, n_kv, d), dtype=torch.bfloat16, device=DEV)
        vp[0, torch.arange(off), 0, torch.arange(off) % d] = 1
        cache.append(kp, vp)
    k = wl.randn_bf16((B, T, n_kv, d), 11, 2).to(DEV)
    v = torch.zeros((B, T, n_kv, d), dtype=torch.bfloat16, device=DEV)
    v[0, torch.arange(T), 0, (off + torch.arange(T)) % d] = 1
    q = torch.zeros((B, T, n_q, d), dtype=torch.bfloat16, device=DEV)
    sinks = torch.zeros(n_q, dtype=torch.float32, device=DEV)
    out, lse = sa.attn_prefill(cache, q, k, v, sinks, window, 0.125, rope_fused=False, return_lse=True)
    torch.cuda.synchronize()
    ok = oatt.allowed_mask(off, T, off + T, window)
    n = ok.sum(axis=1)
    got_n = np.rint(np.exp(to64(lse[0, 0])) - 1).astype(np.int64)
    assert np.array_equal(got_n, n)
    if window:
        j = np.arange(off + T)
        counts = np.stack([np.bincount(j[ok[i]] % d, minlength=d) for i in range(T)])
        got = np.rint(to64(out[0, :, 0]) * (n[:, None] + 1)).astype(np.int64)
        assert np.array_equal(got, counts)


# ---------------------------------------------------------------------------
# Full-size configurations (sampled rows)
# ---------------------------------------------------------------------------

def _sampled_prefill(cfg, layer, n_rows=6, n_heads=3, seed=0):
    window = cfg.layer_window(layer)
    cap = cfg.offset + cfg.T
    cos, sin = _tables(cfg, cap)
    rc, rs = oracle_tables(cfg, cap)
    sinks = wl.sinks(cfg, device="cpu")
    cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV)
    q, k, v = wl.qkv(cfg, cfg.T, layer=layer, device=DEV)
    out = sa.attn_prefill(cache, q, k, v, sinks.to(DEV), window, cfg.sm_scale, cos, sin)
    torch.cuda.synchronize()
    rng = np.random.default_rng(seed)
    rows = sorted(set(rng.integers(0, cfg.T, n_rows).tolist()) | {0, 127, 128, 255, 256, cfg.T - 1})
    heads = sorted(set(rng.integers(0, cfg.n_q, n_heads).tolist()))
    got, want = [], []
    for b in sorted({0, cfg.B - 1}):
        res = oracle_rows(to64(q[b]), None, to64(k[b]), None, to64(v[b]), to64(sinks), 0, rows, heads, b,
                          window, cfg.sm_scale, rc, rs, cfg.q_mult)
        for (i, h), (ro, _) in res.items():
            got.append(out[b, i, h])
            want.append(ro)
    check_bf16_output(torch.stack(got), stack_out(want), f"{cfg.name} sampled rows")


@pytest.mark.parametrize("layer", [0, 1], ids=["band", "full"])
def test_full_size_lite_prefill(cuda_device, layer):
    _sampled_prefill(wl.CONFIGS["lite"], layer)


@pytest.mark.parametrize("layer", [0, 1], ids=["band", "full"])
def test_full_size_gptoss_prefill(cuda_device, layer):
    _sampled_prefill(wl.CONFIGS["gptoss_prefill"], layer)


@pytest.mark.parametrize("layer", [0, 1], ids=["band", "full"])
def test_full_size_long_decode(cuda_device, layer):
    cfg = wl.CONFIGS["long_decode"]
    window = cfg.layer_window(layer)
    cap = cfg.offset + 2
    cos, sin = _tables(cfg, cap)
    rc, rs = oracle_tables(cfg, cap)
    sinks = wl.sinks(cfg, layer=layer)
    kp, vp = wl.prefilled_cache_rows(cfg, layer=layer, device=DEV)
    cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV)
    cache.append(kp, vp)
    q, k, v = wl.qkv(cfg, 1, layer=layer, step=1, device=DEV)
    out, lse = sa.attn_decode(cache, q, k, v, sinks.to(DEV), window, cfg.sm_scale, cos, sin, return_lse=True)
    torch.cuda.synchronize()
    off = cfg.offset
    got, want = [], []
    for h in (0, 9, 63):
        g = h // cfg.q_mult
        # one head at a time: K/V of its group only
        kpre = to64(kp[0, :, g:g + 1])
        vpre = to64(vp[0, :, g:g + 1])
        r = oracle_rows(to64(q[0, :, h:h + 1]), kpre, to64(k[0, :, g:g + 1]), vpre, to64(v[0, :, g:g + 1]),
                        to64(sinks[h:h + 1]), off, [0], [0], 0, window, cfg.sm_scale, rc, rs, 1)
        ro, rl = r[(0, 0)]
        got.append(out[0, 0, h])
        want.append(ro)
        check_lse(lse[0, h, 0], np.array(rl), f"long decode h{h}")
    check_bf16_output(torch.stack(got), stack_out(want), "long decode sampled heads")
    torch.cuda.synchronize()
    assert cache.offset == off + 1


def test_full_size_handoff_sampled(cuda_device):
    cfg = wl.CONFIGS["handoff"]
    cap = cfg.offset + cfg.T + 2
    cos, sin = _tables(cfg, cap)
    rc, rs = oracle_tables(cfg, cap)
    got, want = [], []
    for layer in (0, 1):
        window = cfg.layer_window(layer)
        sinks = wl.sinks(cfg, layer=layer)
        kp, vp = wl.prefilled_cache_rows(cfg, layer=layer, device=DEV)
        cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV)
        cache.append(kp, vp)
        q, k, v = wl.qkv(cfg, cfg.T + 1, layer=layer, device=DEV)
        out = sa.attn_prefill(cache, q[:, :cfg.T], k[:, :cfg.T], v[:, :cfg.T], sinks.to(DEV), window,
                              cfg.sm_scale, cos, sin)
        dec = sa.attn_decode(cache, q[:, cfg.T:], k[:, cfg.T:], v[:, cfg.T:], sinks.to(DEV), window,
                             cfg.sm_scale, cos, sin)
        torch.cuda.synchronize()
        for b in (0, 15):
            for h in (0, 37):
                g = h // cfg.q_mult
                r = oracle_rows(to64(q[b, :, h:h + 1]), to64(kp[b, :, g:g + 1]), to64(k[b, :, g:g + 1]),
                                to64(vp[b, :, g:g + 1]), to64(v[b, :, g:g + 1]), to64(sinks[h:h + 1]),
                                cfg.offset, [0, 255, cfg.T - 1, cfg.T], [0], b, window, cfg.sm_scale,
                                rc, rs, 1)
                for i in (0, 255, cfg.T - 1):
                    got.append(out[b, i, h])
                    want.append(r[(i, 0)][0])
                got.append(dec[b, 0, h])
                want.append(r[(cfg.T, 0)][0])
        del cache, kp, vp
    check_bf16_output(torch.stack(got), stack_out(want), "handoff sampled rows")


def test_many_prefills_in_flight_on_several_streams(cuda_device):
    # More prefill calls in flight than the library has schedule counters for
    # eager launches (64): four streams, 24 calls each, issued without
    # synchronising, so counters are reused while other streams' calls may
    # still run. Every output must equal the one the same call gives alone.
    cfg = wl.scaled(wl.CONFIGS["tiny"], B=1, n_q=8, n_kv=2, d=64)
    T, n_streams, per_stream = 384, 4, 24
    cos, sin = _tables(cfg, T)
    sinks = wl.sinks(cfg).to(DEV)
    inputs = [tuple(t.to(DEV) for t in wl.qkv(cfg, T, step=i)) for i in range(n_streams)]
    ref = []
    for i in range(n_streams):
        c = sa.KVCache(cfg.B, T, cfg.n_kv, cfg.d, device=DEV)
        ref.append(sa.attn_prefill(c, *inputs[i], sinks, 0, cfg.sm_scale, cos, sin))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in range(n_streams)]
    caches = [sa.KVCache(cfg.B, T, cfg.n_kv, cfg.d, device=DEV) for _ in range(n_streams)]
    snaps = [c.snapshot() for c in caches]
    outs = [[torch.empty_like(ref[i]) for _ in range(per_stream)] for i in range(n_streams)]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    for j in range(per_stream):
        for i, s in enumerate(streams):
            with torch.cuda.stream(s):
                caches[i].restore(snaps[i])
                sa.attn_prefill(caches[i], *inputs[i], sinks, 0, cfg.sm_scale, cos, sin, out=outs[i][j])
    torch.cuda.synchronize()
    assert sa.device_status() == "SA_OK"
    for i in range(n_streams):
        for j in range(per_stream):
            assert torch.equal(outs[i][j], ref[i]), (i, j)

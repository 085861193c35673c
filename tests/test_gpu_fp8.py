"""GPU parity of the FP8 (e4m3) KV cache against the oracle.

Bit-exact: the codes and row scales an append or a decode writes (the
quantiser's decision is taken in fp32 on both sides). Outputs: the bf16
tolerance of ``helpers.check_bf16_output`` against the oracle attention over
the dequantised rows, and lse within ``helpers.check_lse``.
"""

import math

import numpy as np
import pytest
import torch

import sink_augmented_gqa_b200 as sa
from oracle import attention as oatt
from oracle import fp8 as ofp8
from oracle import kvcache as okv
from oracle import rope as orope
from oracle.bf16 import round_bf16
from sink_augmented_gqa_b200 import workloads as wl

from helpers import check_bf16_output, check_lse, oracle_tables, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _tables(cfg, max_pos):
    y = cfg.yarn
    return sa.yarn_rope_tables(max_pos, cfg.d, y["theta"], y["scaling"], y["orig_ctx"], y["alpha"], y["beta"],
                               device=DEV)


def _special_rows(shape, seed, shift=0):
    """bf16 rows [B, T, n_kv, d] of mixed magnitudes: in every group of 16
    positions (offset by ``shift``) a zero row, rows scaled by 1e30 and
    1e-30, a row with a single nonzero element, a row of negative zeros but
    one element, and a row scaled by 300; normal rows elsewhere."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    T = shape[1]
    for t in range(T):
        kind = (t + shift) % 16
        if kind == 0:
            x[:, t] = 0.0
        elif kind == 1:
            x[:, t] *= 1e30
        elif kind == 2:
            x[:, t] *= 1e-30
        elif kind == 3:
            x[:, t] = 0.0
            x[:, t, :, 5] = -3.0
        elif kind == 4:
            x[:, t] = -0.0
            x[:, t, :, 0] = 1.0
        elif kind == 5:
            x[:, t] *= 300.0
    return x.to(torch.bfloat16)


def _check_codes(cache, start, stop, k_bf16_rows, v_bf16_rows, what):
    """Codes and scales of positions [start, stop) against the oracle's
    quantisation of the bf16 rows [B, T, n_kv, d] (fp64 values)."""
    kc, ks = ofp8.quantize_rows(k_bf16_rows)
    vc, vs = ofp8.quantize_rows(v_bf16_rows)
    gk = cache.k_rows(start, stop).cpu().numpy()
    gv = cache.v_rows(start, stop).cpu().numpy()
    gks = cache.k_scales(start, stop).cpu().numpy()
    gvs = cache.v_scales(start, stop).cpu().numpy()
    assert np.array_equal(gk, kc), f"{what}: K codes differ at {np.argwhere(gk != kc)[:4].tolist()}"
    assert np.array_equal(gv, vc), f"{what}: V codes differ"
    assert np.array_equal(gks.view(np.uint32), ks.view(np.uint32)), f"{what}: K scales differ"
    assert np.array_equal(gvs.view(np.uint32), vs.view(np.uint32)), f"{what}: V scales differ"


@pytest.mark.parametrize("d", [64, 96, 128])
@pytest.mark.parametrize("ring", [0, 128], ids=["linear", "ring"])
def test_fp8_append_bit_exact(cuda_device, d, ring):
    B, n_kv, T = 2, 3, 45
    cap = 384 if ring else 96
    k = _special_rows((B, T, n_kv, d), 1)
    v = _special_rows((B, T, n_kv, d), 2, shift=5)
    cache = sa.KVCache(B, cap, n_kv, d, device=DEV, ring=ring, fp8=True)
    cache.append(k.to(DEV), v.to(DEV))
    # strided source: a bf16 cache's rows [B, n_kv, cap, d] viewed as [B, T, n_kv, d]
    src = sa.KVCache(B, 64, n_kv, d, device=DEV)
    k2, v2 = _special_rows((B, 20, n_kv, d), 3), _special_rows((B, 20, n_kv, d), 4)
    src.append(k2.to(DEV), v2.to(DEV))
    cache.append(src.k_rows(0, 20), src.v_rows(0, 20))
    torch.cuda.synchronize()
    assert cache.offset == T + 20
    _check_codes(cache, 0, T, to64(k), to64(v), "append")
    _check_codes(cache, T, T + 20, to64(k2), to64(v2), "strided append")


def _check_scaled(gpu, ref, what):
    """The bf16 bar (max 1e-2, mean 1e-3) against the exact (unrounded)
    oracle value, in units of each output row's own magnitude
    max(1, max_d |ref|): rows of values scaled by up to 1e30 make absolute
    bounds meaningless, relative ones keep their sense. (Half a bf16 step is
    at most 2^-9 of a row's magnitude once that exceeds 1, so rounding alone
    never reaches 1e-2 in these units.)"""
    g, r = to64(gpu), np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    scale = np.maximum(1.0, np.abs(r).max(axis=-1, keepdims=True))
    err = np.abs(g - r) / scale
    assert err.max() <= 1e-2, f"{what}: max scaled err {err.max()} at {np.unravel_index(err.argmax(), err.shape)}"
    assert err.mean() <= 1e-3, f"{what}: mean scaled err {err.mean()}"


def _fp8_decode_case(cfg, off, window, ring, n_steps=3, restore=False, special=False):
    n_total = off + n_steps * (2 if restore else 1) + 2
    cos, sin = _tables(cfg, n_total + 8)
    rc, rs = oracle_tables(cfg, n_total + 8)
    sinks = wl.sinks(cfg).to(DEV)
    if ring:
        cap = 384   # the prefix below wraps it
    else:
        cap = ((n_total + 8 + 15) // 16) * 16
    cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV, ring=window if ring else 0, fp8=True)
    ocache = okv.KVCache(cfg.B, n_total + 8, cfg.n_kv, cfg.d)
    if off:
        if special:
            # the V pattern is shifted against K's, so that heavily weighted
            # keys sit next to V rows of very different scale
            kp = _special_rows((cfg.B, off, cfg.n_kv, cfg.d), 11)
            vp = _special_rows((cfg.B, off, cfg.n_kv, cfg.d), 12, shift=3)
        else:
            kp, vp = wl.prefilled_cache_rows(cfg, rows=off)
        step = cap if ring else off
        for s0 in range(0, off, step):
            cache.append(kp[:, s0:s0 + step].to(DEV), vp[:, s0:s0 + step].to(DEV))
        kc, ks = ofp8.quantize_rows(to64(kp))
        vc, vs = ofp8.quantize_rows(to64(vp))
        ocache.append(ofp8.dequantize_rows(kc, ks), ofp8.dequantize_rows(vc, vs))
    ws = sa.decode_workspace(cfg.B, cfg.n_q, cfg.n_kv, cfg.d, device=DEV)

    def steps(first, n):
        for st in range(n):
            q, k, v = wl.qkv(cfg, 1, step=first + st + 1)
            pos = cache.offset
            out, lse = sa.attn_decode(cache, q.to(DEV), k.to(DEV), v.to(DEV), sinks, window, cfg.sm_scale,
                                      cos, sin, workspace=ws, return_lse=True)
            torch.cuda.synchronize()
            ref, ref_lse = ofp8.attend_step_fp8(ocache, to64(q), to64(k), to64(v), to64(sinks.cpu()),
                                                window, cfg.sm_scale, rc, rs)
            if special:
                _check_scaled(out, ref, f"fp8 decode step {first + st}")
                check_lse(lse, ref_lse, f"fp8 decode step {first + st}", rtol=1e-5, atol=2e-4)
            else:
                check_bf16_output(out, ref, f"fp8 decode step {first + st}")
                check_lse(lse, ref_lse, f"fp8 decode step {first + st}")
            # the new row is stored quantised, bit for bit
            k_rot = orope.rotate_bsh(to64(k), pos, rc, rs)
            _check_codes(cache, pos, pos + 1, k_rot, round_bf16(to64(v)), f"fp8 new row {pos}")

    steps(0, n_steps)
    if restore:
        snap, osnap = cache.snapshot(), ocache.snapshot()
        steps(100, n_steps)
        cache.restore(snap)
        ocache.restore(osnap)
        steps(200, n_steps)
    n_cnt = cfg.B * cfg.n_kv
    assert torch.count_nonzero(ws[: 8 * n_cnt]) == 0   # tickets and stage counters


@pytest.mark.parametrize("over", [dict(B=2, n_q=8, n_kv=2, d=64), dict(B=2, n_q=8, n_kv=4, d=96),
                                  dict(B=1, n_q=16, n_kv=2, d=128), dict(B=1, n_q=64, n_kv=8, d=64),
                                  dict(B=3, n_q=3, n_kv=3, d=64)],
                         ids=["d64", "d96", "d128", "gptoss", "mha"])
@pytest.mark.parametrize("layer", [0, 1], ids=["band", "full"])
@pytest.mark.parametrize("off", [0, 37, 5000])
def test_fp8_decode_matches_oracle(cuda_device, over, layer, off):
    cfg = wl.scaled(wl.CONFIGS["tiny"], sm_scale=1 / math.sqrt(over["d"]), **over)
    window = 128 if layer == 0 else 0
    _fp8_decode_case(cfg, off, window, ring=False, restore=(off == 37))


@pytest.mark.parametrize("d", [64, 96, 128])
def test_fp8_ring_decode_matches_oracle(cuda_device, d):
    cfg = wl.scaled(wl.CONFIGS["tiny"], B=2, n_q=8, n_kv=2, d=d, sm_scale=1 / math.sqrt(d))
    _fp8_decode_case(cfg, 900, 128, ring=True, n_steps=3, restore=True)


@pytest.mark.parametrize("layer", [0, 1], ids=["band", "full"])
def test_fp8_decode_mixed_magnitude_rows(cuda_device, layer):
    # zero rows, rows at 1e30 and 1e-30 and single-element rows among normal
    # ones: the per-row scales span ~200 binades inside one split
    cfg = wl.scaled(wl.CONFIGS["tiny"], B=1, n_q=8, n_kv=2, d=64, sm_scale=0.125)
    _fp8_decode_case(cfg, 300, 128 if layer == 0 else 0, ring=False, special=True)


def test_fp8_prefill_is_refused(cuda_device):
    cfg = wl.scaled(wl.CONFIGS["tiny"], B=1, n_q=4, n_kv=2, d=64)
    cos, sin = _tables(cfg, 64)
    cache = sa.KVCache(1, 64, 2, 64, device=DEV, fp8=True)
    q, k, v = wl.qkv(cfg, 8)
    with pytest.raises(sa.SinkAttnError) as e:
        sa.attn_prefill(cache, q.to(DEV), k.to(DEV), v.to(DEV), None, 0, 0.125, cos, sin)
    assert e.value.name == "SA_ERR_UNSUPPORTED" and cache.offset == 0


@pytest.mark.parametrize("layer", [0, 1], ids=["band", "full"])
def test_fp8_full_size_long_decode(cuda_device, layer):
    # 131,072 cached positions, 64 query heads over 8 KV heads, d = 64: the
    # prefix appended (quantised), one decode step, sampled heads against the
    # oracle over the dequantised rows of their KV head.
    cfg = wl.CONFIGS["long_decode"]
    window = cfg.layer_window(layer)
    off = cfg.offset
    cap = ((off + 2 + 15) // 16) * 16
    cos, sin = _tables(cfg, off + 2)
    rc, rs = oracle_tables(cfg, off + 2)
    sinks = wl.sinks(cfg, layer=layer)
    kp, vp = wl.prefilled_cache_rows(cfg, layer=layer, device=DEV)
    cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV, fp8=True)
    cache.append(kp, vp)
    q, k, v = wl.qkv(cfg, 1, layer=layer, step=1, device=DEV)
    out, lse = sa.attn_decode(cache, q, k, v, sinks.to(DEV), window, cfg.sm_scale, cos, sin, return_lse=True)
    torch.cuda.synchronize()
    got, want = [], []
    for h in (0, 9, 63):
        g = h // cfg.q_mult
        lo = max(0, off + 1 - window) if window else 0
        kc, ks = ofp8.quantize_rows(to64(kp[0, lo:, g]))
        vc, vs = ofp8.quantize_rows(to64(vp[0, lo:, g]))
        k_new = orope.rotate_bsh(to64(k[:, :, g:g + 1]), off, rc, rs)[0, 0]
        nkc, nks = ofp8.quantize_rows(k_new)
        nvc, nvs = ofp8.quantize_rows(round_bf16(to64(v[0, 0, g:g + 1])))
        K = np.concatenate([ofp8.dequantize_rows(kc, ks), ofp8.dequantize_rows(nkc, nks)], axis=0)
        V = np.concatenate([ofp8.dequantize_rows(vc, vs), ofp8.dequantize_rows(nvc, nvs)], axis=0)
        qr = orope.rotate_bsh(to64(q[:, :, h:h + 1]), off, rc, rs)
        # keys [lo, off] as a cache of their own: the query sits at position off - lo
        o, l = oatt.sink_attention(qr, K[None, :, None, :], V[None, :, None, :], to64(sinks[h:h + 1]),
                                   off - lo, window, cfg.sm_scale)
        got.append(out[0, 0, h])
        want.append(o[0, 0, 0])
        check_lse(lse[0, h, 0], np.array(l[0, 0, 0]), f"fp8 long decode h{h}")
    check_bf16_output(torch.stack(got), np.stack(want), "fp8 long decode sampled heads")
    assert cache.offset == off + 1

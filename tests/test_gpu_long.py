"""GPU parity of the two long configurations at full size and full length.

* Long-context decode: one band / full layer pair of the 24-layer model, the
  cache pre-filled to offset 131,071, then all 64 decode steps, each appending
  one K/V row per layer (MoE-Xtend README, "TOKEN STREAM (DECODE)": one append
  per layer per step at position = cache offset).
* Prefill-to-decode handoff: 16 sequences sharing offset 65,536, a 512-row
  chunked prefill, then all 32 decode steps, on both layer types (MoE-Xtend
  README, "KV CACHE": prefill once, decode many; "DESIGN CONTRACTS": the
  pre-append offset for RoPE and the mask).

The GPU runs every head of every sequence; the fp64 oracle recomputes sampled
(sequence, head) units row by row -- every decode step, and the chunk's rows
at tile edges -- from the same bits (the pre-filled prefix is generated on the
device and the sampled KV groups copied back).
"""

import numpy as np
import pytest
import torch

import sink_augmented_gqa_b200 as sa
from oracle import attention as oatt
from oracle import bf16 as obf16
from oracle import rope as orope
from sink_augmented_gqa_b200 import workloads as wl

from helpers import OracleOut, check_bf16_output, check_lse, oracle_tables, stack_out, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _tables(cfg, max_pos):
    y = cfg.yarn
    return sa.yarn_rope_tables(max_pos, cfg.d, y["theta"], y["scaling"], y["orig_ctx"], y["alpha"],
                               y["beta"], device=DEV)


class _OracleUnit:
    """The oracle's view of one (sequence b, KV group g): fp64 copies of the
    cache rows, extended by each call's rotated keys and values."""

    def __init__(self, kp, vp, b, g, cap):
        n = kp.shape[1]
        self.K = np.zeros((cap, kp.shape[-1]))
        self.V = np.zeros((cap, kp.shape[-1]))
        self.K[:n] = to64(kp[b, :, g])
        self.V[:n] = to64(vp[b, :, g])
        self.n = n

    def append(self, k_raw, v_raw, rc, rs):
        """k_raw, v_raw: [T, d] fp64 rows of this group, rotated at n, n+1, ..."""
        T = k_raw.shape[0]
        kr = orope.rotate_bsh(k_raw[None, :, None], self.n, rc, rs)[0, :, 0]
        self.K[self.n:self.n + T] = kr
        self.V[self.n:self.n + T] = obf16.round_bf16(v_raw)
        self.n += T
        return kr

    def row(self, q_raw, pos, sink, window, sm_scale, rc, rs):
        """Output and lse of one query row (raw [d]) at position pos."""
        qr = orope.rotate_bsh(q_raw[None, None, None], pos, rc, rs)
        K, V = self.K[None, :pos + 1, None], self.V[None, :pos + 1, None]
        out, lse = oatt.sink_attention(qr, K, V, np.array([sink]), pos, window, sm_scale)
        vabs, _ = oatt.sink_attention(qr, K, np.abs(V), np.array([sink]), pos, window, sm_scale)
        return OracleOut(out[0, 0, 0], vabs[0, 0, 0]), lse[0, 0, 0]


@pytest.mark.parametrize("layer", [0, 1], ids=["band", "full"])
def test_long_decode_all_64_steps(cuda_device, layer):
    cfg = wl.CONFIGS["long_decode"]
    window = cfg.layer_window(layer)
    off, steps = cfg.offset, cfg.decode_steps
    cap = off + steps
    cos, sin = _tables(cfg, cap)
    rc, rs = oracle_tables(cfg, cap)
    sinks = wl.sinks(cfg, layer=layer)
    kp, vp = wl.prefilled_cache_rows(cfg, layer=layer, device=DEV)
    cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV)
    cache.append(kp, vp)
    ws = sa.decode_workspace(cfg.B, cfg.n_q, cfg.n_kv, cfg.d, device=DEV)
    heads = (0, 7, 63)        # both ends of KV group 0, and the last group
    units = {g: _OracleUnit(kp, vp, 0, g, cap) for g in {h // cfg.q_mult for h in heads}}
    del kp, vp
    sk = to64(sinks)
    for st in range(steps):
        q, k, v = wl.qkv(cfg, 1, layer=layer, step=st + 1, device=DEV)
        out, lse = sa.attn_decode(cache, q, k, v, sinks.to(DEV), window, cfg.sm_scale, cos, sin,
                                  workspace=ws, return_lse=True)
        torch.cuda.synchronize()
        pos = off + st
        got, want = [], []
        for g, u in units.items():
            kr = u.append(to64(k[0, :, g]), to64(v[0, :, g]), rc, rs)
            # the row decode wrote into the cache is the oracle's rotated key
            row = to64(cache.k_rows(pos, pos + 1)[0, 0, g])
            assert np.all(np.abs(row - kr[0]) <= obf16.bf16_ulp(kr[0]) * 1.0000001), f"step {st} K row"
            assert np.array_equal(to64(cache.v_rows(pos, pos + 1)[0, 0, g]), u.V[pos])
        for h in heads:
            ro, rl = units[h // cfg.q_mult].row(to64(q[0, 0, h]), pos, sk[h], window, cfg.sm_scale, rc, rs)
            got.append(out[0, 0, h])
            want.append(ro)
            check_lse(lse[0, h, 0], np.array(rl), f"long decode step {st} h{h}")
        check_bf16_output(torch.stack(got), stack_out(want), f"long decode step {st}")
    assert cache.offset == off + steps
    n_cnt = cfg.B * cfg.n_kv   # the split tickets and stage counters end every call at zero
    assert torch.count_nonzero(ws[: 8 * n_cnt]) == 0


@pytest.mark.parametrize("layer", [0, 1], ids=["band", "full"])
def test_handoff_chunk_then_all_32_steps(cuda_device, layer):
    cfg = wl.CONFIGS["handoff"]
    window = cfg.layer_window(layer)
    off, T, steps = cfg.offset, cfg.T, cfg.decode_steps
    cap = off + T + steps
    cos, sin = _tables(cfg, cap)
    rc, rs = oracle_tables(cfg, cap)
    sinks = wl.sinks(cfg, layer=layer)
    sk = to64(sinks)
    kp, vp = wl.prefilled_cache_rows(cfg, layer=layer, device=DEV)
    cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV)
    cache.append(kp, vp)
    seqs, heads = (0, 7, 15), (0, 37, 63)
    units = {(b, g): _OracleUnit(kp, vp, b, g, cap) for b in seqs for g in {h // cfg.q_mult for h in heads}}
    del kp, vp
    torch.cuda.empty_cache()
    # the 512-row chunk at offset 65,536: rows at the 128-row tile edges and a few inside
    q, k, v = wl.qkv(cfg, T, layer=layer, device=DEV)
    out = sa.attn_prefill(cache, q, k, v, sinks.to(DEV), window, cfg.sm_scale, cos, sin)
    torch.cuda.synchronize()
    rows = [0, 1, 63, 127, 128, 200, 255, 256, 383, 384, 450, 510, 511]
    got, want = [], []
    for (b, g), u in units.items():
        u.append(to64(k[b, :, g]), to64(v[b, :, g]), rc, rs)
        for h in heads:
            if h // cfg.q_mult != g:
                continue
            for i in rows:
                ro, _ = u.row(to64(q[b, i, h]), off + i, sk[h], window, cfg.sm_scale, rc, rs)
                got.append(out[b, i, h])
                want.append(ro)
    check_bf16_output(torch.stack(got), stack_out(want), "handoff chunk sampled rows")
    del q, k, v, out
    ws = sa.decode_workspace(cfg.B, cfg.n_q, cfg.n_kv, cfg.d, device=DEV)
    for st in range(steps):
        q, k, v = wl.qkv(cfg, 1, layer=layer, step=st + 1, device=DEV)
        dec, lse = sa.attn_decode(cache, q, k, v, sinks.to(DEV), window, cfg.sm_scale, cos, sin,
                                  workspace=ws, return_lse=True)
        torch.cuda.synchronize()
        pos = off + T + st
        got, want = [], []
        for (b, g), u in units.items():
            u.append(to64(k[b, :, g]), to64(v[b, :, g]), rc, rs)
            for h in heads:
                if h // cfg.q_mult != g:
                    continue
                ro, rl = u.row(to64(q[b, 0, h]), pos, sk[h], window, cfg.sm_scale, rc, rs)
                got.append(dec[b, 0, h])
                want.append(ro)
                check_lse(lse[b, h, 0], np.array(rl), f"handoff step {st} b{b} h{h}")
        check_bf16_output(torch.stack(got), stack_out(want), f"handoff decode step {st}")
    assert cache.offset == off + T + steps

"""The allocation-free decode entry point (sa_attn_decode_static).

Some callers cannot allocate device memory: a runtime embedded in another
process that only hands out device pointers, or a serving loop that must
never call cudaMalloc. For them the library keeps the decode's split scratch
in a fixed array of its own. This file checks, through the C ABI, that the
entry point returns what the workspace-taking decode returns and what the
fp64 oracle computes, on two calls in a row (the shared scratch keeps the
previous call's contents), and that it refuses shapes whose scratch would not
fit. It is collected last on purpose.
"""

import pytest
import torch

import sink_augmented_gqa_b200 as sa
from sink_augmented_gqa_b200 import workloads as wl

from helpers import check_bf16_output, check_lse, oracle_cache, oracle_step, oracle_tables, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _tables(cfg, max_pos):
    y = cfg.yarn
    return sa.yarn_rope_tables(max_pos, cfg.d, y["theta"], y["scaling"], y["orig_ctx"], y["alpha"],
                               y["beta"], device=DEV)


@pytest.mark.parametrize("window", [0, 128])
def test_static_scratch_decode_matches_workspace_decode(cuda_device, window):
    cfg = wl.scaled(wl.CONFIGS["tiny"], B=2, n_q=8, n_kv=2, d=64)
    off = 5000                      # long enough for many splits
    cap = off + 4
    cos, sin = _tables(cfg, cap)
    rc, rs = oracle_tables(cfg, cap)
    sinks = wl.sinks(cfg).to(DEV)
    kp_h, vp_h = wl.prefilled_cache_rows(cfg, rows=off)
    ocache = oracle_cache(cfg.B, cap, cfg.n_kv, cfg.d, kp_h, vp_h)
    kp, vp = kp_h.to(DEV), vp_h.to(DEV)
    ref_cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV)
    new_cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV)
    ref_cache.append(kp, vp)
    new_cache.append(kp, vp)
    ws = sa.decode_workspace(cfg.B, cfg.n_q, cfg.n_kv, cfg.d, device=DEV)
    for step in range(2):           # two calls in a row share the static scratch
        q_h, k_h, v_h = wl.qkv(cfg, 1, step=step + 1)
        q, k, v = q_h.to(DEV), k_h.to(DEV), v_h.to(DEV)
        ref, ref_lse = sa.attn_decode(ref_cache, q, k, v, sinks, window, cfg.sm_scale, cos, sin,
                                      workspace=ws, return_lse=True)
        got, got_lse = sa.attn_decode_static(new_cache, q, k, v, sinks, window, cfg.sm_scale, cos, sin,
                                             return_lse=True)
        torch.cuda.synchronize()
        check_bf16_output(got, to64(ref), f"static-scratch decode, call {step}")
        check_lse(got_lse, to64(ref_lse), f"static-scratch decode lse, call {step}")
        exact, exact_lse = oracle_step(ocache, q_h, k_h, v_h, sinks.cpu(), window, cfg.sm_scale, rc, rs)
        check_bf16_output(got, exact, f"static-scratch decode vs oracle, call {step}")
        check_lse(got_lse, exact_lse, f"static-scratch decode lse vs oracle, call {step}")
        assert new_cache.offset == ref_cache.offset == off + step + 1
    torch.cuda.synchronize()
    assert torch.equal(new_cache.k, ref_cache.k) and torch.equal(new_cache.v, ref_cache.v)


def test_static_scratch_refuses_oversized_shapes(cuda_device):
    # 16 sequences x 8 KV heads x 3 splits, one record of 8 query heads x
    # (128 outputs + m + l) fp32 each: 1.6 MB of scratch, more than the 1 MiB
    # the library holds.
    cfg = wl.scaled(wl.CONFIGS["handoff"], B=16, n_q=64, n_kv=8, d=128, offset=1000, T=0)
    cap = cfg.offset + 2
    cos, sin = _tables(cfg, cap)
    cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV)
    cache.append(cache.k_rows(0, cfg.offset), cache.v_rows(0, cfg.offset))
    q, k, v = wl.qkv(cfg, 1, device=DEV)
    with pytest.raises(sa.SinkAttnError) as e:
        sa.attn_decode_static(cache, q, k, v, None, 0, cfg.sm_scale, cos, sin)
    assert e.value.name == "SA_ERR_WORKSPACE"
    assert cache.offset == cfg.offset        # nothing was enqueued

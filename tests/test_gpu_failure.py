"""Failure detection without faulting the GPU.

Every device-side wait of the library is bounded. With the bound set to zero
cycles, the waits that are not already satisfied give up at once: the
kernels record SA_ERR_TIMEOUT in the device status word, drain the copies and
MMAs they already started, release their memory and return. The host reads
the status, restores the bound, and the same context keeps computing
correct results.
"""

import numpy as np
import pytest
import torch

import sink_augmented_gqa_b200 as sa
from sink_augmented_gqa_b200 import workloads as wl

from helpers import check_bf16_output, oracle_cache, oracle_step, oracle_tables

pytestmark = pytest.mark.gpu
DEV = "cuda"
DEFAULT_LIMIT = 2_000_000_000


def _tables(cfg, max_pos):
    y = cfg.yarn
    return sa.yarn_rope_tables(max_pos, cfg.d, y["theta"], y["scaling"], y["orig_ctx"], y["alpha"],
                               y["beta"], device=DEV)


@pytest.mark.parametrize("window", [0, 16], ids=["full", "band"])
def test_zero_wait_limit_reports_timeout_and_context_survives(cuda_device, window):
    cfg = wl.scaled(wl.CONFIGS["tiny"], B=2)
    off = 3000
    cap = off + 300
    cos, sin = _tables(cfg, cap)
    sinks = wl.sinks(cfg).to(DEV)
    assert sa.device_status() == "SA_OK"
    sa.set_wait_limit(0)
    try:
        cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV)
        kp, vp = wl.prefilled_cache_rows(cfg, rows=off, device=DEV)
        cache.append(kp, vp)
        q, k, v = wl.qkv(cfg, 256, device=DEV)
        sa.attn_prefill(cache, q, k, v, sinks, window, cfg.sm_scale, cos, sin)
        qd, kd, vd = wl.qkv(cfg, 1, step=1, device=DEV)
        sa.attn_decode(cache, qd, kd, vd, sinks, window, cfg.sm_scale, cos, sin)
        torch.cuda.synchronize()
        status = sa.device_status()
    finally:
        sa.set_wait_limit(DEFAULT_LIMIT)
    assert status == "SA_ERR_TIMEOUT"
    assert sa.device_status() == "SA_OK"          # reading the word clears it

    # The context is intact: a fresh call computes the right answer.
    rc, rs = oracle_tables(cfg, cap)
    cache = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=DEV)
    ocache = oracle_cache(cfg.B, cap, cfg.n_kv, cfg.d)
    q, k, v = wl.qkv(cfg, 200, step=5)
    out = sa.attn_prefill(cache, q.to(DEV), k.to(DEV), v.to(DEV), sinks, 16, cfg.sm_scale, cos, sin)
    torch.cuda.synchronize()
    ref, _ = oracle_step(ocache, q, k, v, sinks.cpu(), 16, cfg.sm_scale, rc, rs)
    check_bf16_output(out, ref, "after timeout")
    assert sa.device_status() == "SA_OK"


def test_zero_wait_limit_backward_reports_timeout_and_context_survives(cuda_device):
    # The backward's producer, MMA issuer and P / dS warps give up on their
    # bounded waits, drain what they started (loads, products, reduce-adds)
    # and return; afterwards the same context computes the same gradients as
    # before (dk, dv bit for bit; dq, summed by reduce-adds in a varying
    # order, to rounding).
    import math
    cfg = wl.scaled(wl.CONFIGS["tiny"], B=2, n_q=8, n_kv=2, d=96, sm_scale=1 / math.sqrt(96), seed=900)
    T = 300
    q, k, v = wl.qkv(cfg, T, device=DEV)
    dout = wl.randn_bf16((cfg.B, T, cfg.n_q, cfg.d), cfg.seed, 127, DEV)
    sinks = wl.sinks(cfg, device=DEV)
    cache = sa.KVCache(cfg.B, T, cfg.n_kv, cfg.d, device=DEV)
    out, lse = sa.attn_prefill(cache, q, k, v, sinks, 0, cfg.sm_scale, rope_fused=False, return_lse=True)
    before = sa.attn_backward(q, k, v, out, dout, lse, sinks, 0, cfg.sm_scale)
    torch.cuda.synchronize()
    assert sa.device_status() == "SA_OK"
    sa.set_wait_limit(0)
    try:
        sa.attn_backward(q, k, v, out, dout, lse, sinks, 0, cfg.sm_scale)
        torch.cuda.synchronize()
        status = sa.device_status()
    finally:
        sa.set_wait_limit(DEFAULT_LIMIT)
    assert status == "SA_ERR_TIMEOUT"
    assert sa.device_status() == "SA_OK"
    after = sa.attn_backward(q, k, v, out, dout, lse, sinks, 0, cfg.sm_scale)
    torch.cuda.synchronize()
    assert sa.device_status() == "SA_OK"
    assert torch.equal(before[1], after[1]) and torch.equal(before[2], after[2])
    for x, y in (before[0], after[0]), (before[3], after[3]):
        assert (x - y).abs().amax().item() <= 1e-5 * x.abs().amax().item()


def test_zero_wait_limit_projections_report_timeout_and_context_survives(cuda_device):
    # The projection GEMM (producer, MMA issuer, RMSNorm warps, epilogue) gives
    # up on its bounded waits and returns; afterwards the same context
    # computes bit-identical projections to the ones before the timeout.
    g = torch.Generator().manual_seed(11)
    M, N, K = 600, 1280, 1024
    x = (torch.randn((M, K), generator=g) * 1.0).to(torch.bfloat16).to(DEV)
    w = (torch.randn((N, K), generator=g) / 32).to(torch.bfloat16).to(DEV)
    gamma = (torch.rand(K, generator=g) + 0.5).to(DEV)
    b = (torch.randn((N,), generator=g) * 0.1).to(torch.bfloat16).to(DEV)
    wf = sa.rmsnorm_fold_weight(w, gamma)
    o = (torch.randn((M, K), generator=g)).to(torch.bfloat16).to(DEV)
    w2 = (torch.randn((N, K), generator=g) / 32).to(torch.bfloat16).to(DEV)
    res = (torch.randn((M, N), generator=g)).to(torch.bfloat16).to(DEV)

    def run():
        y = sa.qkv_proj(x, wf, b, 1e-5)
        xr = res.clone()
        sa.out_proj(o, w2, b, xr)
        return y, xr
    y0, r0 = run()
    torch.cuda.synchronize()
    assert sa.device_status() == "SA_OK"
    sa.set_wait_limit(0)
    try:
        run()
        torch.cuda.synchronize()
        status = sa.device_status()
    finally:
        sa.set_wait_limit(DEFAULT_LIMIT)
    assert status == "SA_ERR_TIMEOUT"
    assert sa.device_status() == "SA_OK"
    y1, r1 = run()
    torch.cuda.synchronize()
    assert sa.device_status() == "SA_OK"
    assert torch.equal(y0, y1) and torch.equal(r0, r1)

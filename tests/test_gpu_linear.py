"""GPU parity of the projections around the attention (RMSNorm + fused qkv,
out projection + residual) against ``oracle/linear.py``.

Tolerance, from the arithmetic: the kernel multiplies bf16 operands exactly
and accumulates in fp32; the qkv weight carries RMSNorm's gain folded in and
rounded to bf16 once (relative error <= 2^-9 per weight). With
``S = sum_k |a_k w_nk|`` (exact, in the units of the output), an element may
differ from the exact result rounded to bf16 by one bf16 step plus
``2^-9 S`` (folded weights; qkv only) plus ``2^-12 S`` (fp32 accumulation
over K <= 4096 terms, an order of magnitude above the worst case K 2^-24).
The weight fold itself is bit-exact (one rounding of the exact product).
"""

import math

import numpy as np
import pytest
import torch

import sink_augmented_gqa_b200 as sa
from oracle import attention as oatt
from oracle import bf16 as obf16
from oracle import kvcache as okv
from oracle import linear as olin
from oracle import rope as orope
from sink_augmented_gqa_b200 import workloads as wl

from helpers import check_bf16_output, oracle_attend, oracle_tables, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float32) * scale).to(torch.bfloat16)


def _padded(t, ld):
    """The same values in a [rows, ld'] buffer, ld' = ld rounded up to a
    multiple of 8 (the leading-dimension rule), as a strided view."""
    rows, cols = t.shape
    ld = (ld + 7) // 8 * 8
    buf = torch.zeros((rows, ld), dtype=t.dtype, device=DEV)
    buf[:, :cols] = t.to(DEV)
    return buf[:, :cols]


def _check(gpu, ref, s_abs, rel, what):
    """Against the exact (unrounded) value: the fp32 result lies within
    e = rel * s_abs of it, and its rounding to bf16 adds at most half a bf16
    step at |ref| + e."""
    g = to64(gpu)
    r = np.asarray(ref, dtype=np.float64)
    e = rel * s_abs
    tol = 0.5 * obf16.bf16_ulp(np.abs(r) + e) * 1.0000001 + e
    err = np.abs(g - r)
    bad = np.argwhere(~(err <= tol))
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    assert bad.size == 0, (f"{what}: {len(bad)} elements beyond tolerance; first {bad[:4].tolist()} "
                           f"gpu={g[tuple(bad[0])]} ref={r[tuple(bad[0])]} tol={tol[tuple(bad[0])]}")
    return float((err / (s_abs + 1e-30)).max())


def test_fold_weight_bit_exact(cuda_device):
    N, K = 300, 200
    w = _rand((N, K), 1)
    g = torch.Generator().manual_seed(2)
    gamma = torch.rand(K, generator=g, dtype=torch.float32) * 2 + 0.25
    wd = _padded(w, 208)
    out = torch.full((N, 216), float("nan"), dtype=torch.bfloat16, device=DEV)[:, :K]
    sa.rmsnorm_fold_weight(wd, gamma.to(DEV), out=out)
    torch.cuda.synchronize()
    ref = obf16.round_bf16(to64(w) * to64(gamma)[None, :])
    assert np.array_equal(to64(out), ref)


QKV_CASES = [
    dict(M=1, N=64, K=64),
    dict(M=37, N=600, K=2880),          # ragged N inside a 32-column chunk
    dict(M=300, N=640, K=192, ld=8),     # three M tiles (128, 128, 44), padded rows
    dict(M=129, N=5120, K=2880),         # the gpt-oss qkv width, an M tile of one row
    dict(M=256, N=256, K=4096, bias=False, eps=0.0),
]


@pytest.mark.parametrize("case", QKV_CASES, ids=[f"M{c['M']}N{c['N']}K{c['K']}" for c in QKV_CASES])
def test_qkv_proj_matches_oracle(cuda_device, case):
    M, N, K = case["M"], case["N"], case["K"]
    pad = case.get("ld", 0)
    eps = case.get("eps", 1e-5)
    x = _rand((M, K), 10 + M)
    w = _rand((N, K), 20 + N, scale=1 / math.sqrt(K))
    g = torch.Generator().manual_seed(3)
    gamma = torch.rand(K, generator=g, dtype=torch.float32) + 0.5
    b = _rand((N,), 30) if case.get("bias", True) else None
    wf = sa.rmsnorm_fold_weight(_padded(w, K + pad), gamma.to(DEV))
    y = torch.full((M, (N + pad + 7) // 8 * 8), float("nan"), dtype=torch.bfloat16, device=DEV)[:, :N]
    sa.qkv_proj(_padded(x, K + pad), wf, None if b is None else b.to(DEV), eps, out=y)
    torch.cuda.synchronize()
    x64, w64, g64 = to64(x), to64(w), to64(gamma)
    ref = olin.qkv_proj(x64, g64, eps, w64, None if b is None else to64(b))
    xn = olin.rmsnorm(x64, g64, eps)
    s_abs = np.abs(xn) @ np.abs(w64).T
    _check(y, ref, s_abs, 2.0 ** -9 + 2.0 ** -12, f"qkv_proj {case}")


OUT_CASES = [
    dict(M=5, N=100, K=64),
    dict(M=300, N=2880, K=4096),         # the gpt-oss out projection, ragged N (11 tiles + 64)
    dict(M=200, N=256, K=128, bias=False, ld=16),
]


@pytest.mark.parametrize("case", OUT_CASES, ids=[f"M{c['M']}N{c['N']}K{c['K']}" for c in OUT_CASES])
def test_out_proj_matches_oracle(cuda_device, case):
    M, N, K = case["M"], case["N"], case["K"]
    pad = case.get("ld", 0)
    o = _rand((M, K), 40 + M)
    w = _rand((N, K), 50 + N, scale=1 / math.sqrt(K))
    b = _rand((N,), 60) if case.get("bias", True) else None
    x = _rand((M, N), 70 + M, scale=3.0)
    xd = _padded(x, N + pad)
    sa.out_proj(_padded(o, K + pad), _padded(w, K + pad), None if b is None else b.to(DEV), xd)
    torch.cuda.synchronize()
    ref = olin.out_proj(to64(o), to64(w), None if b is None else to64(b), to64(x))
    s_abs = np.abs(to64(o)) @ np.abs(to64(w)).T
    _check(xd, ref, s_abs, 2.0 ** -12, f"out_proj {case}")


@pytest.mark.parametrize("which", ["qkv", "out"])
def test_full_size_projections_sampled(cuda_device, which):
    # The gpt-oss prefill sizes: T = 8192 rows, 2880 -> 5120 (qkv) and
    # 4096 -> 2880 (out); sampled rows against the oracle.
    T = 8192
    N, K = (5120, 2880) if which == "qkv" else (2880, 4096)
    a = _rand((T, K), 80).to(DEV)
    w = _rand((N, K), 81, scale=1 / math.sqrt(K)).to(DEV)
    b = _rand((N,), 82).to(DEV)
    rows = [0, 1, 127, 128, 4095, 5000, 8190, 8191]
    if which == "qkv":
        g = torch.Generator().manual_seed(83)
        gamma = (torch.rand(K, generator=g, dtype=torch.float32) + 0.5).to(DEV)
        wf = sa.rmsnorm_fold_weight(w, gamma)
        y = sa.qkv_proj(a, wf, b, 1e-5)
        torch.cuda.synchronize()
        xs = to64(a[rows])
        ref = olin.qkv_proj(xs, to64(gamma), 1e-5, to64(w), to64(b))
        s_abs = np.abs(olin.rmsnorm(xs, to64(gamma), 1e-5)) @ np.abs(to64(w)).T
        _check(y[rows], ref, s_abs, 2.0 ** -9 + 2.0 ** -12, "qkv_proj T=8192")
    else:
        x = _rand((T, N), 84, scale=3.0).to(DEV)
        x0 = x[rows].clone()
        sa.out_proj(a, w, b, x)
        torch.cuda.synchronize()
        ref = olin.out_proj(to64(a[rows]), to64(w), to64(b), to64(x0))
        s_abs = np.abs(to64(a[rows])) @ np.abs(to64(w)).T
        _check(x[rows], ref, s_abs, 2.0 ** -12, "out_proj T=8192")


def test_projection_argument_errors(cuda_device):
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((32, 64), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(sa.SinkAttnError):
        sa.qkv_proj(x[:, 1:], w[:, 1:], None, 1e-5)          # misaligned rows
    with pytest.raises(sa.SinkAttnError):
        sa.qkv_proj(x, w, None, -1.0)                        # negative eps
    y = sa.qkv_proj(x[:0], w, None, 1e-5)                    # M = 0: no-op
    assert y.shape == (0, 32)


def test_attention_layer_composition(cuda_device):
    # One gpt-oss attention layer at small T: x -> RMSNorm + qkv (this
    # library) -> prefill on the q|k|v views of the fused output (RoPE fused)
    # -> out projection with the residual add, against the oracle's
    # composition of the same steps (each kernel output rounded to bf16 where
    # the library stores it).
    cfg = wl.scaled(wl.CONFIGS["gptoss_prefill"], T=160)
    T, n_q, n_kv, d = cfg.T, cfg.n_q, cfg.n_kv, cfg.d
    D_model = 2880
    width = d * (n_q + 2 * n_kv)
    x = _rand((T, D_model), 90)
    g = torch.Generator().manual_seed(91)
    gamma = torch.rand(D_model, generator=g, dtype=torch.float32) + 0.5
    wqkv = _rand((width, D_model), 92, scale=1 / math.sqrt(D_model))
    bqkv = _rand((width,), 93)
    wo = _rand((D_model, n_q * d), 94, scale=1 / math.sqrt(n_q * d))
    bo = _rand((D_model,), 95)
    sinks = wl.sinks(cfg, layer=1)
    y = cfg.yarn
    cos, sin = sa.yarn_rope_tables(T, d, y["theta"], y["scaling"], y["orig_ctx"], y["alpha"], y["beta"], device=DEV)
    rc, rs = oracle_tables(cfg, T)
    # library
    wf = sa.rmsnorm_fold_weight(wqkv.to(DEV), gamma.to(DEV))
    qkv = sa.qkv_proj(x.to(DEV), wf, bqkv.to(DEV), 1e-5)
    q = qkv[:, : n_q * d].view(1, T, n_q, d)
    k = qkv[:, n_q * d:(n_q + n_kv) * d].view(1, T, n_kv, d)
    v = qkv[:, (n_q + n_kv) * d:].view(1, T, n_kv, d)
    cache = sa.KVCache(1, T, n_kv, d, device=DEV)
    o = sa.attn_prefill(cache, q, k, v, sinks.to(DEV), 0, cfg.sm_scale, cos, sin)
    xr = x.to(DEV).clone()
    sa.out_proj(o.view(T, n_q * d), wo.to(DEV), bo.to(DEV), xr)
    torch.cuda.synchronize()
    # oracle, fed the library's own bf16 intermediates so each stage is checked on its own
    ref_qkv = olin.qkv_proj(to64(x), to64(gamma), 1e-5, to64(wqkv), to64(bqkv))
    s_abs = np.abs(olin.rmsnorm(to64(x), to64(gamma), 1e-5)) @ np.abs(to64(wqkv)).T
    _check(qkv, ref_qkv, s_abs, 2.0 ** -9 + 2.0 ** -12, "layer: qkv")
    qq, kk, vv = olin.split_qkv(to64(qkv), n_q, n_kv, d)
    oc = okv.KVCache(1, T, n_kv, d)
    ref_o, _ = oracle_attend(oc, qq[None], kk[None], vv[None], to64(sinks), 0, cfg.sm_scale, rc, rs)
    check_bf16_output(o, ref_o, "layer: attention")
    ref_x = olin.out_proj(to64(o.view(T, n_q * d)), to64(wo), to64(bo), to64(x))
    s_abs_o = np.abs(to64(o.view(T, n_q * d))) @ np.abs(to64(wo)).T
    _check(xr, ref_x, s_abs_o, 2.0 ** -12, "layer: out projection")

"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: torch's
scaled_dot_product_attention (an independent formulation of softmax
attention), complex-number rotation, closed forms, the pages' printed values
(``tests/golden``), brute-force counting, and algebraic invariants. Together
they are chosen so a dropped term, a wrong sign or index, or a transposed
operand in the oracle fails at least one of them.
"""

import cmath
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention, bf16, kvcache, rope, yarn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
YARN = dict(theta=150000.0, s=32.0, orig_ctx=4096, alpha=1.0, beta=32.0)


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16_normal(rng, shape, std=1.0):
    return bf16.round_bf16(rng.standard_normal(shape) * std)


# --------------------------------------------------------------------------
# bf16 rounding
# --------------------------------------------------------------------------

def test_bf16_matches_torch_rne_on_fp32_values():
    rng = _rng(0)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-30, 30, 200000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(bf16.round_bf16(x.astype(np.float64)), ref)


def test_bf16_ties_to_even_and_range():
    one = 1.0
    half_ulp = 2.0 ** -8          # bf16 ulp at 1 is 2**-7
    assert bf16.round_bf16(np.array([one + half_ulp]))[0] == 1.0            # tie -> even
    assert bf16.round_bf16(np.array([one + 3 * half_ulp]))[0] == 1.0 + 2 ** -6  # tie -> even (up)
    assert bf16.round_bf16(np.array([one + half_ulp * 1.0000001]))[0] == 1.0 + 2 ** -7
    assert np.isinf(bf16.round_bf16(np.array([3.5e38]))[0])
    assert bf16.round_bf16(np.array([2.0 ** -133]))[0] == 2.0 ** -133       # smallest subnormal
    assert bf16.round_bf16(np.array([2.0 ** -135]))[0] == 0.0
    bits = bf16.to_bits(np.array([1.0, -2.0]))
    assert list(bits) == [0x3F80, 0xC000]


# --------------------------------------------------------------------------
# YaRN / NTK-by-parts
# --------------------------------------------------------------------------

def test_concentration_value():
    # ln 32 = 5 ln 2, so 0.1 * ln 32 + 1 = 0.5 * ln 2 + 1.
    assert yarn.concentration(32.0) == pytest.approx(1.0 + 0.5 * 0.6931471805599453, abs=1e-15)
    assert yarn.concentration(1.0) == 1.0


@pytest.mark.parametrize("d,theta", [(64, 150000.0), (96, 150000.0), (128, 10000.0)])
def test_cutpoints_are_where_the_rotation_count_equals_alpha_beta(d, theta):
    # The page's NTK-by-parts ratio r(i) = L * theta_i / (2 pi), theta_i = b^(-2i/d),
    # counts the rotations of pair i over the training context. The cutpoints
    # are where r equals beta (fast side) and alpha (slow side).
    L = YARN["orig_ctx"]
    i_beta, i_alpha = yarn.cutpoints(d, theta, L, YARN["alpha"], YARN["beta"])

    def r(i):
        return L * theta ** (-2.0 * i / d) / (2.0 * math.pi)

    assert r(i_beta) == pytest.approx(YARN["beta"], rel=1e-12)
    assert r(i_alpha) == pytest.approx(YARN["alpha"], rel=1e-12)
    assert i_beta < i_alpha


def test_inv_freq_three_regimes():
    d, theta, s = 64, YARN["theta"], YARN["s"]
    inv = yarn.inv_freq(d, theta, s, YARN["orig_ctx"], YARN["alpha"], YARN["beta"])
    i_beta, i_alpha = yarn.cutpoints(d, theta, YARN["orig_ctx"], YARN["alpha"], YARN["beta"])
    # Independent base schedule: theta_i = b^(-2i/d) via exp/log.
    base = np.array([math.exp(-2.0 * i / d * math.log(theta)) for i in range(d // 2)])
    fast = np.arange(d // 2) <= math.floor(i_beta)
    slow = np.arange(d // 2) >= math.ceil(i_alpha)
    np.testing.assert_allclose(inv[fast], base[fast], rtol=1e-13)       # untouched
    np.testing.assert_allclose(inv[slow], base[slow] / s, rtol=1e-13)   # stretched by s
    # Between the cutpoints the blend weight falls linearly from 1 to 0.
    mid = ~(fast | slow)
    w = (inv[mid] - base[mid] / s) / (base[mid] - base[mid] / s)
    assert np.all((w > 0) & (w < 1))
    np.testing.assert_allclose(np.diff(w, 2), 0.0, atol=1e-12)
    np.testing.assert_allclose(np.diff(w), -1.0 / (i_alpha - i_beta), rtol=1e-10)
    # Derived at d=64, theta=150000, L=4096, alpha=1, beta=32: pairs 0..8 fast, 18..31 slow.
    assert fast.sum() == 9 and slow.sum() == 14
    # Slower clocks (higher i) never rotate faster.
    assert np.all(np.diff(inv) < 0)


def test_tables_as_complex_rotation():
    d = 64
    c, s = yarn.tables(300, d, YARN["theta"], YARN["s"], YARN["orig_ctx"], YARN["alpha"], YARN["beta"])
    inv = yarn.inv_freq(d, YARN["theta"], YARN["s"], YARN["orig_ctx"], YARN["alpha"], YARN["beta"])
    conc = yarn.concentration(YARN["s"])
    for t in (0, 1, 7, 299):
        for i in (0, 5, 20, 31):
            z = conc * cmath.exp(1j * t * inv[i])
            assert c[t, i] == pytest.approx(z.real, abs=1e-13)
            assert s[t, i] == pytest.approx(z.imag, abs=1e-13)


def _rope_tables(max_pos, d):
    return yarn.tables(max_pos, d, YARN["theta"], YARN["s"], YARN["orig_ctx"], YARN["alpha"], YARN["beta"])


def test_rope_matches_complex_multiplication_half_split():
    d = 64
    c, s = _rope_tables(500, d)
    inv = yarn.inv_freq(d, YARN["theta"], YARN["s"], YARN["orig_ctx"], YARN["alpha"], YARN["beta"])
    conc = yarn.concentration(YARN["s"])
    rng = _rng(1)
    x = rng.standard_normal(d)
    for p in (0, 3, 499):
        y = rope.rotate(x, p, c, s)
        z = (x[: d // 2] + 1j * x[d // 2:]) * conc * np.exp(1j * p * inv)
        np.testing.assert_allclose(y[: d // 2], z.real, atol=1e-12)
        np.testing.assert_allclose(y[d // 2:], z.imag, atol=1e-12)


def test_rope_at_zero_is_concentration_times_identity_and_preserves_norm():
    d = 96
    c, s = _rope_tables(1000, d)
    conc = yarn.concentration(YARN["s"])
    rng = _rng(2)
    x = rng.standard_normal(d)
    np.testing.assert_allclose(rope.rotate(x, 0, c, s), conc * x, atol=1e-14)
    for p in (1, 17, 999):
        y = rope.rotate(x, p, c, s)
        # every pair keeps its length, scaled by conc
        np.testing.assert_allclose(np.hypot(y[:48], y[48:]), conc * np.hypot(x[:48], x[48:]), rtol=1e-12)


def test_rope_scores_depend_only_on_relative_position():
    d = 64
    c, s = _rope_tables(140000, d)
    rng = _rng(3)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    ref = rope.rotate(q, 10, c, s) @ rope.rotate(k, 3, c, s)
    for shift in (1, 1000, 131000):
        got = rope.rotate(q, 10 + shift, c, s) @ rope.rotate(k, 3 + shift, c, s)
        assert got == pytest.approx(ref, rel=1e-9, abs=1e-9)
    # ... and do change with the relative position
    assert abs(rope.rotate(q, 11, c, s) @ rope.rotate(k, 3, c, s) - ref) > 1e-3


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

def _case(seed, B, T, n_q, n_kv, d, off=0, sink_std=1.0):
    rng = _rng(seed)
    n = off + T
    q = _bf16_normal(rng, (B, T, n_q, d))
    K = _bf16_normal(rng, (B, n, n_kv, d))
    V = _bf16_normal(rng, (B, n, n_kv, d))
    sinks = rng.standard_normal(n_q) * sink_std
    return q, K, V, sinks


def _sdpa(q, K, V, off, window, scale, sinks=None):
    """torch SDPA in fp64 with an additive mask; the sink becomes one extra
    key with k = 0, v = 0 and additive bias sigma_h."""
    B, T, n_q, d = q.shape
    n_kv = K.shape[2]
    qm = n_q // n_kv
    n = off + T
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)                       # B,H,T,d
    kt = torch.from_numpy(K[:, :n]).permute(0, 2, 1, 3).repeat_interleave(qm, dim=1)
    vt = torch.from_numpy(V[:, :n]).permute(0, 2, 1, 3).repeat_interleave(qm, dim=1)
    i = torch.arange(T)[:, None] + off
    j = torch.arange(n)[None, :]
    ok = j <= i
    if window > 0:
        ok = ok & (j > i - window)
    bias = torch.zeros(T, n, dtype=torch.float64).masked_fill(~ok, float("-inf"))
    bias = bias.expand(B, n_q, T, n).clone()
    if sinks is not None:
        kt = torch.cat([kt, torch.zeros(B, n_q, 1, d, dtype=torch.float64)], dim=2)
        vt = torch.cat([vt, torch.zeros(B, n_q, 1, d, dtype=torch.float64)], dim=2)
        sb = torch.from_numpy(np.asarray(sinks, dtype=np.float64))[None, :, None, None].expand(B, n_q, T, 1)
        bias = torch.cat([bias, sb], dim=3)
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=bias, scale=scale)
    return out.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("window", [0, 16, 5])
@pytest.mark.parametrize("off", [0, 37])
def test_no_sink_equals_textbook_sdpa(window, off):
    q, K, V, _ = _case(10 + window + off, 2, 23, 8, 2, 64, off)
    out, _ = attention.sink_attention(q, K, V, None, off, window, 0.125)
    np.testing.assert_allclose(out, _sdpa(q, K, V, off, window, 0.125), atol=1e-12)


@pytest.mark.parametrize("window", [0, 16])
@pytest.mark.parametrize("off", [0, 50])
def test_sink_equals_sdpa_with_a_zero_key_biased_by_sigma(window, off):
    q, K, V, sinks = _case(20 + window + off, 2, 19, 8, 4, 32, off, sink_std=2.0)
    out, _ = attention.sink_attention(q, K, V, sinks, off, window, 0.2)
    np.testing.assert_allclose(out, _sdpa(q, K, V, off, window, 0.2, sinks), atol=1e-12)


def test_sink_closed_form_against_plain_lse():
    q, K, V, sinks = _case(30, 1, 12, 4, 2, 16, 5)
    plain, lse_plain = attention.sink_attention(q, K, V, None, 5, 0, 0.3)
    with_sink, lse_sink = attention.sink_attention(q, K, V, sinks, 5, 0, 0.3)
    # out_sink = out_plain / (1 + e^{sigma - LSE_plain});  LSE_sink = logaddexp(LSE_plain, sigma)
    factor = 1.0 / (1.0 + np.exp(sinks[None, :, None] - lse_plain))        # [B, H, T]
    np.testing.assert_allclose(with_sink, plain * factor.transpose(0, 2, 1)[..., None], atol=1e-12)
    np.testing.assert_allclose(lse_sink, np.logaddexp(lse_plain, sinks[None, :, None]), atol=1e-12)


def test_sink_limits_and_first_row():
    q, K, V, sinks = _case(40, 1, 6, 4, 4, 8, 0)
    big = np.full(4, 1e4)
    out, _ = attention.sink_attention(q, K, V, big, 0, 0, 0.5)
    assert np.abs(out).max() == 0.0
    out, lse = attention.sink_attention(q, K, V, np.full(4, np.inf), 0, 0, 0.5)
    assert np.abs(out).max() == 0.0 and np.all(np.isinf(lse))
    # Row p = 0 sees only key 0: out = v0 * sigmoid(s00 - sigma).
    out, _ = attention.sink_attention(q, K, V, sinks, 0, 0, 0.5)
    for h in range(4):
        s00 = 0.5 * float(q[0, 0, h] @ K[0, 0, h])
        w = 1.0 / (1.0 + math.exp(sinks[h] - s00))
        np.testing.assert_allclose(out[0, 0, h], V[0, 0, h] * w, atol=1e-13)


def test_wide_window_equals_full_causal():
    q, K, V, sinks = _case(50, 1, 30, 8, 2, 16, 10)
    full, _ = attention.sink_attention(q, K, V, sinks, 10, 0, 0.25)
    wide, _ = attention.sink_attention(q, K, V, sinks, 10, 40, 0.25)
    np.testing.assert_array_equal(full, wide)
    narrow, _ = attention.sink_attention(q, K, V, sinks, 10, 39, 0.25)
    assert np.abs(narrow - full).max() > 1e-6   # W = off+T-1 drops key 0 for the last row


def test_gqa_equals_mha_with_replicated_kv_and_qmult_one_is_mha():
    q, K, V, sinks = _case(60, 2, 9, 8, 2, 16, 3)
    gqa, _ = attention.sink_attention(q, K, V, sinks, 3, 0, 0.25)
    Kr = np.repeat(K, 4, axis=2)   # head h -> kv head h // 4 (contiguous groups)
    Vr = np.repeat(V, 4, axis=2)
    mha, _ = attention.sink_attention(q, Kr, Vr, sinks, 3, 0, 0.25)
    np.testing.assert_allclose(gqa, mha, atol=1e-14)
    # q_mult = 1 against the SDPA formulation with no expansion
    np.testing.assert_allclose(mha, _sdpa(q, Kr, Vr, 3, 0, 0.25, sinks), atol=1e-12)
    # grouping is contiguous (h // q_mult), not interleaved (h % n_kv)
    Ki = np.tile(K, (1, 1, 4, 1))
    Vi = np.tile(V, (1, 1, 4, 1))
    inter, _ = attention.sink_attention(q, Ki, Vi, sinks, 3, 0, 0.25)
    assert np.abs(inter - gqa).max() > 1e-3


def test_band_counts_brute_force():
    # The study note's band i - W < j <= i admits exactly min(p + 1, W) keys.
    for off, T, W in ((0, 64, 16), (100, 20, 16), (5, 3, 128)):
        ok = attention.allowed_mask(off, T, off + T, W)
        for i in range(T):
            p = off + i
            cnt = sum(1 for j in range(off + T) if p - W < j <= p)
            assert ok[i].sum() == cnt == min(p + 1, W)
            assert ok[i, p] and (p - W < 0 or not ok[i, p - W])
        assert attention.allowed_pairs(off, T, W) == ok.sum()
    assert attention.allowed_pairs(0, 8192, 0) == 8192 * 8193 // 2


def test_layer_alternation():
    assert [attention.layer_window(l) for l in range(4)] == [128, 0, 128, 0]


def test_mask_probe_counts():
    # q = 0 and sigma = 0 make every allowed score 0, so the weights are 1/(n+1);
    # with v_j = e_{j mod d}, out_c * (n + 1) counts the allowed keys j = c mod d.
    B, T, n_q, n_kv, d, off = 1, 40, 2, 1, 8, 13
    q = np.zeros((B, T, n_q, d))
    n = off + T
    V = np.zeros((B, n, n_kv, d))
    V[0, np.arange(n), 0, np.arange(n) % d] = 1.0
    K = _bf16_normal(_rng(7), (B, n, n_kv, d))
    for W in (0, 16):
        out, lse = attention.sink_attention(q, K, V, np.zeros(n_q), off, W, 0.3)
        for i in range(T):
            p = off + i
            js = [j for j in range(n) if j <= p and (W == 0 or j > p - W)]
            cnt = np.bincount(np.array(js) % d, minlength=d)
            np.testing.assert_allclose(out[0, i, 0] * (len(js) + 1), cnt, atol=1e-12)
            assert lse[0, 0, i] == pytest.approx(math.log(len(js) + 1), abs=1e-13)


def _cos_sin(max_pos, d):
    return yarn.stored_tables(max_pos, d, YARN["theta"], YARN["s"], YARN["orig_ctx"], YARN["alpha"], YARN["beta"])


@pytest.mark.parametrize("window", [0, 16])
def test_handoff_prefill_equals_prefix_then_decode(window):
    # Prefill of T rows in one call == prefill of P rows, then T-P one-row
    # decode calls (the prefill -> decode diagonal), also after a restore.
    rng = _rng(70 + window)
    B, T, P, n_q, n_kv, d = 2, 24, 17, 4, 2, 32
    c, s = _cos_sin(64, d)
    q = _bf16_normal(rng, (B, T, n_q, d))
    k = _bf16_normal(rng, (B, T, n_kv, d))
    v = _bf16_normal(rng, (B, T, n_kv, d))
    sinks = rng.standard_normal(n_q)
    full_cache = kvcache.KVCache(B, 64, n_kv, d)
    full, _ = attention.attend_step(full_cache, q, k, v, sinks, window, 0.2, c, s)

    cache = kvcache.KVCache(B, 64, n_kv, d)
    head, _ = attention.attend_step(cache, q[:, :P], k[:, :P], v[:, :P], sinks, window, 0.2, c, s)
    np.testing.assert_allclose(head, full[:, :P], atol=1e-12)
    snap = cache.snapshot()
    for rep in range(2):
        for t in range(P, T):
            o, _ = attention.attend_step(cache, q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1],
                                         sinks, window, 0.2, c, s)
            np.testing.assert_allclose(o[:, 0], full[:, t], atol=1e-12)
        np.testing.assert_array_equal(cache.K[:, :T], full_cache.K[:, :T])
        cache.restore(snap)
        assert cache.offset == P


def test_handoff_detects_post_append_offset_bug():
    # Using the post-append offset for the mask (the named off-by-one) lets
    # every decode row see one extra (future, unwritten) key: the oracle's
    # pre-append convention must differ from it.
    q, K, V, sinks = _case(80, 1, 1, 2, 1, 8, 9)
    good, _ = attention.sink_attention(q, K, V, sinks, 9, 4, 0.5)
    K2 = np.concatenate([K, np.ones_like(K[:, :1])], axis=1)
    V2 = np.concatenate([V, np.ones_like(V[:, :1])], axis=1)
    bad, _ = attention.sink_attention(q, K2, V2, sinks, 10, 4, 0.5)
    assert np.abs(good - bad).max() > 1e-3


# --------------------------------------------------------------------------
# KV cache
# --------------------------------------------------------------------------

def test_kv_bytes_matches_printed_example():
    g = json.load(open(os.path.join(GOLDEN, "kv_cache_example.json")))
    n = kvcache.kv_bytes(g["L"], g["B"], g["T"], g["H_kv"], g["d"], g["dtype_bytes"])
    assert abs(n / 2 ** 30 - g["printed_gib"]) < g["printed_gib_resolution"]
    assert n == 6 * 2 ** 30   # the printed figure is exact here


def test_windowed_kv_reduction_matches_printed_ratios():
    g = json.load(open(os.path.join(GOLDEN, "kv_window_reduction.json")))
    L = 24
    Lw = int(L * g["windowed_fraction"])
    for pt in g["points"]:
        full = kvcache.kv_bytes(L, 1, pt["T"], 8, 96, 2)
        ring = kvcache.kv_bytes_windowed(L, Lw, g["window"], 1, pt["T"], 8, 96, 2)
        ratio = full / ring
        assert abs(ratio - pt["printed_ratio"]) < pt["resolution"], (pt, ratio)
        assert ratio == 2 * pt["T"] / (pt["T"] + g["window"])   # the closed form for half the layers windowed


def test_gqa_shapes_match_printed_values():
    g = json.load(open(os.path.join(GOLDEN, "gqa_shapes.json")))
    assert g["d_h"] * (g["n_q"] + 2 * g["n_kv"]) == g["qkv_width"]
    assert g["n_q"] // g["n_kv"] == g["q_mult"]
    assert g["n_kv"] / g["n_q"] == g["kv_fraction_of_mha"]
    assert 1.0 / math.sqrt(g["d_h"]) == g["sm_scale"]
    from sink_augmented_gqa_b200.workloads import CONFIGS
    c = CONFIGS["gptoss_prefill"]
    assert (c.n_q, c.n_kv, c.d, c.sm_scale, c.window) == (g["n_q"], g["n_kv"], g["d_h"], g["sm_scale"], g["window"])
    assert c.d * (c.n_q + 2 * c.n_kv) == g["qkv_width"]


def test_cache_append_snapshot_restore_and_stale():
    c = kvcache.KVCache(1, 10, 1, 2)
    rows = lambda t, val: np.full((1, t, 1, 2), float(val))
    c.append(rows(4, 1), rows(4, 1))
    s4 = c.snapshot()
    c.append(rows(3, 2), rows(3, 2))
    s7 = c.snapshot()
    c.restore(s4)
    assert c.offset == 4
    c.append(rows(1, 3), rows(1, 3))          # overwrites row 4 < s7.offset
    with pytest.raises(kvcache.StaleSnapshotError):
        c.restore(s7)
    c.restore(s4)                              # still fine: rows < 4 untouched
    assert c.offset == 4 and np.all(c.K[0, :4] == 1)
    with pytest.raises(kvcache.CapacityError):
        c.append(rows(7, 0), rows(7, 0))
    assert c.offset == 4

"""Pins of the FP8 (e4m3) row quantiser in ``oracle/fp8.py``.

The format is OCP FP8 E4M3 ("fn"); PyTorch's ``float8_e4m3fn`` dtype is an
independent implementation of it and serves as the library routine the
decode table and the rounding reduce to. Saturation, the per-row scale and
the dequantisation bound are checked against closed forms and brute force.
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import fp8, kvcache
from oracle.bf16 import round_bf16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _torch_table():
    return (torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn)
            .float().numpy().astype(np.float64))


def test_decode_table_matches_library():
    ours = fp8.e4m3_value(np.arange(256, dtype=np.uint8))
    lib = _torch_table()
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    ok = ~np.isnan(lib)
    assert np.array_equal(ours[ok], lib[ok])
    # the two NaN patterns of the "fn" variant, and the largest finite value
    assert np.flatnonzero(np.isnan(ours)).tolist() == [0x7F, 0xFF]
    assert ours[0x7E] == 448.0 and ours[0xFE] == -448.0
    assert ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def test_bits_round_trip():
    b = np.array([i for i in range(256) if i not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(fp8.e4m3_bits(fp8.e4m3_value(b)), b)


def test_rounding_matches_library_inside_range():
    rng = np.random.default_rng(7)
    y = np.concatenate([
        rng.uniform(-448, 448, 50000),
        rng.standard_normal(50000) * rng.choice([1e-4, 1e-2, 1.0, 30.0], 50000),
    ])
    vals = np.unique(fp8.e4m3_value(np.arange(256, dtype=np.uint8)))
    vals = vals[np.isfinite(vals)]
    mids = (vals[1:] + vals[:-1]) / 2          # exact ties: round half to even
    y = np.concatenate([y, mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf)])
    y32 = y.astype(np.float32)
    lib = torch.from_numpy(y32).to(torch.float8_e4m3fn)
    ours = fp8.e4m3_round(y32.astype(np.float64))
    assert np.array_equal(ours, lib.float().numpy().astype(np.float64))
    assert np.array_equal(fp8.e4m3_bits(ours), lib.view(torch.uint8).numpy())


def test_rounding_is_nearest_by_brute_force():
    vals = fp8.e4m3_value(np.arange(256, dtype=np.uint8))
    finite = np.isfinite(vals)
    codes = np.arange(256)[finite]
    table = vals[finite]
    rng = np.random.default_rng(3)
    y = rng.uniform(-500, 500, 4000) * rng.choice([1e-3, 0.1, 1.0], 4000)
    r = fp8.e4m3_round(y)
    for yi, ri in zip(y, r):
        d = np.abs(table - min(max(yi, -448.0), 448.0))
        best = table[d == d.min()]
        if len(best) > 1:   # a tie: the even mantissa (lowest code bit clear) wins
            even = [t for t, c in zip(table, codes) if t in best and (c & 1) == 0]
            best = np.array(even)
        assert ri in best, (yi, ri, best)


def test_saturation():
    y = np.array([448.0, 449.0, 463.9, 464.0, 479.0, 1e6, 3.0e38])
    assert np.all(fp8.e4m3_round(y) == 448.0)
    assert np.all(fp8.e4m3_round(-y) == -448.0)


def test_signed_zero_and_subnormals():
    assert fp8.e4m3_bits(fp8.e4m3_round(np.array([-0.0])))[0] == 0x80
    assert fp8.e4m3_bits(fp8.e4m3_round(np.array([0.0])))[0] == 0x00
    # below half the smallest subnormal rounds to zero; half of it is a tie to 0
    assert fp8.e4m3_round(np.array([2.0 ** -10]))[0] == 0.0
    assert fp8.e4m3_round(np.array([2.0 ** -10 * 1.01]))[0] == 2.0 ** -9
    assert fp8.e4m3_round(np.array([3 * 2.0 ** -10]))[0] == 2 * 2.0 ** -9   # tie -> even


def test_worked_row():
    """A row worked by hand (format definition above)."""
    with open(os.path.join(GOLDEN, "fp8_row_example.json")) as f:
        ex = json.load(f)
    x = np.array([ex["row"]], dtype=np.float64)
    assert np.array_equal(round_bf16(x), x)
    codes, scale = fp8.quantize_rows(x)
    assert codes[0].tolist() == ex["codes"]
    assert float(scale[0]) == float(np.float32(ex["scale_num"]) / np.float32(ex["scale_den"]))


def test_row_amax_maps_to_448_and_error_bound():
    rng = np.random.default_rng(11)
    x = round_bf16(rng.standard_normal((300, 64)) * rng.choice([1e-30, 1e-3, 1.0, 1e4], (300, 1)))
    codes, scale = fp8.quantize_rows(x)
    deq = fp8.dequantize_rows(codes, scale)
    for r in range(x.shape[0]):
        j = np.argmax(np.abs(x[r]))
        assert abs(fp8.e4m3_value(codes[r, j])) == 448.0
        assert np.sign(fp8.e4m3_value(codes[r, j])) == np.sign(x[r, j])
    # |x - deq| <= half an e4m3 step of |x| / scale (relative 2**-4 for
    # normals, 2**-10 absolute in code units below 2**-6), plus the fp32
    # division's own rounding, all in units of the scale.
    s = scale.astype(np.float64)[:, None]
    bound = np.maximum(np.abs(x) * 2.0 ** -4, s * 2.0 ** -10) + np.abs(x) * 2.0 ** -22
    assert np.all(np.abs(x - deq) <= bound)


def test_zero_row():
    codes, scale = fp8.quantize_rows(np.zeros((2, 3, 64)))
    assert np.all(codes == 0) and np.all(scale == 0)
    assert np.all(fp8.dequantize_rows(codes, scale) == 0)


def test_fp8_kv_bytes_halve_the_printed_bf16_example():
    """The "KV CACHE" estimator's worked example (24 layers, one sequence,
    131,072 tokens, 8 KV heads, d = 64) is 6.0 GiB in bf16; one byte per
    element halves it, and the row scales add 2 * 4 bytes per (layer, token,
    KV head)."""
    bf16 = kvcache.kv_bytes(24, 1, 131072, 8, 64, 2)
    assert bf16 / 2 ** 30 == pytest.approx(6.0)
    f8 = fp8.kv_bytes_fp8(24, 1, 131072, 8, 64)
    assert f8 - 2 * 24 * 131072 * 8 * 4 == bf16 // 2
    assert f8 / 2 ** 30 == pytest.approx(3.1875)


def test_quantised_step_is_lossless_on_representable_rows():
    """Rows whose values are E4M3 values times a power of two whose row
    maximum is 448 times that power quantise without loss, so the quantised
    step reduces to the bf16 step (pre-rotated inputs, no RoPE)."""
    from oracle import attention as oatt
    rng = np.random.default_rng(5)
    B, T, n_kv, q_mult, d = 1, 9, 2, 2, 64
    table = fp8.e4m3_value(np.arange(256, dtype=np.uint8))
    table = table[np.isfinite(table)]

    def rows(shape):
        x = rng.choice(table, size=shape)
        x[..., 0] = 448.0                      # row maximum: scale = 2**e exactly
        e = rng.integers(-8, 8, size=shape[:-1])[..., None]
        return np.ldexp(x, e)

    k, v = rows((B, T, n_kv, d)), rows((B, T, n_kv, d))
    q = round_bf16(rng.standard_normal((B, T, n_kv * q_mult, d)))
    sinks = rng.standard_normal(n_kv * q_mult)
    c1 = kvcache.KVCache(B, T, n_kv, d)
    c2 = kvcache.KVCache(B, T, n_kv, d)
    o1, l1 = oatt.attend_step(c1, q, k, v, sinks, 0, 0.125, None, None, rope_fused=False)
    o2, l2 = fp8.attend_step_fp8(c2, q, k, v, sinks, 0, 0.125, None, None, rope_fused=False)
    assert np.array_equal(c1.K, c2.K) and np.array_equal(c1.V, c2.V)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    # ... while a value between two E4M3 steps is rounded: 0.3 * 448 = 134.4
    # lies between the steps 128 and 144 of its binade
    k2 = k.copy()
    k2[0, 0, 0, 1] = round_bf16(0.3 * k[0, 0, 0, 0])
    c3 = kvcache.KVCache(B, T, n_kv, d)
    fp8.attend_step_fp8(c3, q, k2, v, sinks, 0, 0.125, None, None, rope_fused=False)
    assert c3.K[0, 0, 0, 1] != k2[0, 0, 0, 1]
    assert c3.K[0, 0, 0, 1] / k[0, 0, 0, 0] * 448 in (128.0, 144.0)

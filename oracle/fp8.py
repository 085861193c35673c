"""FP8 (e4m3) KV-cache rows with one fp32 scale per row: quantise, dequantise.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

The MoE-Xtend README lists quantisation-aware long-context runs, with KV and
its dequantisation first because decode is bandwidth bound ("ROADMAP"), and
its "KV CACHE" estimator charges ``dtype_bytes`` per stored element. The pages
fix neither the 8-bit format nor the scale granularity; the reading taken
here is the plainest self-contained one:

* format: OCP FP8 E4M3 ("fn" variant) -- sign, 4 exponent bits with bias 7,
  3 mantissa bits; normals ``2**(e-7) * (1 + m/8)`` for e = 1..15 except the
  all-ones pattern (NaN), subnormals ``m/8 * 2**-6``; largest finite 448; no
  infinities.
* granularity: one fp32 scale per stored row, i.e. per (sequence, position,
  KV head), so an append never has to revisit earlier rows.
* the rows quantised are the bf16 rows the bf16 cache would store (K after
  rotation, V as given); with ``amax`` their largest magnitude,
  ``scale = fl32(amax / 448)`` and ``code = e4m3(fl32(x / scale))``, where
  ``fl32`` is one correctly rounded fp32 division and ``e4m3`` rounds to the
  nearest value, ties to even, saturating at +/-448. A row of zeros stores
  scale 0 and codes 0.
* the value a reader sees is ``e4m3_value(code) * scale`` (exact in fp64).

Both divisions are carried out in fp32 because they decide an integer code:
the oracle takes that decision in the same precision as the kernel.
"""

import numpy as np

from .attention import sink_attention
from .bf16 import round_bf16
from .rope import rotate_bsh

E4M3_MAX = 448.0
# Smallest normal binade exponent and the subnormal quantum (2**-9).
_E4M3_MIN_NORMAL_EXP = -6
_E4M3_SUBNORMAL_QUANTUM_EXP = -9


def e4m3_round(y):
    """Round finite fp64 values to the nearest E4M3 value, ties to even,
    saturating to +/-448. Returns fp64 (every element E4M3-representable)."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    # |y| = f * 2**e with 0.5 <= f < 1: the binade [2**(e-1), 2**e) holds 8
    # steps of 2**(e-4); below 2**-6 the quantum is fixed at 2**-9.
    _, e = np.frexp(np.where(a == 0, 1.0, a))
    q_exp = np.maximum(e - 4, _E4M3_SUBNORMAL_QUANTUM_EXP)
    r = np.ldexp(np.rint(np.ldexp(a, -q_exp)), q_exp)   # np.rint: half to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, y)


def e4m3_bits(v):
    """uint8 E4M3 patterns of E4M3-representable fp64 values (sign of zero kept)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    sign = np.signbit(v).astype(np.uint32) << 7
    _, e = np.frexp(np.where(a == 0, 1.0, a))
    unbiased = e - 1                                   # a = 2**unbiased * (1 + m/8)
    normal = (a != 0) & (unbiased >= _E4M3_MIN_NORMAL_EXP)
    exp_field = np.where(normal, unbiased + 7, 0)
    mant = np.where(normal,
                    np.ldexp(a, -unbiased) * 8 - 8,          # (1 + m/8) * 8 - 8
                    np.ldexp(a, -_E4M3_SUBNORMAL_QUANTUM_EXP))  # m = a / 2**-9
    m_int = np.rint(mant).astype(np.int64)
    if np.any(np.abs(mant - m_int) != 0) or np.any(m_int > 7) or np.any(exp_field > 15):
        raise ValueError("value not representable in E4M3")
    return (sign | (exp_field.astype(np.uint32) << 3) | m_int.astype(np.uint32)).astype(np.uint8)


def e4m3_value(bits):
    """fp64 values of uint8 E4M3 patterns (NaN for the two NaN patterns)."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    s = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    mag = np.where(e == 0, np.ldexp(m.astype(np.float64), _E4M3_SUBNORMAL_QUANTUM_EXP),
                   np.ldexp(1.0 + m / 8.0, e - 7))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return s * mag


def quantize_rows(x):
    """Quantise the last axis of bf16-representable fp64 ``x`` row by row.

    Returns ``(codes uint8, same shape as x; scales float32, x.shape[:-1])``.
    """
    x = np.asarray(x, dtype=np.float64)
    x32 = x.astype(np.float32)                              # exact for bf16 values
    amax = np.max(np.abs(x32), axis=-1)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)  # one fp32 division
    safe = np.where(scale == 0, np.float32(1), scale)
    y = (x32 / safe[..., None]).astype(np.float32)          # one fp32 division
    codes = e4m3_bits(e4m3_round(y.astype(np.float64)))
    codes = np.where((scale == 0)[..., None], np.uint8(0), codes).astype(np.uint8)
    return codes, scale


def dequantize_rows(codes, scales):
    """fp64 values a reader of the quantised cache sees: code value * scale."""
    return e4m3_value(codes) * np.asarray(scales, dtype=np.float64)[..., None]


def attend_step_fp8(cache, q, k, v, sinks, window, sm_scale, cos_tab, sin_tab, rope_fused=True):
    """One call of the hot path on a quantised cache.

    As ``attention.attend_step``, except that the rows stored are the
    quantised bf16 rows (K after rotation) and every key and value read --
    the call's own new rows included -- is the dequantised row. ``cache`` is
    an fp64 ``kvcache.KVCache`` holding dequantised rows.
    """
    off = cache.offset
    if rope_fused:
        q_rot = rotate_bsh(q, off, cos_tab, sin_tab)
        k_rot = rotate_bsh(k, off, cos_tab, sin_tab)
    else:
        q_rot = round_bf16(q)
        k_rot = round_bf16(k)
    kc, ks = quantize_rows(k_rot)
    vc, vs = quantize_rows(round_bf16(v))
    cache.append(dequantize_rows(kc, ks), dequantize_rows(vc, vs))
    return sink_attention(q_rot, cache.K, cache.V, sinks, off, window, sm_scale)


def kv_bytes_fp8(L, B, T, H_kv, d):
    """The "KV CACHE" estimator with one byte per element, plus the fp32 row
    scales this format adds (one per K row and one per V row)."""
    return 2 * L * B * T * H_kv * d * 1 + 2 * L * B * T * H_kv * 4

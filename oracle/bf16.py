"""Exact fp64 -> bfloat16 rounding (round to nearest, ties to even).

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

bfloat16 keeps fp32's 8-bit exponent and 8 significant bits. The cache on the
pages stores rotated K and unrotated V in bf16 (GPT-OSS-Lite visual guide,
"Overview": decode stores rotated K and unchanged V; MoE-Xtend README, "KV
CACHE": ``dtype_bytes`` is 2 for bf16), so the oracle rounds every stored
value with this function, directly from fp64 (no intermediate fp32 step, which
could double-round).
"""

import numpy as np

# Largest finite bf16: (2 - 2**-7) * 2**127.
BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127
# Quantum of the bf16 subnormal range: 2**-133.
_SUBNORMAL_QUANTUM_EXP = -133


def round_bf16(x):
    """Round fp64 array ``x`` to the nearest bf16 value (ties to even).

    Returns an fp64 array whose every element is exactly representable in
    bf16. NaN stays NaN; values beyond the bf16 range become +/-inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    finite = np.isfinite(x)
    xf = x[finite]
    # x = m * 2**e with 0.5 <= |m| < 1, so the bf16 quantum at x is 2**(e-8),
    # but never finer than the subnormal quantum.
    _, e = np.frexp(xf)
    q_exp = np.maximum(e - 8, _SUBNORMAL_QUANTUM_EXP)
    scaled = np.ldexp(xf, -q_exp)            # exact: power-of-two scaling
    r = np.ldexp(np.rint(scaled), q_exp)     # np.rint rounds half to even
    r = np.where(np.abs(r) > BF16_MAX, np.copysign(np.inf, r), r)
    out[finite] = r
    out[~finite] = x[~finite]
    return out


def bf16_ulp(x):
    """Spacing of bf16 values at |x| (the quantum of the binade holding x)."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    _, e = np.frexp(np.where(x == 0, 1.0, x))
    q = np.ldexp(1.0, np.maximum(e - 8, _SUBNORMAL_QUANTUM_EXP))
    return np.where(x == 0, np.ldexp(1.0, _SUBNORMAL_QUANTUM_EXP), q)


def to_bits(x):
    """bf16 bit patterns (uint16) of fp64 values that are bf16-representable."""
    x = np.asarray(x, dtype=np.float64)
    f32 = x.astype(np.float32)  # exact for bf16-representable values
    return (f32.view(np.uint32) >> 16).astype(np.uint16)


def from_bits(bits):
    """fp64 values of uint16 bf16 bit patterns."""
    bits = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)

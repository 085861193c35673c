"""YaRN / NTK-by-parts rotary tables in fp64.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

Restates the MoE-Xtend README, "ROPE + SCALING" (base schedule
``theta_i = b^(-2i/d)`` and the YaRN + NTK-by-parts pseudocode), in the order
the page gives its steps:

1. ``freqs[i] = base ** (i / (d/2))`` for pair index ``i < d/2``;
2. ``extrapolation = 1/freqs`` (original RoPE), ``interpolation = 1/(s*freqs)``
   (context stretched by ``s``);
3. ``concentration = 0.1 * ln(s) + 1`` (the MoE-Xtend project page gives the
   same expression; the log is natural);
4. cutpoints in pair-index space
   ``i_beta  = (d/2) * ln(L / (beta  * 2 pi)) / ln(base)`` and
   ``i_alpha = (d/2) * ln(L / (alpha * 2 pi)) / ln(base)``;
5. ``ramp = (i - i_beta) / (i_alpha - i_beta)``, ``mask = 1 - clip(ramp, 0, 1)``
   (1 in the fast region, 0 in the slow region);
6. ``inv_freq = interpolation * (1 - mask) + extrapolation * mask``;
7. ``cos = concentration * cos(t * inv_freq)``, ``sin = concentration *
   sin(t * inv_freq)`` at integer position ``t``.

Reading: the tables are indexed by the exact global position ``t`` with no
wrap (the "never reset" position contract of the same README's "DESIGN
CONTRACTS" wins over the ``% max_content_length`` lookup in its implementation
note), so callers size them to at least ``offset + T`` rows. The library
stores the tables as fp32; ``stored_tables`` gives that rounding.
"""

import math

import numpy as np


def concentration(s):
    """YaRN attention-temperature factor 0.1*ln(s) + 1 (applied to cos and sin)."""
    return 0.1 * math.log(s) + 1.0


def cutpoints(d, theta, orig_ctx, alpha, beta):
    """Continuous NTK-by-parts cutpoints (i_beta, i_alpha) in pair-index space."""
    half = d / 2.0
    i_beta = half * math.log(orig_ctx / (beta * 2.0 * math.pi)) / math.log(theta)
    i_alpha = half * math.log(orig_ctx / (alpha * 2.0 * math.pi)) / math.log(theta)
    return i_beta, i_alpha


def inv_freq(d, theta, s, orig_ctx, alpha, beta):
    """fp64 inverse frequencies, one per rotary pair (length d/2)."""
    half = d // 2
    i = np.arange(half, dtype=np.float64)
    freqs = np.power(float(theta), i / half)
    extrapolation = 1.0 / freqs
    interpolation = 1.0 / (s * freqs)
    i_beta, i_alpha = cutpoints(d, theta, orig_ctx, alpha, beta)
    ramp = (i - i_beta) / (i_alpha - i_beta)
    mask = 1.0 - np.clip(ramp, 0.0, 1.0)
    return interpolation * (1.0 - mask) + extrapolation * mask


def tables(max_pos, d, theta, s, orig_ctx, alpha, beta):
    """fp64 cos/sin tables [max_pos, d/2] with the concentration folded in."""
    inv = inv_freq(d, theta, s, orig_ctx, alpha, beta)
    t = np.arange(max_pos, dtype=np.float64)
    ang = np.outer(t, inv)
    conc = concentration(s)
    return conc * np.cos(ang), conc * np.sin(ang)


def stored_tables(max_pos, d, theta, s, orig_ctx, alpha, beta):
    """The tables as the library stores them: fp64 values rounded to fp32."""
    c, sn = tables(max_pos, d, theta, s, orig_ctx, alpha, beta)
    return c.astype(np.float32), sn.astype(np.float32)

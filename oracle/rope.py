"""Rotary embedding of Q and K at the global position, fp64.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

* Positions: query/key row ``i`` of a call that starts at cache offset ``off``
  sits at ``t = off + i`` (MoE-Xtend README, "DESIGN CONTRACTS": absolute
  position monotonicity; "TOKEN STREAM (DECODE)": RoPE uses the global token
  index).
* Only Q and K are rotated; V is untouched (GQA Attention study note, "How it
  works"; GPT-OSS-Lite visual guide: decode stores rotated K and unchanged V).
* Pair convention (a reading, not printed on the pages): half-split pairs
  ``(x[c], x[c + d/2])``, rotated by the angle of pair ``c``::

      x1' = x1*cos - x2*sin,   x2' = x2*cos + x1*sin

  with ``cos``/``sin`` already scaled by the YaRN concentration.
* The rotated values are rounded to bf16 because that is how they are stored
  in the cache and fed to the bf16 score contraction.
"""

import numpy as np

from .bf16 import round_bf16


def rotate(x, positions, cos_tab, sin_tab):
    """Exact fp64 rotation of ``x[..., d]`` at integer ``positions``.

    ``positions`` broadcasts against ``x.shape[:-1]``; ``cos_tab``/``sin_tab``
    are [max_pos, d/2] tables (any float dtype, used as fp64 values).
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    pos = np.asarray(positions)
    c = np.asarray(cos_tab, dtype=np.float64)[pos]
    s = np.asarray(sin_tab, dtype=np.float64)[pos]
    x1 = x[..., :half]
    x2 = x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def rotate_bsh(x, offset, cos_tab, sin_tab):
    """Rotate a [B, T, H, d] block whose row i sits at position offset + i,
    then round to bf16 (the stored precision)."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[1]
    pos = (offset + np.arange(T))[None, :, None]
    pos = np.broadcast_to(pos, x.shape[:-1])
    return round_bf16(rotate(x, pos, cos_tab, sin_tab))

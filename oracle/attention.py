"""Sink-augmented grouped-query attention, written out in fp64.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

Definition restated from the pages:

* Scores (GQA Attention study note, "How it works"):
  ``s[t, h, j] = <q[t, h], k[j, g(h)]> * sm_scale + M[t, j]`` where the query
  head ``h = g * q_mult + m`` shares KV head ``g = h // q_mult``
  (``q_mult = n_q / n_kv``), and ``M`` is 0 on allowed keys, -inf elsewhere.
* Mask, aligned to the KV cache (MoE-Xtend README, "ATTENTION STACK", mask
  engineering): with ``offset`` the number of cached rows before this call,
  query row ``i`` sits at ``p = offset + i`` and may see key row ``j`` iff
  ``j <= p`` (causal) and, on windowed layers, ``j > p - W``. The band edge
  follows the study note's ``i - W < j <= i`` (W keys); the README's
  ``k >= offset + q - W`` would admit W + 1 keys -- the oracle takes the
  study note's reading.
* Which layers are windowed (same README, implementation notes):
  ``layer_idx % 2 == 0`` -> band of W = 128, odd layers full causal.
* Sink (same README, "Sink bias"; the study note): one learned logit
  ``sigma_h`` per query head is appended as an extra softmax column after
  masking, and its weight is dropped after normalisation::

      alpha_j = e^{s_j} / (sum_{allowed k} e^{s_k} + e^{sigma_h})
      out[t, h] = sum_j alpha_j v[j, g(h)]

  ``sigma_h`` is a raw logit: it is not multiplied by ``sm_scale``.
  ``sigma_h = -inf`` is ordinary softmax attention.
* ``lse[t, h] = ln(sum_{allowed} e^{s_j} + e^{sigma_h})`` is returned too.

The oracle computes each (b, h) with one library matmul for the scores and one
for the PV mix, and an explicit mask -- no blocking, no online softmax, no
split-KV.
"""

import numpy as np

from .bf16 import round_bf16
from .rope import rotate_bsh

DEFAULT_WINDOW = 128


def layer_window(layer_idx, window=DEFAULT_WINDOW):
    """Even layers use the sliding band, odd layers are full causal (0)."""
    return window if layer_idx % 2 == 0 else 0


def allowed_mask(offset, T, n_keys, window):
    """Boolean [T, n_keys]: query row i (position offset+i) may see key j."""
    p = offset + np.arange(T)[:, None]
    j = np.arange(n_keys)[None, :]
    ok = j <= p
    if window > 0:
        ok &= j > p - window
    return ok


def sink_attention(q_rot, k_cache, v_cache, sinks, offset, window, sm_scale):
    """Attention of T query rows against cache rows [0, offset + T).

    q_rot:   [B, T, n_q, d]  rotated queries (fp64 values of bf16)
    k_cache: [B, >= offset+T, n_kv, d]  rotated keys (rows < offset+T used)
    v_cache: [B, >= offset+T, n_kv, d]
    sinks:   [n_q] sink logits, or None for no sink (-inf)
    Returns (out [B, T, n_q, d], lse [B, n_q, T]) in fp64.
    """
    q_rot = np.asarray(q_rot, dtype=np.float64)
    B, T, n_q, d = q_rot.shape
    n_kv = k_cache.shape[2]
    assert n_q % n_kv == 0
    q_mult = n_q // n_kv
    n_keys = offset + T
    if sinks is None:
        sinks = np.full(n_q, -np.inf)
    sinks = np.asarray(sinks, dtype=np.float64)
    ok = allowed_mask(offset, T, n_keys, window)
    out = np.zeros((B, T, n_q, d))
    lse = np.zeros((B, n_q, T))
    for b in range(B):
        for h in range(n_q):
            g = h // q_mult
            K = np.asarray(k_cache[b, :n_keys, g, :], dtype=np.float64)
            V = np.asarray(v_cache[b, :n_keys, g, :], dtype=np.float64)
            s = (q_rot[b, :, h, :] @ K.T) * sm_scale
            s = np.where(ok, s, -np.inf)
            sig = sinks[h]
            if sig == np.inf:
                # The sink takes all the mass: every kept weight is 0.
                lse[b, h] = np.inf
                continue
            m = np.maximum(s.max(axis=1), sig)
            e = np.exp(s - m[:, None])
            l = e.sum(axis=1) + np.exp(sig - m)
            out[b, :, h, :] = (e @ V) / l[:, None]
            lse[b, h] = m + np.log(l)
    return out, lse


def attend_step(cache, q, k, v, sinks, window, sm_scale, cos_tab, sin_tab,
                rope_fused=True):
    """One prefill (T >= 1) or decode (T == 1) call of the hot path.

    At the cache's current offset: rotate q and k (when ``rope_fused``),
    append rotated k and v to the cache, then attend the T query rows to
    cache rows [0, offset + T). Returns (out, lse) in fp64.
    """
    off = cache.offset
    if rope_fused:
        q_rot = rotate_bsh(q, off, cos_tab, sin_tab)
        k_rot = rotate_bsh(k, off, cos_tab, sin_tab)
    else:
        q_rot = round_bf16(q)
        k_rot = round_bf16(k)
    cache.append(k_rot, round_bf16(v))
    return sink_attention(q_rot, cache.K, cache.V, sinks, off, window, sm_scale)


def allowed_pairs(offset, T, window):
    """Number of (query, key) pairs the mask admits for one (b, h)."""
    p = offset + np.arange(T, dtype=np.int64)
    n = p + 1
    if window > 0:
        n = np.minimum(n, window)
    return int(n.sum())

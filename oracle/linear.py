"""Pre-norm RMSNorm with the fused qkv projection, and the out projection with
the residual add, written out in fp64.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

GQA Attention study note, "How it works": the residual stream x [T, 2880]
passes through RMSNorm, then one fused linear ``qkv`` of width
``d_h (n_q + 2 n_kv) = 5120``, split into Q, K, V; after attention the 64
heads are flattened to [T, 4096], projected by the linear ``out`` back to
[T, 2880] and added to the residual, ``x <- x + out(o)``. Both linears are
bf16 ``nn.Linear`` layers with bias (the note: an official-code detail).
RMSNorm is not spelled out on the pages; the reading taken is the usual one
with a learned per-channel gain::

    rmsnorm(x)[t, k] = x[t, k] / sqrt(mean_k' x[t, k']^2 + eps) * gamma[k]

with ``eps`` a parameter (1e-5 in the benchmarks). ``nn.Linear`` computes
``y = x W^T + b`` with ``W`` stored [out_features, in_features].
"""

import numpy as np


def rmsnorm(x, gamma, eps):
    """fp64 RMSNorm over the last axis."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(gamma, dtype=np.float64)


def linear(x, w, b=None):
    """``x W^T + b`` (nn.Linear), fp64."""
    y = np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T
    if b is not None:
        y = y + np.asarray(b, dtype=np.float64)
    return y


def qkv_proj(x, gamma, eps, w, b):
    """The fused qkv projection of the pre-normed residual stream."""
    return linear(rmsnorm(x, gamma, eps), w, b)


def out_proj(o, w, b, x):
    """The out projection added to the residual stream: x + o W^T + b."""
    return np.asarray(x, dtype=np.float64) + linear(o, w, b)


def split_qkv(y, n_q, n_kv, d_h):
    """Split the fused [..., d_h (n_q + 2 n_kv)] output into q [..., n_q, d_h],
    k and v [..., n_kv, d_h] (q columns first, then k, then v)."""
    lead = y.shape[:-1]
    q = y[..., : n_q * d_h].reshape(*lead, n_q, d_h)
    k = y[..., n_q * d_h: (n_q + n_kv) * d_h].reshape(*lead, n_kv, d_h)
    v = y[..., (n_q + n_kv) * d_h:].reshape(*lead, n_kv, d_h)
    return q, k, v

"""Append-only KV cache with snapshot / restore, and the KV-byte estimator.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

From the MoE-Xtend README:

* "NOTATION": cache per layer ``K, V: [B, T_cache, H_kv, d]``.
* "KV CACHE", implementation notes: ``Cache.extend`` writes new K/V at rows
  ``[offset : offset + t]`` and then increments ``offset``; caches are
  preallocated; ``Cache.snapshot()`` / ``Cache.restore()`` give "prefill
  once, decode many".
* "DESIGN CONTRACTS": append-only -- decode adds exactly one row per layer
  per step and the offset advances once per append.
* "KV CACHE", memory scaling: ``bytes = 2 * L * B * T * H_kv * d *
  dtype_bytes`` (the factor 2 is K and V).

Reading of snapshot / restore (the pages name the methods only): the state is
the offset plus the rows below it. Because the cache is append-only, restoring
only has to roll the offset back, provided no row below the snapshot's offset
was written after the snapshot was taken. That can only happen when a restore
to a lower offset is followed by an append; such a snapshot is stale and
restoring it is an error.
"""

import numpy as np


class CapacityError(ValueError):
    pass


class StaleSnapshotError(ValueError):
    pass


class Snapshot:
    def __init__(self, offset, seq):
        self.offset = offset
        self.seq = seq


class KVCache:
    """fp64 model of one layer's cache [B, cap, n_kv, d]."""

    def __init__(self, B, cap, n_kv, d):
        self.B, self.cap, self.n_kv, self.d = B, cap, n_kv, d
        self.K = np.zeros((B, cap, n_kv, d))
        self.V = np.zeros((B, cap, n_kv, d))
        self.offset = 0
        self.seq = 0
        self.appends = []  # (seq of the append, first row written)

    def append(self, k_rot, v):
        """Write [B, T, n_kv, d] rows at [offset, offset + T), then advance."""
        T = k_rot.shape[1]
        if self.offset + T > self.cap:
            raise CapacityError(f"offset {self.offset} + {T} rows > capacity {self.cap}")
        o = self.offset
        self.K[:, o:o + T] = k_rot
        self.V[:, o:o + T] = v
        self.seq += 1
        self.appends.append((self.seq, o))
        self.offset = o + T

    def snapshot(self):
        return Snapshot(self.offset, self.seq)

    def restore(self, snap):
        for s, first_row in self.appends:
            if s > snap.seq and first_row < snap.offset:
                raise StaleSnapshotError(
                    f"row {first_row} < snapshot offset {snap.offset} was rewritten after the snapshot")
        self.offset = snap.offset
        self.seq += 1


def kv_bytes(L, B, T, H_kv, d, dtype_bytes):
    """Back-of-the-envelope KV-cache size in bytes (K and V, all layers)."""
    return 2 * L * B * T * H_kv * d * dtype_bytes


def kv_bytes_windowed(L, L_windowed, window, B, T, H_kv, d, dtype_bytes):
    """The same when L_windowed of the L layers keep only their last `window`
    tokens (MoE-Xtend project page, "Results": windowed layers cache 128
    tokens regardless of sequence length)."""
    rows = (L - L_windowed) * T + L_windowed * min(T, window)
    return 2 * B * rows * H_kv * d * dtype_bytes

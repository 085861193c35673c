"""CPU-only checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before any launch."""

import ctypes
import os
import re

import pytest

from sink_augmented_gqa_b200 import build as sbuild
from sink_augmented_gqa_b200 import sinkattn as S

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "sinkattn.h")


@pytest.fixture(scope="module")
def L():
    sbuild.build()
    return S.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sa_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert sorted(S.EXPORTS) == names


def test_status_strings(L):
    for code, name in S.STATUS.items():
        assert L.sa_status_string(code).decode() == name


def _fake_cache(B=1, cap=100, n_kv=2, d=64):
    c = S._KVCache()
    # Host-only bookkeeping never dereferences these (16-byte aligned) addresses.
    st = L_.sa_kv_cache_init(ctypes.byref(c), ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000), B, cap, n_kv, d)
    return c, st


L_ = None


@pytest.fixture(autouse=True)
def _bind(L):
    global L_
    L_ = L


def test_cache_init_validation(L):
    c, st = _fake_cache()
    assert st == 0 and c.offset == 0 and c.cap == 100
    c2 = S._KVCache()
    assert L.sa_kv_cache_init(ctypes.byref(c2), ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000), 1, 10, 2, 80) == 2
    assert L.sa_kv_cache_init(ctypes.byref(c2), None, ctypes.c_void_p(0x20000), 1, 10, 2, 64) == 1
    assert L.sa_kv_cache_init(ctypes.byref(c2), ctypes.c_void_p(0x10008), ctypes.c_void_p(0x20000), 1, 10, 2, 64) == 1


def test_snapshot_restore_host_logic(L):
    c, _ = _fake_cache()
    # Simulate the bookkeeping the library does after appends: appends are
    # device work, so drive the fields the way an append would (offset moves,
    # high-water mark, overwrite log) via restore/snapshot only.
    c.offset, c.high_water, c.seq = 40, 40, 1
    s40 = S._Snapshot()
    assert L.sa_kv_snapshot(ctypes.byref(c), ctypes.byref(s40)) == 0
    assert (s40.offset, s40.seq, s40.cap) == (40, 1, 100)
    c.offset, c.high_water, c.seq = 60, 60, 2
    s60 = S._Snapshot()
    L.sa_kv_snapshot(ctypes.byref(c), ctypes.byref(s60))
    assert L.sa_kv_restore(ctypes.byref(c), ctypes.byref(s40)) == 0 and c.offset == 40 and c.seq == 3
    assert L.sa_kv_restore(ctypes.byref(c), ctypes.byref(s60)) == 0 and c.offset == 60   # nothing rewritten
    # record an overwrite at row 45 after s60 (what an append from offset 45 logs)
    c.seq = 5
    c.log_seq[0], c.log_row[0], c.log_len = 5, 45, 1
    assert L.sa_kv_restore(ctypes.byref(c), ctypes.byref(s60)) == 5      # stale
    assert L.sa_kv_restore(ctypes.byref(c), ctypes.byref(s40)) == 0      # rows < 40 untouched
    other = S._Snapshot()
    other.cache_id, other.offset, other.seq, other.cap = 0x999, 10, 1, 100
    assert L.sa_kv_restore(ctypes.byref(c), ctypes.byref(other)) == 1


def _args(offset=0, T=4, n_q=4, B=1, window=0):
    a = S._AttnArgs()
    for f in ("q", "k", "v", "out"):
        setattr(a, f, 0x30000)
    for f in ("q_strides", "k_strides", "v_strides", "out_strides"):
        setattr(a, f, S._I64x3(4096, 256, 64))
    a.B, a.T, a.n_q, a.offset, a.window, a.sm_scale = B, T, n_q, offset, window, 0.125
    a.rope_fused = 0
    return a


def test_attention_argument_errors_return_before_launch(L):
    c, _ = _fake_cache(cap=100)
    stream = ctypes.c_void_p(0)
    assert L.sa_attn_prefill(ctypes.byref(c), ctypes.byref(_args(offset=3)), stream) == 4     # offset mismatch
    assert L.sa_attn_prefill(ctypes.byref(c), ctypes.byref(_args(T=101)), stream) == 3        # capacity
    assert L.sa_attn_prefill(ctypes.byref(c), ctypes.byref(_args(n_q=5)), stream) == 2        # n_q % n_kv
    assert L.sa_attn_prefill(ctypes.byref(c), ctypes.byref(_args(B=2)), stream) == 1          # batch mismatch
    a = _args()
    a.q_strides = S._I64x3(4096, 256, 60)                                                       # misaligned head stride
    assert L.sa_attn_prefill(ctypes.byref(c), ctypes.byref(a), stream) == 1
    a = _args()
    a.rope_fused = 1                                                                            # no tables
    assert L.sa_attn_prefill(ctypes.byref(c), ctypes.byref(a), stream) == 1
    assert L.sa_attn_prefill(ctypes.byref(c), ctypes.byref(_args(T=0)), stream) == 0          # empty: no-op
    assert c.offset == 0
    assert L.sa_attn_decode(ctypes.byref(c), ctypes.byref(_args(T=2)), None, 0, stream) == 1  # decode is T == 1
    assert L.sa_attn_decode(ctypes.byref(c), ctypes.byref(_args(n_q=20, T=1)), None, 0, stream) == 2  # q_mult > 8
    assert c.offset == 0


def test_workspace_size_bound(L):
    n = L.sa_attn_decode_workspace_size(1, 64, 8, 64)
    assert n >= (512 + 8) * 8 * 66 * 4
    assert L.sa_attn_decode_workspace_size(0, 64, 8, 64) == 0


def test_table_argument_errors(L):
    p = ctypes.c_void_p(0x40000)
    assert L.sa_yarn_rope_tables(p, p, 0, 64, 150000.0, 32.0, 4096, 1.0, 32.0, None) == 1
    assert L.sa_yarn_rope_tables(p, p, 10, 63, 150000.0, 32.0, 4096, 1.0, 32.0, None) == 1
    assert L.sa_yarn_rope_tables(p, p, 10, 64, 150000.0, 32.0, 4096, 32.0, 1.0, None) == 1   # alpha >= beta


def test_prefill_event_hook_arguments(L):
    inv = [k for k, v in S.STATUS.items() if v == "SA_ERR_INVALID_ARG"][0]
    assert L.sa_set_prefill_events(ctypes.c_void_p(0x10), None) == inv
    assert L.sa_set_prefill_events(None, ctypes.c_void_p(0x10)) == inv
    assert L.sa_set_prefill_events(None, None) == 0


def test_ring_cache_host_rules(L):
    ring = lambda cap, window: (lambda c: (c, L.sa_kv_cache_init_ring(ctypes.byref(c), ctypes.c_void_p(0x10000),
                                                                      ctypes.c_void_p(0x20000), 1, cap, 2, 64,
                                                                      window)))(S._KVCache())
    assert ring(768, 128)[1] == 0
    assert ring(700, 128)[1] == 2           # capacity not a multiple of 384
    assert ring(384, 500)[1] == 2           # band wider than the ring
    assert ring(768, 0)[1] == 1
    c, _ = ring(768, 128)
    assert c.ring == 128
    stream = ctypes.c_void_p(0)
    # calls on a ring must use its band; a prefill must fit T + W - 1 rows
    assert L.sa_attn_prefill(ctypes.byref(c), ctypes.byref(_args(T=4, window=0)), stream) == 1
    assert L.sa_attn_prefill(ctypes.byref(c), ctypes.byref(_args(T=4, window=64)), stream) == 1
    assert L.sa_attn_prefill(ctypes.byref(c), ctypes.byref(_args(T=642, window=128)), stream) == 3
    # positions are unbounded: an offset beyond cap is valid
    c.offset, c.high_water, c.seq = 5000, 5000, 3
    s = S._Snapshot()
    assert L.sa_kv_snapshot(ctypes.byref(c), ctypes.byref(s)) == 0 and s.offset == 5000
    # rows [offset - 127, offset) of the snapshot survive while the ring has
    # not advanced past offset + cap - 127
    c.offset = c.high_water = 5000 + 768 - 127
    assert L.sa_kv_restore(ctypes.byref(c), ctypes.byref(s)) == 0 and c.offset == 5000
    c.offset = c.high_water = 5000 + 768 - 126
    assert L.sa_kv_restore(ctypes.byref(c), ctypes.byref(s)) == 5       # stale


def test_fp8_cache_host_rules(L):
    def init(cap=96, ks=0x30000, vs=0x40000, window=0):
        c = S._KVCache()
        st = L.sa_kv_cache_init_fp8(ctypes.byref(c), ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000),
                                    ctypes.c_void_p(ks), ctypes.c_void_p(vs), 1, cap, 2, 64, window)
        return c, st
    c, st = init()
    # the struct layout agrees with the header: the library wrote these fields
    assert st == 0 and c.kv_dtype == S.KV_FP8_E4M3 and c.k_scale == 0x30000 and c.v_scale == 0x40000
    assert c.ring == 0
    assert init(ks=0)[1] == 1                  # scales required
    assert init(vs=0x40008)[1] == 1            # 16-byte aligned scales
    assert init(cap=100)[1] == 2               # capacity a multiple of 16
    assert init(cap=768, window=128)[1] == 0   # ring FP8 cache
    assert init(cap=400, window=128)[1] == 2   # ring rule: multiple of 384
    assert init(window=-1)[1] == 1
    stream = ctypes.c_void_p(0)
    # prefill is not provided on an FP8 cache; the check comes before any launch
    assert L.sa_attn_prefill(ctypes.byref(c), ctypes.byref(_args(T=4, window=0)), stream) == 9
    # a bf16 descriptor with an unknown format is rejected
    b, _ = _fake_cache()
    b.kv_dtype = 7
    assert L.sa_kv_snapshot(ctypes.byref(b), ctypes.byref(S._Snapshot())) == 1


def _bwd_args(**kw):
    p = 0x40000   # 16-byte aligned; never dereferenced: every case below fails validation
    a = S._BwdArgs()
    for name in ("q", "k", "v", "out", "d_out"):
        setattr(a, name, p)
        setattr(a, name + "_strides", S._I64x3(4096, 256, 64))
    a.lse = a.dq = a.dk = a.dv = a.dsinks = p
    a.sinks = None
    a.B, a.T, a.n_q, a.n_kv, a.d, a.window, a.sm_scale = 1, 16, 4, 2, 64, 0, 0.125
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_backward_argument_errors_return_before_launch(L):
    codes = {v: k for k, v in S.STATUS.items()}
    ws = ctypes.c_void_p(0x80000)
    need = L.sa_attn_backward_workspace_size(1, 16, 4)
    assert need >= 2 * 384 * 4 * 4                                  # D and lse rows padded to 384 (whole query tiles)
    assert L.sa_attn_backward_workspace_size(0, 16, 4) == 0

    def call(a, nbytes=need):
        return L.sa_attn_backward(ctypes.byref(a), ws, nbytes, None)
    assert call(_bwd_args(B=0)) == codes["SA_ERR_INVALID_ARG"]
    assert call(_bwd_args(d=80)) == codes["SA_ERR_SHAPE"]
    assert call(_bwd_args(n_kv=3)) == codes["SA_ERR_SHAPE"]           # 4 % 3
    assert call(_bwd_args(n_q=8200, n_kv=8200)) == codes["SA_ERR_SHAPE"]  # row pass sums n_q floats in smem
    assert call(_bwd_args(sm_scale=0.0)) == codes["SA_ERR_INVALID_ARG"]
    a = _bwd_args()
    a.q_strides = S._I64x3(4096, 256, 60)                             # misaligned head stride
    assert call(a) == codes["SA_ERR_INVALID_ARG"]
    assert call(_bwd_args(), nbytes=need - 256) == codes["SA_ERR_WORKSPACE"]


def test_prefill_schedule_slots_wrap(L):
    """The prefill's schedule counters: eager calls cycle through 64 slots and
    wrap (the 65th reuses the 1st, after waiting for it on the device);
    captured calls cycle through 64 others, so a graph never shares one with
    an eager call."""
    eager = [L.sa_prefill_sched_slot(i, 0) for i in range(200)]
    graph = [L.sa_prefill_sched_slot(i, 1) for i in range(200)]
    assert eager[:64] == list(range(64)) and graph[:64] == list(range(64, 128))
    assert all(eager[i] == eager[i % 64] for i in range(200))
    assert all(graph[i] == graph[i % 64] for i in range(200))
    assert not set(eager) & set(graph)
    assert L.sa_prefill_sched_slot(2 ** 64 - 1, 0) == (2 ** 64 - 1) % 64


def test_backward_workspace_rows_pad_to_whole_query_tiles(L):
    # D and lse * log2(e) rows per (sequence, query head), padded to a
    # multiple of 384 entries (whole query tiles of 64, 96 and 128 rows),
    # fp32, the total rounded up to 256 bytes
    for B, T, n_q in [(1, 1, 1), (1, 383, 4), (1, 384, 4), (1, 385, 4), (3, 4096, 8), (2, 8192, 64)]:
        Tp = (T + 383) // 384 * 384
        want = (2 * B * n_q * Tp * 4 + 255) // 256 * 256
        assert L.sa_attn_backward_workspace_size(B, T, n_q) == want, (B, T, n_q)

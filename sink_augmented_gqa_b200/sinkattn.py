"""Thin Python binding of libsinkattn (ctypes).

Argument marshalling only: every computation runs in the CUDA library
(``libsinkattn.so``, built in-tree by ``sink_augmented_gqa_b200.build``).
PyTorch supplies device memory and the current stream. There is no CPU or
PyTorch fallback: if the library is missing, every call raises.

Names mirror the C ABI in ``include/sinkattn.h`` without the ``sa_`` prefix:
``yarn_rope_tables``, ``rope_apply_qk``, ``KVCache`` (``kv_append``,
``kv_snapshot``, ``kv_restore``), ``attn_prefill``, ``attn_decode``.
"""

import ctypes
import os
import struct
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsinkattn.so")
KV_LOG_CAP = 32

STATUS = {
    0: "SA_OK", 1: "SA_ERR_INVALID_ARG", 2: "SA_ERR_SHAPE", 3: "SA_ERR_CAPACITY",
    4: "SA_ERR_OFFSET_MISMATCH", 5: "SA_ERR_STALE_SNAPSHOT", 6: "SA_ERR_CUDA",
    7: "SA_ERR_TIMEOUT", 8: "SA_ERR_WORKSPACE", 9: "SA_ERR_UNSUPPORTED",
}

KV_BF16, KV_FP8_E4M3 = 0, 1


class SinkAttnError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        self.name = STATUS.get(code, f"status {code}")
        super().__init__(f"{where}: {self.name}")


class _KVCache(ctypes.Structure):
    _fields_ = [
        ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("B", ctypes.c_int32), ("cap", ctypes.c_int32), ("n_kv", ctypes.c_int32), ("d", ctypes.c_int32),
        ("offset", ctypes.c_int64), ("seq", ctypes.c_int64), ("high_water", ctypes.c_int64),
        ("log_seq", ctypes.c_int64 * KV_LOG_CAP), ("log_row", ctypes.c_int64 * KV_LOG_CAP),
        ("log_len", ctypes.c_int32), ("log_floor_seq", ctypes.c_int64), ("log_floor_row", ctypes.c_int64),
        ("ring", ctypes.c_int32), ("kv_dtype", ctypes.c_int32),
        ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
    ]


class _BwdArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("q_strides", ctypes.c_int64 * 3),
        ("k", ctypes.c_void_p), ("k_strides", ctypes.c_int64 * 3),
        ("v", ctypes.c_void_p), ("v_strides", ctypes.c_int64 * 3),
        ("out", ctypes.c_void_p), ("out_strides", ctypes.c_int64 * 3),
        ("d_out", ctypes.c_void_p), ("d_out_strides", ctypes.c_int64 * 3),
        ("lse", ctypes.c_void_p), ("sinks", ctypes.c_void_p),
        ("B", ctypes.c_int32), ("T", ctypes.c_int32), ("n_q", ctypes.c_int32), ("n_kv", ctypes.c_int32),
        ("d", ctypes.c_int32), ("window", ctypes.c_int32), ("sm_scale", ctypes.c_float),
        ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p), ("dv", ctypes.c_void_p), ("dsinks", ctypes.c_void_p),
    ]


class _Snapshot(ctypes.Structure):
    _fields_ = [("cache_id", ctypes.c_uint64), ("offset", ctypes.c_int64),
                ("seq", ctypes.c_int64), ("cap", ctypes.c_int32)]


_I64x3 = ctypes.c_int64 * 3



class _AttnArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("q_strides", _I64x3),
        ("k", ctypes.c_void_p), ("k_strides", _I64x3),
        ("v", ctypes.c_void_p), ("v_strides", _I64x3),
        ("sinks", ctypes.c_void_p),
        ("B", ctypes.c_int32), ("T", ctypes.c_int32), ("n_q", ctypes.c_int32),
        ("offset", ctypes.c_int64), ("window", ctypes.c_int32), ("sm_scale", ctypes.c_float),
        ("rope_fused", ctypes.c_int32),
        ("cos", ctypes.c_void_p), ("sin", ctypes.c_void_p), ("max_pos", ctypes.c_int32),
        ("out", ctypes.c_void_p), ("out_strides", _I64x3),
        ("lse", ctypes.c_void_p),
    ]

# sa_attn_args packed in one step (C layout, native alignment): the per-call
# marshalling of a decode step is on the host's critical path when layers are
# launched one by one, and building the ctypes structure field by field costs
# several times more than the packing.
_ATTN_FMT = "@P3qP3qP3qPiiiqifiPPiP3qP"
assert struct.calcsize(_ATTN_FMT) == ctypes.sizeof(_AttnArgs)
_tls = threading.local()


# Every symbol include/sinkattn.h declares.
EXPORTS = (
    "sa_status_string", "sa_yarn_rope_tables", "sa_rope_apply_qk", "sa_kv_cache_init",
    "sa_kv_append", "sa_kv_snapshot", "sa_kv_restore", "sa_attn_prefill", "sa_attn_decode",
    "sa_attn_decode_workspace_size", "sa_get_device_status", "sa_set_wait_limit",
    "sa_attn_decode_static", "sa_set_prefill_events", "sa_kv_cache_init_ring",
    "sa_kv_cache_init_fp8", "sa_rmsnorm_fold_weight", "sa_qkv_proj", "sa_out_proj",
    "sa_attn_backward", "sa_attn_backward_workspace_size", "sa_prefill_sched_slot",
)

_lib = None


def lib():
    """The loaded library (loads it on first use; raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libsinkattn.so not found at {LIB_PATH}; build it with "
                "`python -m sink_augmented_gqa_b200.build` (there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, f64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        P = ctypes.POINTER
        L.sa_status_string.restype = ctypes.c_char_p
        L.sa_status_string.argtypes = [ctypes.c_int]
        L.sa_yarn_rope_tables.argtypes = [vp, vp, i32, i32, f64, f64, i32, f64, f64, vp]
        L.sa_rope_apply_qk.argtypes = [vp, P(i64), vp, P(i64), i32, i32, i32, i32, i32, i64, vp, vp, i32, vp]
        L.sa_kv_cache_init.argtypes = [P(_KVCache), vp, vp, i32, i32, i32, i32]
        L.sa_kv_cache_init_ring.argtypes = [P(_KVCache), vp, vp, i32, i32, i32, i32, i32]
        L.sa_kv_append.argtypes = [P(_KVCache), vp, P(i64), vp, P(i64), i32, vp]
        L.sa_kv_snapshot.argtypes = [P(_KVCache), P(_Snapshot)]
        L.sa_kv_restore.argtypes = [P(_KVCache), P(_Snapshot)]
        L.sa_attn_prefill.argtypes = [P(_KVCache), P(_AttnArgs), vp]
        L.sa_attn_decode.argtypes = [P(_KVCache), P(_AttnArgs), vp, ctypes.c_size_t, vp]
        L.sa_attn_decode_static.argtypes = [P(_KVCache), P(_AttnArgs), vp]
        L.sa_attn_decode_workspace_size.restype = ctypes.c_size_t
        L.sa_attn_decode_workspace_size.argtypes = [i32, i32, i32, i32]
        L.sa_get_device_status.argtypes = [P(i32)]
        L.sa_set_wait_limit.argtypes = [i64]
        L.sa_set_prefill_events.argtypes = [vp, vp]
        L.sa_kv_cache_init_fp8.argtypes = [P(_KVCache), vp, vp, vp, vp, i32, i32, i32, i32, i32]
        f32 = ctypes.c_float
        L.sa_rmsnorm_fold_weight.argtypes = [vp, i64, vp, vp, i64, i32, i32, vp]
        L.sa_qkv_proj.argtypes = [vp, i64, vp, i64, vp, f32, vp, i64, i32, i32, i32, vp]
        L.sa_out_proj.argtypes = [vp, i64, vp, i64, vp, vp, i64, i32, i32, i32, vp]
        L.sa_attn_backward.argtypes = [P(_BwdArgs), vp, ctypes.c_size_t, vp]
        L.sa_attn_backward_workspace_size.restype = ctypes.c_size_t
        L.sa_attn_backward_workspace_size.argtypes = [i32, i32, i32]
        L.sa_prefill_sched_slot.argtypes = [ctypes.c_uint64, i32]
        for name in EXPORTS:
            if name not in ("sa_status_string", "sa_attn_decode_workspace_size",
                            "sa_attn_backward_workspace_size"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(code, where):
    if code != 0:
        raise SinkAttnError(code, where)


def _stream(t=None):
    dev = t.device if t is not None else torch.device("cuda")
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _raw_stream(t):
    """The current stream of t's device as a raw handle (no Stream object)."""
    return torch._C._cuda_getCurrentRawStream(t.device.index)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _strides(t):
    """Element strides [batch, token, head] of a [B, T, H, d] view (d contiguous)."""
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("expected a [B, T, H, d] tensor with a contiguous last dimension")
    return _I64x3(t.stride(0), t.stride(1), t.stride(2))


def _require_bf16_cuda(name, t):
    if t.dtype != torch.bfloat16 or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA bf16 tensor")


# ---------------------------------------------------------------------------
# Public API
# ---------------------------------------------------------------------------

def yarn_rope_tables(max_pos, d, theta=150000.0, scaling=32.0, orig_ctx=4096, alpha=1.0, beta=32.0,
                     device="cuda"):
    """fp32 cos/sin tables [max_pos, d/2] (concentration folded in)."""
    cos = torch.empty((max_pos, d // 2), dtype=torch.float32, device=device)
    sin = torch.empty_like(cos)
    _check(lib().sa_yarn_rope_tables(_ptr(cos), _ptr(sin), max_pos, d, float(theta), float(scaling),
                                     int(orig_ctx), float(alpha), float(beta), _stream(cos)),
           "sa_yarn_rope_tables")
    return cos, sin


def rope_apply_qk(q, k, offset, cos, sin):
    """Rotate q [B,T,n_q,d] and k [B,T,n_kv,d] in place at positions offset + t."""
    ref = q if q is not None else k
    B, T, _, d = ref.shape
    n_q = q.shape[2] if q is not None else 0
    n_kv = k.shape[2] if k is not None else 0
    qs = _strides(q) if q is not None else _I64x3(0, 0, 0)
    ks = _strides(k) if k is not None else _I64x3(0, 0, 0)
    _check(lib().sa_rope_apply_qk(_ptr(q), qs, _ptr(k), ks, B, T, n_q, n_kv, d, int(offset),
                                  _ptr(cos), _ptr(sin), cos.shape[0], _stream(ref)),
           "sa_rope_apply_qk")


class Snapshot:
    def __init__(self, raw):
        self.raw = raw

    @property
    def offset(self):
        return self.raw.offset


class KVCache:
    """One layer's KV cache, head-major [B, n_kv, cap, d] (torch-owned device
    memory): bf16 rows, or with ``fp8=True`` e4m3 codes (uint8) plus fp32
    row scales ``k_scale``/``v_scale`` [B, n_kv, cap]. ``k_rows(start,
    stop)`` views rows as [B, T, n_kv, d]; ``k_scales(start, stop)`` the
    scales as [B, T, n_kv]."""

    def __init__(self, B, cap, n_kv, d, device="cuda", k=None, v=None, ring=0, fp8=False):
        shape = (B, n_kv, cap, d)
        dt = torch.uint8 if fp8 else torch.bfloat16
        self.k = k if k is not None else torch.zeros(shape, dtype=dt, device=device)
        self.v = v if v is not None else torch.zeros(shape, dtype=dt, device=device)
        assert tuple(self.k.shape) == shape and self.k.is_contiguous() and self.v.is_contiguous()
        assert self.k.dtype == dt and self.v.dtype == dt
        self.raw = _KVCache()
        self.fp8 = bool(fp8)
        if fp8:
            self.k_scale = torch.zeros((B, n_kv, cap), dtype=torch.float32, device=self.k.device)
            self.v_scale = torch.zeros((B, n_kv, cap), dtype=torch.float32, device=self.k.device)
            _check(lib().sa_kv_cache_init_fp8(ctypes.byref(self.raw), _ptr(self.k), _ptr(self.v),
                                              _ptr(self.k_scale), _ptr(self.v_scale), B, cap, n_kv, d,
                                              int(ring)), "sa_kv_cache_init_fp8")
        elif ring:
            _check(lib().sa_kv_cache_init_ring(ctypes.byref(self.raw), _ptr(self.k), _ptr(self.v), B, cap,
                                               n_kv, d, int(ring)), "sa_kv_cache_init_ring")
        else:
            _check(lib().sa_kv_cache_init(ctypes.byref(self.raw), _ptr(self.k), _ptr(self.v), B, cap, n_kv,
                                          d), "sa_kv_cache_init")

    @property
    def offset(self):
        return self.raw.offset

    def k_rows(self, start=0, stop=None):
        """K rows [start, stop) as a [B, T, n_kv, d] view (a gathered copy
        of positions [start, stop) for a ring cache)."""
        return self._rows(self.k, start, stop)

    def v_rows(self, start=0, stop=None):
        return self._rows(self.v, start, stop)

    def k_scales(self, start=0, stop=None):
        """FP8 caches: K row scales of positions [start, stop) as [B, T, n_kv]."""
        return self._rows(self.k_scale, start, stop)

    def v_scales(self, start=0, stop=None):
        return self._rows(self.v_scale, start, stop)

    def _rows(self, t, start, stop):
        if not self.raw.ring:
            return t[:, :, start:stop].transpose(1, 2)
        stop = self.raw.offset if stop is None else stop
        idx = torch.arange(start, stop, device=t.device) % self.raw.cap
        return t[:, :, idx].transpose(1, 2)

    @property
    def B(self):
        return self.raw.B

    def append(self, k_rot, v):
        """kv_append: copy already-rotated k and v rows at [offset, offset + T)."""
        _check(lib().sa_kv_append(ctypes.byref(self.raw), _ptr(k_rot), _strides(k_rot), _ptr(v),
                                  _strides(v), k_rot.shape[1], _stream(self.k)), "sa_kv_append")

    def snapshot(self):
        s = _Snapshot()
        _check(lib().sa_kv_snapshot(ctypes.byref(self.raw), ctypes.byref(s)), "sa_kv_snapshot")
        return Snapshot(s)

    def restore(self, snap):
        _check(lib().sa_kv_restore(ctypes.byref(self.raw), ctypes.byref(snap.raw)), "sa_kv_restore")


def _view4(name, t):
    """Strides [B, T, H] of a bf16 CUDA [B, T, H, d] view with contiguous d."""
    if t.dtype != torch.bfloat16 or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA bf16 tensor")
    st = t.stride()
    if len(st) != 4 or st[3] != 1:
        raise ValueError("expected a [B, T, H, d] tensor with a contiguous last dimension")
    return st


def _args(cache, q, k, v, sinks, window, sm_scale, cos, sin, rope_fused, out, lse):
    """sa_attn_args for one call, packed into this thread's reusable struct
    (the library reads it only during the call)."""
    qs, ks, vs, os_ = _view4("q", q), _view4("k", k), _view4("v", v), _view4("out", out)
    if sinks is not None and (sinks.dtype != torch.float32 or not sinks.is_contiguous()):
        raise TypeError("sinks must be a contiguous fp32 CUDA tensor")
    a = getattr(_tls, "args", None)
    if a is None:
        a = _tls.args = _AttnArgs()
    struct.pack_into(_ATTN_FMT, a, 0,
                     q.data_ptr(), qs[0], qs[1], qs[2], k.data_ptr(), ks[0], ks[1], ks[2],
                     v.data_ptr(), vs[0], vs[1], vs[2], 0 if sinks is None else sinks.data_ptr(),
                     q.shape[0], q.shape[1], q.shape[2], cache.raw.offset, int(window), float(sm_scale),
                     1 if rope_fused else 0, 0 if cos is None else cos.data_ptr(),
                     0 if sin is None else sin.data_ptr(), 0 if cos is None else cos.shape[0],
                     out.data_ptr(), os_[0], os_[1], os_[2], 0 if lse is None else lse.data_ptr())
    return a


def attn_prefill(cache, q, k, v, sinks, window, sm_scale, cos=None, sin=None, rope_fused=True,
                 out=None, return_lse=False, lse=None):
    """Prefill T rows: append (rotated) k/v to the cache, attend q to rows
    [0, offset + T). Returns out [B,T,n_q,d] bf16 (and lse [B,n_q,T] fp32)."""
    B, T, n_q, d = q.shape
    if out is None:
        out = torch.empty((B, T, n_q, d), dtype=torch.bfloat16, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((B, n_q, T), dtype=torch.float32, device=q.device)
    a = _args(cache, q, k, v, sinks, window, sm_scale, cos, sin, rope_fused, out, lse)
    _check(lib().sa_attn_prefill(ctypes.byref(cache.raw), ctypes.byref(a), _raw_stream(q)), "sa_attn_prefill")
    return (out, lse) if return_lse else out


def decode_workspace_bytes(B, n_q, n_kv, d):
    return int(lib().sa_attn_decode_workspace_size(B, n_q, n_kv, d))


def decode_workspace(B, n_q, n_kv, d, device="cuda"):
    """A zero-filled workspace for attn_decode (reusable across calls)."""
    return torch.zeros(decode_workspace_bytes(B, n_q, n_kv, d), dtype=torch.uint8, device=device)


def attn_decode(cache, q, k, v, sinks, window, sm_scale, cos=None, sin=None, rope_fused=True,
                workspace=None, out=None, return_lse=False, lse=None):
    """One decode step (T == 1): append the new row, attend to the cache."""
    B, T, n_q, d = q.shape
    if workspace is None:
        workspace = decode_workspace(B, n_q, cache.raw.n_kv, d, q.device)
    if out is None:
        out = torch.empty((B, T, n_q, d), dtype=torch.bfloat16, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((B, n_q, T), dtype=torch.float32, device=q.device)
    a = _args(cache, q, k, v, sinks, window, sm_scale, cos, sin, rope_fused, out, lse)
    _check(lib().sa_attn_decode(ctypes.byref(cache.raw), ctypes.byref(a), workspace.data_ptr(),
                                workspace.numel() * workspace.element_size(), _raw_stream(q)),
           "sa_attn_decode")
    return (out, lse) if return_lse else out


def _require_matrix(name, t):
    if not (t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 2 and t.stride(1) == 1):
        raise TypeError(f"{name} must be a 2-D bf16 CUDA tensor with contiguous rows")


def rmsnorm_fold_weight(w, gamma, out=None):
    """w [N, K] bf16, gamma fp32 [K] -> bf16(w * gamma) (RMSNorm gain folded in)."""
    _require_matrix("w", w)
    if out is None:
        out = torch.empty_like(w)
    _check(lib().sa_rmsnorm_fold_weight(_ptr(w), w.stride(0), _ptr(gamma), _ptr(out), out.stride(0),
                                        w.shape[0], w.shape[1], _stream(w)), "sa_rmsnorm_fold_weight")
    return out


def qkv_proj(x, w_folded, bias, eps, out=None):
    """RMSNorm(x) W^T + b with the gain folded into w_folded: x [M, K] -> [M, N]."""
    _require_matrix("x", x)
    _require_matrix("w_folded", w_folded)
    M, K = x.shape
    N = w_folded.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _check(lib().sa_qkv_proj(_ptr(x), x.stride(0), _ptr(w_folded), w_folded.stride(0), _ptr(bias),
                             float(eps), _ptr(out), out.stride(0), M, N, K, _stream(x)), "sa_qkv_proj")
    return out


def out_proj(o, w, bias, x):
    """x += o W^T + b in place (o [M, K], w [N, K], x [M, N]); returns x."""
    for n, t in (("o", o), ("w", w), ("x", x)):
        _require_matrix(n, t)
    M, K = o.shape
    N = w.shape[0]
    _check(lib().sa_out_proj(_ptr(o), o.stride(0), _ptr(w), w.stride(0), _ptr(bias), _ptr(x), x.stride(0),
                             M, N, K, _stream(o)), "sa_out_proj")
    return x


def attn_backward(q, k, v, out, d_out, lse, sinks, window, sm_scale, workspace=None):
    """Gradients of a self-attention call (offset 0) with respect to the
    rotated q, k, v and the sinks. q/k/v/out/d_out [B, T, H, d] bf16 (strided
    views allowed), lse [B, n_q, T] fp32 from the forward. Returns (dq, dk,
    dv, dsinks) fp32 (dsinks None without sinks)."""
    B, T, n_q, d = q.shape
    n_kv = k.shape[2]
    for n, t in (("q", q), ("k", k), ("v", v), ("out", out), ("d_out", d_out)):
        _require_bf16_cuda(n, t)
    dev = q.device
    dq = torch.empty((B, T, n_q, d), dtype=torch.float32, device=dev)
    dk = torch.empty((B, T, n_kv, d), dtype=torch.float32, device=dev)
    dv = torch.empty((B, T, n_kv, d), dtype=torch.float32, device=dev)
    dsinks = None if sinks is None else torch.empty(n_q, dtype=torch.float32, device=dev)
    if workspace is None:
        nb = lib().sa_attn_backward_workspace_size(B, T, n_q)
        workspace = torch.empty(nb, dtype=torch.uint8, device=dev)
    a = _BwdArgs()
    a.q, a.q_strides = q.data_ptr(), _strides(q)
    a.k, a.k_strides = k.data_ptr(), _strides(k)
    a.v, a.v_strides = v.data_ptr(), _strides(v)
    a.out, a.out_strides = out.data_ptr(), _strides(out)
    a.d_out, a.d_out_strides = d_out.data_ptr(), _strides(d_out)
    a.lse = lse.data_ptr()
    a.sinks = 0 if sinks is None else sinks.data_ptr()
    a.B, a.T, a.n_q, a.n_kv, a.d = B, T, n_q, n_kv, d
    a.window = int(window)
    a.sm_scale = float(sm_scale)
    a.dq, a.dk, a.dv = dq.data_ptr(), dk.data_ptr(), dv.data_ptr()
    a.dsinks = 0 if dsinks is None else dsinks.data_ptr()
    _check(lib().sa_attn_backward(ctypes.byref(a), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _stream(q)), "sa_attn_backward")
    return dq, dk, dv, dsinks


def attn_decode_static(cache, q, k, v, sinks, window, sm_scale, cos=None, sin=None, rope_fused=True,
                       out=None, return_lse=False, lse=None):
    """attn_decode for callers that cannot allocate: the split scratch is a
    fixed array inside the library (SA_DECODE_STATIC_SCRATCH_BYTES per device),
    shared by every call -- do not overlap calls on the GPU."""
    B, T, n_q, d = q.shape
    if out is None:
        out = torch.empty((B, T, n_q, d), dtype=torch.bfloat16, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((B, n_q, T), dtype=torch.float32, device=q.device)
    a = _args(cache, q, k, v, sinks, window, sm_scale, cos, sin, rope_fused, out, lse)
    _check(lib().sa_attn_decode_static(ctypes.byref(cache.raw), ctypes.byref(a), _raw_stream(q)),
           "sa_attn_decode_static")
    return (out, lse) if return_lse else out


def device_status():
    """Reads and clears the device status word: 'SA_OK' or 'SA_ERR_TIMEOUT'."""
    code = ctypes.c_int32(0)
    _check(lib().sa_get_device_status(ctypes.byref(code)), "sa_get_device_status")
    return STATUS.get(code.value, str(code.value))


def set_wait_limit(cycles):
    _check(lib().sa_set_wait_limit(int(cycles)), "sa_set_wait_limit")


def set_prefill_events(before=None, after=None):
    """Record torch.cuda.Event `before`/`after` around the attention kernel of
    every later attn_prefill (None, None: stop recording)."""
    h0 = None if before is None else ctypes.c_void_p(before.cuda_event)
    h1 = None if after is None else ctypes.c_void_p(after.cuda_event)
    _check(lib().sa_set_prefill_events(h0, h1), "sa_set_prefill_events")

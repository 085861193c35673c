"""Benchmark of the sink-augmented GQA hot path on B200.

One step = the whole hot path over one batch of the GPT-OSS-Lite attention
workload (B=8, T=4096, 8 query / 4 KV heads of width 96, YaRN to 131072 from
4096): build the YaRN tables, then for one layer pair -- even layer with the
128-key band, odd layer full causal -- snapshot the cache, prefill 4096 rows
(RoPE, append, attention with the sink column), decode one row (the
prefill -> decode handoff), and restore the snapshot.

value = algorithmic TFLOP/s of the step: F = 4 * d * B * n_q * (admitted
(query, key) pairs), masked or skipped pairs never counted.

Also reported on the same line: the roofline of the dominant call (full-layer
prefill), the gpt-oss prefill (T=8192, 64/8/64, full layer) and the
131,072-context decode (24 layers, KV GB/s) as secondary measurements, the
end-to-end number through host buffers, and the oracle timed on host cores.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
(N > 1: launched by torch.distributed.run, one rank per GPU, weak scaling).
"""

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sink_augmented_gqa_b200 import workloads as wl  # noqa: E402

METRIC = "sink-GQA prefill TFLOP/s and decode KV GB/s at 1 B200, % of roofline"
WORKLOAD = "lite"
L2_BYTES = 126 * 2 ** 20


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), tf=float(p["bf16_tflops"]),
                    tf_sus=float(p["bf16_tflops_sustained"]), src="measured")
    except Exception:
        return dict(hbm=6650.0, tf=1590.0, tf_sus=1400.0, src="fallback")


def pairs(off, T, window):
    """Admitted (query, key) pairs of T rows starting at cache offset off."""
    n = 0
    if window <= 0:
        # sum_{i<T} (off + i + 1)
        return T * off + T * (T + 1) // 2
    for i in range(T):
        n += min(off + i + 1, window)
    return n


def profiled_traffic(summary, sources):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    kernel sources changed since that capture (their sha256 no longer matches)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if ":" in line:
            k, _, v = line.partition(":")
            fields[k.strip()] = v.strip()
    h = hashlib.sha256()
    for src in sources:
        with open(os.path.join(ROOT, "sink_augmented_gqa_b200", "csrc", src), "rb") as f:
            h.update(f.read())
    if fields.get("kernel_sources_sha256") != h.hexdigest():
        return None
    try:
        return int(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def flops(cfg, off, T, window):
    return 4 * cfg.d * cfg.B * cfg.n_q * pairs(off, T, window)


class Clocks:
    """nvidia-smi sampler for the timed region."""

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                       "--format=csv,noheader,nounits", "-lms", "20"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except Exception:
                self.p.kill()

    def summary(self):
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        try:
            os.unlink(self.f.name)
        except OSError:
            pass
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
                for nm, val in zip(names, r[5:9]):
                    if val.strip().lower() == "active":
                        reasons.add(nm)
            except (ValueError, IndexError):
                continue
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        top = max(sm)
        loaded = [s for s in sm if s >= 0.5 * top] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# The GPU arm
# ---------------------------------------------------------------------------

class LiteStep:
    """One step of the hot path on the GPT-OSS-Lite workload (device-resident)."""

    def __init__(self, dev, cfg):
        import sink_augmented_gqa_b200 as sa
        self.sa, self.cfg, self.dev = sa, cfg, dev
        self.max_pos = cfg.T + 1
        self.cap = cfg.T + 1
        y = cfg.yarn
        self.yarn = (y["theta"], y["scaling"], y["orig_ctx"], y["alpha"], y["beta"])
        self.cos = torch.empty((self.max_pos, cfg.d // 2), dtype=torch.float32, device=dev)
        self.sin = torch.empty_like(self.cos)
        self.layers = []
        for layer in range(2):
            q, k, v = wl.qkv(cfg, cfg.T + 1, layer=layer, device=dev)
            self.layers.append(dict(
                window=cfg.layer_window(layer), sinks=wl.sinks(cfg, layer, device=dev),
                q=q, k=k, v=v, cache=sa.KVCache(cfg.B, self.cap, cfg.n_kv, cfg.d, device=dev),
                out=torch.empty((cfg.B, cfg.T, cfg.n_q, cfg.d), dtype=torch.bfloat16, device=dev),
                dec=torch.empty((cfg.B, 1, cfg.n_q, cfg.d), dtype=torch.bfloat16, device=dev),
                ws=sa.decode_workspace(cfg.B, cfg.n_q, cfg.n_kv, cfg.d, device=dev)))
        for L in self.layers:
            L["snap"] = L["cache"].snapshot()
        T = cfg.T
        self.flops = sum(flops(cfg, 0, T, L["window"]) + flops(cfg, T, 1, L["window"]) for L in self.layers)
        self.launches = 1 + 3 * len(self.layers)

    def tables(self):
        from sink_augmented_gqa_b200 import sinkattn as S
        import ctypes
        S._check(S.lib().sa_yarn_rope_tables(S._ptr(self.cos), S._ptr(self.sin), self.max_pos, self.cfg.d,
                                             *[float(x) for x in self.yarn[:2]], int(self.yarn[2]),
                                             float(self.yarn[3]), float(self.yarn[4]), S._stream(self.cos)),
                 "sa_yarn_rope_tables")

    def run(self, ev_full=None, q_in=None, outs=None):
        sa, cfg, T = self.sa, self.cfg, self.cfg.T
        self.tables()
        for li, L in enumerate(self.layers):
            c = L["cache"]
            c.restore(L["snap"])
            q, k, v = (L["q"], L["k"], L["v"]) if q_in is None else q_in[li]
            out, dec = (L["out"], L["dec"]) if outs is None else outs[li]
            if ev_full is not None and L["window"] == 0:
                sa.set_prefill_events(*ev_full)   # around the attention kernel alone
            sa.attn_prefill(c, q[:, :T], k[:, :T], v[:, :T], L["sinks"], L["window"], cfg.sm_scale,
                            self.cos, self.sin, out=out)
            if ev_full is not None and L["window"] == 0:
                sa.set_prefill_events()
            sa.attn_decode(c, q[:, T:], k[:, T:], v[:, T:], L["sinks"], L["window"], cfg.sm_scale,
                           self.cos, self.sin, workspace=L["ws"], out=dec)


def _time_loop(fn, steps, warmup, dist=None):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    return max_over_ranks(ms, dist, "cuda")


def max_over_ranks(x, dist, device):
    """The largest of every rank's x (the job's time is its slowest rank's)."""
    if dist is None:
        return x
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_rank_step, ms_per_step):
    """Whole-job rate: every rank processes its own batch (weak scaling), and
    the step takes as long as the slowest rank."""
    return world * units_per_rank_step / (ms_per_step * 1e-3)


def full_prefill_roofline(step, steps, peaks):
    """Average duration of the full-layer attention kernel over `steps` steps
    (CUDA events the library records on its stream around that launch)."""
    pairs_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(steps)]
    for a, b in pairs_ev:   # create the events before handing their handles over
        a.record()
        b.record()
    torch.cuda.synchronize()
    for i in range(steps):
        step.run(ev_full=pairs_ev[i])
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in pairs_ev)
    cfg = step.cfg
    f = flops(cfg, 0, cfg.T, 0)
    achieved = f / (ms * 1e-3) / 1e12
    return ms, achieved


def gptoss_prefill(dev, peaks, reps=10):
    """Full-layer gpt-oss prefill (B=1, T=8192, 64/8/64 from fused qkv)."""
    import sink_augmented_gqa_b200 as sa
    cfg = wl.CONFIGS["gptoss_prefill"]
    y = cfg.yarn
    cos, sin = sa.yarn_rope_tables(cfg.T, cfg.d, y["theta"], y["scaling"], y["orig_ctx"], y["alpha"],
                                   y["beta"], device=dev)
    res = {}
    for layer in (1, 0):
        window = cfg.layer_window(layer)
        q, k, v = wl.qkv(cfg, cfg.T, layer=layer, device=dev)
        sinks = wl.sinks(cfg, layer, device=dev)
        cache = sa.KVCache(cfg.B, cfg.T, cfg.n_kv, cfg.d, device=dev)
        snap = cache.snapshot()
        out = torch.empty((cfg.B, cfg.T, cfg.n_q, cfg.d), dtype=torch.bfloat16, device=dev)

        def once():
            cache.restore(snap)
            sa.attn_prefill(cache, q, k, v, sinks, window, cfg.sm_scale, cos, sin, out=out)
        for _ in range(3):
            once()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in evs:
            a.record()
            once()
            b.record()
        torch.cuda.synchronize()
        ms = statistics.median(a.elapsed_time(b) for a, b in evs)
        f = flops(cfg, 0, cfg.T, window)
        tf = f / (ms * 1e-3) / 1e12
        key = "full" if window == 0 else "band"
        res[key] = {"ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                    "frac_of_bf16_peak": round(tf / peaks["tf"], 4)}
    return res


def projection_inputs(dev, which, T=8192):
    """Seeded inputs of the gpt-oss projections at T rows: ("qkv") x [T, 2880],
    RMSNorm gain, qkv weight [5120, 2880] with bias; ("out") attention output
    [T, 4096], out weight [2880, 4096] with bias, residual x [T, 2880]."""
    seed = wl.CONFIGS["gptoss_prefill"].seed
    N, K = (5120, 2880) if which == "qkv" else (2880, 4096)
    a = wl.randn_bf16((T, K), seed, 70_000, dev)
    w = (wl.randn_bf16((N, K), seed, 70_001, dev).float() / math.sqrt(K)).to(torch.bfloat16)
    b = wl.randn_bf16((N,), seed, 70_002, dev)
    extra = (wl.randn_bf16((K,), seed, 70_003, dev).float().abs() + 0.5 if which == "qkv"
             else wl.randn_bf16((T, N), seed, 70_004, dev))
    return a, w, b, extra


def projections(dev, peaks, reps=20):
    """The dense projections around a gpt-oss attention layer at T = 8192:
    RMSNorm + fused qkv (2880 -> 5120) and the out projection with the
    residual add (4096 -> 2880), on the tensor cores; 2 T N K flops each.
    Back-to-back launches between CUDA events; each call's operands and
    output (138-160 MB) exceed L2."""
    import sink_augmented_gqa_b200 as sa
    T = 8192
    res = {}
    for which in ("qkv", "out"):
        a, w, b, extra = projection_inputs(dev, which, T)
        N, K = w.shape
        if which == "qkv":
            wf = sa.rmsnorm_fold_weight(w, extra)
            y = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
            fn = lambda: sa.qkv_proj(a, wf, b, 1e-5, out=y)
        else:
            fn = lambda: sa.out_proj(a, w, b, extra)
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        tf = 2 * T * N * K / (ms * 1e-3) / 1e12
        res[f"{which}_proj_T8192"] = {"M_N_K": [T, N, K], "ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                                      "frac_of_bf16_peak": round(tf / peaks["tf"], 4),
                                      "traffic": profiled_traffic(f"gemm_gptoss_{which}_proj.md",
                                                                  ("gemm.cuh", "ptx.cuh"))}
    return res


def lite_backward(dev, peaks, reps=10):
    """Backward pass of a Lite training layer (B = 8, T = 4096, 8/4 heads,
    d = 96), full causal and band, after the library's own forward. Work is
    counted as the algorithmic 5 products of the backward (S, dP, dV, dK,
    dQ: 10 d flops per admitted pair and head); the kernels recompute S and
    dP for dQ, which is not counted."""
    import sink_augmented_gqa_b200 as sa
    cfg = wl.CONFIGS["lite"]
    res = {}
    for layer in (1, 0):
        window = cfg.layer_window(layer)
        q, k, v = wl.qkv(cfg, cfg.T, layer=layer, device=dev)
        dout = wl.randn_bf16((cfg.B, cfg.T, cfg.n_q, cfg.d), cfg.seed, 124, dev)
        sinks = wl.sinks(cfg, layer, device=dev)
        cache = sa.KVCache(cfg.B, cfg.T, cfg.n_kv, cfg.d, device=dev)
        out, lse = sa.attn_prefill(cache, q, k, v, sinks, window, cfg.sm_scale, rope_fused=False, return_lse=True)
        ws = torch.empty(sa.sinkattn.lib().sa_attn_backward_workspace_size(cfg.B, cfg.T, cfg.n_q),
                         dtype=torch.uint8, device=dev)

        def once():
            sa.attn_backward(q, k, v, out, dout, lse, sinks, window, cfg.sm_scale, workspace=ws)
        for _ in range(3):
            once()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            once()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        f = 10 * cfg.d * cfg.B * cfg.n_q * pairs(0, cfg.T, window)
        tf = f / (ms * 1e-3) / 1e12
        res["full" if window == 0 else "band"] = {"ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                                                  "frac_of_bf16_peak": round(tf / peaks["tf"], 4)}
        del cache
    return res


def long_decode(dev, peaks, steps=8, layers=24, ring=False, fp8=False):
    """131,072-context decode: 24 layers alternating band / full, one row per
    layer per step, KV bytes actually read / time. ring=True keeps the band
    layers in 384-row ring caches instead of full-length ones; fp8=True keeps
    every layer's cache as e4m3 codes with fp32 row scales (the bytes counted
    are then codes plus scales)."""
    import sink_augmented_gqa_b200 as sa
    cfg = wl.CONFIGS["long_decode"]
    off = cfg.offset
    cap = off + steps + 4
    ring_cap = 384
    y = cfg.yarn
    cos, sin = sa.yarn_rope_tables(cap, cfg.d, y["theta"], y["scaling"], y["orig_ctx"], y["alpha"],
                                   y["beta"], device=dev)
    caches, ins = [], []
    for layer in range(layers):
        w = cfg.layer_window(layer)
        g = torch.Generator(device=dev)
        g.manual_seed(cfg.seed * 1000 + 50_000 + layer)
        if ring and w:
            # a band layer's ring: the last ring_cap positions, up to `off`
            c = sa.KVCache(cfg.B, ring_cap, cfg.n_kv, cfg.d, device=dev, ring=w, fp8=fp8)
            pre_k = torch.empty((cfg.B, ring_cap, cfg.n_kv, cfg.d), dtype=torch.bfloat16, device=dev)
            pre_v = torch.empty_like(pre_k)
            pre_k.normal_(generator=g)
            pre_v.normal_(generator=g)
            while c.offset < off:   # the prefix streamed through the ring, one ring-full at a time
                n = min(ring_cap, off - c.offset)
                c.append(pre_k[:, :n], pre_v[:, :n])
        elif fp8:
            # the prefix generated in bf16, appended (quantised) into the FP8 cache
            c = sa.KVCache(cfg.B, (cap + 15) // 16 * 16, cfg.n_kv, cfg.d, device=dev, fp8=True)
            pre_k = torch.empty((cfg.B, off, cfg.n_kv, cfg.d), dtype=torch.bfloat16, device=dev)
            pre_v = torch.empty_like(pre_k)
            pre_k.normal_(generator=g)
            pre_v.normal_(generator=g)
            c.append(pre_k, pre_v)
            del pre_k, pre_v
        else:
            c = sa.KVCache(cfg.B, cap, cfg.n_kv, cfg.d, device=dev)
            c.k.normal_(generator=g)
            c.v.normal_(generator=g)
            # rows [0, off) stand for an already-filled, rotated prefix: append them
            # in place (a self-copy) so the cache's offset and bookkeeping follow.
            c.append(c.k_rows(0, off), c.v_rows(0, off))
        caches.append(c)
        ins.append(dict(window=cfg.layer_window(layer), sinks=wl.sinks(cfg, layer, device=dev),
                        ws=sa.decode_workspace(cfg.B, cfg.n_q, cfg.n_kv, cfg.d, device=dev),
                        out=torch.empty((cfg.B, 1, cfg.n_q, cfg.d), dtype=torch.bfloat16, device=dev)))
    snaps = [c.snapshot() for c in caches]
    q, k, v = wl.qkv(cfg, steps, device=dev)

    def run_steps():
        for c, s in zip(caches, snaps):
            c.restore(s)
        for st in range(steps):
            for li, c in enumerate(caches):
                I = ins[li]
                sa.attn_decode(c, q[:, st:st + 1], k[:, st:st + 1], v[:, st:st + 1], I["sinks"], I["window"],
                               cfg.sm_scale, cos, sin, workspace=I["ws"], out=I["out"])
    run_steps()
    torch.cuda.synchronize()
    # K and V of one position of every KV head (FP8: codes plus one fp32 scale each)
    row_bytes = cfg.n_kv * (cfg.d + 4 if fp8 else cfg.d * 2) * 2 * cfg.B

    def graph_of(layer_ids):
        """A CUDA graph of one decode call per listed layer (each on its own
        cache, all at offset `off`): replaying it runs the kernels back to back
        with no host work between them."""
        for li in layer_ids:
            caches[li].restore(snaps[li])
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(gr, stream=side):
                for li in layer_ids:
                    I = ins[li]
                    sa.attn_decode(caches[li], q[:, :1], k[:, :1], v[:, :1], I["sinks"], I["window"], cfg.sm_scale,
                                   cos, sin, workspace=I["ws"], out=I["out"])
        torch.cuda.current_stream().wait_stream(side)
        for li in layer_ids:
            caches[li].restore(snaps[li])
        return gr

    def replay_ms(gr, reps):
        for _ in range(3):
            gr.replay()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record()
        for _ in range(reps):
            gr.replay()
        g1.record()
        torch.cuda.synchronize()
        return g0.elapsed_time(g1) / reps

    # the full-layer kernel: the full layers' calls back to back from a graph,
    # each on its own cache, so the data streamed (~1.7-3.2 GB) is far beyond L2
    full_ids = [i for i in range(layers) if ins[i]["window"] == 0]
    gfull = graph_of(full_ids)
    ms_full = replay_ms(gfull, 10) / len(full_ids)
    del gfull
    gbs_full = (off + 1) * row_bytes / (ms_full * 1e-3) / 1e9
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    run_steps()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    nbytes = 0
    for st in range(steps):
        for li in range(layers):
            p = off + st
            w = ins[li]["window"]
            rows = min(p + 1, w) if w else p + 1
            nbytes += rows * row_bytes
    gbs = nbytes / (ms * 1e-3) / 1e9
    # the same token step (24 layers at offset off) replayed from a CUDA graph:
    # no host launch overhead between the layers
    graph = graph_of(list(range(layers)))
    ms_graph = replay_ms(graph, 20)
    gbytes = 0
    for li in range(layers):
        w = ins[li]["window"]
        gbytes += (min(off + 1, w) if w else off + 1) * row_bytes
    gbs_graph = gbytes / (ms_graph * 1e-3) / 1e9
    del graph
    kv_gib = sum(2 * (c.k.numel() * c.k.element_size() + (c.k_scale.numel() * 4 if fp8 else 0))
                 for c in caches) / 2 ** 30
    del caches
    torch.cuda.empty_cache()
    return {"steps": steps, "layers": layers, "ms_per_token_step": round(ms / steps, 4),
            "KV_GB/s": round(gbs, 1), "frac_of_hbm": round(gbs / peaks["hbm"], 4),
            "full_layer_kernel": {"ms": round(ms_full, 4), "KV_GB/s": round(gbs_full, 1),
                                  "frac_of_hbm": round(gbs_full / peaks["hbm"], 4),
                                  "timing": "device time per launch, full layers back to back from a CUDA graph",
                                  "traffic": profiled_traffic(
                                      "decode_long_context_fp8.md" if fp8 else "decode_long_context_full.md",
                                      ("decode.cuh", "fp8.cuh", "ptx.cuh"))},
            "cuda_graph_token_step": {"ms": round(ms_graph, 4), "KV_GB/s": round(gbs_graph, 1),
                                      "frac_of_hbm": round(gbs_graph / peaks["hbm"], 4)},
            "kv_cache_GiB": round(kv_gib, 3),
            "cache_layout": ("head-major [B][n_kv][cap][d]" + (", band layers in 384-row rings" if ring else "")
                             + (", e4m3 codes + fp32 row scales [B][n_kv][cap]" if fp8 else ", bf16"))}


def e2e_lite(step, steps, warmup):
    """Same step through host buffers: every step copies its q/k/v from pinned
    host memory to the device and reads both layers' outputs back to pinned
    host memory. Steps are pipelined over three streams (host-to-device copies,
    compute, device-to-host copies) with two buffer sets, so one step's copies
    overlap its neighbours' work, as a serving loop would run; the timed
    region spans the first step's first copy to the last step's last copy."""
    cfg = step.cfg
    host_in, dev_in, dev_out, host_out = [], [], [], []
    h2d = d2h = 0
    for L in step.layers:
        hq, hk, hv = (L[n].cpu().pin_memory() for n in ("q", "k", "v"))
        host_in.append((hq, hk, hv))
        h2d += sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    for _ in range(2):
        dev_in.append([tuple(torch.empty_like(L[n]) for n in ("q", "k", "v")) for L in step.layers])
        dev_out.append([(torch.empty_like(L["out"]), torch.empty_like(L["dec"])) for L in step.layers])
        host_out.append([(torch.empty(L["out"].shape, dtype=torch.bfloat16).pin_memory(),
                          torch.empty(L["dec"].shape, dtype=torch.bfloat16).pin_memory()) for L in step.layers])
    d2h = sum(a.numel() * 2 + b.numel() * 2 for a, b in host_out[0])
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event(enable_timing=False)
    computed = [ev(), ev()]   # set s: its inputs are consumed
    landed = [ev(), ev()]     # set s: its inputs are on the device
    read = [ev(), ev()]       # set s: its outputs are on the host
    used = [False, False]

    def run(n, first=None, last=None):
        for i in range(n):
            st = i % 2
            with torch.cuda.stream(s_in):
                if used[st]:
                    s_in.wait_event(computed[st])
                if i == 0 and first is not None:
                    first.record(s_in)
                for (hq, hk, hv), (dq, dk, dv) in zip(host_in, dev_in[st]):
                    dq.copy_(hq, non_blocking=True)
                    dk.copy_(hk, non_blocking=True)
                    dv.copy_(hv, non_blocking=True)
                landed[st].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(landed[st])
                if used[st]:
                    s_comp.wait_event(read[st])
                step.run(q_in=dev_in[st], outs=dev_out[st])
                computed[st].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[st])
                for (ho, hd), (do, dd) in zip(host_out[st], dev_out[st]):
                    ho.copy_(do, non_blocking=True)
                    hd.copy_(dd, non_blocking=True)
                read[st].record(s_out)
                if i == n - 1 and last is not None:
                    last.record(s_out)
            used[st] = True
        torch.cuda.synchronize()

    run(warmup)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(steps, e0, e1)
    return e0.elapsed_time(e1) / steps, h2d, d2h


# ---------------------------------------------------------------------------
# The oracle on host cores (CPU baseline / reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(budget_s=12.0, min_units=1):
    """Times the fp64 oracle on a bounded sample of the bench step: whole
    (sequence, query head) units, each the step's work for that unit -- both
    layers (band and full causal), prefill of T rows and the decode row, i.e.
    T + 1 rows per layer (the decode row attends exactly like a prefill row
    at position T) -- until the time budget is spent. Returns (TFLOP/s,
    cores, description)."""
    from oracle import attention as oatt
    from oracle import rope as orope
    from oracle import yarn as oyarn
    cfg = wl.CONFIGS[WORKLOAD]
    y = cfg.yarn
    n = cfg.T + 1
    cos, sin = oyarn.stored_tables(n, cfg.d, y["theta"], y["scaling"], y["orig_ctx"], y["alpha"], y["beta"])
    layers = []
    for layer in range(2):
        q, k, v = wl.qkv(cfg, n, layer=layer)
        layers.append(dict(window=cfg.layer_window(layer), sinks=wl.sinks(cfg, layer).double().numpy(),
                           q=q.to(torch.float64).numpy(), k=k.to(torch.float64).numpy(),
                           v=v.to(torch.float64).numpy()))
    done = 0
    t0 = time.perf_counter()
    units = 0
    while True:
        b, h = divmod(units, cfg.n_q)
        b %= cfg.B
        g = h // cfg.q_mult
        for L in layers:
            qr = orope.rotate_bsh(L["q"][b:b + 1, :, h:h + 1], 0, cos, sin)
            kr = orope.rotate_bsh(L["k"][b:b + 1, :, g:g + 1], 0, cos, sin)
            oatt.sink_attention(qr, kr, L["v"][b:b + 1, :, g:g + 1], L["sinks"][h:h + 1], 0, L["window"],
                                cfg.sm_scale)
            done += 4 * cfg.d * pairs(0, n, L["window"])
        units += 1
        if units >= min_units and time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    threads = int(os.environ.get("OMP_NUM_THREADS", "0")) or os.cpu_count()
    desc = (f"fp64 numpy oracle on {units} of the step's {cfg.B * cfg.n_q} (sequence, head) units: both layers "
            f"(W={cfg.window} band, full causal), {cfg.T} prefill rows + the decode row each, RoPE included, "
            f"{dt:.1f} s")
    return done / dt / 1e12, threads, desc


def step_config(cfg, world, parallelism):
    """The bench step's workload, the same for both arms."""
    return {"workload": "GPT-OSS-Lite attention: B=8, T=4096 prefill + 1 decode row, "
                        "n_q=8, n_kv=4, d=96, W=128 band layer + full causal layer, "
                        "YaRN theta=150000 s=32 from 4096",
            "global_batch": cfg.B * world, "seq_len": cfg.T, "parallelism": parallelism,
            "l2": "inputs larger than L2 (step working set ~300 MB > 126 MB)"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    per = []
    desc = ""
    for _ in range(args.warmup):
        oracle_sample(budget_s=0.5)
    t_all = time.perf_counter()
    for _ in range(args.steps):
        tf, cores, desc = oracle_sample(budget_s=max(2.0, 20.0 / max(1, args.steps)))
        per.append(tf)
    value = statistics.mean(per)
    cfg = wl.CONFIGS[WORKLOAD]
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": (time.perf_counter() - t_all) * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": step_config(cfg, 1, "none (host oracle)"),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# Single-call loops for profilers (ncu): no timing, no output but a summary
# ---------------------------------------------------------------------------

PROFILE_CASES = ("gptoss_prefill_full", "gptoss_prefill_band", "lite_prefill_full", "long_decode_full",
                 "long_decode_fp8", "gptoss_qkv_proj", "gptoss_out_proj", "lite_backward_b2")


def profile_case(name, dev, steps, warmup):
    import sink_augmented_gqa_b200 as sa
    if name == "lite_backward_b2":
        # the Lite training layer with 2 of its 8 sequences (a capture-sized case)
        cfg = wl.scaled(wl.CONFIGS["lite"], B=2)
        q, k, v = wl.qkv(cfg, cfg.T, layer=1, device=dev)
        dout = wl.randn_bf16((cfg.B, cfg.T, cfg.n_q, cfg.d), cfg.seed, 124, dev)
        sinks = wl.sinks(cfg, 1, device=dev)
        cache = sa.KVCache(cfg.B, cfg.T, cfg.n_kv, cfg.d, device=dev)
        out, lse = sa.attn_prefill(cache, q, k, v, sinks, 0, cfg.sm_scale, rope_fused=False, return_lse=True)

        def once():
            sa.attn_backward(q, k, v, out, dout, lse, sinks, 0, cfg.sm_scale)
        units = 10 * cfg.d * cfg.B * cfg.n_q * pairs(0, cfg.T, 0)
    elif name.endswith("_proj"):
        which = "qkv" if "qkv" in name else "out"
        a, w, b, extra = projection_inputs(dev, which)
        N, K = w.shape
        if which == "qkv":
            wf = sa.rmsnorm_fold_weight(w, extra)

            def once():
                sa.qkv_proj(a, wf, b, 1e-5)
        else:
            def once():
                sa.out_proj(a, w, b, extra)
        units = 2 * a.shape[0] * N * K
    elif name.startswith("gptoss") or name.startswith("lite"):
        cfg = wl.CONFIGS["gptoss_prefill" if name.startswith("gptoss") else "lite"]
        window = cfg.window if name.endswith("band") else 0
        y = cfg.yarn
        cos, sin = sa.yarn_rope_tables(cfg.T, cfg.d, y["theta"], y["scaling"], y["orig_ctx"], y["alpha"],
                                       y["beta"], device=dev)
        q, k, v = wl.qkv(cfg, cfg.T, layer=1, device=dev)
        sinks = wl.sinks(cfg, 1, device=dev)
        cache = sa.KVCache(cfg.B, cfg.T, cfg.n_kv, cfg.d, device=dev)
        snap = cache.snapshot()
        out = torch.empty((cfg.B, cfg.T, cfg.n_q, cfg.d), dtype=torch.bfloat16, device=dev)

        def once():
            cache.restore(snap)
            sa.attn_prefill(cache, q, k, v, sinks, window, cfg.sm_scale, cos, sin, out=out)
        units = flops(cfg, 0, cfg.T, window)
    else:
        cfg = wl.CONFIGS["long_decode"]
        off = cfg.offset
        y = cfg.yarn
        cos, sin = sa.yarn_rope_tables(off + 2, cfg.d, y["theta"], y["scaling"], y["orig_ctx"], y["alpha"],
                                       y["beta"], device=dev)
        fp8 = name.endswith("fp8")
        g = torch.Generator(device=dev)
        g.manual_seed(cfg.seed * 1000 + 50_001)
        if fp8:
            cache = sa.KVCache(cfg.B, (off + 2 + 15) // 16 * 16, cfg.n_kv, cfg.d, device=dev, fp8=True)
            pre = torch.empty((2, cfg.B, off, cfg.n_kv, cfg.d), dtype=torch.bfloat16, device=dev)
            pre.normal_(generator=g)
            cache.append(pre[0], pre[1])
            del pre
        else:
            cache = sa.KVCache(cfg.B, off + 2, cfg.n_kv, cfg.d, device=dev)
            cache.k.normal_(generator=g)
            cache.v.normal_(generator=g)
            cache.append(cache.k_rows(0, off), cache.v_rows(0, off))
        snap = cache.snapshot()
        q, k, v = wl.qkv(cfg, 1, device=dev)
        sinks = wl.sinks(cfg, 1, device=dev)
        ws = sa.decode_workspace(cfg.B, cfg.n_q, cfg.n_kv, cfg.d, device=dev)
        out = torch.empty((cfg.B, 1, cfg.n_q, cfg.d), dtype=torch.bfloat16, device=dev)

        def once():
            cache.restore(snap)
            sa.attn_decode(cache, q, k, v, sinks, 0, cfg.sm_scale, cos, sin, workspace=ws, out=out)
        units = (off + 1) * cfg.n_kv * (cfg.d + 4 if fp8 else cfg.d * 2) * 2 * cfg.B
    for _ in range(warmup + steps):
        once()
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": name, "launches": warmup + steps,
                      "algorithmic_units_per_launch": units,
                      "unit": "bytes" if name.startswith("long") else "flop"}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="libsinkattn", choices=["libsinkattn", "reference"])
    ap.add_argument("--no-extras", action="store_true", help="skip the secondary measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--profile-case", choices=PROFILE_CASES, default=None,
                    help="only run this call warmup+steps times (for profilers); prints no bench line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=dev)
        dist = tdist

    from sink_augmented_gqa_b200 import build as sbuild
    if rank == 0:
        sbuild.build()
    if args.profile_case:
        profile_case(args.profile_case, dev, args.steps, args.warmup)
        return
    if dist is not None:
        dist.barrier()

    peaks = _peaks()
    cfg = wl.CONFIGS[WORKLOAD]
    step = LiteStep(dev, cfg)
    with Clocks(local) as clk:
        ms = _time_loop(step.run, args.steps, args.warmup, dist)
        full_ms, full_tf = full_prefill_roofline(step, max(3, min(args.steps, 10)), peaks)
    clocks = clk.summary()
    ms_step = ms / args.steps
    value = job_throughput(world, step.flops, ms_step) / 1e12

    e2e_ms, h2d, d2h = e2e_lite(step, max(3, args.steps // 2), 3)
    e2e_ms = max_over_ranks(e2e_ms, dist, "cuda")
    e2e_val = job_throughput(world, step.flops, e2e_ms) / 1e12

    extras = {}
    if not args.no_extras and rank == 0:
        extras["gptoss_prefill_T8192"] = gptoss_prefill(dev, peaks)
        extras["gptoss_projections"] = projections(dev, peaks)
        extras["lite_backward_T4096"] = lite_backward(dev, peaks)
        extras["long_context_decode_131072"] = long_decode(dev, peaks)
        extras["long_context_decode_131072_ring"] = long_decode(dev, peaks, ring=True)
        extras["long_context_decode_131072_fp8"] = long_decode(dev, peaks, fp8=True)
        extras["long_context_decode_131072_fp8_ring"] = long_decode(dev, peaks, ring=True, fp8=True)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        tf, cores, desc = oracle_sample()
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc}

    if dist is not None:
        dist.barrier()
    if rank == 0:
        traffic = profiled_traffic("prefill_lite_full.md", ("prefill.cuh", "ptx.cuh"))
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 q/k/v, N(0,0.25) fp32 sinks)",
            "config": step_config(cfg, world, f"dp{world}"),
            "roofline": {"bound": "tensor", "kernel": "prefill_kernel (full-causal layer attention; the staging launch before it is not included)",
                         "achieved": round(full_tf, 2), "peak": peaks["tf"], "unit": "TFLOP/s",
                         "frac": round(full_tf / peaks["tf"], 4), "traffic": traffic,
                         "peak_source": f"{peaks['src']} dense bf16 (burst)", "ms": round(full_ms, 4)},
            "clocks": clocks,
            "e2e": {"value": round(e2e_val, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4)},
            "gpu_launches": step.launches * args.steps,
            "cpu_baseline": cpu,
            "secondary": extras,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

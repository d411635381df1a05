#!/usr/bin/env python
"""Benchmark of the ReSA decode hot path (libresa.so) on B200.

One benchmark step is one rectification period of one token position across
`--layers` attention layers: f sparse decode steps (append, score, select,
split-KV attention, merge) on every layer, then one dense rectification of
the last f tokens on every layer. The layers hold independent KV caches that
are visited round-robin, so between two visits of a cache more than the L2
size (126 MB) of other data is read: the inputs are larger than L2 and no
explicit flush is needed.

metric: ReSA decode-step us (one attention layer, rectify amortised over f)
with achieved HBM GB/s against roofline at 128K/256K, and rectify us.
value = step time / (f * layers * n_gpus) in microseconds (lower is better).

With --gpus N > 1 (torchrun) every rank runs an independent replica of the
workload (the path has no exchange step); timing is the max over ranks.
`--impl reference` times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOADS = {"tiny": 0, "32k": 1, "128k": 2, "256k": 3, "64k": 4}
WORKLOAD_NAMES = {
    0: "resa_decode_tiny_fp32", 1: "resa_decode_32k_b4_needles", 2: "resa_decode_128k_b1", 3: "resa_decode_256k_b1",
    4: "resa_decode_64k_b16",
}
METRIC = "ReSA decode-step us & achieved HBM GB/s vs roofline at 128K/256K; rectify us"

# Counters taken from ncu captures of the kernels as they stand, each keyed by
# a hash of the kernel's source files at capture time: a counter is reported
# only while the sources still hash to that value (null once a kernel changes).
#   attention: DRAM read + write bytes per launch of attend_bf16_kernel at the
#     128K workload (--metrics dram__bytes_read.sum,dram__bytes_write.sum);
#   rectify: sm__pipe_tensor_cycles_active (% of peak, active cycles) of
#     rectify_tc_kernel at 128K, f = 32 (--set full, one cold launch).
NCU_COUNTERS = {
    "attention": {"files": ["attend.cu", "attend_core.cuh", "common.cuh", "launch.h"],
                  "source": "21102da51ec3d8a4",
                  "traffic": {"resa_decode_128k_b1": 53964672}},
    "rectify": {"files": ["rectify_tc.cu", "tc.cuh", "common.cuh", "launch.h"], "source": "32e588cf2e8f88a6",
                "tensor_pipe_active_pct": 36.22, "traffic": 544848384},
}


def source_hash(files) -> str:
    """First 16 hex digits of the SHA-256 of the given kernel sources."""
    import hashlib
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(ROOT, "block_sparse_attention_quest_b200", "csrc", name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def counter(kind: str, key: str, workload: str | None = None):
    """A captured counter, or None when the kernel changed since its capture."""
    c = NCU_COUNTERS[kind]
    if c["source"] is None or source_hash(c["files"]) != c["source"]:
        return None
    v = c.get(key)
    if isinstance(v, dict):
        v = v.get(workload)
    return v


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="128k", choices=sorted(WORKLOADS))
    ap.add_argument("--layers", type=int, default=4)
    ap.add_argument("--r", type=float, default=None)
    ap.add_argument("--f", type=int, default=None, help="rectification period (default 32)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="N > 1: independent replicas (weak scaling) or one layer's KV heads "
                         "split over the ranks (strong scaling)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the 256K, 32K x 4 and 64K x 16 workloads of the default run")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        ids = [x.strip() for x in vis.split(",")] if vis else []
        self.index = ids[local_rank] if local_rank < len(ids) else str(local_rank)
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(value: float, dist, device) -> float:
    """The largest value over all ranks (timings are reported as the slowest
    rank's); identity without a process group."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- GPU arm
def device_cache(spec, dev, tdt):
    """K, V [B, Hkv, max_len, d] drawn on the device with the workload recipe
    (N(0, 1) per element plus a N(0, 0.5^2) mean vector per (batch, KV head,
    block), needles shifted by shift * q_dir), rounded to the cache dtype.
    Used for the extra benchmark workloads, whose sizes make the host
    generator slow; the bits differ from the host generator's, the
    distribution does not."""
    import torch
    from workload import needle_layout
    B, H, L, d = spec.batch, spec.n_kv_heads, spec.max_len, spec.head_dim
    g = torch.Generator(device=dev).manual_seed(spec.seed)
    nb = (spec.len0 + 15) // 16
    out = []
    for _ in ("k", "v"):
        arr = torch.zeros(B, H, L, d, dtype=tdt, device=dev)
        for b in range(B):
            mean = 0.5 * torch.randn(H, nb, 1, d, generator=g, device=dev)
            x = torch.randn(H, nb, 16, d, generator=g, device=dev) + mean
            arr[b, :, :spec.len0] = x.view(H, nb * 16, d)[:, :spec.len0].to(tdt)
            del x, mean
        out.append(arr)
    if spec.needles:
        qd, pos = needle_layout(spec)
        qd_t = torch.from_numpy(qd).to(dev)
        for b in range(B):
            for h in range(H):
                for j in pos[b, h]:
                    sl = out[0][b, h, int(j) * 16:(int(j) + 1) * 16]
                    sl.copy_((sl.float() + spec.needle_shift * qd_t[b, h]).to(tdt))
    return out


def measure_workload(args, resa, spec, L, dev, stream, host_cache=True, full=True):
    """Time one workload: a step of f sparse decode positions on L layer caches
    plus L rectifications, as a CUDA graph; per-call decode and rectify
    times; the sparse and dense (r = 1) calls back to back; the attention
    kernel alone. With full=True also the staged split and the end-to-end
    run through the Python API with host buffers."""
    import torch
    from workload import decode_inputs, make_cache, rectify_inputs
    f = spec.f
    tdt = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
    esize = 2 if spec.dtype == "bf16" else 4
    B, Hq, H, d = spec.batch, spec.n_q_heads, spec.n_kv_heads, spec.head_dim

    def dev_t(x):
        return torch.from_numpy(np.ascontiguousarray(x)).to(dev).to(tdt)

    if host_cache:
        K, V = make_cache(spec)
        k0, v0 = dev_t(K), dev_t(V)
        del K, V
    else:
        k0, v0 = device_cache(spec, dev, tdt)
    layers = []
    for li in range(L):
        k = k0 if li == 0 else k0.clone()
        v = v0 if li == 0 else v0.clone()
        desc = torch.zeros(B, H, spec.max_blocks, 2, d, dtype=tdt, device=dev)
        layers.append(dict(k=k, v=v, desc=desc))
    dims = resa.dims_for(k0, Hq)
    ws = [resa.alloc_workspace(dims, spec.max_len, f, device=dev) for _ in range(L)]

    # a1: descriptor build after prefill (timed once per layer, outside the
    # step; a first untimed pass loads the module)
    for ly in layers:
        resa.build_desc(ly["k"], spec.len0, ly["desc"], Hq)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for ly in layers:
        resa.build_desc(ly["k"], spec.len0, ly["desc"], Hq)
    ev[1].record()
    torch.cuda.synchronize()
    build_desc_us = ev[0].elapsed_time(ev[1]) * 1000.0 / L

    # resident per-step inputs: f decode sets, one rectify set
    dec_in = []
    for t in range(f):
        q, kn, vn = decode_inputs(spec, t)
        dec_in.append((dev_t(q), dev_t(kn), dev_t(vn)))
    len_start = spec.len0
    q_f, k_f, v_f = rectify_inputs(spec, 0, len_start + f, f)
    rect_in = (dev_t(q_f), dev_t(k_f), dev_t(v_f))
    n_at = {t: resa.num_selected(len_start + t + 1, spec.r, spec.n_min) for t in range(f)}
    outs = [torch.empty(B, Hq, d, dtype=tdt, device=dev) for _ in range(L)]
    lses = [torch.empty(B, Hq, dtype=torch.float32, device=dev) for _ in range(L)]
    sels = [[torch.empty(B, H, n_at[t], dtype=torch.int32, device=dev) for t in range(f)]
            for _ in range(L)]
    out_f = [torch.empty(B, f, Hq, d, dtype=tdt, device=dev) for _ in range(L)]

    # One step = f decode positions x L layers, then L rectifications. Every
    # replay decodes positions len0 .. len0+f-1 again (the same cache slots are
    # rewritten with the same values), so each replay does identical work.
    def step(timing=None, stages=False):
        for t in range(f):
            length = len_start + t + 1
            q, kn, vn = dec_in[t]
            for li, ly in enumerate(layers):
                if timing is not None:
                    e0, e1, e2 = timing["dec"][t][li]
                    e0.record()
                if not stages:
                    resa.decode_sparse(q, kn, vn, ly["k"], ly["v"], ly["desc"], length, spec.r,
                                       spec.n_min, 1.0, outs[li], ws[li], lse=lses[li],
                                       sel=sels[li][t])
                else:
                    resa.select_blocks(q, kn, vn, ly["k"], ly["v"], ly["desc"], length, spec.r,
                                       spec.n_min, sels[li][t], ws[li])
                    if timing is not None:
                        e1.record()
                    resa.attend_blocks(q, ly["k"], ly["v"], length, sels[li][t], 1.0, outs[li],
                                       ws[li], lse=lses[li])
                if timing is not None:
                    e2.record()
        length = len_start + f
        for li, ly in enumerate(layers):
            if timing is not None:
                timing["rect"][li][0].record()
            resa.rectify(rect_in[0], rect_in[1], rect_in[2], ly["k"], ly["v"], ly["desc"], length,
                         f, 1.0, out_f[li], ws[li])
            if timing is not None:
                timing["rect"][li][1].record()

    torch.cuda.synchronize()
    # eager run once (also validates arguments), then capture
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    for w in ws:
        assert resa.workspace_status(w) == resa.RESA_OK
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    mk = lambda: torch.cuda.Event(enable_timing=True, external=True)  # noqa: E731
    timing = {"dec": [[(mk(), mk(), mk()) for _ in range(L)] for _ in range(f)],
              "rect": [(mk(), mk()) for _ in range(L)]}
    graph_t = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_t, stream=stream):
        step(timing)
    graph_s = timing_s = None
    if full:
        # the same step through the two stage calls (score + select, then
        # attention): the per-stage split
        timing_s = {"dec": [[(mk(), mk(), mk()) for _ in range(L)] for _ in range(f)],
                    "rect": [(mk(), mk()) for _ in range(L)]}
        graph_s = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_s, stream=stream):
            step(timing_s, stages=True)

    res = {"graph": graph, "layers": layers, "ws": ws, "dec_in": dec_in, "rect_in": rect_in,
           "len_start": len_start, "build_desc_us": build_desc_us}

    def timed_region(steps, warmup, dist=None, sampler=None):
        for _ in range(warmup):
            graph.replay()
        torch.cuda.synchronize()
        if sampler is not None:
            sampler.start()
            time.sleep(0.3)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            t0.record(stream)
            for _ in range(steps):
                graph.replay()
            t1.record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        total_ms = t0.elapsed_time(t1)
        clocks = None
        if sampler is not None:
            # keep the GPU busy while the sampler catches a few more readings
            t_end = time.time() + 0.4
            while time.time() < t_end:
                graph.replay()
                torch.cuda.synchronize()
            clocks = sampler.stop()
        return total_ms, clocks
    res["timed_region"] = timed_region

    def breakdown():
        reps = max(3, min(args.steps, 10))
        dec_us, sel_us, att_us, rect_us = [], [], [], []
        for _ in range(reps):
            graph_t.replay()
            torch.cuda.synchronize()
            for t in range(f):
                for li in range(L):
                    e0, _, e2 = timing["dec"][t][li]
                    dec_us.append(e0.elapsed_time(e2) * 1000.0)
            for li in range(L):
                a, b = timing["rect"][li]
                rect_us.append(a.elapsed_time(b) * 1000.0)
            if graph_s is not None:
                graph_s.replay()
                torch.cuda.synchronize()
                for t in range(f):
                    for li in range(L):
                        e0, e1, e2 = timing_s["dec"][t][li]
                        sel_us.append(e0.elapsed_time(e1) * 1000.0)
                        att_us.append(e1.elapsed_time(e2) * 1000.0)
        return dec_us, sel_us, att_us, rect_us

    # the sparse decode calls alone and the dense (r = 1) arm, each as f * L
    # calls back to back in one CUDA graph: the method's gain over dense
    # attention at the same length
    def graph_us(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for t in range(f):
                for li, ly in enumerate(layers):
                    fn(t, li, ly)
        g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        reps = 3
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) * 1000.0 / (reps * f * L)

    def sparse_call(t, li, ly):
        q, kn, vn = dec_in[t]
        resa.decode_sparse(q, kn, vn, ly["k"], ly["v"], ly["desc"], len_start + t + 1, spec.r,
                           spec.n_min, 1.0, outs[li], ws[li], lse=lses[li], sel=sels[li][t])

    def dense_call(t, li, ly):
        q, kn, vn = dec_in[t]
        resa.decode_dense(q, kn, vn, ly["k"], ly["v"], ly["desc"], len_start + t + 1, 1.0,
                          outs[li], ws[li], lse=lses[li])

    def attend_alone():
        # f * L launches back to back (every layer's selected blocks, so
        # consecutive launches read different caches)
        ga = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ga, stream=stream):
            for t in range(f):
                q = dec_in[t][0]
                for li, ly in enumerate(layers):
                    resa.attend_blocks(q, ly["k"], ly["v"], len_start + t + 1, sels[li][t], 1.0,
                                       outs[li], ws[li], lse=lses[li])
        ga.replay()
        torch.cuda.synchronize()
        ta0 = torch.cuda.Event(enable_timing=True)
        ta1 = torch.cuda.Event(enable_timing=True)
        reps_a = max(3, min(args.steps, 10))
        with torch.cuda.stream(stream):
            ta0.record(stream)
            for _ in range(reps_a):
                ga.replay()
            ta1.record(stream)
        torch.cuda.synchronize()
        del ga
        return ta0.elapsed_time(ta1) * 1000.0 / (reps_a * f * L)

    def summary():
        """Per-call and back-to-back figures with their byte counts."""
        hbm_peak, tf_peak, peak_kind = peaks()
        dec_us, sel_us, att_us, rect_us = breakdown()
        sparse_graph_us = graph_us(sparse_call)
        dense_graph_us = graph_us(dense_call)
        attend_launch_us = attend_alone()
        for w in ws:
            assert resa.workspace_status(w) == resa.RESA_OK
        # bytes of the algorithm (descriptors + selected K/V + Q/O)
        n_mid = n_at[f // 2]
        len_mid = len_start + f // 2 + 1
        M_mid = (len_mid + 15) // 16
        qo = 2 * B * Hq * d * esize
        desc_bytes = B * H * M_mid * 2 * d * esize
        sel_kv = B * H * n_mid * 16 * 2 * d * esize
        attend_bytes = sel_kv + qo + B * H * n_mid * 4
        decode_bytes = desc_bytes + sel_kv + qo
        rect_len = len_start + f
        rect_bytes = (B * H * rect_len * 2 * d * esize + 2 * B * f * Hq * d * esize
                      + 2 * B * f * H * d * esize)
        rect_flops = 4.0 * B * Hq * d * (f * rect_len - f * (f - 1) / 2)
        decode_med = statistics.median(dec_us)
        rect_med = statistics.median(rect_us)
        att_gbs = attend_bytes / (attend_launch_us * 1e-6) / 1e9
        out = {
            "decode_us": round(decode_med, 3),
            "decode_us_p10_p90": [round(float(np.percentile(dec_us, 10)), 3),
                                  round(float(np.percentile(dec_us, 90)), 3)],
            "sparse_decode_graph_us": round(sparse_graph_us, 3),
            "dense_decode_graph_us": round(dense_graph_us, 3),
            "speedup_vs_dense": round(dense_graph_us / sparse_graph_us, 2),
            "decode_bytes": decode_bytes,
            "decode_hbm_gbs": round(decode_bytes / (decode_med * 1e-6) / 1e9, 1),
            "decode_frac_of_measured_hbm": round(decode_bytes / (decode_med * 1e-6) / 1e9 / hbm_peak, 4),
            "decode_graph_frac_of_measured_hbm": round(
                decode_bytes / (sparse_graph_us * 1e-6) / 1e9 / hbm_peak, 4),
            "attend_launch_us": round(attend_launch_us, 3),
            "attend_hbm_gbs": round(att_gbs, 1),
            "attend_frac_of_measured_hbm": round(att_gbs / hbm_peak, 4),
            "attend_bytes": attend_bytes,
            "rectify_us": round(rect_med, 3),
            "rectify_amortised_us_per_token": round(rect_med / f, 3),
            "rectify_hbm_gbs": round(rect_bytes / (rect_med * 1e-6) / 1e9, 1),
            "rectify_frac_of_measured_hbm": round(rect_bytes / (rect_med * 1e-6) / 1e9 / hbm_peak, 4),
            "rectify_tflops": round(rect_flops / (rect_med * 1e-6) / 1e12, 2),
            "build_desc_us": round(build_desc_us, 2),
        }
        if sel_us:
            out["staged_decode_us"] = round(statistics.median([a + b for a, b in zip(sel_us, att_us)]), 3)
            out["staged_select_us"] = round(statistics.median(sel_us), 3)
            out["staged_attend_us"] = round(statistics.median(att_us), 3)
        return out
    res["summary"] = summary

    def e2e():
        return run_e2e(args, resa, spec, layers, ws, dec_in, rect_in, len_start, stream, dev, tdt)
    res["e2e"] = e2e
    return res


def extra_workloads(args, resa, dev, stream, L):
    """The other benchmark workloads on the same GPU (amortised step, per-call
    and back-to-back decode, attention alone, rectify, dense arm)."""
    import torch
    from workload import config
    runs = [("resa_decode_256k_b1_r0.1", 3, {}), ("resa_decode_256k_b1_r0.05", 3, {"r": 0.05}),
            ("resa_decode_32k_b4_needles", 1, {}), ("resa_decode_64k_b16_f32_r0.1", 4, {})]
    out = {}
    for name, idx, over in runs:
        spec = config(idx, steps=64, **over)
        m = measure_workload(args, resa, spec, L, dev, stream, host_cache=False, full=False)
        total_ms, _ = m["timed_region"](max(3, args.steps // 4), args.warmup)
        step_ms = total_ms / max(3, args.steps // 4)
        s = m["summary"]()
        s = {"value": round(step_ms * 1000.0 / (spec.f * L), 3), **s,
             "amortised_speedup_vs_dense": round(s["dense_decode_graph_us"] /
                                                 (step_ms * 1000.0 / (spec.f * L)), 2),
             "context": spec.len0, "batch": spec.batch, "r": spec.r, "f": spec.f}
        out[name] = s
        del m
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank):
    import torch
    import __graft_entry__
    __graft_entry__.build()
    import block_sparse_attention_quest_b200 as resa
    from workload import config

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg_idx = WORKLOADS[args.workload]
    over = {"steps": 64}
    if args.r is not None:
        over["r"] = args.r
    if args.f is not None:
        over["f"] = args.f
    spec = config(cfg_idx, **over)
    shard = args.shard == "heads" and world > 1
    if shard:
        # this rank's KV heads of every layer (no exchange inside the path)
        import dataclasses
        from block_sparse_attention_quest_b200.sharding import kv_head_range
        h0, h1 = kv_head_range(spec.n_kv_heads, rank, world)
        spec = dataclasses.replace(spec, n_kv_heads=h1 - h0, n_q_heads=(h1 - h0) * spec.group)
    f, L = spec.f, args.layers
    B, Hq, H = spec.batch, spec.n_q_heads, spec.n_kv_heads
    stream = torch.cuda.Stream(device=dev)
    m = measure_workload(args, resa, spec, L, dev, stream, host_cache=not shard, full=True)

    dist = None
    if world > 1:
        import torch.distributed as dist

    # timed region: exactly K replays of the step graph after W warm-up ones
    total_ms, clocks = m["timed_region"](args.steps, args.warmup, dist, ClockSampler(local_rank))
    total_ms = max_over_ranks(total_ms, dist, dev)
    step_ms = total_ms / args.steps
    summ = m["summary"]()

    # end-to-end through the public API with host buffers (eager calls)
    e2e = None
    if not args.no_e2e:
        e2e = m["e2e"]()
        e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], dist, dev)
        if world > 1:
            e2e["h2d"] *= world
            e2e["d2h"] *= world

    hbm_peak, tf_peak, peak_kind = peaks()
    # replicas: every rank decodes a whole layer; head shards: the ranks
    # decode one layer together
    units = 1 if shard else world
    us_per_decode = step_ms * 1000.0 / (f * L) / units
    tokens_per_s = B * f * L * units / (step_ms * 1e-3) / L
    launches_per_step = f * L * 3 + L * 3
    wl = WORKLOAD_NAMES[cfg_idx]
    custom = args.r is not None or args.f is not None
    res = {
        "metric": METRIC,
        "value": round(us_per_decode, 3),
        "unit": "us",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": False,
        "scaling": "strong" if shard else "weak",
        "vs_baseline": None,
        "dtype": spec.dtype,
        "data": "synthetic (seeded N(0,1) + block means; no dataset, no weights)",
        "config": {
            "workload": wl, "batch": B, "context": spec.len0,
            "q_heads": Hq, "kv_heads": H, "head_dim": spec.head_dim, "block": 16, "r": spec.r,
            "n_min": spec.n_min, "f": f, "layers": L,
            "step": f"{f} sparse decode steps x {L} layers + {L} rectifications",
            "l2": f"inputs larger than L2: {L} independent layer caches visited round-robin",
            "parallelism": (f"KV-head shards x{world} (this rank's heads: {H})" if shard else
                            f"replicas x{world}" if world > 1 else "single GPU"),
            "timing": "CUDA graph replay, CUDA events on the launching stream",
        },
        **summ,
        "amortised_speedup_vs_dense": round(summ["dense_decode_graph_us"] / us_per_decode, 2),
        "decode_kernels": "score_kernel -> select_reg_kernel -> attend_bf16_kernel (PDL chain)",
        "tokens_per_s": round(tokens_per_s, 1),
        "roofline": {
            "kernel": "attend_bf16_kernel (split-KV attention, LSE merge in the last CTA)",
            "timing": "average over f * layers back-to-back launches in one CUDA graph",
            "bound": "hbm", "achieved": summ["attend_hbm_gbs"], "peak": hbm_peak, "unit": "GB/s",
            "frac": round(summ["attend_hbm_gbs"] / hbm_peak, 4),
            "traffic": None if custom else counter("attention", "traffic", wl),
            "peak_kind": f"{peak_kind} copy bandwidth (burst)",
            "bytes_per_launch": summ["attend_bytes"],
            "bytes": "selected K/V + q + out + block ids",
        },
        "rectify": {
            "kernel": "rectify_tc_kernel (tcgen05.mma, TMEM accumulators) + merge_rows_kernel",
            "us": summ["rectify_us"], "hbm_gbs": summ["rectify_hbm_gbs"],
            "frac_of_measured_hbm": summ["rectify_frac_of_measured_hbm"],
            "tflops": summ["rectify_tflops"],
            "tensor_pipe_active_pct": (None if custom or wl != "resa_decode_128k_b1"
                                       else counter("rectify", "tensor_pipe_active_pct")),
            "tensor_pipe_source": "ncu sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_active, "
                                  "one cold launch at 128K, f = 32 (null once the kernel changed)",
        },
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if not args.no_prefill:
        res["prefill"] = run_prefill(resa, stream, dev, tf_peak, peak_kind)
    if e2e is not None:
        res["e2e"] = {"value": round(e2e["ms_per_step"] * 1000.0 / (f * L) / units, 3),
                      "unit": "us", "h2d_bytes_per_step": e2e["h2d"],
                      "d2h_bytes_per_step": e2e["d2h"]}
    del m
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    if not args.no_workloads and world == 1 and not custom and args.workload == "128k":
        res["workloads"] = extra_workloads(args, resa, dev, stream, L)
        try:
            res["workloads"]["resa_decode_ragged_b4"] = run_varlen(resa, stream, dev, hbm_peak)
        except Exception as e:   # reported in the line; the other measurements stand
            res["workloads"]["resa_decode_ragged_b4"] = {"error": f"{type(e).__name__}: {e}"}
    return res, spec


def run_prefill(resa, stream, dev, tf_peak, peak_kind, length=16384):
    """The prefill-side step (causal attention of every prompt position with
    the descriptors from the same pass) on one prompt of `length` tokens at
    the benchmark's head shape; CUDA events around back-to-back calls."""
    import torch
    from workload import Spec, prefill_queries
    spec = Spec(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, len0=length, steps=0)
    g = torch.Generator(device=dev).manual_seed(spec.seed)
    k = torch.randn(1, 8, spec.max_len, 128, device=dev, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 8, spec.max_len, 128, device=dev, generator=g).to(torch.bfloat16)
    q = torch.from_numpy(prefill_queries(spec)).to(dev).to(torch.bfloat16)
    desc = torch.zeros(1, 8, spec.max_blocks, 2, 128, dtype=torch.bfloat16, device=dev)
    out = torch.empty_like(q)
    ws = resa.alloc_workspace(resa.dims_for(k, 32), spec.max_len, 0, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(2):
            resa.prefill(q, k, v, desc, length, 1.0, out, ws)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        reps = 5
        e0.record(stream)
        for _ in range(reps):
            resa.prefill(q, k, v, desc, length, 1.0, out, ws)
        e1.record(stream)
    torch.cuda.synchronize()
    assert resa.workspace_status(ws) == resa.RESA_OK
    us = e0.elapsed_time(e1) * 1000.0 / reps
    # QK^T and PV over the causal triangle: 4 * Hq * d * sum_i (i + 1)
    flops = 4.0 * 32 * 128 * (length * (length + 1) / 2)
    tflops = flops / (us * 1e-6) / 1e12
    return {"workload": f"prefill_{length // 1024}k_b1", "us": round(us, 1),
            "tflops": round(tflops, 1), "frac": round(tflops / tf_peak, 4),
            "peak": tf_peak, "peak_kind": f"{peak_kind} cuBLAS bf16 (burst)",
            "flops": flops, "bound": "tensor",
            "note": "descriptors of the prompt written by the same pass"}


def run_varlen(resa, stream, dev, hbm_peak, lens=(131072, 98304, 65536, 32768), r=0.1,
               n_min=16, f=32, windows=(32, 0, 17, 32)):
    """A ragged batch (continuous batching): one cache length per row, each
    row's descriptors, selection and attention bounded by its own length, and
    a rectification with a window per row (0 = the row is not rectified).
    CUDA events around back-to-back calls of the per-row-length entry points;
    bytes = each row's descriptors + selected K/V + q/out (decode) and each
    rectified row's whole cache (rectify)."""
    import torch
    B, Hq, H, d = len(lens), 32, 8, 128
    max_len = ((max(lens) + 15) // 16) * 16 + 64
    g = torch.Generator(device=dev).manual_seed(20240610)
    k = torch.randn(B, H, max_len, d, device=dev, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, max_len, d, device=dev, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hq, d, device=dev, generator=g).to(torch.bfloat16)
    q_f = torch.randn(B, f, Hq, d, device=dev, generator=g).to(torch.bfloat16)
    k_f = torch.randn(B, f, H, d, device=dev, generator=g).to(torch.bfloat16)
    v_f = torch.randn(B, f, H, d, device=dev, generator=g).to(torch.bfloat16)
    lens_t = torch.tensor(lens, dtype=torch.int32, device=dev)
    win_t = torch.tensor(windows, dtype=torch.int32, device=dev)
    bound = max(lens)
    desc = torch.zeros(B, H, max_len // 16, 2, d, dtype=torch.bfloat16, device=dev)
    out = torch.empty(B, Hq, d, dtype=torch.bfloat16, device=dev)
    out_f = torch.empty(B, f, Hq, d, dtype=torch.bfloat16, device=dev)
    dims = resa.dims_for(k, Hq)
    ws = resa.alloc_workspace(dims, max_len, f, device=dev)

    def timed(call, reps):
        with torch.cuda.stream(stream):
            for _ in range(3):
                call()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                call()
            e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1000.0 / reps

    with torch.cuda.stream(stream):
        resa.build_desc_varlen(k, lens_t, bound, desc, Hq, stream=stream)
    dec_us = timed(lambda: resa.decode_sparse_varlen(q, None, None, k, v, desc, lens_t, bound, r,
                                                     n_min, 1.0, out, ws, stream=stream), 64)
    rect_us = timed(lambda: resa.rectify_varlen(q_f, k_f, v_f, k, v, desc, lens_t, bound, f, 1.0,
                                                out_f, ws, windows=win_t, stream=stream), 8)
    assert resa.workspace_status(ws) == resa.RESA_OK
    esize = 2
    dec_bytes = 2 * B * Hq * d * esize
    rect_bytes = 0
    for L_b, w_b in zip(lens, windows):
        M = (L_b + 15) // 16
        n = resa.num_selected(L_b, r, n_min)
        dec_bytes += H * ((M - 1) * 2 * d * esize + n * 16 * 2 * d * esize)
        if w_b > 0:
            rect_bytes += H * L_b * 2 * d * esize + 2 * w_b * (Hq + H) * d * esize
    del k, v, desc, ws
    torch.cuda.empty_cache()
    dec_gbs = dec_bytes / (dec_us * 1e-6) / 1e9
    rect_gbs = rect_bytes / (rect_us * 1e-6) / 1e9
    return {"lens": list(lens), "r": r, "n_min": n_min, "f": f, "windows": list(windows),
            "decode_us": round(dec_us, 3), "decode_bytes": dec_bytes,
            "decode_hbm_gbs": round(dec_gbs, 1), "decode_frac_of_measured_hbm": round(dec_gbs / hbm_peak, 4),
            "rectify_us": round(rect_us, 3), "rectify_bytes": rect_bytes,
            "rectify_hbm_gbs": round(rect_gbs, 1),
            "rectify_frac_of_measured_hbm": round(rect_gbs / hbm_peak, 4),
            "timing": "CUDA events around back-to-back calls of resa_decode_sparse_varlen and "
                      "resa_rectify_varlen (no append, fixed lengths)"}


def run_e2e(args, resa, spec, layers, ws, dec_in, rect_in, len_start, stream, dev, tdt):
    """The same step through the public calls with host buffers: every step
    copies its inputs (each decode call's q, k_new, v_new for every layer and
    position, and each layer's rectify inputs) from one pinned host buffer to
    the device, runs the calls eagerly, and reads all of the step's outputs
    back into pinned host memory, inside the timed region."""
    import torch
    f, L = spec.f, len(layers)
    B, Hq, H, d = spec.batch, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
    esz = torch.empty(0, dtype=tdt).element_size()

    def nbytes(x):
        return x.numel() * x.element_size()

    # packed input layout: [position][layer][q | k_new | v_new], then
    # [layer][q_f | k_f | v_f]; every piece starts 16-byte aligned
    pieces = [s for _ in range(1) for t in range(f) for _li in range(L) for s in dec_in[t]]
    pieces += [x for _li in range(L) for x in rect_in]
    offs, off = [], 0
    for x in pieces:
        offs.append(off)
        off += (nbytes(x) + 15) // 16 * 16
    h_in = torch.empty(off, dtype=torch.uint8).pin_memory()
    for x, o in zip(pieces, offs):
        h_in[o:o + nbytes(x)].copy_(x.cpu().contiguous().view(-1).view(torch.uint8))
    d_in = torch.empty(off, dtype=torch.uint8, device=dev)

    def view(o, like):
        return d_in[o:o + nbytes(like)].view(tdt).view(like.shape)
    it = iter(zip(pieces, offs))
    d_dec = [[tuple(view(o, x) for x, o in (next(it), next(it), next(it))) for _li in range(L)]
             for _t in range(f)]
    d_rect = [tuple(view(o, x) for x, o in (next(it), next(it), next(it))) for _li in range(L)]
    # every call writes its own slice of one output buffer, read back once
    n_out = L * f * B * Hq * d
    n_out_f = L * B * f * Hq * d
    d_out = torch.empty(n_out + n_out_f, dtype=tdt, device=dev)
    h_out = torch.empty(n_out + n_out_f, dtype=tdt).pin_memory()
    out = d_out[:n_out].view(L, f, B, Hq, d)
    out_f = d_out[n_out:].view(L, B, f, Hq, d)
    h2d = off
    d2h = nbytes(h_out)

    def step():
        d_in.copy_(h_in, non_blocking=True)
        for t in range(f):
            length = len_start + t + 1
            for li, ly in enumerate(layers):
                q, kn, vn = d_dec[t][li]
                resa.decode_sparse(q, kn, vn, ly["k"], ly["v"], ly["desc"], length, spec.r,
                                   spec.n_min, 1.0, out[li, t], ws[li])
        for li, ly in enumerate(layers):
            q_f, k_f, v_f = d_rect[li]
            resa.rectify(q_f, k_f, v_f, ly["k"], ly["v"], ly["desc"], len_start + f, f, 1.0,
                         out_f[li], ws[li])
        h_out.copy_(d_out, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(max(1, args.warmup)):
            step()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        n = max(2, min(args.steps, 10))
        t0.record(stream)
        for _ in range(n):
            step()
        t1.record(stream)
    torch.cuda.synchronize()
    return {"ms_per_step": t0.elapsed_time(t1) / n, "h2d": h2d, "d2h": d2h}


# ----------------------------------------------------------------- CPU oracle
def host_info() -> dict:
    """Core count and CPU model of the host the oracle runs on."""
    model = None
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model}


class OracleSample:
    """The CPU oracle on a bounded sample of the workload. One sample step is
    one decode step of the whole batch plus the rectification of one (batch,
    KV head) group; the rectification time, scaled by the number of groups
    and amortised over f, is added to the decode time to give microseconds
    per amortised decode step (the benchmark's unit). The wall time of the
    sample step itself is kept too."""

    def __init__(self, spec):
        import oracle as orc
        from workload import make_cache
        self.orc = orc
        self.spec = spec
        K, V = make_cache(spec)
        self.st = orc.State(K, V, spec.len0, spec.group)
        self.groups = spec.batch * spec.n_kv_heads
        self.n = 0

    @staticmethod
    def threads() -> int:
        """Threads the oracle's BLAS calls use under the current limits."""
        try:
            from threadpoolctl import threadpool_info
            return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        except Exception:
            return os.cpu_count() or 1

    def step(self):
        """Returns (us per amortised decode step, wall seconds of the sample)."""
        from workload import decode_inputs, rectify_inputs
        spec, st, orc = self.spec, self.st, self.orc
        q, kn, vn = decode_inputs(spec, self.n % spec.steps)
        t0 = time.perf_counter()
        st.decode(q, kn, vn, spec.r, spec.n_min, 1.0)
        dec_s = time.perf_counter() - t0
        f, G = spec.f, spec.group
        q_f, k_f, v_f = rectify_inputs(spec, 0, st.length, f)
        sub = orc.State.__new__(orc.State)
        sub.K, sub.V = st.K[:1, :1].copy(), st.V[:1, :1].copy()
        sub.lo, sub.hi = st.lo[:1, :1].copy(), st.hi[:1, :1].copy()
        sub.length, sub.group = st.length, G
        t0 = time.perf_counter()
        sub.rectify(q_f[:1, :, :G], k_f[:1, :, :1], v_f[:1, :, :1], f, 1.0)
        rect1_s = time.perf_counter() - t0
        self.n += 1
        return (dec_s + rect1_s * self.groups / f) * 1e6, dec_s + rect1_s

    def describe(self, steps):
        return (f"{steps} sample steps, each = 1 oracle decode step (whole batch) + rectify of 1 "
                f"of {self.groups} (batch, KV head) groups; value = decode + rectify x{self.groups} "
                f"/ f={self.spec.f}; context {self.spec.len0}")

    def timed(self, steps: int, single_thread: bool = False):
        """Median us per amortised decode step and median sample wall ms over
        `steps` sample steps (after one warm-up), on all cores or one."""
        import contextlib
        ctx = contextlib.nullcontext()
        if single_thread:
            from threadpoolctl import threadpool_limits
            ctx = threadpool_limits(limits=1)
        with ctx:
            threads = self.threads()
            self.step()
            runs = [self.step() for _ in range(steps)]
        return (statistics.median(r[0] for r in runs), statistics.median(r[1] for r in runs) * 1e3,
                threads)


def cpu_baseline(spec, steps: int = 3) -> dict:
    """The oracle on this host, on all cores and on one thread."""
    smp = OracleSample(spec)
    us, _, threads = smp.timed(steps)
    us1, _, _ = smp.timed(steps, single_thread=True)
    return {"value": round(us, 1), "unit": "us", "cores": threads, "kind": "oracle",
            "sample": smp.describe(steps), **host_info(),
            "single_thread": {"value": round(us1, 1), "unit": "us", "cores": 1}}


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle as it stands, timed on this host's cores."""
    from workload import config
    cfg_idx = WORKLOADS[args.workload]
    over = {"steps": 64}
    if args.r is not None:
        over["r"] = args.r
    if args.f is not None:
        over["f"] = args.f
    spec = config(cfg_idx, **over)
    if rank != 0:
        return None
    smp = OracleSample(spec)
    threads = smp.threads()
    for _ in range(args.warmup):
        smp.step()
    runs = [smp.step() for _ in range(args.steps)]
    us = statistics.median(r[0] for r in runs)
    wall_ms = statistics.median(r[1] for r in runs) * 1e3
    return {
        "impl": "reference", "metric": METRIC, "value": round(us, 1), "unit": "us",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(wall_ms, 3),
        "ms_per_step_is": "measured wall time of one sample step (1 decode + 1 group's rectify)",
        "value_is": "us per amortised decode step computed from the sample "
                    "(decode + rectify x groups / f)",
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) + block means; no dataset, no weights)",
        "config": {"workload": WORKLOAD_NAMES[cfg_idx], "batch": spec.batch,
                   "context": spec.len0, "r": spec.r, "f": spec.f, "layers": args.layers},
        "cpu_baseline": {"value": round(us, 1), "unit": "us", "cores": threads,
                         "kind": "oracle", "sample": smp.describe(args.steps), **host_info()},
        "e2e": {"value": round(us, 1), "unit": "us", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res, spec = run_ours(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(spec)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()

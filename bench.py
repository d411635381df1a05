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

# DRAM bytes (read + write) per launch of the attention kernel from one ncu
# capture of this workload (profiles/attend_bf16_kernel_128k.md). Reset an
# entry to None whenever attend_bf16_kernel changes.
NCU_TRAFFIC = {"resa_decode_128k_b1": 53982720}


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
def run_ours(args, rank, world, local_rank):
    import torch
    import __graft_entry__
    __graft_entry__.build()
    import block_sparse_attention_quest_b200 as resa
    from workload import config, decode_inputs, make_cache, rectify_inputs

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg_idx = WORKLOADS[args.workload]
    over = {"steps": 64}
    if args.r is not None:
        over["r"] = args.r
    if args.f is not None:
        over["f"] = args.f
    spec = config(cfg_idx, **over)
    f, L = spec.f, args.layers
    tdt = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
    esize = 2 if spec.dtype == "bf16" else 4
    B, Hq, H, d = spec.batch, spec.n_q_heads, spec.n_kv_heads, spec.head_dim

    def dev_t(x):
        return torch.from_numpy(np.ascontiguousarray(x)).to(dev).to(tdt)

    K, V = make_cache(spec)
    k0, v0 = dev_t(K), dev_t(V)
    del K, V
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

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    # eager run once (also validates arguments), then capture
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    assert resa.workspace_status(ws[0]) == resa.RESA_OK
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    mk = lambda: torch.cuda.Event(enable_timing=True, external=True)  # noqa: E731
    timing = {"dec": [[(mk(), mk(), mk()) for _ in range(L)] for _ in range(f)],
              "rect": [(mk(), mk()) for _ in range(L)]}
    graph_t = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_t, stream=stream):
        step(timing)
    # the same step through the two stage calls (score + select, then
    # attention): the per-stage split and the attention kernel on its own
    timing_s = {"dec": [[(mk(), mk(), mk()) for _ in range(L)] for _ in range(f)],
                "rect": [(mk(), mk()) for _ in range(L)]}
    graph_s = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_s, stream=stream):
        step(timing_s, stages=True)

    dist = None
    if world > 1:
        import torch.distributed as dist

    def barrier():
        if dist is not None:
            dist.barrier()

    # warm-up
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()

    # timed region: exactly K replays of the step graph
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    total_ms = t0.elapsed_time(t1)
    # keep the GPU busy while the sampler catches a few more readings
    t_end = time.time() + 0.4
    while time.time() < t_end:
        graph.replay()
        torch.cuda.synchronize()
    clocks = sampler.stop()
    total_ms = max_over_ranks(total_ms, dist, dev)
    step_ms = total_ms / args.steps

    # per-stage breakdown (graph with captured timing events)
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
        graph_s.replay()
        torch.cuda.synchronize()
        for t in range(f):
            for li in range(L):
                e0, e1, e2 = timing_s["dec"][t][li]
                sel_us.append(e0.elapsed_time(e1) * 1000.0)
                att_us.append(e1.elapsed_time(e2) * 1000.0)

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
    sparse_graph_us = graph_us(sparse_call)
    dense_graph_us = graph_us(dense_call)

    # the attention kernel on its own: f * L launches back to back (every
    # layer's selected blocks, so consecutive launches read different caches)
    graph_a = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_a, stream=stream):
        for t in range(f):
            q = dec_in[t][0]
            for li, ly in enumerate(layers):
                resa.attend_blocks(q, ly["k"], ly["v"], len_start + t + 1, sels[li][t], 1.0,
                                   outs[li], ws[li], lse=lses[li])
    graph_a.replay()
    torch.cuda.synchronize()
    ta0 = torch.cuda.Event(enable_timing=True)
    ta1 = torch.cuda.Event(enable_timing=True)
    reps_a = max(3, min(args.steps, 10))
    with torch.cuda.stream(stream):
        ta0.record(stream)
        for _ in range(reps_a):
            graph_a.replay()
        ta1.record(stream)
    torch.cuda.synchronize()
    attend_launch_us = ta0.elapsed_time(ta1) * 1000.0 / (reps_a * f * L)

    # end-to-end through the public API with host buffers (eager calls)
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, resa, spec, layers, ws, dec_in, rect_in, len_start, stream, dev, tdt)
        e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], dist, dev)

    assert resa.workspace_status(ws[0]) == resa.RESA_OK
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
    rect_bytes = B * H * rect_len * 2 * d * esize + 2 * B * f * Hq * d * esize + 2 * B * f * H * d * esize
    rect_flops = 4.0 * B * Hq * d * (f * rect_len - f * (f - 1) / 2)

    hbm_peak, tf_peak, peak_kind = peaks()
    sel_med = statistics.median(sel_us)
    att_med = statistics.median(att_us)
    rect_med = statistics.median(rect_us)
    decode_med = statistics.median(dec_us)
    staged_med = statistics.median([a + b for a, b in zip(sel_us, att_us)])
    dec_gbs = decode_bytes / (decode_med * 1e-6) / 1e9
    att_gbs = attend_bytes / (attend_launch_us * 1e-6) / 1e9
    us_per_decode = step_ms * 1000.0 / (f * L) / world
    tokens_per_s = B * f * L * world / (step_ms * 1e-3) / L
    launches_per_step = f * L * 3 + L * 3
    res = {
        "metric": METRIC,
        "value": round(us_per_decode, 3),
        "unit": "us",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": spec.dtype,
        "data": "synthetic (seeded N(0,1) + block means; no dataset, no weights)",
        "config": {
            "workload": WORKLOAD_NAMES[cfg_idx], "batch": B, "context": spec.len0,
            "q_heads": Hq, "kv_heads": H, "head_dim": d, "block": 16, "r": spec.r,
            "n_min": spec.n_min, "f": f, "layers": L,
            "step": f"{f} sparse decode steps x {L} layers + {L} rectifications",
            "l2": f"inputs larger than L2: {L} independent layer caches visited round-robin",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "timing": "CUDA graph replay, CUDA events on the launching stream",
        },
        "decode_us": round(decode_med, 3),
        "decode_us_p10_p90": [round(float(np.percentile(dec_us, 10)), 3),
                              round(float(np.percentile(dec_us, 90)), 3)],
        "sparse_decode_graph_us": round(sparse_graph_us, 3),
        "dense_decode_graph_us": round(dense_graph_us, 3),
        "speedup_vs_dense": round(dense_graph_us / sparse_graph_us, 2),
        "amortised_speedup_vs_dense": round(dense_graph_us / us_per_decode, 2),
        "decode_kernels": "score_kernel -> select_reg_kernel -> attend_bf16_kernel (PDL chain)",
        "staged_decode_us": round(staged_med, 3),
        "staged_select_us": round(sel_med, 3),
        "staged_attend_us": round(att_med, 3),
        "attend_launch_us": round(attend_launch_us, 3),
        "attend_hbm_gbs": round(att_gbs, 1),
        "decode_hbm_gbs": round(decode_bytes / (decode_med * 1e-6) / 1e9, 1),
        "decode_bytes": decode_bytes,
        "decode_frac_of_measured_hbm": round(decode_bytes / (decode_med * 1e-6) / 1e9 / hbm_peak, 4),
        "rectify_us": round(rect_med, 3),
        "rectify_amortised_us_per_token": round(rect_med / f, 3),
        "rectify_hbm_gbs": round(rect_bytes / (rect_med * 1e-6) / 1e9, 1),
        "rectify_tflops": round(rect_flops / (rect_med * 1e-6) / 1e12, 2),
        "build_desc_us": round(build_desc_us, 2),
        "tokens_per_s": round(tokens_per_s, 1),
        "roofline": {
            "kernel": "attend_bf16_kernel (split-KV attention, LSE merge in the last CTA)",
            "timing": "average over f * layers back-to-back launches in one CUDA graph",
            "bound": "hbm", "achieved": round(att_gbs, 1), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(att_gbs / hbm_peak, 4),
            "traffic": (NCU_TRAFFIC.get(WORKLOAD_NAMES[cfg_idx])
                        if args.r is None and args.f is None else None),
            "peak_kind": f"{peak_kind} copy bandwidth",
            "bytes_per_launch": attend_bytes,
            "bytes": "selected K/V + q + out + block ids",
        },
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if not args.no_prefill:
        res["prefill"] = run_prefill(resa, stream, dev, tf_peak, peak_kind)
    if e2e is not None:
        res["e2e"] = {"value": round(e2e["ms_per_step"] * 1000.0 / (f * L) / world, 3),
                      "unit": "us", "h2d_bytes_per_step": e2e["h2d"],
                      "d2h_bytes_per_step": e2e["d2h"]}
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
class OracleSample:
    """The CPU oracle on a bounded sample of the workload. One sample step is
    one decode step of the whole batch plus the rectification of one (batch,
    KV head) group, the latter scaled by the number of groups; amortised over
    f it gives microseconds per decode step in the benchmark's unit."""

    def __init__(self, spec):
        import oracle as orc
        from workload import make_cache
        self.orc = orc
        self.spec = spec
        try:
            from threadpoolctl import threadpool_info
            self.threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        except Exception:
            self.threads = os.cpu_count() or 1
        K, V = make_cache(spec)
        self.st = orc.State(K, V, spec.len0, spec.group)
        self.groups = spec.batch * spec.n_kv_heads
        self.n = 0

    def step(self):
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
        rect_s = (time.perf_counter() - t0) * self.groups
        self.n += 1
        return (dec_s + rect_s / f) * 1e6

    def describe(self, steps):
        return (f"{steps} sample steps, each = 1 oracle decode step (whole batch) + rectify of 1 "
                f"of {self.groups} (batch, KV head) groups scaled x{self.groups}, amortised over "
                f"f={self.spec.f}; context {self.spec.len0}")


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
    for _ in range(args.warmup):
        smp.step()
    per = [smp.step() for _ in range(args.steps)]
    us = statistics.median(per)
    return {
        "impl": "reference", "metric": METRIC, "value": round(us, 1), "unit": "us",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(us * spec.f * args.layers / 1000.0, 3),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) + block means; no dataset, no weights)",
        "config": {"workload": WORKLOAD_NAMES[cfg_idx], "batch": spec.batch,
                   "context": spec.len0, "r": spec.r, "f": spec.f, "layers": args.layers},
        "cpu_baseline": {"value": round(us, 1), "unit": "us", "cores": smp.threads,
                         "kind": "oracle", "sample": smp.describe(args.steps)},
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
        smp = OracleSample(spec)
        smp.step()                       # warm-up (page-in, BLAS threads)
        per = [smp.step() for _ in range(3)]
        res["cpu_baseline"] = {"value": round(statistics.median(per), 1), "unit": "us",
                               "cores": smp.threads, "kind": "oracle",
                               "sample": smp.describe(3)}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()

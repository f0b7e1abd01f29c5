"""Benchmark of the DSA hot path: indexer -> top-2048 -> absorbed sparse MLA.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: the indexer scores
every earlier position of every query, the top-k kernel selects 2,048 per
query, and every layer of the configuration attends over that selection (one
attention launch for all layers).  The default configuration is the largest
that fits one GPU: 4 sequences x 2^20 positions, one selection reused by 3 RoPE
layers and 1 NoPE layer (1.11 GB of compulsory HBM traffic per step).  The
metric is per layer, so `value` counts query-layers per second.  Inputs are
resident in HBM when the timed region starts; every step streams more than
the 126 MB L2 holds, so no flush is needed between steps.

Timing: the K steps are captured into one CUDA graph; the timed region replays
that graph R times (R chosen so the region lasts at least --min-seconds,
default 1 s, long enough for a clock record), bracketed by a barrier and
synchronisation, timed with CUDA events on the launching stream, max over
ranks.  `ms_per_step` = region / (K x R).

The same run also measures the 64 x 32,768 decode batch and the chunked
prefill (8,192 queries over 40,960 positions; the indexer's tensor-core rate)
as extra keys.

Multi-GPU: `--gpus N` without torchrun spawns N processes itself (one per GPU,
NCCL); under torchrun each rank is one process.  Decode sequences are
independent, so each rank runs its own batch with no collective on the data
path; the only collectives are the barrier and the max-over-ranks reduction of
the device time ("scaling": "weak").

The reference arm (--impl reference) times the fp64 CPU oracle on a bounded
sample of the same workload (one query per step) on the host cores.
"""

from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_attention_16_b200 import accounting as acc  # noqa: E402
from sparse_attention_16_b200 import replicas  # noqa: E402
from sparse_attention_16_b200.workloads import (CONFIGS, make_workload, quantize_e4m3_rows, quantize_latent_fp8,  # noqa: E402
                                                small_case)

HEADLINE = "decode_b4_1m_4layers"
EXTRAS = ("decode_b64_32k", "prefill_32k_plus_8k", "decode_b16_32k_4queries")
METRIC = "sparse-MLA+DSA decode queries/s per layer; achieved HBM TB/s vs peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {"indexer": ["indexer.cuh", "ptx.cuh"], "indexer_fp8": ["indexer.cuh", "ptx.cuh"],
                  "topk": ["topk.cuh", "ptx.cuh"], "attend": ["attend.cuh", "ptx.cuh"]}


def kernel_source_hash(kernel):
    """Hash of the source files that define one kernel (its profile is void once they change)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_attention_16_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload):
    """dram bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    m_h = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    if not m_b or not m_h or m_h.group(1) != kernel_source_hash(kernel):
        return None
    return float(m_b.group(1))


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"dsa_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- our arm

def query_group(case):
    """Queries scored together per key tile: 8 in chunked prefill, 4 when a
    sequence decodes 4 queries at once, else 1."""
    if case.kind == "prefill":
        return 8
    return 4 if case.per_seq % 4 == 0 else 1


def measure(name, dev, steps, warmup, rank, world, local, min_seconds=0.0, sample_clocks=False, fp8=False,
            eager=False, e2e=False, e2e_steps=20, fp8_cache=False):
    """Times `steps` steps of configuration `name` (see the module docstring).
    Returns a dict with the timing, the per-kernel breakdown and the rooflines."""
    from sparse_attention_16_b200 import ops

    case = CONFIGS[name]
    # each rank owns an independent batch of the same shape (its own seed)
    case = dataclasses.replace(case, seed=replicas.rank_seed(case.seed, rank))
    wl = make_workload(case, dev)
    T, ld, k = wl.T, case.ld, case.topk
    n_layers = len(wl.layers)
    q_group = query_group(case)

    scores = torch.empty((T, ld), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    cnt = torch.empty((T,), dtype=torch.int32, device=dev)
    outs = [torch.empty((T, 64, 512), dtype=torch.bfloat16, device=dev) for _ in wl.layers]
    lses = [torch.empty((T, 64), dtype=torch.float32, device=dev) for _ in wl.layers]
    if fp8_cache:
        # FP8 latent rows (E4M3 codes + block scales) of the same seeded caches (input preparation, untimed)
        caches = [quantize_latent_fp8(L.cache, L.d_rope) for L in wl.layers]
        for L in wl.layers:
            L.cache = None
        torch.cuda.empty_cache()
    else:
        caches = [L.cache for L in wl.layers]
    layers = [dict(q_nope=L.q_nope, q_pe=L.q_pe, qmul=L.qmul, cache=c, d_rope=L.d_rope, out=o, lse=l)
              for L, c, o, l in zip(wl.layers, caches, outs, lses)]
    n_rows = caches[0].shape[0]
    att_ws = ops.workspace(ops.layers_workspace_bytes(T, n_layers, k), dev)
    # decode: the indexer also counts its scores into a histogram that the top-k's first pass reads
    hist = torch.empty((T, 2048), dtype=torch.int32, device=dev) if q_group == 1 else None
    topk_ws = ops.workspace(ops.topk_workspace_bytes(T, ld, k), dev) if q_group == 1 else None
    stream = torch.cuda.current_stream()
    if fp8:
        # E4M3 codes + per-row scales of the same seeded keys/queries (input preparation, untimed)
        q8, q8_scale = quantize_e4m3_rows(wl.q_idx)
        k8, k8_scale = quantize_e4m3_rows(wl.k_idx)

    # events around each kernel of every step of the breakdown graph (same stream)
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)] for _ in range(steps)]
    fw_ws = ops.workspace(ops.forward_workspace_bytes(T, ld, k, q_group, n_layers), dev)

    def step(i=None):
        if i is None:
            # the timed step: the public fused call (indexer, top-k, attention of every layer)
            if fp8:
                ops.sparse_mla_forward_fp8(q8, q8_scale, wl.w, k8, k8_scale, wl.seq_row_start, wl.q_seq, wl.q_pos,
                                           layers, ld, k=k, q_group=q_group, idx_out=idx, count_out=cnt, ws=fw_ws)
            else:
                ops.sparse_mla_forward(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos, layers, ld,
                                       k=k, q_group=q_group, idx_out=idx, count_out=cnt, ws=fw_ws)
            return
        # the breakdown step: the three calls separately, events between them
        e = ev[i]
        if e:
            e[0].record(stream)
        if fp8:
            ops.index_scores_fp8(q8, q8_scale, wl.w, k8, k8_scale, wl.seq_row_start, wl.q_seq, wl.q_pos, scores,
                                 q_group=q_group, hist=hist)
        else:
            ops.index_scores(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos, scores,
                             q_group=q_group, hist=hist)
        if e:
            e[1].record(stream)
        ops.topk(scores, wl.q_pos, k, idx, cnt, hist=hist, ws=topk_ws)
        if e:
            e[2].record(stream)
        ops.sparse_mla_attend_layers(layers, n_rows, wl.seq_row_start, wl.q_seq, idx, cnt, q_pos=wl.q_pos,
                                     ws=att_ws)
        if e:
            e[3].record(stream)

    for _ in range(max(warmup, 3)):
        step()
    step(0)   # the breakdown's separate calls, once before they are captured
    torch.cuda.synchronize()
    ops.check_errors()

    # The K timed steps are captured once into a CUDA graph, so host launch
    # overhead does not leak into the device timings; every kernel of every step
    # still runs.  The timed graph has no event nodes between kernels; a second
    # graph of the same steps with events around each kernel gives the
    # per-kernel breakdown, replayed after the timed region.
    graph = graph_ev = None
    n0 = ops.launch_count()
    if not eager:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(steps):
                step()
        launches_per_graph = ops.launch_count() - n0
        graph_ev = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_ev):
            stream = torch.cuda.current_stream()
            for i in range(steps):
                step(i)
        stream = torch.cuda.current_stream()
        # one untimed replay, timed to size the region
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        graph.replay()
        b.record(stream)
        torch.cuda.synchronize()
        one = a.elapsed_time(b) / 1e3
        replays = max(1, math.ceil(1.1 * min_seconds / max(one, 1e-6)))
        replays = int(replicas.max_over_ranks(float(replays), device=dev)) if world > 1 else replays
    else:
        replays = 1

    sampler = ClockSampler(local) if (sample_clocks and rank == 0) else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    if graph is not None:
        for _ in range(replays):
            graph.replay()
    else:
        n0 = ops.launch_count()
        for _ in range(steps):
            step()
    t1.record(stream)
    torch.cuda.synchronize()
    launches = (launches_per_graph * replays) if graph is not None else ops.launch_count() - n0
    elapsed = t0.elapsed_time(t1) / 1e3
    elapsed = replicas.max_over_ranks(elapsed, device=dev)
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if sampler else None
    ops.check_errors()
    # per-kernel breakdown (outside the timed region)
    if graph_ev is not None:
        graph_ev.replay()
    else:
        for i in range(steps):
            step(i)
    torch.cuda.synchronize()
    idx_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    topk_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    att_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)

    # ---- algorithmic bytes / flops and rooflines
    peaks, peak_src = load_peaks()
    q_pos = wl.q_pos.to("cpu").numpy().astype(np.int64)
    n_scored = int((q_pos + 1).sum())
    idx_bytes = acc.indexer_bytes(n_scored, T, T * ld, fp8=fp8)
    n_rows_att = int(np.minimum(q_pos + 1, k).sum())
    att_bytes = sum(acc.attend_bytes(n_rows_att, T, L.d_rope, row_bytes=c.shape[1] if fp8_cache else None)
                    for L, c in zip(wl.layers, caches))
    step_bytes = idx_bytes + acc.topk_bytes(n_scored, T, k) + att_bytes
    timed_steps = steps * replays
    step_s = elapsed / timed_steps
    idx_name = "indexer_kernel<{},{}>".format(q_group, "fp8" if fp8 else "bf16")
    idx_kernel = "indexer_fp8" if fp8 else "indexer"
    res = {
        "config": case.name, "T": T, "n_layers": n_layers, "ld": ld, "q_group": q_group, "steps": steps,
        "graph_replays": replays,
        "timed_steps": timed_steps, "timed_region_s": round(elapsed, 4), "ms_per_step": round(step_s * 1e3, 4),
        "queries_per_s": T * world / step_s, "query_layers_per_s": T * n_layers * world / step_s,
        "launches": launches, "clocks": clocks,
        "kernel_ms": {"indexer": round(idx_ms, 4), "topk": round(topk_ms, 4),
                      "attention_all_layers": round(att_ms, 4)},
        "step_hbm": {"algorithmic_bytes": step_bytes, "achieved_tbs": round(step_bytes / step_s / 1e12, 3),
                     "frac_of_measured_copy": round(step_bytes / step_s / 1e9 / peaks["hbm_gbs"], 4),
                     "frac_of_8tbs": round(step_bytes / step_s / 8e12, 4)},
        "attention_hbm": {"algorithmic_bytes": att_bytes,
                          "achieved_tbs": round(att_bytes / (att_ms / 1e3) / 1e12, 3),
                          "frac_of_measured_copy": round(att_bytes / (att_ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4)},
    }
    idx_dur = idx_ms / 1e3
    if q_group == 1:
        achieved = idx_bytes / idx_dur / 1e9
        res["roofline"] = {"kernel": idx_name, "bound": "hbm", "achieved": round(achieved, 1),
                           "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                           "peak_source": f"{peak_src} hbm_gbs", "traffic": profiled_traffic(idx_kernel, case.name),
                           "algorithmic_bytes_per_launch": idx_bytes, "avg_launch_ms": round(idx_ms, 4)}
    else:
        flops = acc.indexer_flops(n_scored)
        achieved = flops / idx_dur / 1e12
        # an FP8 contraction is measured against the bf16 peak x 2 (the nominal fp8 : bf16 ratio, 4.5 : 2.25)
        ratio = 2.0 if fp8 else 1.0
        peak_tf = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * ratio
        res["roofline"] = {"kernel": idx_name, "bound": "tensor", "achieved": round(achieved, 1), "peak": peak_tf,
                           "unit": "TFLOP/s", "frac": round(achieved / peak_tf, 4),
                           "frac_of_burst_peak": round(achieved / (peaks["bf16_tflops"] * ratio), 4),
                           "peak_source": (f"{peak_src} bf16_tflops_sustained"
                                           + (" x 2 (nominal fp8:bf16)" if fp8 else "")
                                           + " (kernel timed inside a multi-ms step)"),
                           "traffic": profiled_traffic(idx_kernel, case.name),
                           "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": idx_bytes,
                           "avg_launch_ms": round(idx_ms, 4)}
    plan = ops.plan_attend(T, min(n_layers, 8), k)
    res["attend_plan"] = {"n_split": plan.n_split, "rows_per_split": plan.rows_per_split, "merge": bool(plan.merge),
                          "workspace_bytes": int(plan.workspace_bytes)}
    if e2e:
        res["e2e"] = run_e2e(wl, ld, k, q_group, dev, e2e_steps,
                             fp8=(q8, q8_scale, k8, k8_scale) if fp8 else None, caches=caches)
    del graph, graph_ev
    return res


def run_e2e(wl, ld, k, q_group, dev, steps, fp8=None, caches=None, min_seconds=0.5):
    """Same metric through dsa_sparse_mla_forward (dsa_sparse_mla_forward_fp8 with
    `fp8` = (q8, q_scale, k8, k_scale)) with pinned host inputs and outputs: every
    step copies that step's queries host->device into one of two device input
    slots, runs the fused call, and copies the outputs device->host.  The copies
    run on their own streams, ordered by events: step s+1's upload and step s-1's
    download overlap step s's compute; a slot is refilled only after the compute
    that read it, an output only after its download.  The `steps` steps are
    captured once as a CUDA graph (host launch overhead excluded, every copy and
    kernel of every step included) and replayed for at least `min_seconds`."""
    from sparse_attention_16_b200 import ops

    T = wl.T
    n_layers = len(wl.layers)
    if fp8 is None:
        host_in = {"q_idx": wl.q_idx, "w": wl.w, "q_seq": wl.q_seq, "q_pos": wl.q_pos}
    else:
        host_in = {"q8": fp8[0], "q_scale": fp8[1], "w": wl.w, "q_seq": wl.q_seq, "q_pos": wl.q_pos}
    for i, L in enumerate(wl.layers):
        host_in[f"q_nope{i}"] = L.q_nope
        if L.q_pe is not None:
            host_in[f"q_pe{i}"] = L.q_pe
        host_in[f"qmul{i}"] = L.qmul
    pinned = {n: t.to("cpu").pin_memory() for n, t in host_in.items()}
    slots = [{n: torch.empty_like(t) for n, t in host_in.items()} for _ in range(2)]
    outs = [[torch.empty((T, 64, 512), dtype=torch.bfloat16, device=dev) for _ in wl.layers] for _ in range(2)]
    host_out = [[torch.empty((T, 64, 512), dtype=torch.bfloat16).pin_memory() for _ in wl.layers] for _ in range(2)]
    ws = ops.workspace(ops.forward_workspace_bytes(T, ld, k, q_group, n_layers), dev)
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0])
    s_up, s_comp, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_up = [torch.cuda.Event() for _ in range(steps)]
    ev_comp = [torch.cuda.Event() for _ in range(steps)]
    ev_down = [torch.cuda.Event() for _ in range(steps)]

    def forward(sl):
        d = slots[sl]
        layers = [dict(q_nope=d[f"q_nope{i}"], q_pe=d.get(f"q_pe{i}"), qmul=d[f"qmul{i}"],
                       cache=caches[i] if caches is not None else L.cache, d_rope=L.d_rope, out=outs[sl][i], lse=None)
                  for i, L in enumerate(wl.layers)]
        if fp8 is None:
            ops.sparse_mla_forward(d["q_idx"], d["w"], wl.k_idx, wl.seq_row_start, d["q_seq"], d["q_pos"], layers, ld,
                                   k=k, q_group=q_group, ws=ws, stream=s_comp)
        else:
            ops.sparse_mla_forward_fp8(d["q8"], d["q_scale"], d["w"], fp8[2], fp8[3], wl.seq_row_start, d["q_seq"],
                                       d["q_pos"], layers, ld, k=k, q_group=q_group, ws=ws, stream=s_comp)

    def issue():
        # the three streams fork from the compute stream and join it at the end
        root = torch.cuda.Event()
        root.record(s_comp)
        s_up.wait_event(root)
        s_down.wait_event(root)
        for i in range(steps):
            sl = i % 2
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(ev_comp[i - 2])   # the compute that read this slot is done
                for n in pinned:
                    slots[sl][n].copy_(pinned[n], non_blocking=True)
                ev_up[i].record(s_up)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_up[i])
                if i >= 2:
                    s_comp.wait_event(ev_down[i - 2])   # this slot's outputs have been downloaded
                forward(sl)
                ev_comp[i].record(s_comp)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev_comp[i])
                for o, h in zip(outs[sl], host_out[sl]):
                    h.copy_(o, non_blocking=True)
                ev_down[i].record(s_down)
        s_comp.wait_event(ev_up[steps - 1])
        s_comp.wait_event(ev_down[steps - 1])

    torch.cuda.synchronize()
    issue()   # warm-up, eager
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s_comp):
        issue()
    with torch.cuda.stream(s_comp):
        graph.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_comp)
    with torch.cuda.stream(s_comp):
        graph.replay()
    b.record(s_comp)
    torch.cuda.synchronize()
    replays = max(1, math.ceil(min_seconds / max(a.elapsed_time(b) / 1e3, 1e-6)))
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_comp)
    with torch.cuda.stream(s_comp):
        for _ in range(replays):
            graph.replay()
    t1.record(s_comp)
    torch.cuda.synchronize()
    el = t0.elapsed_time(t1) / 1e3
    n = steps * replays
    del graph
    return {"value": round(T * n_layers * n / el, 1), "unit": "query-layers/s", "queries_per_s": round(T * n / el, 1),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(el / n * 1e3, 4),
            "steps": n, "api": "dsa_sparse_mla_forward" + ("_fp8" if fp8 is not None else ""),
            "how": ("every step: pinned host->device upload of its queries, the fused call, device->host download "
                    "of its outputs, on three streams ordered by events (uploads and downloads overlap the "
                    "neighbouring steps' compute); captured once as a CUDA graph of the steps and replayed")}


def run_ours(args, rank, world, local):
    from sparse_attention_16_b200 import ops

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    ops.load_library()
    head = measure(args.config, dev, args.steps, args.warmup, rank, world, local, min_seconds=args.min_seconds,
                   sample_clocks=True, fp8=args.fp8_keys, eager=args.eager, e2e=not args.no_e2e,
                   fp8_cache=args.fp8_cache)
    torch.cuda.empty_cache()
    case = CONFIGS[args.config]
    wl_T = head["T"]
    line = {
        "metric": METRIC, "value": round(head["query_layers_per_s"], 1), "unit": "query-layers/s",
        "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded, shapes/distributions of the configuration)",
        "config": {"workload": args.config + ("+fp8_index_keys" if args.fp8_keys else "")
                   + ("+fp8_latent_cache" if args.fp8_cache else ""),
                   "queries_per_gpu": wl_T, "context": list(case.seq_lengths)[:1],
                   "layers": [("rope" if d else "nope") for d in case.layers], "topk": case.topk,
                   "parallelism": f"replicas{world}" if world > 1 else "1gpu",
                   "l2": f"inputs larger than L2 ({head['step_hbm']['algorithmic_bytes'] / 1e6:.0f} MB per step)"},
        "queries_per_s": round(head["queries_per_s"], 1),
        "timing": {"graph_steps": args.steps, "graph_replays": head["graph_replays"],
                   "timed_steps": head["timed_steps"], "timed_region_s": head["timed_region_s"],
                   "how": ("CUDA graph of K steps of dsa_sparse_mla_forward (the fused call) replayed R times "
                           "inside one event-timed region; kernel_ms from a second graph of the same steps as three "
                           "separate calls (indexer, top-k, attention) with events between them")},
        "step_hbm": head["step_hbm"], "attention_hbm": head["attention_hbm"], "kernel_ms": head["kernel_ms"],
        "roofline": head["roofline"], "gpu_launches": head["launches"], "clocks": head["clocks"],
        "e2e": head.get("e2e"), "attend_plan": head["attend_plan"],
    }
    props = ops.device_props()
    line["device"] = {"sms": props.sms, "attend_max_clusters": {c: props.max_clusters[c] for c in range(2, 9)}}
    if world == 1 and not args.no_extras:
        extras = {}
        for name in EXTRAS:
            if name == args.config:
                continue
            r = measure(name, dev, 3 if CONFIGS[name].kind == "prefill" else args.steps, 3, rank, world, local,
                        min_seconds=0.0 if CONFIGS[name].kind == "prefill" else 0.3, fp8=args.fp8_keys,
                        fp8_cache=args.fp8_cache)
            torch.cuda.empty_cache()
            keep = ("ms_per_step", "queries_per_s", "query_layers_per_s", "kernel_ms", "step_hbm", "attention_hbm",
                    "roofline", "timed_steps", "attend_plan", "q_group")
            extras[name] = {k_: (round(v, 4) if isinstance(v, float) else v) for k_, v in r.items() if k_ in keep}
        line["extra_configs"] = extras
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.config, budget_s=args.cpu_seconds)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- oracle (CPU) arm

SAMPLE_CACHE_LIMIT = 1 << 30   # host bytes of latent cache beyond which the sample draws only the selected rows


def _oracle_sample(config, n_queries):
    """A bounded slice of the configuration: ``n_queries`` sequences (or prefill
    queries) of the same shape and distributions, drawn on the CPU.  Returns
    (indexer workload, attention workload or None).  When the sequences' latent
    caches would exceed SAMPLE_CACHE_LIMIT (the 2^20-position configuration:
    4.7 GB per sequence), the attention side is drawn as `topk` rows per query
    and layer (iid rows of the same distribution) that stand for the selected
    positions: the oracle does the same arithmetic on them."""
    case = CONFIGS[config]
    if case.kind == "decode":
        sub = small_case(config + "_sample", case.lengths[:n_queries], layers=case.layers, qmul=case.qmul,
                         mla_q_std=case.mla_q_std, seed=case.seed, planted=case.planted, per_seq=case.per_seq)
    else:
        sub = small_case(config + "_sample", kind="prefill", cached=case.cached + case.new - n_queries,
                         new=n_queries, layers=case.layers, qmul=case.qmul, mla_q_std=case.mla_q_std,
                         seed=case.seed)
    cache_bytes = sum(sub.seq_lengths) * sum(512 + d for d in case.layers) * 2
    if cache_bytes <= SAMPLE_CACHE_LIMIT:
        return make_workload(sub, "cpu"), None
    idx_part = make_workload(dataclasses.replace(sub, layers=()), "cpu")
    att_part = make_workload(small_case(config + "_rows", (case.topk,) * idx_part.T, layers=case.layers,
                                        qmul=case.qmul, mla_q_std=case.mla_q_std, seed=case.seed + 1), "cpu")
    return idx_part, att_part


def _oracle_step(sample):
    import oracle
    from sparse_attention_16_b200.workloads import SOFTMAX_SCALE, to_numpy

    wl, att = sample
    if att is None:
        layers = [dict(q_nope=to_numpy(L.q_nope), q_pe=None if L.q_pe is None else to_numpy(L.q_pe),
                       qmul=to_numpy(L.qmul), cache=to_numpy(L.cache), d_rope=L.d_rope) for L in wl.layers]
        return oracle.forward(to_numpy(wl.q_idx), to_numpy(wl.w), to_numpy(wl.k_idx), to_numpy(wl.seq_row_start),
                              to_numpy(wl.q_seq), to_numpy(wl.q_pos), layers, SOFTMAX_SCALE, k=wl.case.topk)
    q_pos = to_numpy(wl.q_pos)
    scores = oracle.index_scores(to_numpy(wl.q_idx), to_numpy(wl.w), to_numpy(wl.k_idx), to_numpy(wl.seq_row_start),
                                 to_numpy(wl.q_seq), q_pos, int(q_pos.max()) + 1)
    idx, count = oracle.topk_select(scores, q_pos, wl.case.topk)
    # the i-th selected position of query t is row i of its drawn rows
    local = np.where(idx >= 0, np.arange(idx.shape[1])[None, :], -1).astype(np.int32)
    outs = []
    for L in att.layers:
        outs.append(oracle.sparse_mla(to_numpy(L.q_nope), None if L.q_pe is None else to_numpy(L.q_pe),
                                      to_numpy(L.qmul), SOFTMAX_SCALE, to_numpy(L.cache), L.d_rope,
                                      to_numpy(att.seq_row_start), to_numpy(att.q_seq), local, count))
    return idx, count, outs


def _threads_used():
    try:
        from threadpoolctl import threadpool_info

        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def _time_oracle(sample, budget_s):
    t = time.perf_counter()
    reps = 0
    while True:
        _oracle_step(sample)
        reps += 1
        if time.perf_counter() - t > budget_s or reps >= 50:
            break
    return reps, time.perf_counter() - t


def cpu_baseline(config, budget_s=20.0, n_queries=1):
    """The oracle on the host cores (numpy's default thread pool), then on one thread."""
    sample = _oracle_sample(config, n_queries)
    n_layers = len(CONFIGS[config].layers)
    T = sample[0].T
    reps, el = _time_oracle(sample, budget_s)
    how = "attention rows drawn at the selected positions only" if sample[1] is not None else "full caches"
    res = {"value": round(reps * T * n_layers / el, 4), "unit": "query-layers/s",
           "queries_per_s": round(reps * T / el, 4), "cores": _threads_used(), "kind": "oracle",
           "sample": f"{reps} x {T} queries of {config} (same shape, CPU-drawn, {how}), fp64 numpy oracle"}
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:
        return res
    with threadpool_limits(limits=1):
        reps1, el1 = _time_oracle(sample, budget_s / 2)
    res["single_thread"] = {"value": round(reps1 * T * n_layers / el1, 4), "unit": "query-layers/s", "cores": 1,
                            "sample": f"{reps1} x {T} queries, the same sample"}
    return res


def run_reference(args, rank, world):
    if rank != 0:
        return
    sample = _oracle_sample(args.config, 1)
    n_layers = len(CONFIGS[args.config].layers)
    for _ in range(args.warmup):
        _oracle_step(sample)
    t = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(sample)
    el = time.perf_counter() - t
    T = sample[0].T
    value = args.steps * T * n_layers / el
    cores = _threads_used()
    how = "attention rows drawn at the selected positions only" if sample[1] is not None else "full caches"
    desc = f"each step = {T} query of {args.config} (same shape, {how}), fp64 numpy oracle on host cores"
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "query-layers/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.config},
            "cpu_baseline": {"value": round(value, 4), "unit": "query-layers/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(value, 4), "unit": "query-layers/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- launcher

def _spawned_rank(local, world, port, argv):
    os.environ.update(RANK=str(local), LOCAL_RANK=str(local), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port), LOCAL_WORLD_SIZE=str(world))
    sys.argv = [sys.argv[0]] + argv
    main()


def spawn_ranks(n, argv):
    """`--gpus N` without torchrun: one process per GPU (spawn), ranks 0..N-1 on
    this node, rendezvous on 127.0.0.1.  Rank 0 prints the JSON line."""
    import socket

    import torch.multiprocessing as mp

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    mp.start_processes(_spawned_rank, args=(n, port, argv), nprocs=n, start_method="spawn")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=HEADLINE, choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--min-seconds", type=float, default=1.0, help="shortest timed region (graph replays)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--eager", action="store_true", help="launch every step from the host instead of a CUDA graph")
    ap.add_argument("--fp8-keys", action="store_true",
                    help="score with FP8 (E4M3) index keys and queries, per-row scales (dsa_index_scores_fp8); "
                         "the selection and attention are unchanged")
    ap.add_argument("--fp8-cache", action="store_true",
                    help="keep every layer's latent cache as FP8 rows (E4M3 codes, one fp32 scale per 128 values "
                         "and one for the rotary key); the attention widens the selected rows on chip")
    args = ap.parse_args()
    rank, world, local = dist_env()
    if args.gpus > 1 and "RANK" not in os.environ:
        spawn_ranks(args.gpus, sys.argv[1:])
        return
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()

"""Benchmark of the DSA hot path: indexer -> top-2048 -> absorbed sparse MLA.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: the indexer scores
every earlier position of every query, the top-k kernel selects 2,048 per
query, and every layer of the configuration attends over that selection.  The
default configuration is the decode batch the headline metric is quoted on: 64
sequences x 32,768 positions, one RoPE layer.  Inputs are resident in HBM when
the timed region starts (698 MB per step, larger than the 126 MB L2, so every
step streams from HBM).

Multi-GPU (torchrun, one process per GPU): decode sequences are independent,
so each rank runs its own batch with no collective on the data path; the only
collectives are the barrier and the max-over-ranks reduction of the device
time ("scaling": "weak").

The reference arm (--impl reference) times the fp64 CPU oracle on a bounded
sample of the same workload (a few queries per step) on the host cores.
"""

from __future__ import annotations

import argparse
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
from sparse_attention_16_b200.workloads import CONFIGS, make_workload, quantize_e4m3_rows, small_case  # noqa: E402

HEADLINE = "decode_b64_32k"
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

def run_ours(args, rank, world, local):
    from sparse_attention_16_b200 import ops

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    case = CONFIGS[args.config]
    # each rank owns an independent batch of the same shape (its own seed)
    case = type(case)(**{**case.__dict__, "seed": replicas.rank_seed(case.seed, rank)})
    wl = make_workload(case, dev)
    T, ld, k = wl.T, case.ld, case.topk
    q_group = 8 if case.kind == "prefill" else 1
    ops.load_library()

    scores = torch.empty((T, ld), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    cnt = torch.empty((T,), dtype=torch.int32, device=dev)
    outs = [torch.empty((T, 64, 512), dtype=torch.bfloat16, device=dev) for _ in wl.layers]
    lses = [torch.empty((T, 64), dtype=torch.float32, device=dev) for _ in wl.layers]
    att_ws = ops.workspace(ops.attend_workspace_bytes(T, k), dev)
    stream = torch.cuda.current_stream()
    if args.fp8_keys:
        # E4M3 codes + per-row scales of the same seeded keys/queries (input preparation, untimed)
        q8, q8_scale = quantize_e4m3_rows(wl.q_idx)
        k8, k8_scale = quantize_e4m3_rows(wl.k_idx)
        wl.k_idx = None          # the bf16 keys are not read in this mode
        torch.cuda.empty_cache()

    # events around the indexer launch of every timed step (same stream)
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)] for _ in range(args.steps)]

    def step(i=None):
        e = ev[i] if i is not None else None
        if e:
            e[0].record(stream)
        if args.fp8_keys:
            ops.index_scores_fp8(q8, q8_scale, wl.w, k8, k8_scale, wl.seq_row_start, wl.q_seq, wl.q_pos, scores,
                                 q_group=q_group)
        else:
            ops.index_scores(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos, scores,
                             q_group=q_group)
        if e:
            e[1].record(stream)
        ops.topk(scores, wl.q_pos, k, idx, cnt)
        if e:
            e[2].record(stream)
        for L, o, l in zip(wl.layers, outs, lses):
            ops.sparse_mla_attend(L.q_nope, L.q_pe, L.qmul, L.cache, L.d_rope, wl.seq_row_start,
                                  wl.q_seq, idx, cnt, o, l, ws=att_ws)
        if e:
            e[3].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    ops.check_errors()

    # The K timed steps are captured once into a CUDA graph and replayed, so
    # host-side launch overhead does not leak into the device timings.  Every
    # kernel of every step still runs.  The timed graph has no event nodes
    # between kernels (they would stop each kernel from being scheduled while
    # the previous one drains); a second graph of the same steps with events
    # around each kernel gives the per-kernel breakdown, after the timed region.
    graph = graph_ev = None
    n0 = ops.launch_count()
    if not args.eager:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(args.steps):
                step()
        launches = ops.launch_count() - n0
        graph_ev = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_ev):
            stream = torch.cuda.current_stream()
            for i in range(args.steps):
                step(i)
        stream = torch.cuda.current_stream()
        graph.replay()            # one untimed replay
        torch.cuda.synchronize()

    sampler = ClockSampler(local) if rank == 0 else None
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
        graph.replay()
    else:
        n0 = ops.launch_count()
        for i in range(args.steps):
            step()
    t1.record(stream)
    torch.cuda.synchronize()
    if graph is None:
        launches = ops.launch_count() - n0
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
        for i in range(args.steps):
            step(i)
    torch.cuda.synchronize()

    idx_ms = [e[0].elapsed_time(e[1]) for e in ev]
    topk_ms = [e[1].elapsed_time(e[2]) for e in ev]
    att_ms = [e[2].elapsed_time(e[3]) for e in ev]

    # ---- roofline of the dominant kernel: the indexer (HBM-bound in decode,
    # tensor-bound in chunked prefill, where 8 queries share each key tile)
    peaks, peak_src = load_peaks()
    q_pos = wl.q_pos.to("cpu").numpy().astype(np.int64)
    n_scored = int((q_pos + 1).sum())
    idx_bytes = acc.indexer_bytes(n_scored, T, T * ld, fp8=args.fp8_keys)
    idx_kernel = "indexer_fp8" if args.fp8_keys else "indexer"
    idx_name = "indexer_kernel<{},{}>".format(q_group, "fp8" if args.fp8_keys else "bf16")
    idx_dur = statistics.mean(idx_ms) / 1e3
    if q_group == 1:
        achieved_gbs = idx_bytes / idx_dur / 1e9
        roofline = {"kernel": idx_name, "bound": "hbm",
                    "achieved": round(achieved_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(achieved_gbs / peaks["hbm_gbs"], 4), "peak_source": f"{peak_src} hbm_gbs",
                    "traffic": profiled_traffic(idx_kernel, args.config),
                    "algorithmic_bytes_per_launch": idx_bytes, "avg_launch_ms": round(idx_dur * 1e3, 4)}
    else:
        flops = acc.indexer_flops(n_scored)
        achieved_tf = flops / idx_dur / 1e12
        # an FP8 contraction is measured against the bf16 peak x 2 (the nominal fp8 : bf16 ratio, 4.5 : 2.25)
        ratio = 2.0 if args.fp8_keys else 1.0
        peak_tf = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * ratio
        roofline = {"kernel": idx_name, "bound": "tensor",
                    "achieved": round(achieved_tf, 1), "peak": peak_tf, "unit": "TFLOP/s",
                    "frac": round(achieved_tf / peak_tf, 4),
                    "frac_of_burst_peak": round(achieved_tf / (peaks["bf16_tflops"] * ratio), 4),
                    "peak_source": (f"{peak_src} bf16_tflops_sustained" + (" x 2 (nominal fp8:bf16)" if args.fp8_keys
                                                                          else "")
                                    + " (kernel timed inside a multi-ms step)"),
                    "traffic": profiled_traffic(idx_kernel, args.config),
                    "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": idx_bytes,
                    "avg_launch_ms": round(idx_dur * 1e3, 4)}

    # whole-step algorithmic bytes (all kernels) and the fraction of HBM peak they imply
    n_rows_att = int(np.minimum(q_pos + 1, k).sum())
    step_bytes = idx_bytes + acc.topk_bytes(n_scored, T, k)
    for L in wl.layers:
        step_bytes += acc.attend_bytes(n_rows_att, T, L.d_rope)

    # ---- end to end through the C ABI with host buffers
    # the fused C-ABI call takes bf16 index keys; no end-to-end line in FP8-key mode
    e2e = run_e2e(args, wl, ld, k, q_group, dev) if not (args.no_e2e or args.fp8_keys) else None

    value = replicas.job_throughput(T, world, args.steps, elapsed)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": round(elapsed / args.steps * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded, shapes/distributions of the configuration)",
        "config": {"workload": args.config + ("+fp8_index_keys" if args.fp8_keys else ""),
                   "queries_per_gpu": T, "context": list(case.seq_lengths)[:1],
                   "layers": [("rope" if L.d_rope else "nope") for L in wl.layers], "topk": k,
                   "parallelism": f"replicas{world}" if world > 1 else "1gpu",
                   "l2": f"inputs larger than L2 ({step_bytes / 1e6:.0f} MB per step)"},
        "step_hbm": {"algorithmic_bytes": step_bytes,
                     "achieved_tbs": round(step_bytes / (elapsed / args.steps) / 1e12, 3),
                     "frac_of_measured_copy": round(step_bytes / (elapsed / args.steps) / 1e9 / peaks["hbm_gbs"], 4),
                     "frac_of_8tbs": round(step_bytes / (elapsed / args.steps) / 8e12, 4)},
        "kernel_ms": {"indexer": round(statistics.mean(idx_ms), 4), "topk": round(statistics.mean(topk_ms), 4),
                      "attention_all_layers": round(statistics.mean(att_ms), 4)},
        "roofline": roofline, "gpu_launches": launches, "clocks": clocks, "e2e": e2e,
        "timing": ("CUDA graph of the timed steps, one replay; kernel_ms from a second graph of the same "
                   "steps with events around each kernel" if graph is not None else "eager launches"),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.config, budget_s=args.cpu_seconds)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(args, wl, ld, k, q_group, dev):
    """Same metric through dsa_sparse_mla_forward with pinned host inputs/outputs:
    each step copies the step's queries host->device and the outputs back."""
    from sparse_attention_16_b200 import ops

    T = wl.T
    host_in = {"q_idx": wl.q_idx, "w": wl.w, "q_seq": wl.q_seq, "q_pos": wl.q_pos}
    for i, L in enumerate(wl.layers):
        host_in[f"q_nope{i}"] = L.q_nope
        if L.q_pe is not None:
            host_in[f"q_pe{i}"] = L.q_pe
        host_in[f"qmul{i}"] = L.qmul
    pinned = {n: t.to("cpu").pin_memory() for n, t in host_in.items()}
    dev_in = {n: torch.empty_like(t) for n, t in host_in.items()}
    outs = [torch.empty((T, 64, 512), dtype=torch.bfloat16, device=dev) for _ in wl.layers]
    host_out = [torch.empty((T, 64, 512), dtype=torch.bfloat16).pin_memory() for _ in wl.layers]
    ws = ops.workspace(ops.forward_workspace_bytes(T, ld, k, q_group), dev)
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out)

    def step():
        for n in pinned:
            dev_in[n].copy_(pinned[n], non_blocking=True)
        layers = [dict(q_nope=dev_in[f"q_nope{i}"], q_pe=dev_in.get(f"q_pe{i}"), qmul=dev_in[f"qmul{i}"],
                       cache=L.cache, d_rope=L.d_rope, out=outs[i], lse=None) for i, L in enumerate(wl.layers)]
        ops.sparse_mla_forward(dev_in["q_idx"], dev_in["w"], wl.k_idx, wl.seq_row_start, dev_in["q_seq"],
                               dev_in["q_pos"], layers, ld, k=k, q_group=q_group, ws=ws)
        for o, h in zip(outs, host_out):
            h.copy_(o, non_blocking=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s)
    for _ in range(args.steps):
        step()
    t1.record(s)
    torch.cuda.synchronize()
    el = t0.elapsed_time(t1) / 1e3
    return {"value": round(T * args.steps / el, 1), "unit": "queries/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(el / args.steps * 1e3, 4),
            "api": "dsa_sparse_mla_forward"}


# --------------------------------------------------------------------------- oracle (CPU) arm

def _oracle_sample_workload(config, n_queries):
    """A bounded slice of the configuration: ``n_queries`` sequences (or prefill
    queries) of the same shape and distributions, drawn on the CPU."""
    case = CONFIGS[config]
    if case.kind == "decode":
        sub = small_case(config + "_sample", case.lengths[:n_queries], layers=case.layers, qmul=case.qmul,
                         mla_q_std=case.mla_q_std, seed=case.seed, planted=case.planted)
    else:
        sub = small_case(config + "_sample", kind="prefill", cached=case.cached + case.new - n_queries,
                         new=n_queries, layers=case.layers, qmul=case.qmul, mla_q_std=case.mla_q_std,
                         seed=case.seed)
    return make_workload(sub, "cpu")


def _oracle_step(wl):
    import oracle
    from sparse_attention_16_b200.workloads import SOFTMAX_SCALE, to_numpy

    layers = [dict(q_nope=to_numpy(L.q_nope), q_pe=None if L.q_pe is None else to_numpy(L.q_pe),
                   qmul=to_numpy(L.qmul), cache=to_numpy(L.cache), d_rope=L.d_rope) for L in wl.layers]
    return oracle.forward(to_numpy(wl.q_idx), to_numpy(wl.w), to_numpy(wl.k_idx), to_numpy(wl.seq_row_start),
                          to_numpy(wl.q_seq), to_numpy(wl.q_pos), layers, SOFTMAX_SCALE, k=wl.case.topk)


def _threads_used():
    try:
        from threadpoolctl import threadpool_info

        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(config, budget_s=20.0, n_queries=1):
    wl = _oracle_sample_workload(config, n_queries)
    t = time.perf_counter()
    reps = 0
    while True:
        _oracle_step(wl)
        reps += 1
        if time.perf_counter() - t > budget_s or reps >= 50:
            break
    el = time.perf_counter() - t
    return {"value": round(reps * wl.T / el, 4), "unit": "queries/s", "cores": _threads_used(), "kind": "oracle",
            "sample": f"{reps} x {wl.T} queries of {config} (same shape, CPU-drawn), fp64 numpy oracle"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    wl = _oracle_sample_workload(args.config, 1)
    for _ in range(args.warmup):
        _oracle_step(wl)
    t = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(wl)
    el = time.perf_counter() - t
    value = args.steps * wl.T / el
    cores = _threads_used()
    sample = f"each step = {wl.T} query of {args.config} (same shape), fp64 numpy oracle on host cores"
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "queries/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.config},
            "cpu_baseline": {"value": round(value, 4), "unit": "queries/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "queries/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=HEADLINE, choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--eager", action="store_true", help="launch every step from the host instead of a CUDA graph")
    ap.add_argument("--fp8-keys", action="store_true",
                    help="score with FP8 (E4M3) index keys and queries, per-row scales (dsa_index_scores_fp8); "
                         "the selection and attention are unchanged")
    args = ap.parse_args()
    rank, world, local = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()

"""Runs one kernel of the hot path a few times on a configuration's inputs, for
profiler captures (ncu) of that kernel alone.

    python -m sparse_attention_16_b200.profile_case --kernel indexer --config decode_b64_32k --launches 3

Only the inputs the chosen kernel reads are drawn (the indexer and top-k never
touch the latent caches), so a capture holds little device memory.  The
selection fed to the attention kernel comes from one untimed indexer + top-k
pass.  Prints the mean CUDA-event time per launch.
"""

from __future__ import annotations

import argparse
import dataclasses

import torch

from sparse_attention_16_b200 import ops
from sparse_attention_16_b200.workloads import CONFIGS, make_workload, quantize_e4m3_rows


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", choices=["indexer", "topk", "attend"], required=True)
    ap.add_argument("--config", default="decode_b64_32k", choices=sorted(CONFIGS))
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--layer", type=int, default=-1,
                    help="attention: one layer of the configuration (default: all its layers in one launch)")
    ap.add_argument("--fp8", action="store_true", help="indexer: FP8 (E4M3) keys and queries, per-row scales")
    ap.add_argument("--context", type=int, default=0,
                    help="decode configurations: every sequence this long instead (a smaller capture of the same "
                         "launch shape)")
    a = ap.parse_args()

    case = CONFIGS[a.config]
    if a.context:
        assert case.kind == "decode", "--context applies to decode configurations"
        case = dataclasses.replace(case, lengths=(a.context,) * len(case.lengths))
    if a.kernel != "attend":
        case = dataclasses.replace(case, layers=())
    dev = torch.device("cuda", 0)
    wl = make_workload(case, dev)
    T, ld, k = wl.T, case.ld, case.topk
    q_group = 8 if case.kind == "prefill" else 1
    scores = torch.empty((T, ld), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    cnt = torch.empty((T,), dtype=torch.int32, device=dev)
    # decode: the indexer's score histogram feeds the top-k's first pass (as in the fused call)
    hist = torch.empty((T, 2048), dtype=torch.int32, device=dev) if q_group == 1 else None
    topk_ws = ops.workspace(ops.topk_workspace_bytes(T, ld, k), dev) if q_group == 1 else None

    if a.fp8:
        q8, q8_scale = quantize_e4m3_rows(wl.q_idx)
        k8, k8_scale = quantize_e4m3_rows(wl.k_idx)

    def indexer():
        if a.fp8:
            ops.index_scores_fp8(q8, q8_scale, wl.w, k8, k8_scale, wl.seq_row_start, wl.q_seq, wl.q_pos, scores,
                                 q_group=q_group, hist=hist)
        else:
            ops.index_scores(wl.q_idx, wl.w, wl.k_idx, wl.seq_row_start, wl.q_seq, wl.q_pos, scores,
                             q_group=q_group, hist=hist)

    def topk():
        ops.topk(scores, wl.q_pos, k, idx, cnt, hist=hist, ws=topk_ws)

    if a.kernel in ("topk", "attend"):
        indexer()
        topk()
    run = {"indexer": indexer, "topk": topk}.get(a.kernel)
    if a.kernel == "attend":
        chosen = wl.layers if a.layer < 0 else [wl.layers[a.layer]]
        outs = [torch.empty((T, 64, 512), dtype=torch.bfloat16, device=dev) for _ in chosen]
        lses = [torch.empty((T, 64), dtype=torch.float32, device=dev) for _ in chosen]
        layers = [dict(q_nope=L.q_nope, q_pe=L.q_pe, qmul=L.qmul, cache=L.cache, d_rope=L.d_rope, out=o, lse=l)
                  for L, o, l in zip(chosen, outs, lses)]
        ws = ops.workspace(ops.layers_workspace_bytes(T, len(layers), k), dev)

        def run():
            ops.sparse_mla_attend_layers(layers, chosen[0].cache.shape[0], wl.seq_row_start, wl.q_seq, idx, cnt,
                                         q_pos=wl.q_pos, ws=ws)

    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.launches):
        run()
    e1.record()
    torch.cuda.synchronize()
    ops.check_errors()
    print(f"{a.kernel} on {a.config}: {e0.elapsed_time(e1) / a.launches:.4f} ms per launch "
          f"({a.launches} launches)", flush=True)


if __name__ == "__main__":
    main()

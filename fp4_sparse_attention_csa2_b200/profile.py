"""Run a few launches of one libcsa2 kernel group on a workload, for a profiler
to capture (``ncu ... python -m fp4_sparse_attention_csa2_b200.profile``).

    --kernel score   Full-layer scoring only (csa2_index_scores)
    --kernel attn    sparse + window attention (csa2_sparse_swa_attn) on the
                     top-k of one Full layer
    --kernel stack   whole decode steps of the layer pattern
    --kernel cp      one rank's device work of an 8-way context-parallel step
                     (runner.CpRankStep, the last rank's shard; no exchange)
"""
import argparse

import torch

import fp4_sparse_attention_csa2_b200 as csa2
from fp4_sparse_attention_csa2_b200 import workloads as wl
from fp4_sparse_attention_csa2_b200.runner import CpRankStep, Stack, build_replicas, new_workspace


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", default="score", choices=["score", "attn", "stack", "cp"])
    ap.add_argument("--workload", default="ctx1m", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--seed", type=int, default=0)
    args = ap.parse_args()
    w = wl.WORKLOADS[args.workload]
    lens = wl.seq_lens(w, args.seed)
    layers = [wl.layer_queries(w, l, args.seed) for l in range(len(w.pattern))]
    cache = build_replicas(w, 1, args.seed, lens)[0]
    ws = new_workspace(cache, w)
    stack = Stack(w, layers, ws)
    L0 = stack.layers[0]
    torch.cuda.synchronize()
    if args.kernel == "score":
        for _ in range(args.launches):
            csa2.index_scores(cache, L0["q_idx"], L0["w"], ws)
    elif args.kernel == "attn":
        csa2.index_full(cache, L0["q_idx"], L0["w"], w.pool_k, w.top_k, stack.pool, stack.topk, ws)
        for _ in range(args.launches):
            csa2.sparse_swa_attn(cache, stack.layers[1]["q"], stack.topk, w.window, stack.out[1], stack.lse[1], ws)
    elif args.kernel == "cp":
        cp = CpRankStep(w, lens, layers, [cache])
        for _ in range(args.launches):
            cp.step(cp.shards[-1])
        torch.cuda.synchronize()
        cp.check("after the profiled steps")
    else:
        for _ in range(args.launches):
            stack.step(cache)
    torch.cuda.synchronize()
    st = csa2.read_device_status(ws)
    print("profile run done: %s x%d on %s, device status %s" % (args.kernel, args.launches, w.name,
                                                               csa2.status_string(st)))
    if st != csa2.OK:
        raise SystemExit(1)


if __name__ == "__main__":
    main()

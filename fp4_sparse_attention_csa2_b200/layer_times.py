"""Warm device time of each layer type and each C-ABI call of a decode step:
every entry is captured N times into one CUDA graph (rotating over the cache
replicas, so the keys do not sit in L2 from the previous call), the graph is
replayed a few times, and CUDA events on the launching stream give the time
per call.

    python -m fp4_sparse_attention_csa2_b200.layer_times [--workload ctx1m]
"""
import argparse

import torch

import fp4_sparse_attention_csa2_b200 as csa2
from fp4_sparse_attention_csa2_b200 import workloads as wl
from fp4_sparse_attention_csa2_b200.runner import Stack, build_replicas, new_workspace


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="ctx1m", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--replicas", type=int, default=3)
    ap.add_argument("--calls", type=int, default=30, help="calls captured per graph")
    ap.add_argument("--replays", type=int, default=5)
    ap.add_argument("--seed", type=int, default=0)
    args = ap.parse_args()
    w = wl.WORKLOADS[args.workload]
    lens = wl.seq_lens(w, args.seed)
    layers = [wl.layer_queries(w, l, args.seed) for l in range(len(w.pattern))]
    reps = build_replicas(w, args.replicas, args.seed, lens)
    ws = new_workspace(reps[0], w)
    st = Stack(w, layers, ws)
    first = {m: w.pattern.index(m) for m in set(w.pattern)}
    L0 = st.layers[first["F"]]
    csa2.index_full(reps[0], L0["q_idx"], L0["w"], w.pool_k, w.top_k, st.pool, st.topk, ws)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()

    def layer(c, l):
        m = st.modes[l]
        L = st.layers[l]
        idx = m != csa2.REUSE
        csa2.layer_step(c, m, L["q"], st.topk, st.out[l], ws, w.window, q_idx=L["q_idx"] if idx else None,
                        head_w=L["w"] if idx else None, pool_idx=st.pool, lse=st.lse[l], pool_k=w.pool_k)

    ops = {"layer " + m: (lambda c, l=first[m]: layer(c, l)) for m in "FRU" if m in first}
    ops["index_scores"] = lambda c: csa2.index_scores(c, L0["q_idx"], L0["w"], ws)
    ops["index_full"] = lambda c: csa2.index_full(c, L0["q_idx"], L0["w"], w.pool_k, w.top_k, st.pool, st.topk, ws)
    if "R" in first:
        L1 = st.layers[first["R"]]
        ops["index_reindex"] = lambda c: csa2.index_reindex(c, L1["q_idx"], L1["w"], st.pool, w.top_k, st.topk, ws)
    ops["sparse_swa_attn"] = lambda c: csa2.sparse_swa_attn(c, L0["q"], st.topk, w.window, st.out[0], st.lse[0], ws)
    ops["whole step"] = lambda c: st.step(c)

    n, r = args.calls, len(reps)
    for name, fn in ops.items():
        with torch.cuda.stream(stream):
            for i in range(3):                               # warm-up, eager
                fn(reps[i % r])
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
            for i in range(n):
                fn(reps[i % r])
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            for _ in range(args.replays):
                g.replay()
            b.record(stream)
        torch.cuda.synchronize()
        print("%-16s %8.2f us" % (name, a.elapsed_time(b) * 1e3 / (args.replays * n)))
        del g
    st_code = csa2.read_device_status(ws)
    print("status", csa2.status_string(st_code))
    if st_code != csa2.OK:
        raise SystemExit(1)


if __name__ == "__main__":
    main()

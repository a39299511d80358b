"""Benchmark: CSA2 decode layer-steps/s on the 1M-context stack, with the
kernels' roofline fractions, an end-to-end number through the public binding
with host buffers, the other four synthetic workloads beside it, and the CPU
oracle as a reported baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload ctx1m] [--no-extra-workloads]

One step = one decode step of the whole layer stack (ctx1m: Full, Reindex and
six Reuse layers for one 1,048,576-token sequence).  The metric counts layer
executions per second over all ranks.  Under torchrun every rank runs its own
sequence (weak scaling over independent sequences, no data-path collective).
The K-step timed region is repeated (at least five times and about half a
second in all) and the median region is reported, with the SM clock sampled
throughout.
"""
import argparse
import ctypes
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fp4_sparse_attention_csa2_b200 import workloads as wl  # noqa: E402
from fp4_sparse_attention_csa2_b200.runner import Stack, build_replicas  # noqa: E402

METRIC = "CSA2 decode layer-steps/s at 1M ctx; FP4-KV achieved HBM GB/s vs 8 TB/s"
PROFILE = os.path.join(ROOT, "profiles", "index_score_ctx1m.md")
SCORE_SOURCES = ["fp4_sparse_attention_csa2_b200/csrc/index_tc.cu", "fp4_sparse_attention_csa2_b200/csrc/tc.cuh",
                 "fp4_sparse_attention_csa2_b200/csrc/common.cuh"]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p["hbm_gbs"], "measured"
    return 6650.0, "fallback"


# --------------------------------------------------------------------------- distributed plumbing
def dist_backend():
    """NCCL between GPUs; gloo when no GPU is visible (the host-side plumbing
    is then exercised on CPU processes), or as CSA2_DIST_BACKEND says."""
    return os.environ.get("CSA2_DIST_BACKEND") or ("nccl" if torch.cuda.is_available() else "gloo")


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if dist_backend() == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """The slowest rank's value (device times are taken per rank; the job's
    time is the maximum)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, layers_per_step, steps, ms_max):
    """Layer executions per second of the whole job: every rank runs its own
    sequence's steps (weak scaling), over the slowest rank's time."""
    return world * layers_per_step * steps / (ms_max / 1e3)


def rank_seed(seed, rank):
    """Each rank decodes its own independent sequence."""
    return seed + rank


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """NVML sampling of SM clock and throttle reasons while the timed region runs."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index, period=0.02):
        self.samples, self.reasons = [], set()
        self.period = period
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- our arm
def kernel_nodes(graph):
    """Number of kernel nodes in a captured CUDA graph (all of them are libcsa2's)."""
    try:
        import cuda.bindings.runtime as rt
        g = rt.cudaGraph_t(init_value=graph.raw_cuda_graph())
        err, _, n = rt.cudaGraphGetNodes(g, 0)
        err, nodes, n = rt.cudaGraphGetNodes(g, n)
        k = 0
        for nd in nodes[:n]:
            err, t = rt.cudaGraphNodeGetType(nd)
            if t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                k += 1
        return k
    except Exception as e:  # counting is best effort; the JSON then says null
        print("kernel node count unavailable: %r" % (e,), file=sys.stderr)
        return None


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_hash):
    """Per-launch DRAM bytes of the scoring kernel from the committed ncu
    summary, if it was taken on the current source of that kernel."""
    if not os.path.exists(PROFILE):
        return None
    vals = {}
    with open(PROFILE) as f:
        for line in f:
            if ":" in line and line.strip().startswith("-"):
                k, v = line.strip()[1:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_hash") != kernel_hash:
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def replay_regions(graphs, K, stream, world, min_total_s=0.5, min_reps=5):
    """Time exactly K steps (graph replays, round robin over the cache
    replicas) as one region, bracketed by a barrier and a synchronisation,
    repeated until at least min_reps regions and about min_total_s seconds;
    returns each region's device time in ms (max over ranks)."""
    times, spent = [], 0.0
    while len(times) < min_reps or spent < min_total_s * 1e3:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(K):
                graphs[i % len(graphs)].replay()
            e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ms = max_over_ranks(e0.elapsed_time(e1), world)
        times.append(ms)
        spent += ms
        if len(times) >= 10000:
            break
    return times


def capture_steps(stack, reps, stream):
    graphs = []
    for r in reps:
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
            stack.step(r)
        graphs.append(g)
    launches = kernel_nodes(graphs[0])
    for g in graphs:
        g.instantiate()
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    return graphs, launches


def timed_launches(fn, reps, stream, calls_per_rep=3, replays=None):
    """Mean device time of one call of fn(cache): a graph of calls rotating
    over the cache replicas, replayed after a warm-up replay."""
    R = calls_per_rep * len(reps)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        for i in range(R):
            fn(reps[i % len(reps)])
    g.replay()
    torch.cuda.synchronize()
    n = replays or 10
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        s0.record(stream)
        for _ in range(n):
            g.replay()
        s1.record(stream)
    torch.cuda.synchronize()
    return s0.elapsed_time(s1) / (n * R)


def replicas_for(w, lens):
    """Cache replicas rotated by the timed loop: at least three, and enough
    that together they exceed three times the L2 (the previous step's keys and
    rows are then not in L2), up to 64."""
    n_slots, _, _ = wl.cache_geometry(w, lens)
    key_bytes = 64 if w.idx_key_dtype == wl.E4M3 else 256
    one = n_slots * (w.row_stride + key_bytes)
    l2 = torch.cuda.get_device_properties(0).L2_cache_size if torch.cuda.is_available() else 126 << 20
    return int(min(64, max(3, -(-3 * l2 // max(one, 1)))))


def workload_line(w, seed, layers, args, stream, world, cpu_budget):
    """Layer-steps/s of one workload's decode step (CUDA graphs over rotating
    replicas, median of repeated K-step regions), its algorithmic bytes and
    roofline fractions, and the oracle timed beside it."""
    import fp4_sparse_attention_csa2_b200 as csa2
    from fp4_sparse_attention_csa2_b200.runner import new_workspace
    lens = wl.seq_lens(w, seed)
    if w.append_n:
        # (a) quantise-and-append of the last append_n positions of every
        # sequence in one batched call, timed on its own
        app = append_line(w, seed, lens, stream)
    reps = build_replicas(w, replicas_for(w, lens), seed, lens)
    ws = new_workspace(reps[0], w)
    stack = Stack(w, layers, ws)
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            stack.step(reps[i % len(reps)])
    stream.synchronize()
    st = csa2.read_device_status(ws, stream)
    if st != csa2.OK:
        raise RuntimeError("%s: device status after warm-up: %s" % (w.name, csa2.status_string(st)))
    graphs, launches = capture_steps(stack, reps, stream)
    K = max(1, min(args.steps, 200))
    times = replay_regions(graphs, K, stream, world, min_total_s=0.2, min_reps=3)
    ms = statistics.median(times) / K
    hbm, _ = peaks()
    sb = step_bytes(w, lens)
    line = {"layer_steps_per_s": round(world * len(w.pattern) / (ms / 1e3), 1), "ms_per_step": round(ms, 5),
            "batch": w.batch, "query_tokens": w.T, "context": int(lens.max()), "layers": w.pattern,
            "replicas": len(reps), "step_bytes_algorithmic": sb,
            "step_frac_of_8TBps": round(sb / (ms / 1e3) / 8e12, 4),
            "step_frac_of_measured_hbm": round(sb / (ms / 1e3) / (hbm * 1e9), 4), "gpu_launches_per_step": launches}
    if w.append_n:
        line["append"] = app
    if cpu_budget > 0:
        line["cpu_baseline"] = cpu_baseline(w, seed, layers, budget_s=cpu_budget)
    st = csa2.read_device_status(ws, stream)
    if st != csa2.OK:
        raise RuntimeError("%s: device status after timing: %s" % (w.name, csa2.status_string(st)))
    del graphs, stack, reps
    torch.cuda.empty_cache()
    return line


def append_line(w, seed, lens, stream):
    """Throughput of csa2_kv_append_quant for the workload's append step:
    every sequence's last append_n positions (bf16 latents and index keys) in
    one batched call.  Algorithmic bytes: the bf16 inputs read and the FP4 rows
    and E4M3 keys written."""
    import fp4_sparse_attention_csa2_b200 as csa2
    n_slots, table, stride = wl.cache_geometry(w, lens, seed)
    q0 = wl.layer_queries(w, 0, seed)["q_idx"]
    n_cached = int(lens.min()) - w.append_n
    cache = csa2.Cache(w.batch, n_slots, w.D, w.D_I, w.row_stride, w.idx_key_dtype, lens, table, w.page_size, stride)
    x = torch.stack([wl.latent(w, b, int(lens[b]), seed, t0=int(lens[b]) - w.append_n) for b in range(w.batch)])
    keys = torch.stack([wl.index_keys(w, b, int(lens[b]), q0[b, w.T - 1], seed, t0=int(lens[b]) - w.append_n)[0]
                        for b in range(w.batch)])
    x, keys = x.cuda(), keys.cuda()
    sp = torch.full((w.batch,), n_cached, dtype=torch.int32, device="cuda")
    fn = lambda c: csa2.kv_append_quant(c, x, sp, keys)
    ms = timed_launches(fn, [cache], stream, calls_per_rep=20)
    R = w.D // 2 + w.D // 16
    nbytes = w.batch * w.append_n * (2 * w.D + R + 2 * w.D_I + w.D_I)
    hbm, _ = peaks()
    del cache, x, keys
    torch.cuda.empty_cache()
    return {"positions_per_s": round(w.batch * w.append_n / (ms / 1e3), 1), "ms_per_call": round(ms, 5),
            "algorithmic_bytes_per_call": nbytes, "achieved_GBps": round(nbytes / (ms / 1e3) / 1e9, 1),
            "frac_of_8TBps": round(nbytes / (ms / 1e3) / 8e12, 4),
            "frac_of_measured_hbm": round(nbytes / (ms / 1e3) / (hbm * 1e9), 4)}


def run_ours(args, world, rank):
    import fp4_sparse_attention_csa2_b200 as csa2
    from fp4_sparse_attention_csa2_b200.runner import E2ERunner
    csa2.lib()
    w = wl.WORKLOADS[args.workload]
    seed = rank_seed(args.seed, rank)
    lens = wl.seq_lens(w, seed)
    layers = [wl.layer_queries(w, l, seed) for l in range(len(w.pattern))]
    reps = build_replicas(w, args.replicas, seed, lens)
    n_ws = csa2.workspace_bytes(reps[0], w.T, w.H, w.pool_k, w.top_k, w.window)
    ws = torch.empty(n_ws, dtype=torch.uint8, device="cuda")
    csa2.workspace_init(ws)
    stack = Stack(w, layers, ws)
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            stack.step(reps[i % len(reps)])
    stream.synchronize()
    st = csa2.read_device_status(ws, stream)
    if st != csa2.OK:
        raise RuntimeError("device status after warm-up: " + csa2.status_string(st))

    graphs, launches_per_step = capture_steps(stack, reps, stream)
    K = args.steps
    # the timed region: exactly K steps, repeated; the median region is the value
    with ClockSampler(torch.cuda.current_device()) as clk:
        times = replay_regions(graphs, K, stream, world)
    ms = statistics.median(times)
    st = csa2.read_device_status(ws, stream)
    if st != csa2.OK:
        raise RuntimeError("device status after timing: " + csa2.status_string(st))
    value = job_throughput(world, len(w.pattern), K, ms)
    hbm, peak_kind = peaks()

    # the dominant kernel by bytes (Full-layer scoring over every cached
    # position) timed on its own: a graph of launches over the rotating replicas
    L0 = stack.layers[0]
    score_ms = timed_launches(lambda c: csa2.index_scores(c, L0["q_idx"], L0["w"], ws), reps, stream)
    key_bytes = 64 if w.idx_key_dtype == wl.E4M3 else 256
    alg_bytes = int(np.sum(lens.astype(np.int64))) * w.T * key_bytes if w.T == 1 else int(np.sum(lens)) * key_bytes
    achieved = alg_bytes / (score_ms / 1e3) / 1e9
    traffic = profiled_traffic(source_hash(SCORE_SOURCES))

    # the attention call (the largest share of the step's time) on its own:
    # tensor-core bound at 64 heads (4 H D flop per attended row), also as bytes
    csa2.index_full(reps[0], L0["q_idx"], L0["w"], w.pool_k, w.top_k, stack.pool, stack.topk, ws)
    L1 = stack.layers[1]
    attn_ms = timed_launches(lambda c: csa2.sparse_swa_attn(c, L1["q"], stack.topk, w.window, stack.out[1],
                                                            stack.lse[1], ws), reps, stream)
    n_att = w.batch * w.T * (w.window + w.top_k)
    row = w.D // 2 + w.D // 16
    attn_flop = 4.0 * w.H * w.D * n_att
    with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) \
            else open(os.devnull) as f:
        txt = f.read()
    tf_peak = json.loads(txt)["bf16_tflops"] if txt else 1590.0
    attn_roof = {"kernel": "sparse + window attention and its split-softmax merge (one layer)", "bound": "tensor",
                 "achieved": round(attn_flop / (attn_ms / 1e3) / 1e12, 2), "peak": tf_peak,
                 "peak_kind": "measured bf16 burst (fp16 runs at the same nominal rate)" if txt else "fallback",
                 "unit": "TFLOP/s", "frac": round(attn_flop / (attn_ms / 1e3) / 1e12 / tf_peak, 5),
                 "flop_per_launch": attn_flop, "ms_per_launch": round(attn_ms, 5),
                 "algorithmic_bytes_per_launch": n_att * row,
                 "achieved_GBps": round(n_att * row / (attn_ms / 1e3) / 1e9, 1),
                 "frac_of_measured_hbm": round(n_att * row / (attn_ms / 1e3) / (hbm * 1e9), 5)}

    # end to end through the public binding with host buffers: per step the
    # step's inputs (every layer's queries; index queries and head weights of
    # the Full and Reindex layers) copied from pinned host memory, the step's
    # kernels as one graph replay, every layer's output and log-sum-exp read
    # back into pinned host memory; two device buffer sets alternate so that
    # the copies of neighbouring steps overlap the compute
    runner = E2ERunner(w, layers, ws, reps, stream)
    host_in, h_out0 = runner.stacks[0].host_buffers(layers)
    _, h_out1 = runner.stacks[1].host_buffers(layers)
    h2d, d2h = runner.bytes_per_step()
    Ke = max(3, min(K, 200))
    runner.run(host_in, (h_out0, h_out1), 4)
    torch.cuda.synchronize()
    e2e_times = []
    for _ in range(5):
        barrier(world)
        torch.cuda.synchronize()
        x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        runner.run(host_in, (h_out0, h_out1), Ke, x0, x1)
        torch.cuda.synchronize()
        barrier(world)
        e2e_times.append(max_over_ranks(x0.elapsed_time(x1), world))
    e2e_value = job_throughput(world, len(w.pattern), Ke, statistics.median(e2e_times))
    st = csa2.read_device_status(ws, stream)
    if st != csa2.OK:
        raise RuntimeError("device status after the end-to-end run: " + csa2.status_string(st))
    del runner, graphs
    torch.cuda.empty_cache()

    # the same step with layer-local window state: every layer appends its T
    # new bf16 rows to its own ring and attends over the ring's window rows
    local = local_window_line(w, lens, seed, layers, ws, reps, stream, world, K)
    # the append-time pool update of an in-flight request (its pool kept current
    # as tokens are appended), for one and for 64 appended positions
    pool_update = pool_update_line(w, lens, stack, ws, reps, stream)
    # prefill / verification of 64 query tokens through the same stack
    prefill = prefill_line(w, lens, seed, reps, stream, world, T=64)
    # one rank's device work in an 8-way context-parallel step of the same stack
    cp = cp_decode_line(w, lens, layers, reps, stream) if world == 1 else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, seed, layers, budget_s=args.cpu_budget)

    # the other synthetic workloads, each with its own numbers (one GPU only)
    extra = {}
    if world == 1 and not args.no_extra_workloads:
        for name in ("tiny4k", "long64k", "batch32_paged", "append_mq"):
            if name == w.name:
                continue
            we = wl.WORKLOADS[name]
            le = [wl.layer_queries(we, l, seed) for l in range(len(we.pattern))]
            extra[name] = workload_line(we, seed, le, args, stream, world,
                                        0.0 if args.no_cpu_baseline else args.extra_cpu_budget)

    if rank == 0:
        ms_step = ms / K
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "layer-steps/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp32-accum (E2M1/E4M3 storage, bf16 queries)",
            "data": "synthetic (seeded N(0,1) latents and keys, planted positions; no dataset)",
            "config": {"workload": w.name, "batch": w.batch, "context": int(lens.max()), "query_tokens": w.T,
                       "layers": w.pattern, "heads": w.H, "dim": w.D, "indexer": "%dx%d" % (w.H_I, w.D_I),
                       "pool_k": w.pool_k, "top_k": w.top_k, "window": w.window,
                       "parallelism": "dp%d (independent sequences per rank)" % world,
                       "l2": "%d rotating cache replicas, %.0f MB each (> 126 MB L2 together)" % (
                           len(reps), (reps[0].rows.numel() + reps[0].idx_keys.numel() *
                                       reps[0].idx_keys.element_size()) / 1e6),
                       "timing": "CUDA graph per step, CUDA events, max over ranks; %d timed regions of exactly %d "
                                 "steps, the median region reported (min %.5f, max %.5f ms per step)" % (
                                     len(times), K, min(times) / K, max(times) / K)},
            "roofline": {"kernel": "index scoring (Full layer, every cached position)", "bound": "hbm",
                         "achieved": round(achieved, 1), "peak": hbm, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": round(achieved / hbm, 4), "traffic": traffic,
                         "algorithmic_bytes_per_launch": alg_bytes, "ms_per_launch": round(score_ms, 5),
                         "frac_of_8TBps": round(achieved / 8000.0, 4)},
            "roofline_attention": attn_roof,
            "step_bytes_algorithmic": step_bytes(w, lens),
            "e2e": {"value": round(e2e_value, 1), "unit": "layer-steps/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": Ke,
                    "path": "python binding -> C ABI; each step one CUDA-graph replay of its csa2_layer_step calls; "
                            "inputs copied from pinned host memory and every output and lse read back to pinned "
                            "host memory every step, on side streams, two device buffer sets alternating so "
                            "neighbouring steps' copies overlap the compute; median of 5 runs"},
            "gpu_launches": None if launches_per_step is None else launches_per_step * K,
            "gpu_launches_per_step": launches_per_step,
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
            "local_window": local,
            "pool_update": pool_update,
            "prefill": prefill,
            "context_parallel": cp,
            "workloads": extra,
        }
        line["roofline"]["step_frac_of_8TBps"] = round(line["step_bytes_algorithmic"] / (ms_step / 1e3) / 8e12, 4)
        print(json.dumps(line))
        sys.stdout.flush()


def local_window_line(w, lens, seed, layers, ws, reps, stream, world, K):
    """Layer-steps/s of the decode step with a bf16 window ring per layer (the
    ring append of each layer's T new rows is inside the step), and the
    attention call over the ring alone."""
    import fp4_sparse_attention_csa2_b200 as csa2
    stack = Stack(w, layers, ws)
    stack.attach_rings(reps, lens, seed)
    with torch.cuda.stream(stream):
        for i in range(3):
            stack.step(reps[i % len(reps)])
    stream.synchronize()
    st = csa2.read_device_status(ws, stream)
    if st != csa2.OK:
        raise RuntimeError("local window: device status after warm-up: " + csa2.status_string(st))
    graphs, launches = capture_steps(stack, reps, stream)
    times = replay_regions(graphs, K, stream, world, min_total_s=0.3, min_reps=3)
    ms = statistics.median(times) / K
    L0, L1 = stack.layers[0], stack.layers[1]
    csa2.index_full(reps[0], L0["q_idx"], L0["w"], w.pool_k, w.top_k, stack.pool, stack.topk, ws)
    attn_ms = timed_launches(lambda c: csa2.sparse_swa_attn_local(c, stack.rings[id(c)][1], L1["q"], stack.topk,
                                                                  w.window, stack.out[1], stack.lse[1], ws),
                             reps, stream)
    st = csa2.read_device_status(ws, stream)
    if st != csa2.OK:
        raise RuntimeError("local window: device status after timing: " + csa2.status_string(st))
    n_q = w.batch * w.T
    sb = step_bytes(w, lens, local=True)
    hbm, _ = peaks()
    del graphs
    line = {"layer_steps_per_s": round(world * len(w.pattern) / (ms / 1e3), 1), "ms_per_step": round(ms, 5),
            "ring_rows": stack.ring_len, "ring_bytes_per_layer": w.batch * stack.ring_len * w.D * 2,
            "gpu_launches_per_step": launches, "attention_ms_per_launch": round(attn_ms, 5),
            "attention_tflops": round(4.0 * w.H * w.D * n_q * (w.window + w.top_k) / (attn_ms / 1e3) / 1e12, 2),
            "step_bytes_algorithmic": sb, "step_frac_of_measured_hbm": round(sb / (ms / 1e3) / (hbm * 1e9), 4),
            "path": "per layer csa2_ring_append of the step's T rows, then csa2_layer_step with the layer's ring "
                    "(window rows bf16 from the ring, top-k rows FP4 from the shared cache)"}
    del stack
    torch.cuda.empty_cache()
    return line


def pool_update_line(w, lens, stack, ws, reps, stream):
    """csa2_index_pool_update timed alone (graph of calls over the replicas):
    the Full layer's pool, without the positions about to be appended, updated
    with the last n_new positions under the Reindex layer's query.
    Algorithmic bytes: the index keys of every candidate (64 B each, E4M3)."""
    import fp4_sparse_attention_csa2_b200 as csa2
    L0, L1 = stack.layers[0], stack.layers[1]
    csa2.index_full(reps[0], L0["q_idx"], L0["w"], w.pool_k, w.top_k, stack.pool, stack.topk, ws)
    torch.cuda.synchronize()
    out = {}
    key = 64 if w.idx_key_dtype == wl.E4M3 else 256
    for n_new in (1, 64):
        t_new0 = torch.as_tensor(lens.astype(np.int64) - n_new, device="cuda").view(-1, 1, 1)
        prev = torch.where(stack.pool >= t_new0, torch.full_like(stack.pool, -1), stack.pool).contiguous()
        pool = torch.empty_like(prev)
        topk = torch.empty_like(stack.topk)
        ms = timed_launches(lambda c: csa2.index_pool_update(c, L1["q_idx"], L1["w"], prev, n_new, w.top_k, pool,
                                                             topk, ws), reps, stream)
        st = csa2.read_device_status(ws, stream)
        if st != csa2.OK:
            raise RuntimeError("pool update: device status " + csa2.status_string(st))
        n_q = w.batch * w.T
        out["n_new_%d" % n_new] = {"us_per_call": round(ms * 1e3, 2),
                                   "candidates": w.pool_k + n_new,
                                   "updates_per_s": round(n_q / (ms / 1e3), 1),
                                   "algorithmic_bytes_per_call": n_q * (w.pool_k + n_new) * key}
    return out


def prefill_line(w, lens, seed, reps, stream, world, T):
    """The stack for T query tokens per sequence (the last T positions, as in
    verifying T drafted tokens or a prefill chunk) through csa2_prefill_layer,
    one CUDA graph per replica; token-layer steps per second."""
    import dataclasses
    import fp4_sparse_attention_csa2_b200 as csa2
    wt = dataclasses.replace(w, T=T)
    layers = [{k: v.cuda() for k, v in wl.layer_queries(wt, l, seed).items()} for l in range(len(w.pattern))]
    B = w.batch
    n = csa2.prefill_workspace_bytes(reps[0], T, w.H, w.H_I, w.pool_k, w.top_k, w.window)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    csa2.workspace_init(ws)
    pool = torch.zeros((B, T, w.pool_k), dtype=torch.int32, device="cuda")
    topk = torch.zeros((B, T, w.top_k), dtype=torch.int32, device="cuda")
    out = torch.empty((B, T, w.H, w.D), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, T, w.H), dtype=torch.float32, device="cuda")
    modes = [{"F": csa2.FULL, "R": csa2.REINDEX, "U": csa2.REUSE}[m] for m in w.pattern]

    def step(c):
        for L, m in zip(layers, modes):
            idx = m != csa2.REUSE
            csa2.prefill_layer(c, m, L["q"], topk, out, ws, w.window, q_idx=L["q_idx"] if idx else None,
                               head_w=L["w"] if idx else None, pool_idx=pool, lse=lse, pool_k=w.pool_k,
                               H_I=w.H_I)

    with torch.cuda.stream(stream):
        for i in range(3):
            step(reps[i % len(reps)])
    stream.synchronize()
    st = csa2.read_device_status(ws, stream)
    if st != csa2.OK:
        raise RuntimeError("prefill: device status after warm-up: " + csa2.status_string(st))
    graphs = []
    for r in reps:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
            step(r)
        graphs.append(g)
    times = replay_regions(graphs, 3, stream, world, min_total_s=0.3, min_reps=3)
    ms = statistics.median(times) / 3
    st = csa2.read_device_status(ws, stream)
    if st != csa2.OK:
        raise RuntimeError("prefill: device status after timing: " + csa2.status_string(st))
    del graphs
    torch.cuda.empty_cache()
    return {"query_tokens": T, "ms_per_step": round(ms, 4),
            "token_layer_steps_per_s": round(world * B * T * len(w.pattern) / (ms / 1e3), 1),
            "chunk_tokens": min(T, 128 // ((w.H_I + 15) // 16 * 16)),
            "path": "csa2_prefill_layer per layer: the tokens in chunks through the decode kernels, causal per token"}


def cp_decode_line(w, lens, layers, reps, stream, R=8):
    """One rank's device work in an R-way context-parallel decode step of the
    stack (runner.CpRankStep: the sequence's positions in R shards of L / R;
    its shard calls, the merge selections over all R ranks' candidates and the
    log-sum-exp merges of all R attention parts).  The all-gathers between
    ranks are not in the timed region (one GPU here).  The timed steps rotate
    over every shard of every replica (R x replicas shards, more key bytes than
    the L2 holds)."""
    from fp4_sparse_attention_csa2_b200.runner import CpRankStep
    try:
        cp = CpRankStep(w, lens, layers, reps, R)
    except ValueError:
        return None
    with torch.cuda.stream(stream):
        ms = timed_launches(cp.step, cp.shards, stream, calls_per_rep=1, replays=5)
        # the step's pieces: a Full layer's indexing share (shard scoring and
        # pool, merge of all ranks' pools), a Reindex layer's, one layer's attention
        f_ms = timed_launches(cp.full_part, cp.shards, stream, calls_per_rep=1, replays=5)
        r_ms = timed_launches(cp.reindex_part, cp.shards, stream, calls_per_rep=1, replays=5) \
            if "R" in w.pattern else None
        a_ms = timed_launches(cp.attn_part, cp.shards, stream, calls_per_rep=1, replays=5)
    cp.check("after timing")
    key = 64 if w.idx_key_dtype == wl.E4M3 else 256
    n_f, n_r = w.pattern.count("F"), w.pattern.count("R")
    gathered = R * (n_f * w.pool_k * 8 + len(w.pattern) * w.H * (w.D + 1) * 4)    # all-gathers
    reduced = n_r * w.pool_k * 4                                                   # the Reindex all-reduce
    line = {"ranks": R, "shard_positions": cp.n, "us_per_step_rank": round(ms * 1e3, 2),
            "us_full_index_share": round(f_ms * 1e3, 2),
            "us_reindex_share": None if r_ms is None else round(r_ms * 1e3, 2),
            "us_attention_layer": round(a_ms * 1e3, 2),
            "layer_steps_per_s_compute": round(len(w.pattern) / (ms / 1e3), 1),
            "shard_key_bytes_per_step": cp.n * key * n_f,
            "allgather_bytes_per_step_rank": gathered,
            "allreduce_bytes_per_step": reduced,
            "collectives_per_step": n_f + n_r + len(w.pattern),
            "path": "per rank: csa2_cp_index_local on its shard + csa2_cp_merge_select over all ranks' candidates "
                    "(Full), csa2_cp_reindex_local + csa2_cp_reindex_select on the summed pool scores (Reindex), "
                    "csa2_cp_sparse_swa_attn on its shard + csa2_lse_merge of all parts (every layer); the NCCL "
                    "collectives between these are not timed (one GPU)"}
    del cp
    torch.cuda.empty_cache()
    return line


def step_bytes(w, lens, local=False):
    """Algorithmic bytes of one step: index keys scored (every visible key of
    every sequence once: the scorer reads a key once for all of a sequence's
    query tokens), pool keys rescored and FP4 rows attended (upper bound
    |S| = window + top_k per query token).  local: the window rows are bf16
    rows of the layer's ring and each layer appends its T new rows."""
    key = 64 if w.idx_key_dtype == wl.E4M3 else 256
    L = lens.astype(np.int64)
    full = int(np.sum(L)) * key
    n_q = w.batch * w.T
    re = n_q * min(w.pool_k, int(L.min())) * key
    S = n_q * (w.window + w.top_k) * (w.D // 2 + w.D // 16)
    if local:
        # window rows bf16 from the layer's ring, plus the append of the
        # step's T rows (read and written)
        S = n_q * (w.window * 2 * w.D + w.top_k * (w.D // 2 + w.D // 16)) + 2 * n_q * 2 * w.D
    n_f = w.pattern.count("F")
    n_r = w.pattern.count("R")
    return n_f * full + n_r * re + len(w.pattern) * S


# --------------------------------------------------------------------------- the oracle
def oracle_step_timer(w, seed, layers, budget_s, max_steps=1000, warmup=0):
    """Time the CPU oracle on decode steps of the workload for about budget_s
    seconds (setup -- key encoding, row quantisation -- excluded).  Returns
    (layer-steps per second, steps run, seconds, sample description)."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from harness import attended_positions, build_ref_cache, fill_ref_rows, host_layer
    lens = wl.seq_lens(w, seed)
    ref = build_ref_cache(w, seed=seed, rows=False, layers=layers, batches=[0])
    hl = [host_layer(L) for L in layers]
    lat = wl.latent(w, 0, int(lens[0]), seed)
    # rows of every position any layer may attend: quantised once, untimed
    j = w.T - 1
    p = int(lens[0]) - w.T + j
    pool, topk, _ = oracle.index_full(ref, 0, w.T, j, hl[0]["q_idx"][0, j], w.q_idx_dtype, hl[0]["w"][0, j],
                                      w.pool_k, w.top_k)
    need = attended_positions(topk, p, w.window)
    for l, m in enumerate(w.pattern):
        if m == "R":
            tk, _ = oracle.index_reindex(ref, 0, w.T, j, hl[l]["q_idx"][0, j], w.q_idx_dtype, hl[l]["w"][0, j],
                                         pool, w.top_k)
            need |= attended_positions(tk, p, w.window)
    fill_ref_rows(ref, w, 0, need, lat)
    for _ in range(warmup):
        oracle.run_stack(ref, w.pattern, hl, w.T, w.pool_k, w.top_k, w.window, w.q_idx_dtype, batches=[0],
                         tokens=[j])
    steps, t0 = 0, time.perf_counter()
    while True:
        oracle.run_stack(ref, w.pattern, hl, w.T, w.pool_k, w.top_k, w.window, w.q_idx_dtype, batches=[0],
                         tokens=[j])
        steps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or steps >= max_steps:
            break
    sample = ("sequence 0, query token %d of the %s stack (%s): %d full decode step(s), single-threaded C "
              "oracle, fp64" % (j, w.name, w.pattern, steps))
    # one (sequence, token) of the batch; the metric's step covers batch*T of them
    per_step = el / steps * (w.batch * w.T)
    return len(w.pattern) / per_step, steps, el, sample


def cpu_baseline(w, seed, layers, budget_s):
    v, steps, el, sample = oracle_step_timer(w, seed, layers, budget_s)
    return {"value": round(v, 4), "unit": "layer-steps/s", "cores": 1, "kind": "oracle", "sample": sample,
            "seconds": round(el, 2)}


def oracle_piece_timer(w, seed, layers, budget_s, steps, warmup):
    """The reference arm: the oracle's decode step of one (sequence, token) cut
    into pieces -- the Full layer's scoring in slices of positions, then each
    selection, Reindex and layer attention whole (the calls the step makes) --
    with the slices sized so that `steps` pieces take about budget_s seconds.  Warm-up steps run pieces untimed; timed step i runs piece
    (warmup + i) mod P (consecutive pieces are grouped when there are more
    pieces than steps, so each is timed at least once).  One decode step costs
    the sum of the pieces' mean times.  Returns (layer-steps per second,
    seconds of the timed steps, sample description, seconds per layer of each
    type for one (sequence, token) -- None when pieces were grouped)."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from harness import attended_positions, build_ref_cache, fill_ref_rows, host_layer
    lens = wl.seq_lens(w, seed)
    ref = build_ref_cache(w, seed=seed, rows=False, layers=layers, batches=[0])
    hl = [host_layer(L) for L in layers]
    j = w.T - 1
    p = int(lens[0]) - w.T + j
    # the indices every layer attends with, and the rows they need (untimed set-up)
    topk_of, pools = {}, {}
    pool = topk = None
    scores = {}
    for l, m in enumerate(w.pattern):
        if m == "F":
            pool, topk, scores[l] = oracle.index_full(ref, 0, w.T, j, hl[l]["q_idx"][0, j], w.q_idx_dtype,
                                                      hl[l]["w"][0, j], w.pool_k, w.top_k, want_scores=True)
            pools[l] = pool
        elif m == "R":
            pools[l] = pool
            topk, _ = oracle.index_reindex(ref, 0, w.T, j, hl[l]["q_idx"][0, j], w.q_idx_dtype, hl[l]["w"][0, j],
                                           pool, w.top_k)
        topk_of[l] = topk
    need = set()
    for tk in topk_of.values():
        need |= attended_positions(tk, p, w.window)
    fill_ref_rows(ref, w, 0, need, wl.latent(w, 0, int(lens[0]), seed))
    positions = np.arange(p + 1, dtype=np.int32)

    def run(piece):
        kind, l, a, b = piece
        if kind == "score":
            oracle.index_scores(ref, 0, positions[a:b], hl[l]["q_idx"][0, j], w.q_idx_dtype, hl[l]["w"][0, j])
        elif kind == "select":
            oracle.select_top(scores[l], None, w.pool_k)
            oracle.select_top(scores[l], None, w.top_k)
        elif kind == "reindex":
            oracle.index_reindex(ref, 0, w.T, j, hl[l]["q_idx"][0, j], w.q_idx_dtype, hl[l]["w"][0, j], pools[l],
                                 w.top_k)
        else:
            oracle.sparse_swa_attn(ref, 0, w.T, j, hl[l]["q"][0, j][a:b], topk_of[l], w.window)

    def timed(piece):
        t0 = time.perf_counter()
        run(piece)
        return time.perf_counter() - t0

    # piece sizes from untimed probes: every piece is a whole oracle call as
    # the decode step makes it (a layer's attention, a selection, a Reindex),
    # except the Full scoring, cut into as many position slices as it takes
    # for `steps` pieces to fit in budget_s
    probe = min(8192, p + 1)
    t_pos = timed(("score", 0, 0, probe)) / probe
    t_rest = sum(timed(("attn", l, 0, w.H)) for l in range(len(w.pattern)))
    t_rest += sum(timed(("select", l, 0, 0)) for l, m in enumerate(w.pattern) if m == "F")
    t_rest += sum(timed(("reindex", l, 0, 0)) for l, m in enumerate(w.pattern) if m == "R")
    n_f = w.pattern.count("F")
    t_step = n_f * t_pos * (p + 1) + t_rest
    n_other = len(w.pattern) + n_f + w.pattern.count("R")
    want = int(np.ceil(max(steps, 1) * t_step / max(budget_s, 1e-9)))
    n_slices = max(1, -(-max(want - n_other, n_f) // max(n_f, 1)))
    slice_n = int(max(min(-(-(p + 1) // n_slices), p + 1), min(1024, p + 1)))
    pieces = []
    for l, m in enumerate(w.pattern):
        if m == "F":
            pieces += [("score", l, a, min(a + slice_n, p + 1)) for a in range(0, p + 1, slice_n)]
            pieces.append(("select", l, 0, 0))
        elif m == "R":
            pieces.append(("reindex", l, 0, 0))
        pieces.append(("attn", l, 0, w.H))
    n_groups = min(len(pieces), max(steps, 1))
    groups = [pieces[g * len(pieces) // n_groups:(g + 1) * len(pieces) // n_groups] for g in range(n_groups)]
    for i in range(warmup):
        for pc in groups[i % n_groups]:
            run(pc)
    acc = [0.0] * n_groups
    cnt = [0] * n_groups
    t_all = time.perf_counter()
    for i in range(steps):
        g = (warmup + i) % n_groups
        t0 = time.perf_counter()
        for pc in groups[g]:
            run(pc)
        acc[g] += time.perf_counter() - t0
        cnt[g] += 1
    el = time.perf_counter() - t_all
    per_seq_token = sum(a / c for a, c in zip(acc, cnt) if c)
    # seconds per layer type (one (sequence, token)), when every piece was timed on its own
    per_type = None
    if n_groups == len(pieces) and all(cnt):
        per_type = {}
        for m in sorted(set(w.pattern)):
            layers_m = [l for l, x in enumerate(w.pattern) if x == m]
            tot = sum(acc[g] / cnt[g] for g in range(n_groups) if groups[g][0][1] in layers_m)
            per_type[m] = round(tot / len(layers_m), 4)
    # one (sequence, token) of the batch; the metric's step covers batch*T of them
    per_step = per_seq_token * (w.batch * w.T)
    sample = ("sequence 0, query token %d of the %s stack (%s), single-threaded C oracle, fp64: one decode step cut "
              "into %d pieces (Full scoring in slices of %d positions; each selection, Reindex and layer attention "
              "whole), %d timed step(s) of one group of consecutive pieces each, round robin over %d groups; a "
              "decode step costs the sum of the groups' mean times (%.2f s)"
              % (j, w.name, w.pattern, len(pieces), slice_n, steps, n_groups, per_seq_token))
    return len(w.pattern) / per_step, el, sample, per_type


def run_reference(args, world, rank):
    """The oracle as the reference arm (rank 0 only): exactly `warmup` untimed
    and `steps` timed steps, each a bounded piece of the workload's decode
    step (see oracle_piece_timer), the value scaled to whole decode steps."""
    if rank != 0:
        return
    w = wl.WORKLOADS[args.workload]
    layers = [wl.layer_queries(w, l, args.seed) for l in range(len(w.pattern))]
    v, el, sample, per_type = oracle_piece_timer(w, args.seed, layers, args.ref_budget, args.steps, args.warmup)
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "layer-steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / max(args.steps, 1) * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded, same generator as the CUDA arm)",
            "config": {"workload": w.name, "context": int(wl.seq_lens(w, args.seed).max()), "layers": w.pattern},
            "cpu_baseline": {"kind": "oracle", "cores": 1, "sample": sample, "value": round(v, 4),
                             "seconds_per_layer": per_type},
            "e2e": {"value": round(v, 4), "unit": "layer-steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="ctx1m", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--replicas", type=int, default=3)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=120.0, help="seconds of timed oracle work in the reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="report the headline workload only (one GPU otherwise adds the other four)")
    ap.add_argument("--extra-cpu-budget", type=float, default=3.0,
                    help="seconds of oracle time per extra workload")
    args = ap.parse_args()
    world, rank, _ = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Device-side set-up and stepping of a CSA2 layer stack through the C ABI:
fill a cache with csa2_kv_append_quant from the seeded inputs, and run one
decode step (every layer of the pattern) with csa2_layer_step."""
import torch

import fp4_sparse_attention_csa2_b200 as csa2
from fp4_sparse_attention_csa2_b200 import workloads as wl

APPEND_CHUNK = 1 << 16


def build_replicas(w, n_rep, seed, lens):
    """One cache filled through csa2_kv_append_quant, then copied into n_rep
    independent buffers (rotated by the benchmark so that no step finds its
    inputs in L2)."""
    n_slots, table, stride = wl.cache_geometry(w, lens, seed)
    base = csa2.Cache(w.batch, n_slots, w.D, w.D_I, w.row_stride, w.idx_key_dtype, lens, table, w.page_size, stride)
    q0 = wl.layer_queries(w, 0, seed)["q_idx"]
    sp = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b in range(w.batch):
        L = int(lens[b])
        x = wl.latent(w, b, L, seed)
        keys, _ = wl.index_keys(w, b, L, q0[b, w.T - 1], seed)
        v = base.view(b)
        for t0 in range(0, L, APPEND_CHUNK):
            sp.fill_(t0)
            csa2.kv_append_quant(v, x[t0:t0 + APPEND_CHUNK][None].cuda(), sp,
                                 keys[t0:t0 + APPEND_CHUNK][None].cuda())
        torch.cuda.synchronize()
    reps = [base]
    for _ in range(n_rep - 1):
        c = csa2.Cache(w.batch, n_slots, w.D, w.D_I, w.row_stride, w.idx_key_dtype, lens, table, w.page_size,
                       stride)
        c.rows.copy_(base.rows)
        c.idx_keys.copy_(base.idx_keys)
        reps.append(c)
    torch.cuda.synchronize()
    return reps


FLAT_ALIGN = 256   # every tensor of a flat buffer starts on this byte boundary (the C ABI wants 16)


def flat_views(specs, device, pin=False):
    """One uint8 buffer holding tensors of the given (shape, dtype) specs, each
    starting on a FLAT_ALIGN-byte boundary; returns (buffer, [views]).  One
    copy of the buffer moves all of them (a step's inputs or outputs)."""
    offs, off = [], 0
    for shape, dtype in specs:
        n = 1
        for d in shape:
            n *= int(d)
        offs.append((off, n * torch.empty((), dtype=dtype).element_size()))
        off = (off + offs[-1][1] + FLAT_ALIGN - 1) // FLAT_ALIGN * FLAT_ALIGN
    buf = torch.zeros(max(off, 1), dtype=torch.uint8, device=device)
    if pin:
        buf = buf.pin_memory()
    views = [buf[o:o + nb].view(dtype).view(shape) for (o, nb), (shape, dtype) in zip(offs, specs)]
    return buf, views


class Stack:
    """Device buffers of one decode step and the C-ABI calls that run it.

    The inputs a step consumes (every layer's q; q_idx and head weights of
    the Full and Reindex layers) live in one flat device buffer, `inputs`, and
    every layer's out and lse in another, `outputs`, so a host round trip of a
    step is one copy each way (`host_buffers` gives matching pinned host
    buffers)."""

    def __init__(self, w, layers, ws):
        self.w, self.ws = w, ws
        B, T = w.batch, w.T
        self.modes = [{"F": csa2.FULL, "R": csa2.REINDEX, "U": csa2.REUSE}[m] for m in w.pattern]
        self.in_keys = [[k for k in L if k == "q" or m != csa2.REUSE] for L, m in zip(layers, self.modes)]
        in_specs = [(tuple(L[k].shape), L[k].dtype) for L, ks in zip(layers, self.in_keys) for k in ks]
        self.inputs, views = flat_views(in_specs, "cuda")
        it = iter(views)
        self.layers = []
        for L, ks in zip(layers, self.in_keys):
            d = {}
            for k, v in L.items():
                if k in ks:
                    d[k] = next(it)
                    d[k].copy_(v)
                else:
                    d[k] = v.cuda()
            self.layers.append(d)
        self.pool = torch.zeros((B, T, w.pool_k), dtype=torch.int32, device="cuda")
        self.topk = torch.zeros((B, T, w.top_k), dtype=torch.int32, device="cuda")
        n = len(w.pattern)
        out_specs = [((B, T, w.H, w.D), torch.float32)] * n + [((B, T, w.H), torch.float32)] * n
        self.outputs, views = flat_views(out_specs, "cuda")
        self.out, self.lse = views[:n], views[n:]
        self.rings = None

    def attach_rings(self, reps, lens, seed=0):
        """Give every layer its own bf16 window ring ([B, window + T - 1, D],
        filled with the layer's rows of the window positions) on every cache
        replica: each step then appends the layer's T new rows
        (csa2_ring_append) and attends over the ring's window rows."""
        w = self.w
        B, T = w.batch, w.T
        ring_len = w.window + T - 1
        self.ring_len = ring_len
        start = torch.as_tensor(lens, dtype=torch.int32) - ring_len
        self.fill_start = start.cuda()
        self.start = (torch.as_tensor(lens, dtype=torch.int32) - T).cuda()
        self.x_local = []
        fill = []
        for l in range(len(self.modes)):
            rows = torch.stack([wl.window_rows(w, l, b, int(start[b]), ring_len, seed) for b in range(B)])
            fill.append(rows.cuda())
            self.x_local.append(rows[:, ring_len - T:].contiguous().cuda())   # the step's own T rows
        self.rings = {}
        for c in reps:
            rl = []
            for l in range(len(self.modes)):
                r = torch.zeros((B, ring_len, w.D), dtype=torch.bfloat16, device="cuda")
                csa2.ring_append(c, r, fill[l], self.fill_start)
                rl.append(r)
            self.rings[id(c)] = rl
        torch.cuda.synchronize()

    def host_buffers(self, layers):
        """Pinned host copies of `inputs` (filled from the host-side layers)
        and of `outputs` (to be read back into)."""
        in_specs = [(tuple(L[k].shape), L[k].dtype) for L, ks in zip(layers, self.in_keys) for k in ks]
        h_in, views = flat_views(in_specs, "cpu", pin=True)
        it = iter(views)
        for L, ks in zip(layers, self.in_keys):
            for k in ks:
                next(it).copy_(L[k])
        h_out = torch.empty(self.outputs.numel(), dtype=torch.uint8).pin_memory()
        return h_in, h_out

    def step(self, cache):
        rings = None if self.rings is None else self.rings[id(cache)]
        for l, m in enumerate(self.modes):
            L = self.layers[l]
            idx = m != csa2.REUSE
            ring = None
            if rings is not None:
                ring = rings[l]
                csa2.ring_append(cache, ring, self.x_local[l], self.start)
            csa2.layer_step(cache, m, L["q"], self.topk, self.out[l], self.ws, self.w.window,
                            q_idx=L["q_idx"] if idx else None, head_w=L["w"] if idx else None, pool_idx=self.pool,
                            lse=self.lse[l], pool_k=self.w.pool_k, ring=ring)


def new_workspace(cache, w):
    ws = torch.empty(csa2.workspace_bytes(cache, w.T, w.H, w.pool_k, w.top_k, w.window), dtype=torch.uint8,
                     device="cuda")
    csa2.workspace_init(ws)
    return ws


class E2ERunner:
    """Decode steps end to end through the public binding, as a serving loop
    would run them: every step's inputs are copied from pinned host memory and
    every step's outputs read back into pinned host memory, while the kernels
    of a step are one CUDA-graph replay.  Two Stacks (two sets of device input
    and output buffers) alternate, so step i + 1's inputs are on their way in
    and step i - 1's outputs on their way out while step i computes: the
    host-to-device copies run on one side stream, the device-to-host copies on
    another, ordered against the compute stream by events."""

    def __init__(self, w, layers, ws, reps, stream):
        self.w, self.reps, self.stream = w, reps, stream
        self.stacks = [Stack(w, layers, ws), Stack(w, layers, ws)]
        self.h2d = torch.cuda.Stream()
        self.d2h = torch.cuda.Stream()
        self.graphs = {}
        for s, st in enumerate(self.stacks):
            for r, c in enumerate(reps):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
                    st.step(c)
                self.graphs[(r, s)] = g
        self.ev_in = [torch.cuda.Event() for _ in range(2)]
        self.ev_done = [torch.cuda.Event() for _ in range(2)]
        self.ev_out = [torch.cuda.Event() for _ in range(2)]

    def bytes_per_step(self):
        st = self.stacks[0]
        return st.inputs.numel(), st.outputs.numel()

    def run(self, host_in, host_outs, n, t0=None, t1=None):
        """n steps; host_in: pinned uint8 copy of a Stack's inputs; host_outs:
        two pinned uint8 buffers the outputs alternate into.  t0 / t1
        (optional CUDA events) are recorded before the first copy and after
        the last read-back."""
        if t0 is not None:
            t0.record(self.h2d)
        for i in range(n):
            s = i % 2
            st = self.stacks[s]
            with torch.cuda.stream(self.h2d):
                if i >= 2:
                    self.h2d.wait_event(self.ev_done[s])          # step i - 2 no longer reads these inputs
                st.inputs.copy_(host_in, non_blocking=True)
                self.ev_in[s].record(self.h2d)
            self.stream.wait_event(self.ev_in[s])
            if i >= 2:
                self.stream.wait_event(self.ev_out[s])            # step i - 2's outputs have left the device
            with torch.cuda.stream(self.stream):
                self.graphs[(i % len(self.reps), s)].replay()
            self.ev_done[s].record(self.stream)
            with torch.cuda.stream(self.d2h):
                self.d2h.wait_event(self.ev_done[s])
                host_outs[s].copy_(st.outputs, non_blocking=True)
                self.ev_out[s].record(self.d2h)
        if t1 is not None:
            self.d2h.wait_stream(self.stream)
            t1.record(self.d2h)


class CpRankStep:
    """One rank's device work in an R-way context-parallel decode step of the
    stack, on one GPU: the sequence (batch 1, one query token) is split into R
    shards of L / R positions, taken as shard views of the given caches.  The
    candidates and attention parts of all R ranks are computed once from the
    first cache's shards; step(shard) then runs one rank's calls of a step --
    its shard calls, the selections over all ranks' candidates (Full) and
    summed pool scores (Reindex), the log-sum-exp merges of all ranks' parts
    -- with no exchange in between."""

    def __init__(self, w, lens, layers, caches, R=8):
        L = int(lens[0])
        n = L // R
        if w.batch != 1 or w.T != 1 or w.paged or n % 64 or n * R != L:
            raise ValueError("an even split of one contiguous sequence into 64-aligned shards")
        self.w, self.R, self.n = w, R, n
        H, D, B = w.H, w.D, 1
        dev = "cuda"
        self.shards = [(c.shard_view(0, r * n, n), r) for c in caches for r in range(R)]
        self.pos0 = [torch.tensor([r * n], dtype=torch.int32, device=dev) for r in range(R)]
        self.glens = torch.tensor([L], dtype=torch.int32, device=dev)
        self.ws = torch.empty(csa2.workspace_bytes(self.shards[0][0], 1, H, w.pool_k, w.top_k, w.window),
                              dtype=torch.uint8, device=dev)
        csa2.workspace_init(self.ws)
        self.mws = torch.empty(csa2.cp_merge_workspace_bytes(R, B, w.pool_k), dtype=torch.uint8, device=dev)
        csa2.workspace_init(self.mws)
        self.dl = [{k: v.cuda() for k, v in x.items()} for x in layers]
        self.pool = torch.empty((B, w.pool_k), dtype=torch.int32, device=dev)
        self.topk = torch.empty((B, w.top_k), dtype=torch.int32, device=dev)
        self.gpool = torch.empty((R, B, w.pool_k, 2), dtype=torch.int32, device=dev)
        self.rscores = torch.empty((R, B, w.pool_k), dtype=torch.float32, device=dev)
        self.gscores = torch.empty((B, w.pool_k), dtype=torch.float32, device=dev)
        self.gout = torch.empty((len(w.pattern), R, B, H, D), dtype=torch.float32, device=dev)
        self.glse = torch.empty((len(w.pattern), R, B, H), dtype=torch.float32, device=dev)
        self.cand_pool = torch.empty((B, w.pool_k, 2), dtype=torch.int32, device=dev)
        self.pool_scores = torch.empty((B, w.pool_k), dtype=torch.float32, device=dev)
        self.part_o = torch.empty((B, H, D), dtype=torch.float32, device=dev)
        self.part_l = torch.empty((B, H), dtype=torch.float32, device=dev)
        self.out = torch.empty((B, H, D), dtype=torch.float32, device=dev)
        self.lse = torch.empty((B, H), dtype=torch.float32, device=dev)
        # every rank's candidates and attention parts, from the first cache's shards
        for l, m in enumerate(w.pattern):
            q = self.dl[l]
            if m == "F":
                for r in range(R):
                    csa2.cp_index_local(self.shards[r][0], self.pos0[r], q["q_idx"], q["w"], w.pool_k, self.gpool[r],
                                        self.ws)
                csa2.cp_merge_select(self.gpool, self.glens, w.pool_k, self.pool, self.mws, n_b=w.top_k,
                                     out_b=self.topk)
            elif m == "R":
                for r in range(R):
                    csa2.cp_reindex_local(self.shards[r][0], self.pos0[r], q["q_idx"], q["w"], self.pool,
                                          self.rscores[r], self.ws)
                torch.sum(self.rscores, dim=0, out=self.gscores)      # the all-reduce
                csa2.cp_reindex_select(self.pool, self.gscores, self.glens, w.top_k, self.topk)
            for r in range(R):
                csa2.cp_sparse_swa_attn(self.shards[r][0], self.pos0[r], self.glens, q["q"], self.topk, w.window,
                                        self.gout[l, r], self.glse[l, r], self.ws)
        torch.cuda.synchronize()
        self.check("after the set-up")

    def check(self, when):
        for x in (self.ws, self.mws):
            st = csa2.read_device_status(x)
            if st != csa2.OK:
                raise RuntimeError("context parallel %s: device status %s" % (when, csa2.status_string(st)))

    def full_part(self, sh, l=None):
        w, q = self.w, self.dl[self.w.pattern.index("F") if l is None else l]
        csa2.cp_index_local(sh[0], self.pos0[sh[1]], q["q_idx"], q["w"], w.pool_k, self.cand_pool, self.ws)
        csa2.cp_merge_select(self.gpool, self.glens, w.pool_k, self.pool, self.mws, n_b=w.top_k, out_b=self.topk)

    def reindex_part(self, sh, l=None):
        w, q = self.w, self.dl[self.w.pattern.index("R") if l is None else l]
        csa2.cp_reindex_local(sh[0], self.pos0[sh[1]], q["q_idx"], q["w"], self.pool, self.pool_scores, self.ws)
        csa2.cp_reindex_select(self.pool, self.gscores, self.glens, w.top_k, self.topk)

    def attn_part(self, sh, l=None):
        w = self.w
        l = len(w.pattern) - 1 if l is None else l
        csa2.cp_sparse_swa_attn(sh[0], self.pos0[sh[1]], self.glens, self.dl[l]["q"], self.topk, w.window,
                                self.part_o, self.part_l, self.ws)
        csa2.lse_merge(self.gout[l], self.glse[l], self.out, self.lse)

    def step(self, sh):
        for l, m in enumerate(self.w.pattern):
            if m == "F":
                self.full_part(sh, l)
            elif m == "R":
                self.reindex_part(sh, l)
            self.attn_part(sh, l)

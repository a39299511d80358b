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


class Stack:
    """Device buffers of one decode step and the C-ABI calls that run it."""

    def __init__(self, w, layers, ws):
        self.w, self.ws = w, ws
        B, T = w.batch, w.T
        self.layers = [{k: v.cuda() for k, v in L.items()} for L in layers]
        self.pool = torch.zeros((B, T, w.pool_k), dtype=torch.int32, device="cuda")
        self.topk = torch.zeros((B, T, w.top_k), dtype=torch.int32, device="cuda")
        self.out = [torch.empty((B, T, w.H, w.D), dtype=torch.float32, device="cuda") for _ in w.pattern]
        self.lse = [torch.empty((B, T, w.H), dtype=torch.float32, device="cuda") for _ in w.pattern]
        self.modes = [{"F": csa2.FULL, "R": csa2.REINDEX, "U": csa2.REUSE}[m] for m in w.pattern]

    def step(self, cache):
        for l, m in enumerate(self.modes):
            L = self.layers[l]
            idx = m != csa2.REUSE
            csa2.layer_step(cache, m, L["q"], self.topk, self.out[l], self.ws, self.w.window,
                            q_idx=L["q_idx"] if idx else None, head_w=L["w"] if idx else None, pool_idx=self.pool,
                            lse=self.lse[l], pool_k=self.w.pool_k)


def new_workspace(cache, w):
    ws = torch.empty(csa2.workspace_bytes(cache, w.T, w.H, w.pool_k, w.top_k, w.window), dtype=torch.uint8,
                     device="cuda")
    csa2.workspace_init(ws)
    return ws

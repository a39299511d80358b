"""GPU-side test helpers: fill a device cache through the library's own
append call from the seeded inputs, and run layer stacks through the C ABI."""
import numpy as np
import torch

import fp4_sparse_attention_csa2_b200 as csa2
from fp4_sparse_attention_csa2_b200 import workloads as wl
from harness import cache_geometry

APPEND_CHUNK = 1 << 16


def build_gpu_cache(w, seed=0, lens=None, q_idx0=None, upto=None):
    """Device cache whose positions [0, upto[b]) (default: all of L_b) are
    written through csa2_kv_append_quant from the seeded bf16 inputs."""
    lens = wl.seq_lens(w, seed) if lens is None else np.asarray(lens, dtype=np.int32)
    n_slots, table, stride = cache_geometry(w, lens, seed)
    cache = csa2.Cache(w.batch, n_slots, w.D, w.D_I, w.row_stride, w.idx_key_dtype, lens, table, w.page_size,
                       stride)
    if q_idx0 is None:
        q_idx0 = wl.layer_queries(w, 0, seed)["q_idx"]
    sp = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b in range(w.batch):
        L = int(lens[b])
        end = L if upto is None else int(upto[b])
        x = wl.latent(w, b, L, seed)
        keys, _ = wl.index_keys(w, b, L, q_idx0[b, w.T - 1], seed)
        v = cache.view(b)
        for t0 in range(0, end, APPEND_CHUNK):
            t1 = min(end, t0 + APPEND_CHUNK)
            sp.fill_(t0)
            csa2.kv_append_quant(v, x[t0:t1][None].cuda(), sp, keys[t0:t1][None].cuda())
        torch.cuda.synchronize()
    return cache


def device_layer(layer):
    return {k: v.cuda() for k, v in layer.items()}


def new_ws(cache, w):
    n = csa2.workspace_bytes(cache, w.T, w.H, w.pool_k, w.top_k, w.window)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    csa2.workspace_init(ws)
    return ws


def run_gpu_stack(cache, w, layers, ws=None):
    """Run w.pattern through csa2_layer_step; returns per layer (pool|None,
    topk, out, lse) as host numpy arrays, plus the final device status."""
    B, T = w.batch, w.T
    ws = new_ws(cache, w) if ws is None else ws
    pool = torch.full((B, T, w.pool_k), -7, dtype=torch.int32, device="cuda")
    topk = torch.full((B, T, w.top_k), -7, dtype=torch.int32, device="cuda")
    res = []
    for l, mode in enumerate(w.pattern):
        L = device_layer(layers[l])
        out = torch.empty((B, T, w.H, w.D), dtype=torch.float32, device="cuda")
        lse = torch.empty((B, T, w.H), dtype=torch.float32, device="cuda")
        m = {"F": csa2.FULL, "R": csa2.REINDEX, "U": csa2.REUSE}[mode]
        csa2.layer_step(cache, m, L["q"], topk, out, ws, w.window, q_idx=L["q_idx"] if mode != "U" else None,
                        head_w=L["w"] if mode != "U" else None, pool_idx=pool, lse=lse, pool_k=w.pool_k)
        res.append((pool.cpu().numpy().copy() if mode == "F" else None, topk.cpu().numpy().copy(),
                    out.cpu().numpy(), lse.cpu().numpy()))
    status = csa2.read_device_status(ws)
    return res, status


def attn_errors(got, want):
    d = np.abs(np.asarray(got, dtype=np.float64) - want)
    return float(d.max()), float(d.mean())


def build_gpu_shards(w, R, seed=0, lens=None, q_idx0=None):
    """The cache of every rank of an R-way context-parallel split: shard r of
    sequence b holds positions wl.shard_bounds(L_b, R)[r] of the seeded inputs
    (written through csa2_kv_append_quant into a contiguous cache of its own).
    Returns [(cache, pos0 int32 [B] on the device)] per rank."""
    lens = wl.seq_lens(w, seed) if lens is None else np.asarray(lens, dtype=np.int32)
    if q_idx0 is None:
        q_idx0 = wl.layer_queries(w, 0, seed)["q_idx"]
    bounds = [wl.shard_bounds(int(lens[b]), R) for b in range(w.batch)]
    xs = [wl.latent(w, b, int(lens[b]), seed) for b in range(w.batch)]
    ks = [wl.index_keys(w, b, int(lens[b]), q_idx0[b, w.T - 1], seed)[0] for b in range(w.batch)]
    shards = []
    sp = torch.zeros(1, dtype=torch.int32, device="cuda")
    for r in range(R):
        n = [bounds[b][r][1] for b in range(w.batch)]
        cap = max(64, (max(n) + 63) // 64 * 64)
        cache = csa2.Cache(w.batch, w.batch * cap, w.D, w.D_I, w.row_stride, w.idx_key_dtype, n, None, w.page_size,
                           cap)
        for b in range(w.batch):
            p0, nb = bounds[b][r]
            v = cache.view(b)
            for t0 in range(0, nb, APPEND_CHUNK):
                t1 = min(nb, t0 + APPEND_CHUNK)
                sp.fill_(t0)
                csa2.kv_append_quant(v, xs[b][p0 + t0:p0 + t1][None].cuda(), sp, ks[b][p0 + t0:p0 + t1][None].cuda())
        pos0 = torch.tensor([bounds[b][r][0] for b in range(w.batch)], dtype=torch.int32, device="cuda")
        shards.append((cache, pos0))
    torch.cuda.synchronize()
    return shards

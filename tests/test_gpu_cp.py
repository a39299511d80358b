"""Context-parallel decode on the GPU: the shard calls (csa2_cp_index_local,
csa2_cp_reindex_local, csa2_cp_sparse_swa_attn), the selections after the
exchange (csa2_cp_merge_select, csa2_cp_reindex_select) and the log-sum-exp
merge, with R ranks emulated one after another on one GPU (each rank's shard
is a cache of its own; the all-gathers become stacked buffers, the all-reduce
a sum).
The merged results are checked against the oracle run on the whole sequence
(tldrocket.com "DeepSeek AI Released DeepSeek-V4.1-Flash ...", paragraphs 1
and 3; zerohour.day: a context of one million tokens): the Full layer's pool
and top-k with the cutoff-band rule, the Reindex of the GPU's pool, and every
layer's out and lse against the oracle's attention over the GPU's top-k.  The
per-shard attention parts are checked against the oracle's attention over the
explicit set S ∩ shard, and the merge against the oracle's ref_lse_merge."""
import numpy as np
import pytest
import torch

import fp4_sparse_attention_csa2_b200 as csa2
import oracle
from fp4_sparse_attention_csa2_b200 import workloads as wl
from gpu_harness import attn_errors, build_gpu_shards, device_layer
from harness import attended_positions, build_ref_cache
from test_gpu_stack import MAX_ABS, MEAN_ABS, compare_stack

pytestmark = pytest.mark.gpu


def _shard_ws(w, shards):
    out = []
    for cache, _ in shards:
        ws = torch.empty(csa2.workspace_bytes(cache, 1, w.H, w.pool_k, w.top_k, w.window), dtype=torch.uint8,
                         device="cuda")
        csa2.workspace_init(ws)
        out.append(ws)
    return out


def run_cp_stack(w, shards, layers, lens):
    """w.pattern over R emulated ranks; per layer (pool|None, topk, out, lse)
    as host arrays shaped like run_gpu_stack's (T = 1), plus every status."""
    R, B = len(shards), w.batch
    glens = torch.as_tensor(np.asarray(lens, dtype=np.int32)).cuda()
    wss = _shard_ws(w, shards)
    mws = torch.empty(csa2.cp_merge_workspace_bytes(R, B, w.pool_k), dtype=torch.uint8, device="cuda")
    csa2.workspace_init(mws)
    pool = torch.full((B, w.pool_k), -7, dtype=torch.int32, device="cuda")
    topk = torch.full((B, w.top_k), -7, dtype=torch.int32, device="cuda")
    cand_pool = torch.empty((R, B, w.pool_k, 2), dtype=torch.int32, device="cuda")
    pool_scores = torch.empty((R, B, w.pool_k), dtype=torch.float32, device="cuda")
    res = []
    for l, mode in enumerate(w.pattern):
        L = device_layer(layers[l])
        if mode == "F":
            for r, (cache, pos0) in enumerate(shards):
                csa2.cp_index_local(cache, pos0, L["q_idx"], L["w"], w.pool_k, cand_pool[r], wss[r])
            csa2.cp_merge_select(cand_pool, glens, w.pool_k, pool, mws, n_b=w.top_k, out_b=topk)
        elif mode == "R":
            for r, (cache, pos0) in enumerate(shards):
                csa2.cp_reindex_local(cache, pos0, L["q_idx"], L["w"], pool, pool_scores[r], wss[r])
            # the all-reduce: each entry's owner adds its score, every other rank a zero
            summed = pool_scores.sum(dim=0).contiguous()
            csa2.cp_reindex_select(pool, summed, glens, w.top_k, topk)
        outs = torch.empty((R, B, w.H, w.D), dtype=torch.float32, device="cuda")
        lses = torch.empty((R, B, w.H), dtype=torch.float32, device="cuda")
        for r, (cache, pos0) in enumerate(shards):
            csa2.cp_sparse_swa_attn(cache, pos0, glens, L["q"], topk, w.window, outs[r], lses[r], wss[r])
        out = torch.empty((B, w.H, w.D), dtype=torch.float32, device="cuda")
        lse = torch.empty((B, w.H), dtype=torch.float32, device="cuda")
        csa2.lse_merge(outs, lses, out, lse)
        res.append((pool[:, None].cpu().numpy().copy() if mode == "F" else None, topk[:, None].cpu().numpy().copy(),
                    out[:, None].cpu().numpy(), lse[:, None].cpu().numpy()))
    status = [csa2.read_device_status(ws) for ws in wss] + [csa2.read_device_status(mws)]
    return res, status


@pytest.mark.parametrize("name,L,R,kw", [
    ("long64k", 20000, 2, {}),                                   # 20,000 merged candidates: the two-pass select
    ("long64k", 50000, 2, {}),                                   # shards over 16,384 positions: two-pass shard pools
    ("long64k", 50000, 3, {"pool_k": 4096, "top_k": 512}),       # 12,288 candidates: the one-CTA select
    ("tiny4k", 4096, 4, {}),                                     # fp32 keys (CUDA-core scoring), 16 x 128 heads
    ("batch32_paged", 30000, 2, {"batch": 3}),                   # ragged sequences, each split over the ranks
    ("ctx1m", 40000, 8, {}),                                     # eight ranks, the ctx1m stack
])
def test_cp_stack_matches_oracle(name, L, R, kw):
    w = wl.scaled(wl.WORKLOADS[name], L, T=1, **kw)
    layers = [wl.layer_queries(w, l) for l in range(len(w.pattern))]
    lens = wl.seq_lens(w)
    ref = build_ref_cache(w, layers=layers)
    shards = build_gpu_shards(w, R, q_idx0=layers[0]["q_idx"])
    got, status = run_cp_stack(w, shards, layers, lens)
    assert all(s == csa2.OK for s in status), status
    compare_stack(w, ref, got, layers, [(b, 0) for b in range(w.batch)])


def test_cp_full_size_ctx1m_eight_ranks():
    # the 1,048,576-position sequence over 8 ranks of 131,072 positions
    w = wl.WORKLOADS["ctx1m"]
    layers = [wl.layer_queries(w, l) for l in range(3)]
    w3 = wl.Workload(**{**w.__dict__, "pattern": "FRU"})
    lens = wl.seq_lens(w)
    shards = build_gpu_shards(w, 8, q_idx0=layers[0]["q_idx"])
    got, status = run_cp_stack(w3, shards, layers, lens)
    del shards
    assert all(s == csa2.OK for s in status), status
    ref = build_ref_cache(w, rows=False, layers=layers)
    lat = wl.latent(w, 0, int(lens[0]))
    n_band = compare_stack(w3, ref, got, layers, [(0, 0)], lambda b: lat)
    print("ctx1m over 8 ranks: %d index differences inside the cutoff band" % n_band)


@pytest.mark.parametrize("H", [64, 48])
def test_cp_parts_are_attention_over_each_shards_share(H):
    # each rank's (out, lse) is the attention over S ∩ shard: the oracle's
    # attention over that explicit set (no window of its own); 64 heads run the
    # tensor-core kernel with the shard mapping inside it, 48 heads the
    # CUDA-core kernel over the shard's list
    w = wl.scaled(wl.WORKLOADS["long64k"], 9000, T=1, H=H)
    R = 3
    lens = wl.seq_lens(w)
    l0 = wl.layer_queries(w, 0)
    ref = build_ref_cache(w, layers=[l0])
    shards = build_gpu_shards(w, R, q_idx0=l0["q_idx"])
    p = int(lens[0]) - 1
    rng = np.random.default_rng(7)
    topk = rng.choice(p + 1, w.top_k, replace=False).astype(np.int32)
    topk[:50] = -1                                              # padding
    topk[50:60] = np.arange(p - 9, p + 1)                       # inside the window: counted once
    glens = torch.as_tensor(lens).cuda()
    q = l0["q"].cuda()
    S = attended_positions(topk, p, w.window)
    bounds = wl.shard_bounds(int(lens[0]), R)
    wss = _shard_ws(w, shards)
    for r, (cache, pos0) in enumerate(shards):
        out = torch.empty((1, w.H, w.D), dtype=torch.float32, device="cuda")
        lse = torch.empty((1, w.H), dtype=torch.float32, device="cuda")
        csa2.cp_sparse_swa_attn(cache, pos0, glens, q, torch.from_numpy(topk[None]).cuda(), w.window, out, lse, wss[r])
        assert csa2.read_device_status(wss[r]) == csa2.OK
        lo, n = bounds[r]
        part = np.array(sorted(t for t in S if lo <= t < lo + n), dtype=np.int32)
        assert part.size > 0
        ro, rl = oracle.sparse_swa_attn(ref, 0, 1, 0, wl.bf16_bits(l0["q"])[0, 0], part, 0)
        mx, mean = attn_errors(out.cpu().numpy()[0], ro)
        assert mx <= MAX_ABS and mean <= MEAN_ABS, (r, mx, mean)
        lmx, _ = attn_errors(lse.cpu().numpy()[0], rl)
        assert lmx <= MAX_ABS, (r, lmx)


def test_cp_empty_parts_and_bad_topk_entries():
    # no top-k entries: every rank but the last holds nothing of S (out 0,
    # lse -inf) and the merge is the window alone; an entry beyond the global
    # length is flagged and skipped
    w = wl.scaled(wl.WORKLOADS["long64k"], 6000, T=1)
    lens = wl.seq_lens(w)
    l0 = wl.layer_queries(w, 0)
    ref = build_ref_cache(w, layers=[l0])
    shards = build_gpu_shards(w, 3, q_idx0=l0["q_idx"])
    glens = torch.as_tensor(lens).cuda()
    topk = torch.full((1, w.top_k), -1, dtype=torch.int32, device="cuda")
    topk[0, 3] = int(lens[0]) + 5
    wss = _shard_ws(w, shards)
    outs = torch.empty((3, 1, w.H, w.D), dtype=torch.float32, device="cuda")
    lses = torch.empty((3, 1, w.H), dtype=torch.float32, device="cuda")
    for r, (cache, pos0) in enumerate(shards):
        csa2.cp_sparse_swa_attn(cache, pos0, glens, l0["q"].cuda(), topk, w.window, outs[r], lses[r], wss[r])
    assert [csa2.read_device_status(ws) for ws in wss] == [csa2.ERR_DEVICE_BOUNDS] * 3
    for r in range(2):
        assert torch.all(outs[r] == 0) and torch.all(torch.isneginf(lses[r]))
    out = torch.empty((1, w.H, w.D), dtype=torch.float32, device="cuda")
    lse = torch.empty((1, w.H), dtype=torch.float32, device="cuda")
    csa2.lse_merge(outs, lses, out, lse)
    ro, rl = oracle.sparse_swa_attn(ref, 0, 1, 0, wl.bf16_bits(l0["q"])[0, 0], np.full(1, -1, np.int32), w.window)
    mx, mean = attn_errors(out.cpu().numpy()[0], ro)
    assert mx <= MAX_ABS and mean <= MEAN_ABS
    assert attn_errors(lse.cpu().numpy()[0], rl)[0] <= MAX_ABS


@pytest.mark.parametrize("R,B,H,D", [(1, 1, 16, 128), (3, 2, 64, 512), (8, 1, 64, 512), (5, 4, 32, 96)])
def test_lse_merge_matches_oracle(R, B, H, D):
    g = torch.Generator().manual_seed(R * 100 + B)
    outs = torch.randn((R, B, H, D), generator=g, dtype=torch.float32)
    lses = torch.randn((R, B, H), generator=g, dtype=torch.float32) * 8
    if R > 1:
        lses[0, 0, :4] = -float("inf")                          # empty parts
    lses[:, -1, H - 1] = -float("inf")                          # a head whose every part is empty
    # both in one buffer per rank, as an all-gather leaves them
    buf = torch.cat([outs.reshape(R, -1), lses.reshape(R, -1)], dim=1).cuda()
    o_view = buf[:, :B * H * D].view(R, B, H, D)
    l_view = buf[:, B * H * D:].view(R, B, H)
    out = torch.empty((B, H, D), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    csa2.lse_merge(o_view, l_view, out, lse)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for b in range(B):
        ro, rl = oracle.lse_merge(outs[:, b].numpy(), lses[:, b].numpy())
        if b == B - 1:
            assert np.all(out[b, H - 1] == 0) and np.isneginf(lse[b, H - 1])
        fin = np.isfinite(rl)
        assert np.array_equal(np.isneginf(lse[b]), np.isneginf(rl))
        assert np.max(np.abs(lse[b][fin] - rl[fin])) <= 1e-5 * max(1.0, np.max(np.abs(rl[fin])))
        assert np.max(np.abs(out[b] - ro)) <= 2e-6 * max(1.0, np.max(np.abs(ro)))


def test_stack_class_on_one_rank():
    # ContextParallelStack over a one-rank NCCL group: the library's shard
    # calls through the class, every exchange an all-gather of one part
    import torch.distributed as dist
    from fp4_sparse_attention_csa2_b200.cp import ContextParallelStack
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0, world_size=1)
    try:
        w = wl.scaled(wl.WORKLOADS["long64k"], 12000, T=1)
        layers = [wl.layer_queries(w, l) for l in range(len(w.pattern))]
        lens = wl.seq_lens(w)
        ref = build_ref_cache(w, layers=layers)
        (cache, pos0), = build_gpu_shards(w, 1, q_idx0=layers[0]["q_idx"])
        st = ContextParallelStack(cache, pos0, torch.as_tensor(lens).cuda(), w.H, w.pool_k, w.top_k, w.window)
        pool = torch.full((1, w.pool_k), -7, dtype=torch.int32, device="cuda")
        topk = torch.full((1, w.top_k), -7, dtype=torch.int32, device="cuda")
        got = []
        for l, mode in enumerate(w.pattern):
            L = device_layer(layers[l])
            out = torch.empty((1, w.H, w.D), dtype=torch.float32, device="cuda")
            lse = torch.empty((1, w.H), dtype=torch.float32, device="cuda")
            m = {"F": csa2.FULL, "R": csa2.REINDEX, "U": csa2.REUSE}[mode]
            st.layer(m, L["q"], topk, out, lse, q_idx=L["q_idx"], head_w=L["w"], pool=pool)
            got.append((pool[:, None].cpu().numpy().copy() if mode == "F" else None,
                        topk[:, None].cpu().numpy().copy(), out[:, None].cpu().numpy(), lse[:, None].cpu().numpy()))
        assert csa2.read_device_status(st.ws) == csa2.OK
        compare_stack(w, ref, got, layers, [(0, 0)])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,L,R,kw", [
    ("long64k", 50000, 3, {}),                                   # contiguous cache
    ("batch32_paged", 40000, 2, {"batch": 1, "lens": ("fixed", 40000)}),   # paged cache, page-aligned shards
])
def test_cp_on_shard_views_of_one_cache(name, L, R, kw):
    # the shards as views of one cache (Cache.shard_view): the same results
    # as the oracle on the whole sequence
    from gpu_harness import build_gpu_cache
    w = wl.scaled(wl.WORKLOADS[name], L, T=1, **kw)
    layers = [wl.layer_queries(w, l) for l in range(len(w.pattern))]
    lens = wl.seq_lens(w)
    ref = build_ref_cache(w, layers=layers)
    dev = build_gpu_cache(w, q_idx0=layers[0]["q_idx"])
    step = (L + R - 1) // R // 64 * 64 + 64
    shards = []
    for r in range(R):
        p0 = min(r * step, L)
        v = dev.shard_view(0, p0, min(step, L - p0))
        shards.append((v, torch.tensor([p0], dtype=torch.int32, device="cuda")))
    got, status = run_cp_stack(w, shards, layers, lens)
    assert all(s == csa2.OK for s in status), status
    compare_stack(w, ref, got, layers, [(0, 0)])

"""Indexer parity: Full-layer pool / top-k sets and Reindex top-k sets from the
CUDA path against the oracle, exact outside the 1e-5 relative band around the
cutoff score (tldrocket.com "DeepSeek AI Released DeepSeek-V4.1-Flash ...",
paragraph 3; hackernews.kjhq.dev post 49735410, key points 2-3)."""
import numpy as np
import pytest
import torch

import fp4_sparse_attention_csa2_b200 as csa2
import oracle
from fp4_sparse_attention_csa2_b200 import workloads as wl
from gpu_harness import build_gpu_cache, device_layer, new_ws
from harness import band_set_check, build_ref_cache, host_layer

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny4k", 4096, {}),
    ("tiny4k", 333, {}),                        # L < pool: -1 padding
    ("long64k", 20000, {}),
    ("long64k", 5000, {"T": 3}),                # causal among 3 query tokens
    ("batch32_paged", 30000, {"batch": 5}),     # paged, ragged lengths
    ("append_mq", 9000, {"batch": 2}),          # T = 4
    ("tiny4k", 512, {}),                        # L = K: the pool is every position
    ("long64k", 16384, {}),                     # L = K = 16,384, the largest pool
    ("long64k", 16385, {}),                     # one position more than the largest pool
    ("long64k", 20000, {"pool_k": 2048}),       # k = K: both targets cut at the same place
    ("long64k", 20000, {"pool_k": 64, "top_k": 1}),   # k = 1
]


def _run_full(w, layer, cache, ws):
    L = device_layer(layer)
    pool = torch.full((w.batch, w.T, w.pool_k), -7, dtype=torch.int32, device="cuda")
    topk = torch.full((w.batch, w.T, w.top_k), -7, dtype=torch.int32, device="cuda")
    csa2.index_full(cache, L["q_idx"], L["w"], w.pool_k, w.top_k, pool, topk, ws)
    return pool.cpu().numpy(), topk.cpu().numpy()


@pytest.mark.parametrize("name,L,kw", CASES)
def test_full_pool_and_topk_sets(name, L, kw):
    w = wl.scaled(wl.WORKLOADS[name], L, **kw)
    layer = wl.layer_queries(w, 0)
    ref = build_ref_cache(w, rows=False, layers=[layer])
    dev = build_gpu_cache(w, q_idx0=layer["q_idx"])
    ws = new_ws(dev, w)
    pool, topk = _run_full(w, layer, dev, ws)
    assert csa2.read_device_status(ws) == csa2.OK
    hl = host_layer(layer)
    for b in range(w.batch):
        for j in range(w.T):
            rp, rt, s = oracle.index_full(ref, b, w.T, j, hl["q_idx"][b, j], w.q_idx_dtype, hl["w"][b, j],
                                          w.pool_k, w.top_k, want_scores=True)
            band_set_check(pool[b, j], rp, lambda t: s[t], s.size)
            band_set_check(topk[b, j], rt, lambda t: s[t], s.size)
            # k is a subset of K on the device too
            assert set(topk[b, j][topk[b, j] >= 0]) <= set(pool[b, j][pool[b, j] >= 0])


@pytest.mark.parametrize("name,L,kw", CASES)
def test_reindex_sets_on_oracle_pool(name, L, kw):
    w = wl.scaled(wl.WORKLOADS[name], L, **kw)
    l0, l1 = wl.layer_queries(w, 0), wl.layer_queries(w, 1)
    ref = build_ref_cache(w, rows=False, layers=[l0])
    dev = build_gpu_cache(w, q_idx0=l0["q_idx"])
    ws = new_ws(dev, w)
    h0, h1 = host_layer(l0), host_layer(l1)
    pools = np.zeros((w.batch, w.T, w.pool_k), dtype=np.int32)
    for b in range(w.batch):
        for j in range(w.T):
            pools[b, j], _, _ = oracle.index_full(ref, b, w.T, j, h0["q_idx"][b, j], w.q_idx_dtype, h0["w"][b, j],
                                                  w.pool_k, w.top_k)
    # shuffle the pool order: the device must not rely on it
    rng = np.random.default_rng(3)
    for b in range(w.batch):
        for j in range(w.T):
            pools[b, j] = rng.permutation(pools[b, j])
    D1 = device_layer(l1)
    topk = torch.full((w.batch, w.T, w.top_k), -7, dtype=torch.int32, device="cuda")
    pool_d = torch.from_numpy(pools).cuda()
    csa2.index_reindex(dev, D1["q_idx"], D1["w"], pool_d, w.top_k, topk, ws)
    topk = topk.cpu().numpy()
    assert csa2.read_device_status(ws) == csa2.OK
    assert np.array_equal(pool_d.cpu().numpy(), pools)          # the pool is only read
    for b in range(w.batch):
        for j in range(w.T):
            rt, s = oracle.index_reindex(ref, b, w.T, j, h1["q_idx"][b, j], w.q_idx_dtype, h1["w"][b, j],
                                         pools[b, j], w.top_k, want_scores=True)
            by_pos = {int(t): float(v) for t, v in zip(pools[b, j], s) if t >= 0}
            band_set_check(topk[b, j], rt, lambda t: by_pos[t], len(by_pos))


def test_all_equal_scores_select_exactly_k():
    # every key is zero: all scores tie at 0, any min(K, p+1) distinct positions are right
    w = wl.scaled(wl.WORKLOADS["long64k"], 40000)
    cache = csa2.Cache(1, 40000 // 64 * 64 + 64, w.D, 64, w.row_stride, csa2.E4M3, [40000],
                       seq_stride_slots=40000 // 64 * 64 + 64)
    ws = new_ws(cache, w)
    pool, topk = _run_full(w, wl.layer_queries(w, 0), cache, ws)
    for arr, k in ((pool, w.pool_k), (topk, w.top_k)):
        v = arr[0, 0]
        assert np.all(v[:k] >= 0) and np.unique(v).size == k and v.max() < 40000
    # the top-k is a subset of the pool even when both cut inside one group of ties
    assert set(topk[0, 0]) <= set(pool[0, 0])


@pytest.mark.parametrize("pattern", ["thirds", "two_thirds_top"])
def test_tied_score_groups_give_nested_sets(pattern):
    # 40,000 positions whose index keys take three values k0, ~k0 / 2 and 0, so
    # the scores take three values s0 > s1 > 0 (equal keys give bit-identical
    # scores); every cutoff falls inside a group of equal scores.  "thirds": the pool takes group 0 whole and part of group 1,
    # the top-k part of group 0.  "two_thirds_top": group 0 alone is larger
    # than the pool, so both cut inside the same group of ties.
    L = 40000
    w = wl.scaled(wl.WORKLOADS["long64k"], L)
    slots = (L + 63) // 64 * 64
    cache = csa2.Cache(1, slots, w.D, 64, w.row_stride, csa2.E4M3, [L], seq_stride_slots=slots)
    layer = wl.layer_queries(w, 0)
    q = layer["q_idx"][0, 0].float()                       # [H_I, 64]
    k0 = q.sum(0)
    k0 = (k0 / k0.abs().max() * 8).to(torch.bfloat16)     # largest entry 8, inside the E4M3 range
    keys = torch.zeros((L, 64), dtype=torch.bfloat16)
    t = torch.arange(L)
    g = (t % 3) if pattern == "thirds" else torch.where(t % 3 == 2, 2, 0)
    keys[g == 0] = k0
    keys[g == 1] = (k0.float() / 2).to(torch.bfloat16)
    x = torch.zeros((1, L, w.D), dtype=torch.bfloat16, device="cuda")
    sp = torch.zeros(1, dtype=torch.int32, device="cuda")
    csa2.kv_append_quant(cache, x, sp, keys[None].cuda())
    ws = new_ws(cache, w)
    pool, topk = _run_full(w, layer, cache, ws)
    assert csa2.read_device_status(ws) == csa2.OK
    # k0 is along the sum of the indexer queries, so its dot products sum to a
    # positive number: group 0 scores above group 2 (score 0)
    s0 = float((layer["w"][0, 0].float() * torch.relu(q @ k0.float())).sum())
    assert s0 > 0
    gp, gt = g.numpy()[pool[0, 0]], g.numpy()[topk[0, 0]]
    n0 = int((g == 0).sum())
    assert np.unique(pool[0, 0]).size == w.pool_k and np.unique(topk[0, 0]).size == w.top_k
    assert set(topk[0, 0]) <= set(pool[0, 0])
    assert np.all(gt == 0)
    if n0 <= w.pool_k:
        assert np.sum(gp == 0) == n0 and np.all(gp[gp != 0] == 1)
    else:
        assert np.all(gp == 0)


def test_reuse_touches_no_index_buffer():
    w = wl.scaled(wl.WORKLOADS["long64k"], 6000)
    dev = build_gpu_cache(w)
    ws = new_ws(dev, w)
    rng = np.random.default_rng(0)
    topk = torch.from_numpy(rng.choice(6000, (1, 1, w.top_k), replace=False).astype(np.int32)).cuda()
    pool = torch.full((1, 1, w.pool_k), 12345, dtype=torch.int32, device="cuda")
    before = (topk.clone(), pool.clone())
    q = wl.layer_queries(w, 3)["q"].cuda()
    out = torch.empty((1, 1, w.H, w.D), dtype=torch.float32, device="cuda")
    csa2.layer_step(dev, csa2.REUSE, q, topk, out, ws, w.window, pool_idx=pool)
    torch.cuda.synchronize()
    assert torch.equal(topk, before[0]) and torch.equal(pool, before[1])


def test_out_of_range_pool_entry_flags_status():
    w = wl.scaled(wl.WORKLOADS["long64k"], 3000)
    dev = build_gpu_cache(w)
    ws = new_ws(dev, w)
    l1 = device_layer(wl.layer_queries(w, 1))
    pool = torch.arange(w.pool_k, dtype=torch.int32, device="cuda").view(1, 1, -1) % 3000
    pool[0, 0, 5] = 3000                        # beyond p
    pool[0, 0, 6] = -1
    topk = torch.empty((1, 1, w.top_k), dtype=torch.int32, device="cuda")
    csa2.index_reindex(dev, l1["q_idx"], l1["w"], pool, w.top_k, topk, ws)
    assert csa2.read_device_status(ws) == csa2.ERR_DEVICE_BOUNDS
    assert 3000 not in topk.cpu().numpy()

"""Pins of the oracle's indexer (Full / Reindex / Reuse selection) against
library routines and the bounds the pages print: the candidate pool holds at
most 16,384 positions and Reuse layers take the indices unchanged
(tldrocket.com "DeepSeek AI Released DeepSeek-V4.1-Flash ...", paragraph 3;
hackernews.kjhq.dev post 49735410, key point 2)."""
import numpy as np
import pytest
import torch

import oracle
from fp4_sparse_attention_csa2_b200 import workloads as wl
from harness import band_set_check, build_ref_cache, host_layer


def _small(name, L, **kw):
    return wl.scaled(wl.WORKLOADS[name], L, **kw)


def _keys_f64(cache, b, n):
    """Stored index keys of positions 0..n-1 decoded by the library (torch fp8)."""
    slots = np.array([cache.slot(b, t) for t in range(n)])
    k = cache.idx_keys[slots]
    if cache.idx_key_dtype == oracle.E4M3:
        return torch.from_numpy(k.copy()).view(torch.float8_e4m3fn).double().numpy()
    return k.astype(np.float64)


def _q_f64(q):
    return q.double().numpy() if isinstance(q, torch.Tensor) else np.asarray(q, dtype=np.float64)


@pytest.mark.parametrize("name,L", [("tiny4k", 1000), ("long64k", 3000)])
def test_scores_equal_numpy_gemm_relu_weighted_sum(name, L):
    w = _small(name, L)
    cache = build_ref_cache(w, rows=False)
    lay = wl.layer_queries(w, 0)
    qi, hw = lay["q_idx"][0, 0], lay["w"][0, 0]
    pos = np.arange(L, dtype=np.int32)
    s = oracle.index_scores(cache, 0, pos, wl.host_array(qi), w.q_idx_dtype, hw.numpy())
    K = _keys_f64(cache, 0, L)
    want = np.maximum(K @ _q_f64(qi).T, 0.0) @ hw.double().numpy()   # BLAS GEMM
    assert np.allclose(s, want, rtol=1e-12, atol=1e-12)


def test_single_head_positive_dot_is_plain_dot():
    w = _small("tiny4k", 300, H_I=1)
    cache = build_ref_cache(w, rows=False)
    q = torch.randn(1, 64, generator=torch.Generator().manual_seed(5))
    K = _keys_f64(cache, 0, 300)
    pos = np.arange(300, dtype=np.int32)
    s = oracle.index_scores(cache, 0, pos, q.numpy(), oracle.F32, np.ones(1, np.float32))
    dots = K @ q.double().numpy()[0]
    assert np.allclose(s[dots > 0], dots[dots > 0], rtol=1e-13, atol=0)
    assert np.all(s[dots <= 0] == 0)


def test_select_top_equals_full_sort():
    rng = np.random.default_rng(0)
    for n, k in [(10, 3), (1000, 128), (5000, 5000), (50, 80)]:
        s = rng.standard_normal(n)
        s[rng.integers(0, n, n // 5)] = 0.5          # plenty of exact ties
        got = oracle.select_top(s, None, k)
        order = np.lexsort((np.arange(n), -s))       # score desc, position asc
        want = np.full(k, -1, dtype=np.int32)
        want[:min(k, n)] = order[:k]
        assert np.array_equal(got, want)


@pytest.mark.parametrize("T", [1, 3])
def test_full_pool_and_topk_bounds(T):
    w = _small("tiny4k", 2000, T=T)
    cache = build_ref_cache(w, rows=False)
    lay = wl.layer_queries(w, 0)
    for j in range(T):
        p = 2000 - T + j
        pool, topk, s = oracle.index_full(cache, 0, T, j, wl.host_array(lay["q_idx"][0, j]), w.q_idx_dtype,
                                          lay["w"][0, j].numpy(), w.pool_k, w.top_k, want_scores=True)
        assert s.size == p + 1                                 # causal: t <= p_j only
        assert np.sum(pool >= 0) == min(w.pool_k, p + 1)
        assert np.sum(topk >= 0) == min(w.top_k, p + 1)
        assert set(topk[topk >= 0]) <= set(pool[pool >= 0])   # k is a subset of K
        assert pool.max() <= p
        order = np.lexsort((np.arange(p + 1), -s))
        assert np.array_equal(pool, order[:w.pool_k])


def test_pool_shorter_than_k_is_padded():
    w = _small("tiny4k", 100)
    cache = build_ref_cache(w, rows=False)
    lay = wl.layer_queries(w, 0)
    pool, topk, _ = oracle.index_full(cache, 0, 1, 0, wl.host_array(lay["q_idx"][0, 0]), w.q_idx_dtype,
                                      lay["w"][0, 0].numpy(), 512, 128)
    assert np.sum(pool >= 0) == 100 and np.all(pool[100:] == -1)
    assert np.sum(topk >= 0) == 100


def test_pool_bound_16384():
    w = _small("tiny4k", 100)
    cache = build_ref_cache(w, rows=False)
    lay = wl.layer_queries(w, 0)
    with pytest.raises(RuntimeError):
        oracle.index_full(cache, 0, 1, 0, wl.host_array(lay["q_idx"][0, 0]), w.q_idx_dtype,
                          lay["w"][0, 0].numpy(), 16385, 128)
    with pytest.raises(RuntimeError):
        oracle.index_full(cache, 0, 1, 0, wl.host_array(lay["q_idx"][0, 0]), w.q_idx_dtype,
                          lay["w"][0, 0].numpy(), 64, 128)


def test_reindex_with_whole_context_pool_equals_full_selection():
    # pool = every position (L <= K): Reindex == Full selection with the Reindex query
    w = _small("long64k", 1500)
    cache = build_ref_cache(w, rows=False)
    l0, l1 = wl.layer_queries(w, 0), wl.layer_queries(w, 1)
    pool, _, _ = oracle.index_full(cache, 0, 1, 0, wl.host_array(l0["q_idx"][0, 0]), w.q_idx_dtype,
                                   l0["w"][0, 0].numpy(), w.pool_k, w.top_k)
    assert np.sum(pool >= 0) == 1500
    re_topk, _ = oracle.index_reindex(cache, 0, 1, 0, wl.host_array(l1["q_idx"][0, 0]), w.q_idx_dtype,
                                      l1["w"][0, 0].numpy(), pool, w.top_k)
    _, full_topk, _ = oracle.index_full(cache, 0, 1, 0, wl.host_array(l1["q_idx"][0, 0]), w.q_idx_dtype,
                                        l1["w"][0, 0].numpy(), w.pool_k, w.top_k)
    assert np.array_equal(re_topk, full_topk)


def test_reindex_scores_only_the_pool():
    w = _small("tiny4k", 3000)
    cache = build_ref_cache(w, rows=False)
    l0, l1 = wl.layer_queries(w, 0), wl.layer_queries(w, 1)
    pool, _, _ = oracle.index_full(cache, 0, 1, 0, wl.host_array(l0["q_idx"][0, 0]), w.q_idx_dtype,
                                   l0["w"][0, 0].numpy(), w.pool_k, w.top_k)
    topk, s = oracle.index_reindex(cache, 0, 1, 0, wl.host_array(l1["q_idx"][0, 0]), w.q_idx_dtype,
                                   l1["w"][0, 0].numpy(), pool, w.top_k, want_scores=True)
    assert set(topk) <= set(pool)
    order = np.lexsort((pool, -s))
    assert np.array_equal(topk, pool[order[:w.top_k]])


def test_planted_keys_are_selected():
    # the planted positions (cosine 0.9 with the query direction) score far
    # above the N(0,1) background, so every one of them lands in the top-k
    w = _small("long64k", 8192)
    cache = build_ref_cache(w, rows=False)
    l0 = wl.layer_queries(w, 0)
    _, planted = wl.index_keys(w, 0, 8192, l0["q_idx"][0, 0])
    _, topk, _ = oracle.index_full(cache, 0, 1, 0, wl.host_array(l0["q_idx"][0, 0]), w.q_idx_dtype,
                                   l0["w"][0, 0].numpy(), w.pool_k, w.top_k)
    assert set(planted.tolist()) <= set(topk.tolist())


def test_reuse_passes_indices_through_unchanged():
    w = _small("tiny4k", 1200)
    cache = build_ref_cache(w)
    layers = [host_layer(wl.layer_queries(w, l)) for l in range(3)]
    res = oracle.run_stack(cache, "FRU", layers, 1, w.pool_k, w.top_k, w.window, w.q_idx_dtype)
    assert np.array_equal(res[1][(0, 0)][1], res[2][(0, 0)][1])
    assert res[1][(0, 0)][1].tobytes() == res[2][(0, 0)][1].tobytes()


def test_cache_stores_index_keys_as_e4m3_of_the_input():
    # the oracle cache's index keys equal torch's round-to-nearest-even
    # float8_e4m3fn conversion of the bf16 key inputs (an encoder other than
    # the oracle's own; the inputs stay far inside the E4M3 range)
    w = wl.scaled(wl.WORKLOADS["long64k"], 3000)
    layers = [wl.layer_queries(w, 0)]
    cache = build_ref_cache(w, rows=False, layers=layers)
    keys, _ = wl.index_keys(w, 0, 3000, layers[0]["q_idx"][0, w.T - 1])
    assert keys.dtype == torch.bfloat16 and float(keys.float().abs().max()) < 448
    want = keys.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    slots = [cache.slot(0, t) for t in range(3000)]
    assert np.array_equal(cache.idx_keys[slots], want)


# ------------------------------------------------------------------ append-time pool maintenance
# (the Full layer's candidate pool of tldrocket.com "DeepSeek AI Released
# DeepSeek-V4.1-Flash ...", paragraph 3, kept current for an in-flight request)

def _pool_case(L0, L, pool_k=1024, top_k=128):
    w = wl.scaled(wl.WORKLOADS["long64k"], L, pool_k=pool_k, top_k=top_k)
    layer = wl.layer_queries(w, 0)
    cache = build_ref_cache(w, rows=False, layers=[layer])
    h = host_layer(layer)
    return w, cache, h["q_idx"][0, 0], h["w"][0, 0]


def test_pool_update_equals_full_selection_over_the_longer_context():
    # top-K(S ∪ N) = top-K(top-K(S) ∪ N): updating the pool of the first L0
    # positions with the appended ones equals selecting over all L
    L0, L = 5000, 6000
    w, cache, q, hw = _pool_case(L0, L)
    cache.set_seq_lens([L0])
    prev, _, _ = oracle.index_full(cache, 0, 1, 0, q, w.q_idx_dtype, hw, w.pool_k, w.top_k)
    cache.set_seq_lens([L])
    pool, topk = oracle.index_pool_update(cache, 0, 1, 0, q, w.q_idx_dtype, hw, prev, L0, w.top_k)
    fp, ft, s = oracle.index_full(cache, 0, 1, 0, q, w.q_idx_dtype, hw, w.pool_k, w.top_k, want_scores=True)
    band_set_check(pool, fp, lambda t: s[t], s.size)
    band_set_check(topk, ft, lambda t: s[t], s.size)
    assert set(topk[topk >= 0]) <= set(pool[pool >= 0])


def test_pool_update_without_new_positions_keeps_the_pool():
    w, cache, q, hw = _pool_case(3000, 3000)
    prev, _, _ = oracle.index_full(cache, 0, 1, 0, q, w.q_idx_dtype, hw, w.pool_k, w.top_k)
    pool, _ = oracle.index_pool_update(cache, 0, 1, 0, q, w.q_idx_dtype, hw, prev, 3000, w.top_k)
    assert set(pool.tolist()) == set(prev.tolist())


def test_pool_update_from_an_empty_pool_is_the_full_selection():
    w, cache, q, hw = _pool_case(0, 2500)
    empty = np.full(w.pool_k, -1, dtype=np.int32)
    pool, topk = oracle.index_pool_update(cache, 0, 1, 0, q, w.q_idx_dtype, hw, empty, 0, w.top_k)
    fp, ft, s = oracle.index_full(cache, 0, 1, 0, q, w.q_idx_dtype, hw, w.pool_k, w.top_k, want_scores=True)
    band_set_check(pool, fp, lambda t: s[t], s.size)
    band_set_check(topk, ft, lambda t: s[t], s.size)


def test_pool_update_rejects_previous_entries_among_the_new_positions():
    w, cache, q, hw = _pool_case(0, 2000)
    prev = np.full(w.pool_k, -1, dtype=np.int32)
    prev[0] = 1500
    with pytest.raises(RuntimeError):
        oracle.index_pool_update(cache, 0, 1, 0, q, w.q_idx_dtype, hw, prev, 1200, w.top_k)


def test_pool_update_below_the_pool_size_keeps_every_position():
    # fewer candidates than pool_k: the pool is every position 0..p, the
    # newest one included
    w, cache, q, hw = _pool_case(0, 900)
    prev = np.full(w.pool_k, -1, dtype=np.int32)
    prev[:600] = np.arange(600)
    pool, topk = oracle.index_pool_update(cache, 0, 1, 0, q, w.q_idx_dtype, hw, prev, 600, w.top_k)
    assert set(pool[pool >= 0].tolist()) == set(range(900)) and np.all(pool[900:] == -1)
    assert np.sum(topk >= 0) == w.top_k


def test_top_k_of_shard_top_ks_is_the_global_top_k():
    # a context sharded over devices selects globally from the union of the
    # shards' local selections: top-K(∪ S_g) = top-K(∪ top-K(S_g))
    w = wl.scaled(wl.WORKLOADS["long64k"], 9000, pool_k=1024, top_k=128)
    layer = wl.layer_queries(w, 0)
    cache = build_ref_cache(w, rows=False, layers=[layer])
    h = host_layer(layer)
    fp, _, s = oracle.index_full(cache, 0, 1, 0, h["q_idx"][0, 0], w.q_idx_dtype, h["w"][0, 0], w.pool_k, w.top_k,
                                 want_scores=True)
    for G in (2, 4, 7):
        bounds = np.linspace(0, 9000, G + 1).astype(np.int64)
        cand = []
        for g in range(G):
            pos = np.arange(bounds[g], bounds[g + 1], dtype=np.int32)
            loc = oracle.select_top(s[pos], pos, w.pool_k)
            cand.append(loc[loc >= 0])
        cand = np.concatenate(cand)
        glob = oracle.select_top(s[cand], cand, w.pool_k)
        band_set_check(glob, fp, lambda t: s[t], s.size)


def test_token_j_of_T_equals_a_single_token_at_its_own_length():
    # causal multi-token decode / prefill: token j of T sees exactly what a
    # lone query token sees when the sequence ends at p_j = L - T + j
    T, L = 5, 3000
    w = wl.scaled(wl.WORKLOADS["long64k"], L, T=T, pool_k=512, top_k=64)
    layer = wl.layer_queries(w, 0)
    cache = build_ref_cache(w, rows=False, layers=[layer])
    h = host_layer(layer)
    for j in range(T):
        cache.set_seq_lens([L])
        pool, topk, _ = oracle.index_full(cache, 0, T, j, h["q_idx"][0, j], w.q_idx_dtype, h["w"][0, j],
                                          w.pool_k, w.top_k)
        cache.set_seq_lens([L - T + j + 1])
        pool1, topk1, _ = oracle.index_full(cache, 0, 1, 0, h["q_idx"][0, j], w.q_idx_dtype, h["w"][0, j],
                                            w.pool_k, w.top_k)
        assert np.array_equal(pool, pool1) and np.array_equal(topk, topk1), j

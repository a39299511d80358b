"""The workspace-free Reindex entry point.

Some callers cannot hand the library a workspace: code that runs while a
framework captures a CUDA graph under a no-allocation policy, plugins that are
given tensors but no allocator, real-time paths that cannot pay for
cudaMalloc's implicit synchronisation.  For them, csa2_index_reindex_noalloc
keeps its scratch in a fixed array inside the library.  These tests call it
through the C ABI twice in a row (the second call finds the first call's
scores in the shared array) and check each result against the CPU oracle's
Reindex of the same pool (the index-set rule of every other index test:
exact outside the 1e-5 band around the cutoff score) and against the
workspace-based csa2_index_reindex on the same inputs.  They build all of
their inputs, so they pass alone in a fresh process and after the rest of the
suite.
"""
import numpy as np
import pytest
import torch

import fp4_sparse_attention_csa2_b200 as csa2
import oracle
from fp4_sparse_attention_csa2_b200 import workloads as wl
from gpu_harness import build_gpu_cache, device_layer, new_ws
from harness import band_set_check, build_ref_cache, host_layer

pytestmark = pytest.mark.gpu


def _check_against_oracle(ref, w, layer, pool, got):
    hl = host_layer(layer)
    for b in range(w.batch):
        for j in range(w.T):
            want, s = oracle.index_reindex(ref, b, w.T, j, hl["q_idx"][b, j], w.q_idx_dtype, hl["w"][b, j],
                                           pool[b, j], w.top_k, want_scores=True)
            by_pos = {int(t): float(v) for t, v in zip(pool[b, j], s) if t >= 0}
            band_set_check(got[b, j], want, lambda t: by_pos[t], len(by_pos))


def test_noalloc_reindex_matches_oracle_and_workspace_reindex_twice():
    w = wl.scaled(wl.WORKLOADS["batch32_paged"], 24000, batch=3, T=2)
    l0 = wl.layer_queries(w, 0)
    dev = build_gpu_cache(w, q_idx0=l0["q_idx"])
    ref = build_ref_cache(w, rows=False, layers=[l0])
    ws = new_ws(dev, w)
    L0 = device_layer(l0)
    pool = torch.empty((w.batch, w.T, w.pool_k), dtype=torch.int32, device="cuda")
    topk0 = torch.empty((w.batch, w.T, w.top_k), dtype=torch.int32, device="cuda")
    csa2.index_full(dev, L0["q_idx"], L0["w"], w.pool_k, w.top_k, pool, topk0, ws)
    pool_h = pool.cpu().numpy()
    for layer in (1, 2):                                # two calls in a row share the scratch
        lq = wl.layer_queries(w, layer)
        Ll = device_layer(lq)
        want = torch.full((w.batch, w.T, w.top_k), -7, dtype=torch.int32, device="cuda")
        got = torch.full((w.batch, w.T, w.top_k), -7, dtype=torch.int32, device="cuda")
        csa2.index_reindex(dev, Ll["q_idx"], Ll["w"], pool, w.top_k, want, ws)
        csa2.index_reindex_noalloc(dev, Ll["q_idx"], Ll["w"], pool, w.top_k, got)
        torch.cuda.synchronize()
        assert csa2.read_device_status(ws) == csa2.OK
        a, g = want.cpu().numpy(), got.cpu().numpy()
        _check_against_oracle(ref, w, lq, pool_h, g)
        for bb in range(w.batch):
            for j in range(w.T):
                assert np.array_equal(np.sort(a[bb, j]), np.sort(g[bb, j])), (layer, bb, j)
                assert np.all(g[bb, j] >= 0)        # the pools hold more than top_k positions


def test_noalloc_reindex_skips_a_page_outside_the_cache():
    # A page id outside the cache makes the scorer skip that page's pool
    # entries.  The scratch is first filled by a call on the intact table, so a
    # skipped entry whose score slot were left unwritten would be ranked by
    # that earlier call's score; the result must be the oracle's Reindex of the
    # pool without the skipped entries.
    w = wl.scaled(wl.WORKLOADS["batch32_paged"], 20000, batch=2, T=1)
    l0, l1 = wl.layer_queries(w, 0), wl.layer_queries(w, 1)
    dev = build_gpu_cache(w, q_idx0=l0["q_idx"])
    ref = build_ref_cache(w, rows=False, layers=[l0])
    ws = new_ws(dev, w)
    L0, L1 = device_layer(l0), device_layer(l1)
    pool = torch.empty((w.batch, w.T, w.pool_k), dtype=torch.int32, device="cuda")
    topk = torch.empty((w.batch, w.T, w.top_k), dtype=torch.int32, device="cuda")
    csa2.index_full(dev, L0["q_idx"], L0["w"], w.pool_k, w.top_k, pool, topk, ws)
    out = torch.full((w.batch, w.T, w.top_k), -7, dtype=torch.int32, device="cuda")
    csa2.index_reindex_noalloc(dev, L1["q_idx"], L1["w"], pool, w.top_k, out)     # fills the scratch
    torch.cuda.synchronize()
    pool_h = pool.cpu().numpy()
    # the page holding sequence 0's best Reindex entry now points outside the cache
    first = out.cpu().numpy()[0, 0]
    bad_page = int(first[0]) // w.page_size
    table = dev.page_table.clone()
    n_pages = dev.n_slots // w.page_size
    dev.page_table[0, bad_page] = n_pages + 3
    torch.cuda.synchronize()
    try:
        out2 = torch.full((w.batch, w.T, w.top_k), -7, dtype=torch.int32, device="cuda")
        csa2.index_reindex_noalloc(dev, L1["q_idx"], L1["w"], pool, w.top_k, out2)
        torch.cuda.synchronize()
        got = out2.cpu().numpy()
    finally:
        dev.page_table.copy_(table)
        torch.cuda.synchronize()
    kept = pool_h.copy()
    on_bad = (kept[0, 0] >= 0) & (kept[0, 0] // w.page_size == bad_page)
    assert on_bad.any()
    kept[0, 0][on_bad] = -1
    assert not np.isin(got[0, 0], pool_h[0, 0][on_bad]).any()
    _check_against_oracle(ref, w, l1, kept, got)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    w = wl.scaled(wl.WORKLOADS["long64k"], 4096, batch=1)
    dev = build_gpu_cache(w)
    T = 80                                              # 80 * 16384 pool entries > 4 MiB of scratch
    q = torch.zeros((1, T, 1, 64), dtype=torch.bfloat16, device="cuda")
    hw = torch.ones((1, T, 1), dtype=torch.float32, device="cuda")
    pool = torch.zeros((1, T, 16384), dtype=torch.int32, device="cuda")
    out = torch.zeros((1, T, 16), dtype=torch.int32, device="cuda")
    with pytest.raises(csa2.CSA2Error) as ei:
        csa2.index_reindex_noalloc(dev, q, hw, pool, 16, out)
    assert ei.value.code == csa2.ERR_UNSUPPORTED

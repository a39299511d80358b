"""Append-time pool update on the GPU (csa2_index_pool_update) against the
oracle's ref_index_pool_update: the new pool and top-k sets exact outside the
1e-5 relative band around each cutoff score (tldrocket.com "DeepSeek AI
Released DeepSeek-V4.1-Flash ...", paragraphs 3-4: the candidate pool of at
most 16,384 positions kept current as quantised tokens are appended)."""
import numpy as np
import pytest
import torch

import fp4_sparse_attention_csa2_b200 as csa2
import oracle
from fp4_sparse_attention_csa2_b200 import workloads as wl
from gpu_harness import build_gpu_cache, device_layer, new_ws
from harness import band_set_check, build_ref_cache, host_layer


def _prev_pools(w, lens, n_new, seed, fill=0.9):
    """A previous pool per (sequence, token): distinct positions before the
    append (a seeded fraction `fill` of pool_k, or all of them when fewer
    exist), -1 padding, in shuffled order."""
    rng = np.random.default_rng(seed)
    prev = np.full((w.batch, w.T, w.pool_k), -1, dtype=np.int32)
    for b in range(w.batch):
        t_new0 = int(lens[b]) - n_new
        for j in range(w.T):
            n = min(t_new0, int(fill * w.pool_k))
            if n > 0:
                prev[b, j, :n] = rng.choice(t_new0, n, replace=False)
            prev[b, j] = rng.permutation(prev[b, j])
    return prev


def _run(w, n_new, in_place=False, prev=None, seed=0):
    lens = wl.seq_lens(w)
    l0, l1 = wl.layer_queries(w, 0), wl.layer_queries(w, 1)
    ref = build_ref_cache(w, rows=False, layers=[l0])
    dev = build_gpu_cache(w, q_idx0=l0["q_idx"])
    ws = new_ws(dev, w)
    prev = _prev_pools(w, lens, n_new, seed) if prev is None else prev
    D1 = device_layer(l1)
    prev_d = torch.from_numpy(prev).cuda()
    pool = prev_d if in_place else torch.full_like(prev_d, -7)
    topk = torch.full((w.batch, w.T, w.top_k), -7, dtype=torch.int32, device="cuda")
    csa2.index_pool_update(dev, D1["q_idx"], D1["w"], prev_d, n_new, w.top_k, pool, topk, ws)
    st = csa2.read_device_status(ws)
    return w, ref, lens, prev, pool.cpu().numpy(), topk.cpu().numpy(), st, host_layer(l1)


def _check(w, ref, lens, prev, pool, topk, h1, n_new):
    for b in range(w.batch):
        for j in range(w.T):
            t_new0 = int(lens[b]) - n_new
            rp, rt = oracle.index_pool_update(ref, b, w.T, j, h1["q_idx"][b, j], w.q_idx_dtype, h1["w"][b, j],
                                              prev[b, j], t_new0, w.top_k)
            # every candidate's score under this query: the Full-layer scores
            _, _, s = oracle.index_full(ref, b, w.T, j, h1["q_idx"][b, j], w.q_idx_dtype, h1["w"][b, j],
                                        w.pool_k, w.top_k, want_scores=True)
            n_cand = int(np.sum(prev[b, j] >= 0)) + max(0, int(lens[b]) - w.T + j + 1 - t_new0)
            band_set_check(pool[b, j], rp, lambda t: s[t], n_cand)
            band_set_check(topk[b, j], rt, lambda t: s[t], n_cand)
            assert set(topk[b, j][topk[b, j] >= 0]) <= set(pool[b, j][pool[b, j] >= 0])


pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,L,n_new,kw", [
    ("long64k", 20000, 64, {"pool_k": 2048, "top_k": 256}),    # 2,112 candidates: the one-CTA select
    ("long64k", 20000, 64, {}),                                 # 16,448 candidates: the two-pass select
    ("long64k", 5000, 8, {"T": 4}),                             # 4 tokens, causal among the new positions
    ("batch32_paged", 30000, 16, {"batch": 3, "pool_k": 4096}), # paged, ragged lengths
    ("tiny4k", 600, 100, {}),                                   # the previous pool is every earlier position
    ("long64k", 9000, 0, {"pool_k": 1024, "top_k": 128}),       # nothing appended: the best of the previous pool
])
def test_pool_update_sets(name, L, n_new, kw):
    w, ref, lens, prev, pool, topk, st, h1 = _run(wl.scaled(wl.WORKLOADS[name], L, **kw), n_new)
    assert st == csa2.OK
    _check(w, ref, lens, prev, pool, topk, h1, n_new)


def test_pool_update_in_place():
    n_new = 32
    w, ref, lens, prev, pool, topk, st, h1 = _run(wl.scaled(wl.WORKLOADS["long64k"], 12000, pool_k=2048, top_k=256),
                                                  n_new, in_place=True)
    assert st == csa2.OK
    _check(w, ref, lens, prev, pool, topk, h1, n_new)


def test_previous_pool_entry_after_the_append_is_a_device_error():
    w = wl.scaled(wl.WORKLOADS["long64k"], 6000, pool_k=512, top_k=64)
    lens = wl.seq_lens(w)
    n_new = 16
    prev = _prev_pools(w, lens, n_new, 1)
    prev[0, 0, 3] = int(lens[0]) - 1          # a position the append just wrote
    w, ref, lens, prev2, pool, topk, st, h1 = _run(w, n_new, prev=prev)
    assert st == csa2.ERR_DEVICE_BOUNDS
    # the entry is dropped; the rest is the update of the remaining pool
    prev[0, 0, 3] = -1
    _check(w, ref, lens, prev, pool, topk, h1, n_new)

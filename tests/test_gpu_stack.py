"""End-to-end parity of whole CSA2 stacks (Full, Reindex, Reuse layers run
through csa2_layer_step exactly as the benchmark runs them) against the oracle
(tldrocket.com "DeepSeek AI Released DeepSeek-V4.1-Flash ...", paragraph 3;
fanout.sh lesson, "What you will learn" item 2)."""
import numpy as np
import pytest
import torch

import fp4_sparse_attention_csa2_b200 as csa2
import oracle
from fp4_sparse_attention_csa2_b200 import workloads as wl
from gpu_harness import attn_errors, build_gpu_cache, run_gpu_stack
from harness import attended_positions, band_set_check, build_ref_cache, fill_ref_rows, host_layer

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-3, 2e-4


def compare_stack(w, ref, got, layers, pairs, latents=None):
    """Check every layer of `got` (from run_gpu_stack) for the (b, j) pairs,
    each step on the GPU's own inputs so that no step's check depends on an
    earlier step matching exactly: the Full layer's pool and top-k against the
    oracle's Full selection; the Reindex layer's top-k against the oracle's
    Reindex of the GPU's pool; Reuse indices byte-identical to the layer
    before; every layer's out and lse against the oracle's attention over the
    GPU's own top-k.  With `latents`, oracle rows are quantised on demand for
    the attended sets.  Returns the number of index differences that lie
    inside the cutoff band (information only; outside it a check fails)."""
    hl = [host_layer(L) for L in layers]
    n_band = 0
    for (b, j) in pairs:
        p = int(ref.seq_lens[b]) - w.T + j
        gpool_cur = None
        for l, mode in enumerate(w.pattern):
            gpool, gtopk, gout, glse = got[l]
            if mode == "F":
                pool, topk, s = oracle.index_full(ref, b, w.T, j, hl[l]["q_idx"][b, j], w.q_idx_dtype,
                                                  hl[l]["w"][b, j], w.pool_k, w.top_k, want_scores=True)
                n_band += band_set_check(gpool[b, j], pool, lambda t: s[t], s.size)
                n_band += band_set_check(gtopk[b, j], topk, lambda t: s[t], s.size)
                gpool_cur = gpool[b, j]
            elif mode == "R":
                # the oracle's Reindex of the pool the GPU's Full layer produced
                topk, s = oracle.index_reindex(ref, b, w.T, j, hl[l]["q_idx"][b, j], w.q_idx_dtype,
                                               hl[l]["w"][b, j], gpool_cur, w.top_k, want_scores=True)
                by_pos = {int(t): float(v) for t, v in zip(gpool_cur, s) if t >= 0}
                n_band += band_set_check(gtopk[b, j], topk, lambda t: by_pos[t], len(by_pos))
            else:
                # Reuse: the device passes the indices on unchanged
                assert np.array_equal(gtopk[b, j], got[l - 1][1][b, j]), (l, b, j)
            # this layer's attention over the GPU's own top-k
            if latents is not None:
                fill_ref_rows(ref, w, b, attended_positions(gtopk[b, j], p, w.window), latents(b))
            ro, rl = oracle.sparse_swa_attn(ref, b, w.T, j, wl.bf16_bits(layers[l]["q"])[b, j], gtopk[b, j],
                                            w.window)
            mx, mean = attn_errors(gout[b, j], ro)
            assert mx <= MAX_ABS and mean <= MEAN_ABS, (l, b, j, mx, mean)
            lmx, lmean = attn_errors(glse[b, j], rl)
            assert lmx <= MAX_ABS and lmean <= MEAN_ABS, (l, b, j, "lse", lmx, lmean)
    return n_band


@pytest.mark.parametrize("name,L,kw", [
    ("tiny4k", 4096, {}),
    ("long64k", 12000, {}),
    ("batch32_paged", 12000, {"batch": 3}),
    ("ctx1m", 30000, {}),
    ("append_mq", 6000, {"batch": 2}),
])
def test_stack_small(name, L, kw):
    w = wl.scaled(wl.WORKLOADS[name], L, **kw)
    layers = [wl.layer_queries(w, l) for l in range(len(w.pattern))]
    ref = build_ref_cache(w, layers=layers)
    dev = build_gpu_cache(w, q_idx0=layers[0]["q_idx"])
    got, status = run_gpu_stack(dev, w, layers)
    assert status == csa2.OK
    pairs = [(b, j) for b in range(w.batch) for j in range(w.T)]
    compare_stack(w, ref, got, layers, pairs)


# ----------------------------------------------------------------------------- full sizes
def _full_size(name, pairs_of, sample_rows=20000):
    w = wl.WORKLOADS[name]
    layers = [wl.layer_queries(w, l) for l in range(len(w.pattern))]
    dev = build_gpu_cache(w, q_idx0=layers[0]["q_idx"])
    got, status = run_gpu_stack(dev, w, layers)
    assert status == csa2.OK
    pairs = pairs_of(w)
    ref = build_ref_cache(w, rows=False, layers=layers, batches=sorted(set(b for b, _ in pairs)))
    cache_lat = {}

    def latents(b):
        if b not in cache_lat:
            cache_lat.clear()
            cache_lat[b] = wl.latent(w, b, int(ref.seq_lens[b]))
        return cache_lat[b]

    n_band = compare_stack(w, ref, got, layers, pairs, latents)
    print("%s: %d (b, j) pairs checked at every layer, %d index differences inside the cutoff band"
          % (name, len(pairs), n_band))
    # a sample of FP4 rows, bit-exact
    rng = np.random.default_rng(1)
    b = pairs[0][0]
    L = int(ref.seq_lens[b])
    ts = np.sort(rng.choice(L, min(sample_rows, L), replace=False))
    x = latents(b)
    want = oracle.quantize_rows(wl.bf16_bits(x[torch.from_numpy(ts)]), w.row_stride)
    slots = [ref.slot(b, int(t)) for t in ts]
    gotr = dev.rows[torch.tensor(slots, device="cuda")].cpu().numpy()
    D = w.D
    assert np.array_equal(gotr[:, :D // 2 + D // 16], want[:, :D // 2 + D // 16])


def test_full_size_long64k():
    _full_size("long64k", lambda w: [(0, 0)])


def test_full_size_ctx1m():
    _full_size("ctx1m", lambda w: [(0, 0)])


def test_full_size_batch32_paged():
    # eight of the 32 sequences, the shortest and the longest among them
    def pairs(w):
        lens = wl.seq_lens(w)
        order = [int(b) for b in np.argsort(lens)]
        pick = sorted(set([order[0], order[-1]] + list(range(0, w.batch, 5))))[:8]
        return [(b, 0) for b in pick]
    _full_size("batch32_paged", pairs)


def test_full_size_append_mq():
    w = wl.WORKLOADS["append_mq"]
    layers = [wl.layer_queries(w, l) for l in range(len(w.pattern))]
    n_cached = w.lens[1] - w.append_n
    # (a) the cache holds n_cached positions; the last append_n positions of
    # every sequence are appended in one batched call
    dev = build_gpu_cache(w, q_idx0=layers[0]["q_idx"], upto=[n_cached] * w.batch)
    x = torch.stack([wl.latent(w, b, w.lens[1], t0=n_cached) for b in range(w.batch)])
    keys = torch.stack([wl.index_keys(w, b, w.lens[1], layers[0]["q_idx"][b, w.T - 1], t0=n_cached)[0]
                        for b in range(w.batch)])
    sp = torch.full((w.batch,), n_cached, dtype=torch.int32, device="cuda")
    csa2.kv_append_quant(dev, x.cuda(), sp, keys.cuda())
    torch.cuda.synchronize()
    for b in (0, w.batch - 1):
        want = oracle.quantize_rows(wl.bf16_bits(x[b]), w.row_stride)
        slots = torch.arange(n_cached, w.lens[1], device="cuda") + b * dev.seq_stride_slots
        assert np.array_equal(dev.rows[slots].cpu().numpy()[:, :288], want[:, :288])
        wk = oracle.e4m3_encode(keys[b].float().numpy())
        assert np.array_equal(dev.idx_keys[slots].cpu().numpy(), wk)
    # (b) 4 query tokens per sequence through F, R, U, U
    got, status = run_gpu_stack(dev, w, layers)
    assert status == csa2.OK
    checked = (0, 3, 5, w.batch - 1)
    ref = build_ref_cache(w, rows=False, layers=layers, batches=list(checked))
    pairs = [(b, j) for b in checked for j in range(w.T)]
    lat = {}

    def latents(b):
        if b not in lat:
            lat.clear()
            lat[b] = wl.latent(w, b, w.lens[1])
        return lat[b]

    n_band = compare_stack(w, ref, got, layers, pairs, latents)
    print("append_mq: %d (b, j) pairs checked at every layer, %d index differences inside the cutoff band"
          % (len(pairs), n_band))

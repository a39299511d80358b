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
    """Check every layer of `got` (from run_gpu_stack) for the (b, j) pairs.
    With `latents`, oracle rows are quantised on demand for the attended sets."""
    hl = [host_layer(L) for L in layers]
    n_exact = 0
    for (b, j) in pairs:
        p = int(ref.seq_lens[b]) - w.T + j
        pool_ok = True
        pool = topk = None
        for l, mode in enumerate(w.pattern):
            gpool, gtopk, gout, glse = got[l]
            if mode == "F":
                pool, topk, s = oracle.index_full(ref, b, w.T, j, hl[l]["q_idx"][b, j], w.q_idx_dtype,
                                                  hl[l]["w"][b, j], w.pool_k, w.top_k, want_scores=True)
                d1 = band_set_check(gpool[b, j], pool, lambda t: s[t], s.size)
                d2 = band_set_check(gtopk[b, j], topk, lambda t: s[t], s.size)
                pool_ok = d1 == 0 and d2 == 0
            elif mode == "R":
                if not pool_ok:
                    break
                topk, s = oracle.index_reindex(ref, b, w.T, j, hl[l]["q_idx"][b, j], w.q_idx_dtype,
                                               hl[l]["w"][b, j], pool, w.top_k, want_scores=True)
                by_pos = {int(t): float(v) for t, v in zip(pool, s) if t >= 0}
                pool_ok = band_set_check(gtopk[b, j], topk, lambda t: by_pos[t], len(by_pos)) == 0
            else:
                # Reuse: the device passes the indices on unchanged
                assert np.array_equal(gtopk[b, j], got[l - 1][1][b, j])
            if not pool_ok:
                break
            if latents is not None:
                fill_ref_rows(ref, w, b, attended_positions(topk, p, w.window), latents(b))
            ro, rl = oracle.sparse_swa_attn(ref, b, w.T, j, wl.bf16_bits(layers[l]["q"])[b, j], topk, w.window)
            mx, mean = attn_errors(gout[b, j], ro)
            assert mx <= MAX_ABS and mean <= MEAN_ABS, (l, b, j, mx, mean)
            assert np.allclose(glse[b, j], rl, atol=MAX_ABS, rtol=0)
        n_exact += pool_ok
    return n_exact


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
    assert compare_stack(w, ref, got, layers, pairs) == len(pairs)


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

    n_exact = compare_stack(w, ref, got, layers, pairs, latents)
    assert n_exact >= len(pairs) - 1, "too many (b, j) with index-set differences inside the band"
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
    _full_size("batch32_paged", lambda w: [(0, 0), (17, 0), (31, 0)])


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
    ref = build_ref_cache(w, rows=False, layers=layers, batches=[0, w.batch - 1])
    pairs = [(b, j) for b in (0, w.batch - 1) for j in range(w.T)]
    lat = {}

    def latents(b):
        if b not in lat:
            lat.clear()
            lat[b] = wl.latent(w, b, w.lens[1])
        return lat[b]

    n_exact = compare_stack(w, ref, got, layers, pairs, latents)
    assert n_exact >= len(pairs) - 1

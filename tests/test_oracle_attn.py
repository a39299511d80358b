"""Pins of the oracle's sparse + sliding-window attention against textbook
special cases (hackernews.kjhq.dev post 49735410, key point 2: local sliding
windows plus global sparse retrieval; tldrocket.com "DeepSeek AI Released
DeepSeek-V4.1-Flash ...", paragraph 2: a 128-token window in every layer)."""
import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden
from fp4_sparse_attention_csa2_b200 import workloads as wl
from harness import build_ref_cache

E2M1 = {int(c, 16): float(v) for c, v in read_golden("e2m1_values.txt")}


def _decode_rows_lib(cache, b, positions, D):
    """Rows decoded without the oracle: golden E2M1 table x torch's E4M3 scale."""
    out = np.zeros((len(positions), D))
    for i, t in enumerate(positions):
        row = cache.rows[cache.slot(b, int(t))]
        sc = torch.from_numpy(row[D // 2:D // 2 + D // 16].copy()).view(torch.float8_e4m3fn).double().numpy()
        codes = np.empty(D, dtype=np.int64)
        codes[0::2] = row[:D // 2] & 0xF
        codes[1::2] = row[:D // 2] >> 4
        out[i] = np.array([E2M1[c] for c in codes]) * np.repeat(sc, 16)
    return out


def _numpy_attn(q_bf16, V, scale):
    q = q_bf16.double().numpy()
    z = scale * (q @ V.T)                                # [H, n]
    p = torch.softmax(torch.from_numpy(z), dim=1).numpy()
    lse = torch.logsumexp(torch.from_numpy(z), dim=1).numpy()
    return p @ V, lse


def _setup(L=700, T=1, **kw):
    w = wl.scaled(wl.WORKLOADS["tiny4k"], L, T=T, **kw)
    cache = build_ref_cache(w)
    q = wl.layer_queries(w, 2)["q"]
    return w, cache, q


def test_topk_covering_context_equals_dense():
    w, cache, q = _setup(700)
    p = 699
    topk = np.arange(p + 1, dtype=np.int32)[::-1].copy()
    out, lse = oracle.sparse_swa_attn(cache, 0, 1, 0, wl.bf16_bits(q[0, 0]), topk, w.window)
    dout, dlse = oracle.dense_attn(cache, 0, 1, 0, wl.bf16_bits(q[0, 0]))
    V = _decode_rows_lib(cache, 0, range(p + 1), w.D)
    nout, nlse = _numpy_attn(q[0, 0], V, 1 / np.sqrt(w.D))
    assert np.allclose(out, dout, rtol=0, atol=1e-12) and np.allclose(lse, dlse, atol=1e-12)
    assert np.allclose(out, nout, rtol=0, atol=1e-12) and np.allclose(lse, nlse, atol=1e-12)


def test_empty_topk_is_dense_over_window():
    w, cache, q = _setup(700)
    topk = np.full(w.top_k, -1, dtype=np.int32)
    out, lse = oracle.sparse_swa_attn(cache, 0, 1, 0, wl.bf16_bits(q[0, 0]), topk, w.window)
    V = _decode_rows_lib(cache, 0, range(700 - w.window, 700), w.D)
    nout, nlse = _numpy_attn(q[0, 0], V, 1 / np.sqrt(w.D))
    assert np.allclose(out, nout, atol=1e-12) and np.allclose(lse, nlse, atol=1e-12)


def test_sparse_plus_window_equals_numpy_over_union():
    w, cache, q = _setup(900)
    rng = np.random.default_rng(1)
    topk = rng.choice(900, w.top_k, replace=False).astype(np.int32)
    topk[:10] = -1
    out, lse = oracle.sparse_swa_attn(cache, 0, 1, 0, wl.bf16_bits(q[0, 0]), topk, w.window, 0.07)
    S = sorted(set(range(900 - w.window, 900)) | set(int(t) for t in topk if t >= 0))
    V = _decode_rows_lib(cache, 0, S, w.D)
    nout, nlse = _numpy_attn(q[0, 0], V, 0.07)
    assert np.allclose(out, nout, atol=1e-12) and np.allclose(lse, nlse, atol=1e-12)
    assert max(np.sum(topk >= 0), w.window) <= len(S) <= np.sum(topk >= 0) + w.window


def test_invariant_under_permutation_and_window_duplicates():
    w, cache, q = _setup(900)
    rng = np.random.default_rng(2)
    topk = rng.choice(700, w.top_k, replace=False).astype(np.int32)
    base, blse = oracle.sparse_swa_attn(cache, 0, 1, 0, wl.bf16_bits(q[0, 0]), topk, w.window)
    perm = rng.permutation(topk)
    out, lse = oracle.sparse_swa_attn(cache, 0, 1, 0, wl.bf16_bits(q[0, 0]), perm, w.window)
    assert np.array_equal(out, base) and np.array_equal(lse, blse)
    dup = topk.copy()
    dup[:20] = np.arange(880, 900)                    # window positions repeated in top-k
    a, _ = oracle.sparse_swa_attn(cache, 0, 1, 0, wl.bf16_bits(q[0, 0]), dup, w.window)
    b, _ = oracle.sparse_swa_attn(cache, 0, 1, 0, wl.bf16_bits(q[0, 0]), topk[20:].copy(), w.window)
    assert np.array_equal(a, b)


def test_window_shorter_than_context_start():
    # p + 1 < W: the window is [0, p]
    w, cache, q = _setup(50)
    topk = np.full(w.top_k, -1, dtype=np.int32)
    out, _ = oracle.sparse_swa_attn(cache, 0, 1, 0, wl.bf16_bits(q[0, 0]), topk, w.window)
    dout, _ = oracle.dense_attn(cache, 0, 1, 0, wl.bf16_bits(q[0, 0]))
    assert np.allclose(out, dout, atol=1e-12)


def test_multi_token_causal():
    # token j of T sees positions <= p_j = L - T + j only, in top-k and window
    T = 4
    w, cache, q = _setup(600, T=T)
    topk = np.arange(600, dtype=np.int32)              # includes the later tokens' positions
    for j in range(T):
        out, _ = oracle.sparse_swa_attn(cache, 0, T, j, wl.bf16_bits(q[0, j]), topk, w.window)
        dout, _ = oracle.dense_attn(cache, 0, T, j, wl.bf16_bits(q[0, j]))
        assert np.allclose(out, dout, atol=1e-12)


def test_out_of_range_index_is_an_error():
    w, cache, q = _setup(300)
    topk = np.zeros(w.top_k, dtype=np.int32)
    topk[5] = 300
    with pytest.raises(RuntimeError):
        oracle.sparse_swa_attn(cache, 0, 1, 0, wl.bf16_bits(q[0, 0]), topk, w.window)


def test_paged_equals_contiguous():
    base = wl.scaled(wl.WORKLOADS["batch32_paged"], 900, batch=3, lens=("uniform", 300, 900))
    contig = wl.Workload(**{**base.__dict__, "paged": False, "name": "contig"})
    cp = build_ref_cache(base)
    cc = build_ref_cache(contig)
    assert np.array_equal(cp.seq_lens, cc.seq_lens)
    layers = [wl.layer_queries(base, l) for l in range(2)]
    hl = [{k: wl.host_array(v) for k, v in L.items()} for L in layers]
    rp = oracle.run_stack(cp, "FR", hl, 1, base.pool_k, base.top_k, base.window, base.q_idx_dtype)
    rc = oracle.run_stack(cc, "FR", hl, 1, base.pool_k, base.top_k, base.window, base.q_idx_dtype)
    for l in range(2):
        for key in rp[l]:
            assert np.array_equal(rp[l][key][1], rc[l][key][1])
            assert np.array_equal(rp[l][key][2], rc[l][key][2])


def test_future_topk_entries_are_not_attended_without_window():
    # window 0, token 0 of 2: an index of the later token's position (legal,
    # < L) must be ignored, not clipped onto p; only the past entries count
    T = 2
    w, cache, q = _setup(500, T=T)
    p = 500 - T
    past = np.array([3, 17, 250, p], dtype=np.int32)
    topk = np.concatenate([past, np.array([p + 1], dtype=np.int32)])
    out, lse = oracle.sparse_swa_attn(cache, 0, T, 0, wl.bf16_bits(q[0, 0]), topk, 0, 0.05)
    V = _decode_rows_lib(cache, 0, sorted(past.tolist()), w.D)
    nout, nlse = _numpy_attn(q[0, 0], V, 0.05)
    assert np.allclose(out, nout, atol=1e-12) and np.allclose(lse, nlse, atol=1e-12)
    # without p itself the set is the three earlier positions only
    out2, _ = oracle.sparse_swa_attn(cache, 0, T, 0, wl.bf16_bits(q[0, 0]),
                                     np.array([3, 17, 250, p + 1], dtype=np.int32), 0, 0.05)
    V2 = _decode_rows_lib(cache, 0, [3, 17, 250], w.D)
    assert np.allclose(out2, _numpy_attn(q[0, 0], V2, 0.05)[0], atol=1e-12)


# ------------------------------------------------------------------ layer-local window state
# ([FANOUT] item 2: queries and the sliding-window state stay layer-local;
# [TLDR] paragraph 2: the window runs in every layer)

def _ring(w, L, ring_len, seed):
    g = torch.Generator().manual_seed(seed)
    ring = torch.randn((w.batch, ring_len, w.D), generator=g).to(torch.bfloat16)
    return ring, wl.bf16_bits(ring)


def test_local_window_holding_the_cache_rows_equals_shared_rows():
    # a ring that holds the window positions' dequantised FP4 rows (exact in
    # bf16) gives exactly the shared-cache result
    w, cache, q = _setup(900)
    p, ring_len = 899, 160
    rows = _decode_rows_lib(cache, 0, range(900), w.D)
    ring = torch.zeros((1, ring_len, w.D), dtype=torch.float64)
    for t in range(p - w.window + 1, p + 1):
        ring[0, t % ring_len] = torch.from_numpy(rows[t])
    assert torch.equal(ring.to(torch.bfloat16).double(), ring)          # exact in bf16
    rng = np.random.default_rng(4)
    topk = rng.choice(900, w.top_k, replace=False).astype(np.int32)
    a, al = oracle.sparse_swa_attn(cache, 0, 1, 0, wl.bf16_bits(q[0, 0]), topk, w.window)
    b, bl = oracle.sparse_swa_attn_local(cache, wl.bf16_bits(ring.to(torch.bfloat16)), 0, 1, 0,
                                         wl.bf16_bits(q[0, 0]), topk, w.window)
    assert np.array_equal(a, b) and np.array_equal(al, bl)


def test_local_window_only_is_dense_over_the_ring_rows():
    w, cache, q = _setup(700)
    p, ring_len = 699, 200                                               # 700 % 200 != 0: the ring wraps
    ring, bits = _ring(w, 700, ring_len, 5)
    topk = np.full(w.top_k, -1, dtype=np.int32)
    out, lse = oracle.sparse_swa_attn_local(cache, bits, 0, 1, 0, wl.bf16_bits(q[0, 0]), topk, w.window, 0.03)
    V = np.stack([ring[0, t % ring_len].double().numpy() for t in range(p - w.window + 1, p + 1)])
    nout, nlse = _numpy_attn(q[0, 0], V, 0.03)
    assert np.allclose(out, nout, atol=1e-12) and np.allclose(lse, nlse, atol=1e-12)


def test_local_window_mixed_with_shared_topk_rows():
    # window rows from the ring, the other attended rows from the FP4 cache; a
    # top-k entry inside the window uses the ring row once
    w, cache, q = _setup(900)
    p, ring_len = 899, 128
    ring, bits = _ring(w, 900, ring_len, 6)
    rng = np.random.default_rng(7)
    topk = rng.choice(700, w.top_k, replace=False).astype(np.int32)
    topk[:5] = [899, 880, 850, -1, 772]                                  # three of them in the window
    out, lse = oracle.sparse_swa_attn_local(cache, bits, 0, 1, 0, wl.bf16_bits(q[0, 0]), topk, w.window, 0.04)
    win = list(range(p - w.window + 1, p + 1))
    far = sorted(set(int(t) for t in topk if 0 <= t < p - w.window + 1))
    V = np.concatenate([_decode_rows_lib(cache, 0, far, w.D),
                        np.stack([ring[0, t % ring_len].double().numpy() for t in win])])
    nout, nlse = _numpy_attn(q[0, 0], V, 0.04)
    assert np.allclose(out, nout, atol=1e-12) and np.allclose(lse, nlse, atol=1e-12)


def test_local_ring_shorter_than_the_window_is_an_error():
    w, cache, q = _setup(300)
    _, bits = _ring(w, 300, w.window - 1, 8)
    with pytest.raises(RuntimeError):
        oracle.sparse_swa_attn_local(cache, bits, 0, 1, 0, wl.bf16_bits(q[0, 0]),
                                     np.full(w.top_k, -1, dtype=np.int32), w.window)


# ------------------------------------------------------------------ partials over disjoint parts
# (the attention of a context sharded over devices: each attends over its part
# of S, the parts' (output, log-sum-exp) pairs are merged)

def test_lse_merge_of_disjoint_parts_equals_attention_over_the_union():
    w, cache, q = _setup(900)
    rng = np.random.default_rng(9)
    S = rng.choice(900, 300, replace=False).astype(np.int32)
    qb = wl.bf16_bits(q[0, 0])
    full, flse = oracle.sparse_swa_attn(cache, 0, 1, 0, qb, S, 0, 0.05)
    for n_parts in (2, 3, 5):
        parts = np.array_split(rng.permutation(S), n_parts)
        res = [oracle.sparse_swa_attn(cache, 0, 1, 0, qb, part, 0, 0.05) for part in parts]
        out, lse = oracle.lse_merge(np.stack([r[0] for r in res]), np.stack([r[1] for r in res]))
        assert np.allclose(out, full, atol=1e-12) and np.allclose(lse, flse, atol=1e-12)
    # the merge itself against its definition written with numpy
    outs, lses = np.stack([r[0] for r in res]), np.stack([r[1] for r in res])
    L = np.logaddexp.reduce(lses, axis=0)
    assert np.allclose(lse, L, atol=1e-12)
    assert np.allclose(out, np.einsum("ih,ihd->hd", np.exp(lses - L), outs), atol=1e-12)


def test_lse_merge_with_empty_parts():
    w, cache, q = _setup(600)
    qb = wl.bf16_bits(q[0, 0])
    S = np.arange(100, 160, dtype=np.int32)
    full, flse = oracle.sparse_swa_attn(cache, 0, 1, 0, qb, S, 0)
    empty = oracle.sparse_swa_attn(cache, 0, 1, 0, qb, np.full(4, -1, dtype=np.int32), 0)
    assert np.all(np.isneginf(empty[1])) and np.all(empty[0] == 0)
    out, lse = oracle.lse_merge(np.stack([empty[0], full, empty[0]]), np.stack([empty[1], flse, empty[1]]))
    assert np.allclose(out, full, atol=1e-15) and np.allclose(lse, flse, atol=1e-15)
    out, lse = oracle.lse_merge(np.stack([empty[0], empty[0]]), np.stack([empty[1], empty[1]]))
    assert np.all(out == 0) and np.all(np.isneginf(lse))

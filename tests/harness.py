"""Test-side helpers: build the oracle's host cache for a workload from the
seeded inputs, and compare index sets under the cutoff-band rule."""
import numpy as np

import oracle
from fp4_sparse_attention_csa2_b200 import workloads as wl


cache_geometry = wl.cache_geometry


def build_ref_cache(w, seed=0, lens=None, rows=True, layers=None, batches=None):
    """Oracle host cache with every position of the sequences in `batches`
    (default: all) written: index keys encoded by the oracle and, with rows=True,
    latent rows quantised by the oracle."""
    lens = wl.seq_lens(w, seed) if lens is None else np.asarray(lens, dtype=np.int32)
    n_slots, table, stride = cache_geometry(w, lens, seed)
    cache = oracle.RefCache(w.batch, n_slots, w.D, w.D_I, w.row_stride, w.idx_key_dtype, lens,
                            page_table=table, page_size=w.page_size, seq_stride_slots=stride)
    q0 = (layers[0] if layers else wl.layer_queries(w, 0, seed))["q_idx"]
    for b in (range(w.batch) if batches is None else batches):
        L = int(lens[b])
        keys, _ = wl.index_keys(w, b, L, q0[b, w.T - 1], seed)
        x = wl.bf16_bits(wl.latent(w, b, L, seed)) if rows else None
        cache.write(b, 0, x, wl.host_array(keys), wl.F32 if w.idx_key_dtype == wl.F32 else wl.BF16)
    return cache


def band_set_check(got, want_sorted, scores_by_pos, n_valid, rel=1e-5):
    """Index-set parity: `got` (any order, -1 padding) must hold exactly
    min(n_out, n_valid) positions; it may differ from the oracle's ordered
    selection `want_sorted` only at positions whose oracle score lies within
    rel * |c*| of the cutoff score c* (the last selected oracle score)."""
    got = np.asarray(got)
    n_sel = int(np.sum(np.asarray(want_sorted) >= 0))
    g = got[got >= 0]
    assert g.size == n_sel, "cardinality %d != %d" % (g.size, n_sel)
    assert np.unique(g).size == g.size, "duplicate positions"
    assert np.all(got[:n_sel] >= 0) and np.all(got[n_sel:] == -1), "padding must come last"
    if n_sel == 0:
        return 0
    w = set(int(x) for x in want_sorted[:n_sel])
    gs = set(int(x) for x in g)
    cstar = scores_by_pos(int(want_sorted[n_sel - 1]))
    tol = rel * abs(cstar)
    for t in w ^ gs:
        assert abs(scores_by_pos(t) - cstar) <= tol, "position %d outside the cutoff band" % t
    return len(w ^ gs)


def host_layer(layer):
    """A layer's query tensors as the oracle takes them (bf16 -> uint16 bits)."""
    return {k: wl.host_array(v) for k, v in layer.items()}


def fill_ref_rows(ref, w, b, positions, latent_b):
    """Quantise (with the oracle) the latent rows of the given positions of
    sequence b into the oracle cache; latent_b is the bf16 [L_b, D] input."""
    pos = np.unique(np.asarray([int(t) for t in positions if t >= 0], dtype=np.int64))
    bits = wl.bf16_bits(latent_b)
    for t in pos:
        ref.write(b, int(t), bits[t:t + 1])


def attended_positions(topk, p, window):
    """Positions of window ∪ top-k for a query at p (the oracle's reading)."""
    s = set(range(max(0, p - window + 1), p + 1))
    s.update(int(t) for t in topk if 0 <= t <= p)
    return s

"""Python access to the CPU oracle (``oracle/csa2_ref.c``).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference legs may import this package.  It never
imports the CUDA library and the CUDA library never imports it.

Everything here is argument marshalling around the C oracle plus the plain
layer-pattern driver (Full -> Reindex -> Reuse ..., as the CSA2 modes are
described in the tldrocket.com retelling "DeepSeek AI Released
DeepSeek-V4.1-Flash with 1M Context, FP4 KV Cache, and Cross-Layer Attention
Reuse", paragraph 3: Full layers build fresh indices, Reindex layers rescore the
shared candidate set, Reuse layers take what came before).
"""
import ctypes
import os

import numpy as np

from . import build as _build

F32, BF16, E4M3 = 0, 1, 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        c_p = ctypes.c_void_p
        i64 = ctypes.c_int64
        i32 = ctypes.c_int
        L.ref_e4m3_value.restype = ctypes.c_double
        L.ref_e4m3_value.argtypes = [ctypes.c_uint8]
        L.ref_e2m1_value.restype = ctypes.c_double
        L.ref_e2m1_value.argtypes = [ctypes.c_uint8]
        L.ref_e4m3_encode.restype = ctypes.c_uint8
        L.ref_e4m3_encode.argtypes = [ctypes.c_float]
        L.ref_e2m1_encode.restype = ctypes.c_uint8
        L.ref_e2m1_encode.argtypes = [ctypes.c_float]
        L.ref_e2m1_encode_array.argtypes = [c_p, i64, c_p]
        L.ref_encode_e4m3_array.argtypes = [i32, c_p, i64, c_p]
        L.ref_quantize_block16.argtypes = [c_p, c_p, c_p]
        L.ref_quantize_rows.argtypes = [c_p, i64, i32, i32, c_p]
        L.ref_dequant_row.argtypes = [c_p, i32, c_p]
        L.ref_slot.restype = i64
        L.ref_slot.argtypes = [c_p, i32, i64]
        L.ref_kv_append.argtypes = [c_p, c_p, i32, c_p, c_p, i32]
        L.ref_kv_write.argtypes = [c_p, i32, i64, i64, c_p, i32, c_p]
        L.ref_index_scores.argtypes = [c_p, i32, i64, c_p, i32, c_p, i32, c_p, c_p]
        L.ref_select_top.argtypes = [c_p, c_p, i64, i32, c_p]
        L.ref_index_full.argtypes = [c_p, i32, i32, i32, i32, c_p, c_p, i32, i32, i32, c_p, c_p, c_p]
        L.ref_index_reindex.argtypes = [c_p, i32, i32, i32, i32, c_p, c_p, i32, c_p, i32, i32, c_p, c_p]
        L.ref_sparse_swa_attn.argtypes = [c_p, i32, i32, i32, i32, c_p, c_p, i32, i32, ctypes.c_double,
                                          c_p, c_p]
        L.ref_dense_attn.argtypes = [c_p, i32, i32, i32, i32, c_p, ctypes.c_double, c_p, c_p]
        L.ref_lse_merge.argtypes = [i32, i32, i32, c_p, c_p, c_p, c_p]
        L.ref_index_pool_update.argtypes = [c_p, i32, i32, i32, i32, c_p, c_p, i32, c_p, i32, i64, i32, c_p, c_p]
        L.ref_sparse_swa_attn_local.argtypes = [c_p, c_p, i64, i32, i32, i32, i32, c_p, c_p, i32, i32,
                                                ctypes.c_double, c_p, c_p]
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError("oracle %s failed with status %d" % (what, rc))


# --------------------------------------------------------------------------- formats
def e4m3_value(code):
    return lib().ref_e4m3_value(int(code) & 0xFF)


def e2m1_value(code):
    return lib().ref_e2m1_value(int(code) & 0xF)


def e4m3_encode(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    _check(lib().ref_encode_e4m3_array(F32, _ptr(x), x.size, _ptr(out)), "e4m3_encode")
    return out


def e2m1_encode(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    _check(lib().ref_e2m1_encode_array(_ptr(x), x.size, _ptr(out)), "e2m1_encode")
    return out


def quantize_block16(x):
    """One 16-channel block -> (16 unpacked E2M1 codes, E4M3 scale code)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    assert x.size == 16
    codes = np.zeros(16, dtype=np.uint8)
    sc = np.zeros(1, dtype=np.uint8)
    _check(lib().ref_quantize_block16(_ptr(x), _ptr(codes), _ptr(sc)), "quantize_block16")
    return codes, int(sc[0])


def quantize_rows(x_bf16_u16, row_stride):
    """bf16 bit patterns [n, D] (uint16) -> FP4 rows [n, row_stride] (uint8)."""
    x = np.ascontiguousarray(x_bf16_u16, dtype=np.uint16)
    n, D = x.shape
    rows = np.zeros((n, row_stride), dtype=np.uint8)
    _check(lib().ref_quantize_rows(_ptr(x), n, D, row_stride, _ptr(rows)), "quantize_rows")
    return rows


def dequant_row(row, D):
    row = np.ascontiguousarray(row, dtype=np.uint8)
    out = np.zeros(D, dtype=np.float64)
    _check(lib().ref_dequant_row(_ptr(row), D, _ptr(out)), "dequant_row")
    return out


# --------------------------------------------------------------------------- cache
class _RefCacheStruct(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_void_p),
        ("idx_keys", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p),
        ("batch", ctypes.c_int32),
        ("max_pages", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("dim", ctypes.c_int32),
        ("idx_dim", ctypes.c_int32),
        ("row_stride", ctypes.c_int32),
        ("seq_stride_slots", ctypes.c_int64),
        ("n_slots", ctypes.c_int64),
        ("idx_key_dtype", ctypes.c_int32),
    ]


class RefCache:
    """Host-side copy of the global cache: FP4 rows, index keys, page table."""

    def __init__(self, batch, n_slots, dim, idx_dim, row_stride, idx_key_dtype, seq_lens,
                 page_table=None, page_size=64, seq_stride_slots=0):
        self.rows = np.zeros((n_slots, row_stride), dtype=np.uint8)
        kd = np.uint8 if idx_key_dtype == E4M3 else np.float32
        self.idx_keys = np.zeros((n_slots, idx_dim), dtype=kd)
        self.seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
        self.page_table = None if page_table is None else np.ascontiguousarray(page_table, dtype=np.int32)
        self.s = _RefCacheStruct(
            self.rows.ctypes.data, self.idx_keys.ctypes.data,
            None if self.page_table is None else self.page_table.ctypes.data,
            self.seq_lens.ctypes.data, batch,
            0 if self.page_table is None else self.page_table.shape[1], page_size, dim, idx_dim,
            row_stride, seq_stride_slots, n_slots, idx_key_dtype)
        self.batch, self.dim, self.idx_dim, self.idx_key_dtype = batch, dim, idx_dim, idx_key_dtype

    @property
    def ref(self):
        return ctypes.byref(self.s)

    def set_seq_lens(self, seq_lens):
        self.seq_lens[:] = seq_lens

    def slot(self, b, t):
        return lib().ref_slot(self.ref, b, t)

    def append(self, x_bf16_u16, idx_new=None, idx_src_dtype=BF16, start_pos=None):
        """x: uint16 [B, n_new, D] bf16 bit patterns; idx_new: [B, n_new, D_I]."""
        x = np.ascontiguousarray(x_bf16_u16, dtype=np.uint16)
        B, n_new, D = x.shape
        sp = np.ascontiguousarray(start_pos, dtype=np.int32)
        idx = None
        if idx_new is not None:
            idx = np.ascontiguousarray(idx_new, dtype=np.float32 if idx_src_dtype == F32 else np.uint16)
        _check(lib().ref_kv_append(self.ref, _ptr(x), idx_src_dtype, _ptr(idx), _ptr(sp), n_new), "kv_append")


    def write(self, b, t0, x_bf16_u16=None, idx=None, idx_src_dtype=BF16):
        """Write positions t0.. of sequence b (rows [n, D] and/or keys [n, D_I])."""
        x = None if x_bf16_u16 is None else np.ascontiguousarray(x_bf16_u16, dtype=np.uint16)
        k = None
        if idx is not None:
            k = np.ascontiguousarray(idx, dtype=np.float32 if idx_src_dtype == F32 else np.uint16)
        n = x.shape[0] if x is not None else k.shape[0]
        _check(lib().ref_kv_write(self.ref, b, t0, n, _ptr(x), idx_src_dtype, _ptr(k)), "kv_write")


def _qarr(q, q_dtype):
    return np.ascontiguousarray(q, dtype=np.float32 if q_dtype == F32 else np.uint16)


def index_scores(cache, b, positions, q, q_dtype, w):
    q = _qarr(q, q_dtype)
    w = np.ascontiguousarray(w, dtype=np.float32)
    pos = np.ascontiguousarray(positions, dtype=np.int32)
    out = np.zeros(pos.size, dtype=np.float64)
    _check(lib().ref_index_scores(cache.ref, b, pos.size, _ptr(pos), q_dtype, _ptr(q), q.shape[0], _ptr(w),
                                  _ptr(out)), "index_scores")
    return out


def select_top(scores, positions, n_out):
    s = np.ascontiguousarray(scores, dtype=np.float64)
    pos = None if positions is None else np.ascontiguousarray(positions, dtype=np.int32)
    out = np.zeros(n_out, dtype=np.int32)
    _check(lib().ref_select_top(_ptr(s), _ptr(pos), s.size, n_out, _ptr(out)), "select_top")
    return out


def index_full(cache, b, T, j, q, q_dtype, w, pool_k, top_k, want_scores=False):
    """Full mode for query token j of sequence b: (pool_idx, topk_idx, scores|None)."""
    q = _qarr(q, q_dtype)
    w = np.ascontiguousarray(w, dtype=np.float32)
    pool = np.zeros(pool_k, dtype=np.int32)
    topk = np.zeros(top_k, dtype=np.int32)
    p = int(cache.seq_lens[b]) - T + j
    scores = np.zeros(max(p + 1, 1), dtype=np.float64) if want_scores else None
    _check(lib().ref_index_full(cache.ref, b, T, j, q_dtype, _ptr(q), _ptr(w), q.shape[0], pool_k, top_k,
                                _ptr(pool), _ptr(topk), _ptr(scores)), "index_full")
    return pool, topk, scores


def index_reindex(cache, b, T, j, q, q_dtype, w, pool_idx, top_k, want_scores=False):
    q = _qarr(q, q_dtype)
    w = np.ascontiguousarray(w, dtype=np.float32)
    pool = np.ascontiguousarray(pool_idx, dtype=np.int32)
    topk = np.zeros(top_k, dtype=np.int32)
    scores = np.zeros(pool.size, dtype=np.float64) if want_scores else None
    _check(lib().ref_index_reindex(cache.ref, b, T, j, q_dtype, _ptr(q), _ptr(w), q.shape[0], _ptr(pool),
                                   pool.size, top_k, _ptr(topk), _ptr(scores)), "index_reindex")
    return topk, scores


def index_pool_update(cache, b, T, j, q, q_dtype, w, pool_prev, t_new0, top_k):
    """The pool of an in-flight request after positions t_new0.. were appended:
    the best of the previous pool and the new positions -> (pool_idx, topk_idx)."""
    q = _qarr(q, q_dtype)
    w = np.ascontiguousarray(w, dtype=np.float32)
    prev = np.ascontiguousarray(pool_prev, dtype=np.int32)
    pool = np.zeros(prev.size, dtype=np.int32)
    topk = np.zeros(top_k, dtype=np.int32)
    _check(lib().ref_index_pool_update(cache.ref, b, T, j, q_dtype, _ptr(q), _ptr(w), q.shape[0], _ptr(prev),
                                       prev.size, t_new0, top_k, _ptr(pool), _ptr(topk)), "index_pool_update")
    return pool, topk


def sparse_swa_attn(cache, b, T, j, q_bf16_u16, topk_idx, window, sm_scale=0.0):
    """q: uint16 [H, D] bf16 bit patterns -> (out fp64 [H, D], lse fp64 [H])."""
    q = np.ascontiguousarray(q_bf16_u16, dtype=np.uint16)
    H, D = q.shape
    tk = np.ascontiguousarray(topk_idx, dtype=np.int32)
    out = np.zeros((H, D), dtype=np.float64)
    lse = np.zeros(H, dtype=np.float64)
    _check(lib().ref_sparse_swa_attn(cache.ref, b, T, j, H, _ptr(q), _ptr(tk), tk.size, window, sm_scale,
                                     _ptr(out), _ptr(lse)), "sparse_swa_attn")
    return out, lse


def sparse_swa_attn_local(cache, ring_bf16_u16, b, T, j, q_bf16_u16, topk_idx, window, sm_scale=0.0):
    """Sparse attention whose window rows come from a layer-local bf16 ring:
    ring uint16 [batch, ring_len, D] (position t at slot t % ring_len);
    q uint16 [H, D] -> (out fp64 [H, D], lse fp64 [H])."""
    ring = np.ascontiguousarray(ring_bf16_u16, dtype=np.uint16)
    q = np.ascontiguousarray(q_bf16_u16, dtype=np.uint16)
    H, D = q.shape
    tk = np.ascontiguousarray(topk_idx, dtype=np.int32)
    out = np.zeros((H, D), dtype=np.float64)
    lse = np.zeros(H, dtype=np.float64)
    _check(lib().ref_sparse_swa_attn_local(cache.ref, _ptr(ring), ring.shape[1], b, T, j, H, _ptr(q), _ptr(tk),
                                           tk.size, window, sm_scale, _ptr(out), _ptr(lse)),
           "sparse_swa_attn_local")
    return out, lse


def lse_merge(outs, lses):
    """Merge attention partials over disjoint parts of one attended set:
    outs [n, H, D], lses [n, H] -> (out [H, D], lse [H])."""
    outs = np.ascontiguousarray(outs, dtype=np.float64)
    lses = np.ascontiguousarray(lses, dtype=np.float64)
    n, H, D = outs.shape
    out = np.zeros((H, D), dtype=np.float64)
    lse = np.zeros(H, dtype=np.float64)
    _check(lib().ref_lse_merge(n, H, D, _ptr(outs), _ptr(lses), _ptr(out), _ptr(lse)), "lse_merge")
    return out, lse


def dense_attn(cache, b, T, j, q_bf16_u16, sm_scale=0.0):
    q = np.ascontiguousarray(q_bf16_u16, dtype=np.uint16)
    H, D = q.shape
    out = np.zeros((H, D), dtype=np.float64)
    lse = np.zeros(H, dtype=np.float64)
    _check(lib().ref_dense_attn(cache.ref, b, T, j, H, _ptr(q), sm_scale, _ptr(out), _ptr(lse)), "dense_attn")
    return out, lse


# --------------------------------------------------------------------------- layer stack
FULL, REINDEX, REUSE = "F", "R", "U"


def run_stack(cache, pattern, layers, T, pool_k, top_k, window, q_idx_dtype, sm_scale=0.0, tokens=None,
              batches=None):
    """Run a layer pattern (e.g. "FRUU") for every sequence b and query token j.

    layers[l] is a dict with 'q' (uint16 [B, T, H, D]), and for F/R layers
    'q_idx' ([B, T, H_I, D_I]) and 'w' (float32 [B, T, H_I]).  A Reindex layer
    rescores the pool of the most recent Full layer; a Reuse layer attends with
    the top-k of the most recent Full or Reindex layer, unchanged.
    Returns per layer a dict of {(b, j): (pool|None, topk, out, lse)}.
    """
    batches = range(cache.batch) if batches is None else batches
    tokens = range(T) if tokens is None else tokens
    results = []
    pool = {}
    topk = {}
    for l, mode in enumerate(pattern):
        L = layers[l]
        res = {}
        for b in batches:
            for j in tokens:
                key = (b, j)
                if mode == FULL:
                    pool[key], topk[key], _ = index_full(cache, b, T, j, L["q_idx"][b, j], q_idx_dtype,
                                                         L["w"][b, j], pool_k, top_k)
                elif mode == REINDEX:
                    topk[key], _ = index_reindex(cache, b, T, j, L["q_idx"][b, j], q_idx_dtype, L["w"][b, j],
                                                 pool[key], top_k)
                out, lse = sparse_swa_attn(cache, b, T, j, L["q"][b, j], topk[key], window, sm_scale)
                res[key] = (pool.get(key) if mode == FULL else None, topk[key].copy(), out, lse)
        results.append(res)
    return results

"""Python binding of libcsa2 (include/csa2.h): the CSA2 decode-time attention
step over an FP4 global KV cache on one B200.

The binding only marshals arguments: torch tensors provide device memory and
streams, every step of the path runs in the CUDA library.  Function names match
the C ABI without the ``csa2_`` prefix.  There is no CPU fallback: without the
built library every call raises.
"""
import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# CSA2_LIBRARY=debug selects the debug build (NVTX ranges, device-side bounds
# checks); it is never loaded otherwise
LIB_PATH = os.path.join(HERE, "libcsa2_debug.so" if os.environ.get("CSA2_LIBRARY") == "debug" else "libcsa2.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE_BOUNDS = range(6)
FULL, REINDEX, REUSE = 0, 1, 2
F32, BF16, E4M3 = 0, 1, 2

ABI_FUNCTIONS = (
    "csa2_workspace_bytes", "csa2_workspace_init", "csa2_kv_append_quant", "csa2_kv_export_rows",
    "csa2_kv_import_rows", "csa2_index_scores", "csa2_index_full",
    "csa2_index_reindex", "csa2_index_reindex_noalloc", "csa2_index_pool_update", "csa2_sparse_swa_attn",
    "csa2_ring_append",
    "csa2_sparse_swa_attn_local", "csa2_layer_step", "csa2_prefill_workspace_bytes", "csa2_prefill_layer",
    "csa2_cp_index_local", "csa2_cp_reindex_local", "csa2_cp_reindex_select", "csa2_cp_merge_workspace_bytes",
    "csa2_cp_merge_select",
    "csa2_cp_sparse_swa_attn", "csa2_lse_merge",
    "csa2_read_device_status", "csa2_status_string", "csa2_debug_set_wait_limit", "csa2_debug_default_wait_limit",
    "csa2_debug_encode",
)


class CSA2Error(RuntimeError):
    def __init__(self, code, what):
        super().__init__("%s: %s" % (what, status_string(code)))
        self.code = code


class csa2_cache(ctypes.Structure):
    _fields_ = [
        ("kv_rows", ctypes.c_void_p), ("idx_keys", ctypes.c_void_p), ("page_table", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p), ("batch", ctypes.c_int32), ("max_pages", ctypes.c_int32),
        ("page_size", ctypes.c_int32), ("dim", ctypes.c_int32), ("idx_dim", ctypes.c_int32),
        ("row_stride", ctypes.c_int32), ("seq_stride_slots", ctypes.c_int64), ("n_slots", ctypes.c_int64),
        ("idx_key_dtype", ctypes.c_int),
    ]


class csa2_layer_args(ctypes.Structure):
    _fields_ = [
        ("mode", ctypes.c_int), ("q", ctypes.c_void_p), ("q_idx", ctypes.c_void_p), ("q_idx_dtype", ctypes.c_int),
        ("head_w", ctypes.c_void_p), ("T", ctypes.c_int), ("H", ctypes.c_int), ("H_I", ctypes.c_int),
        ("pool_k", ctypes.c_int), ("top_k", ctypes.c_int), ("window", ctypes.c_int), ("sm_scale", ctypes.c_float),
        ("pool_idx", ctypes.c_void_p), ("topk_idx", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("lse", ctypes.c_void_p), ("ring", ctypes.c_void_p), ("ring_len", ctypes.c_int64),
    ]


_lib = None


def lib():
    """The loaded libcsa2.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("%s is not built; run `python -m fp4_sparse_attention_csa2_b200.build%s`"
                               % (os.path.basename(LIB_PATH), " --debug" if "debug" in LIB_PATH else ""))
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        cp = ctypes.POINTER(csa2_cache)
        L.csa2_workspace_bytes.restype = sz
        L.csa2_workspace_bytes.argtypes = [cp, i32, i32, i32, i32, i32]
        L.csa2_workspace_init.argtypes = [vp, sz, vp]
        L.csa2_kv_append_quant.argtypes = [cp, vp, vp, i32, vp, i32, vp, vp]
        L.csa2_kv_export_rows.argtypes = [cp, vp, i32, vp, vp, vp, vp]
        L.csa2_kv_import_rows.argtypes = [cp, vp, i32, vp, vp, vp, vp]
        L.csa2_index_scores.argtypes = [cp, vp, i32, vp, i32, i32, vp, vp, sz, vp]
        L.csa2_index_full.argtypes = [cp, vp, i32, vp, i32, i32, i32, i32, vp, vp, vp, sz, vp]
        L.csa2_index_reindex.argtypes = [cp, vp, i32, vp, i32, i32, vp, i32, i32, vp, vp, sz, vp]
        L.csa2_index_reindex_noalloc.argtypes = [cp, vp, i32, vp, i32, i32, vp, i32, i32, vp, vp]
        L.csa2_index_pool_update.argtypes = [cp, vp, i32, vp, i32, i32, vp, i32, i32, i32, vp, vp, vp, sz, vp]
        L.csa2_sparse_swa_attn.argtypes = [cp, vp, i32, i32, vp, i32, i32, ctypes.c_float, vp, vp, vp, sz, vp]
        L.csa2_ring_append.argtypes = [cp, vp, ctypes.c_int64, vp, vp, i32, vp]
        L.csa2_sparse_swa_attn_local.argtypes = [cp, vp, ctypes.c_int64, vp, i32, i32, vp, i32, i32, ctypes.c_float,
                                                 vp, vp, vp, sz, vp]
        L.csa2_layer_step.argtypes = [cp, ctypes.POINTER(csa2_layer_args), vp, sz, vp]
        L.csa2_prefill_workspace_bytes.restype = sz
        L.csa2_prefill_workspace_bytes.argtypes = [cp, i32, i32, i32, i32, i32, i32]
        L.csa2_prefill_layer.argtypes = [cp, ctypes.POINTER(csa2_layer_args), vp, sz, vp]
        L.csa2_cp_index_local.argtypes = [cp, vp, vp, i32, vp, i32, i32, vp, vp, sz, vp]
        L.csa2_cp_reindex_local.argtypes = [cp, vp, vp, i32, vp, i32, vp, i32, vp, vp, sz, vp]
        L.csa2_cp_reindex_select.argtypes = [vp, vp, i32, i32, vp, i32, vp, vp]
        L.csa2_cp_merge_workspace_bytes.restype = sz
        L.csa2_cp_merge_workspace_bytes.argtypes = [i32, i32, i32]
        L.csa2_cp_merge_select.argtypes = [vp, i32, i32, i32, vp, i32, vp, i32, vp, vp, sz, vp]
        L.csa2_cp_sparse_swa_attn.argtypes = [cp, vp, vp, vp, i32, vp, i32, i32, ctypes.c_float, vp, vp, vp, sz, vp]
        L.csa2_lse_merge.argtypes = [i32, i32, i32, i32, vp, ctypes.c_int64, vp, ctypes.c_int64, vp, vp, vp]
        L.csa2_read_device_status.argtypes = [vp, vp]
        L.csa2_status_string.restype = ctypes.c_char_p
        L.csa2_status_string.argtypes = [i32]
        L.csa2_debug_set_wait_limit.argtypes = [ctypes.c_uint32]
        L.csa2_debug_default_wait_limit.restype = ctypes.c_uint32
        L.csa2_debug_default_wait_limit.argtypes = []
        L.csa2_debug_encode.argtypes = [i32, vp, ctypes.c_int64, vp, vp]
        for name in ("csa2_workspace_init", "csa2_kv_append_quant", "csa2_kv_export_rows", "csa2_kv_import_rows",
                     "csa2_index_scores", "csa2_index_full",
                     "csa2_index_reindex", "csa2_index_reindex_noalloc", "csa2_index_pool_update",
                     "csa2_sparse_swa_attn", "csa2_ring_append", "csa2_sparse_swa_attn_local",
                     "csa2_layer_step", "csa2_prefill_layer", "csa2_read_device_status",
                     "csa2_debug_set_wait_limit", "csa2_cp_index_local", "csa2_cp_reindex_local", "csa2_cp_reindex_select",
                     "csa2_cp_merge_select", "csa2_cp_sparse_swa_attn", "csa2_lse_merge",
                     "csa2_debug_encode"):
            getattr(L, name).restype = i32
        _lib = L
    return _lib


def status_string(code):
    return lib().csa2_status_string(int(code)).decode()


def _check(code, what):
    if code != OK:
        raise CSA2Error(code, what)


def _p(t):
    """Device pointer of a tensor the library reads or writes: a contiguous
    CUDA tensor (a host tensor would hand the kernels a host address)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libcsa2 takes CUDA tensors; got one on %s" % t.device)
    if not t.is_contiguous():
        raise ValueError("libcsa2 takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _addr(t):
    p = _p(t)
    return None if p is None else p.value


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class Cache:
    """The global cache of one stack on one device: FP4 rows, index keys, page
    table and sequence lengths (all device tensors owned by this object)."""

    def __init__(self, batch, n_slots, dim, idx_dim, row_stride, idx_key_dtype, seq_lens, page_table=None,
                 page_size=64, seq_stride_slots=0, device="cuda"):
        if torch.device(device).type != "cuda":
            raise ValueError("the cache lives in device memory; got device %s" % device)
        self.rows = torch.zeros((n_slots, row_stride), dtype=torch.uint8, device=device)
        kd = torch.uint8 if idx_key_dtype == E4M3 else torch.float32
        self.idx_keys = torch.zeros((n_slots, idx_dim), dtype=kd, device=device)
        self.seq_lens = torch.as_tensor(seq_lens, dtype=torch.int32).to(device).contiguous()
        self.page_table = None if page_table is None else \
            torch.as_tensor(page_table, dtype=torch.int32).to(device).contiguous()
        self.batch, self.dim, self.idx_dim, self.idx_key_dtype = batch, dim, idx_dim, idx_key_dtype
        self.page_size, self.row_stride, self.n_slots = page_size, row_stride, n_slots
        self.seq_stride_slots = seq_stride_slots
        self.c = csa2_cache(
            self.rows.data_ptr(), self.idx_keys.data_ptr(),
            None if self.page_table is None else self.page_table.data_ptr(), self.seq_lens.data_ptr(), batch,
            0 if self.page_table is None else self.page_table.shape[1], page_size, dim, idx_dim, row_stride,
            seq_stride_slots, n_slots, idx_key_dtype)

    @property
    def ref(self):
        return ctypes.byref(self.c)

    def view(self, b):
        """A batch-1 cache of sequence b sharing this cache's memory."""
        v = _View()
        c = self.c
        if self.page_table is None:
            st = self.seq_stride_slots
            v.c = csa2_cache(c.kv_rows + b * st * self.row_stride,
                             c.idx_keys + b * st * self.idx_dim * self.idx_keys.element_size(), None,
                             c.seq_lens + 4 * b, 1, 0, c.page_size, c.dim, c.idx_dim, c.row_stride, st, st,
                             c.idx_key_dtype)
        else:
            v.c = csa2_cache(c.kv_rows, c.idx_keys, c.page_table + 4 * b * c.max_pages, c.seq_lens + 4 * b, 1,
                             c.max_pages, c.page_size, c.dim, c.idx_dim, c.row_stride, 0, c.n_slots,
                             c.idx_key_dtype)
        v.owner = self
        return v

    def shard_view(self, b, pos0, n):
        """A batch-1 cache whose positions 0 .. n-1 are positions pos0 ..
        pos0 + n - 1 of sequence b of this cache (sharing its memory; its own
        seq_lens = [n]): one rank's shard for the context-parallel calls.
        pos0 must be a multiple of 64 (of the page size when paged)."""
        c = self.c
        v = _View()
        v.lens = torch.tensor([n], dtype=torch.int32, device=self.rows.device)
        if self.page_table is None:
            if pos0 % 64 or pos0 + n > self.seq_stride_slots:
                raise ValueError("shard outside the sequence or not 64-aligned")
            st = self.seq_stride_slots - pos0
            base = b * self.seq_stride_slots + pos0
            v.c = csa2_cache(c.kv_rows + base * self.row_stride,
                             c.idx_keys + base * self.idx_dim * self.idx_keys.element_size(), None,
                             v.lens.data_ptr(), 1, 0, c.page_size, c.dim, c.idx_dim, c.row_stride, st,
                             self.n_slots - base, c.idx_key_dtype)
        else:
            if pos0 % self.page_size or pos0 + n > self.capacity:
                raise ValueError("a paged shard starts on a page boundary and ends within the sequence's pages")
            first = pos0 // self.page_size
            v.c = csa2_cache(c.kv_rows, c.idx_keys, c.page_table + 4 * (b * c.max_pages + first), v.lens.data_ptr(),
                             1, c.max_pages - first, c.page_size, c.dim, c.idx_dim, c.row_stride, 0, c.n_slots,
                             c.idx_key_dtype)
        v.owner = self
        v.batch, v.dim = 1, self.dim
        return v

    @property
    def capacity(self):
        return self.page_table.shape[1] * self.page_size if self.page_table is not None else self.seq_stride_slots


class _View:
    @property
    def ref(self):
        return ctypes.byref(self.c)


def workspace_bytes(cache, T, H, pool_k, top_k, window):
    n = lib().csa2_workspace_bytes(cache.ref, T, H, pool_k, top_k, window)
    if n == 0:
        raise CSA2Error(ERR_INVALID_ARG, "workspace_bytes")
    return n


def workspace_init(ws, stream=None):
    _check(lib().csa2_workspace_init(_p(ws), ws.numel() * ws.element_size(), _stream(stream)), "workspace_init")


def kv_append_quant(cache, x, start_pos, idx_new=None, ws=None, stream=None):
    """x: bf16 [B, n_new, dim]; idx_new: bf16/fp32 [B, n_new, idx_dim]; start_pos: int32 [B] (device)."""
    dt = F32 if (idx_new is not None and idx_new.dtype == torch.float32) else BF16
    _check(lib().csa2_kv_append_quant(cache.ref, _p(x), _p(idx_new), dt, _p(start_pos), x.shape[1], _p(ws),
                                      _stream(stream)), "kv_append_quant")


def kv_export_rows(cache, start_pos, n, rows, keys=None, ws=None, stream=None):
    """Stored rows [B, n, dim/2 + dim/16] uint8 (and keys [B, n, key bytes])
    of positions start_pos[b] + i, copied out of the cache."""
    _check(lib().csa2_kv_export_rows(cache.ref, _p(start_pos), n, _p(rows), _p(keys), _p(ws), _stream(stream)),
           "kv_export_rows")


def kv_import_rows(cache, start_pos, n, rows, keys=None, ws=None, stream=None):
    """The inverse of kv_export_rows: the buffers written back into the cache."""
    _check(lib().csa2_kv_import_rows(cache.ref, _p(start_pos), n, _p(rows), _p(keys), _p(ws), _stream(stream)),
           "kv_import_rows")


def _qdt(q_idx):
    return F32 if q_idx.dtype == torch.float32 else BF16


def index_scores(cache, q_idx, head_w, ws, scores=None, stream=None):
    """Full-layer scores of every visible position: into `scores` (fp32
    [B, T, capacity]) or, when None, into the workspace."""
    B, T, H_I, _ = q_idx.shape
    _check(lib().csa2_index_scores(cache.ref, _p(q_idx), _qdt(q_idx), _p(head_w), T, H_I, _p(scores), _p(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)), "index_scores")


def index_full(cache, q_idx, head_w, pool_k, top_k, pool_idx, topk_idx, ws, stream=None):
    """q_idx [B, T, H_I, idx_dim]; head_w fp32 [B, T, H_I]; writes pool_idx [B, T, pool_k], topk_idx [B, T, top_k]."""
    B, T, H_I, _ = q_idx.shape
    _check(lib().csa2_index_full(cache.ref, _p(q_idx), _qdt(q_idx), _p(head_w), T, H_I, pool_k, top_k, _p(pool_idx),
                                 _p(topk_idx), _p(ws), ws.numel() * ws.element_size(), _stream(stream)), "index_full")


def index_reindex(cache, q_idx, head_w, pool_idx, top_k, topk_idx, ws, stream=None):
    B, T, H_I, _ = q_idx.shape
    _check(lib().csa2_index_reindex(cache.ref, _p(q_idx), _qdt(q_idx), _p(head_w), T, H_I, _p(pool_idx),
                                    pool_idx.shape[-1], top_k, _p(topk_idx), _p(ws), ws.numel() * ws.element_size(),
                                    _stream(stream)), "index_reindex")


def index_reindex_noalloc(cache, q_idx, head_w, pool_idx, top_k, topk_idx, stream=None):
    """csa2_index_reindex for callers that cannot hand over a workspace: the
    scratch is a fixed array inside the library (see include/csa2.h)."""
    B, T, H_I, _ = q_idx.shape
    _check(lib().csa2_index_reindex_noalloc(cache.ref, _p(q_idx), _qdt(q_idx), _p(head_w), T, H_I, _p(pool_idx),
                                            pool_idx.shape[-1], top_k, _p(topk_idx), _stream(stream)),
           "index_reindex_noalloc")


def index_pool_update(cache, q_idx, head_w, pool_prev, n_new, top_k, pool_idx, topk_idx, ws, stream=None):
    """The pool of an in-flight request after its last n_new positions were
    appended: the best of pool_prev [B, T, pool_k] and the new positions, into
    pool_idx [B, T, pool_k] (may be pool_prev) and topk_idx [B, T, top_k]."""
    B, T, H_I, _ = q_idx.shape
    _check(lib().csa2_index_pool_update(cache.ref, _p(q_idx), _qdt(q_idx), _p(head_w), T, H_I, _p(pool_prev),
                                        pool_prev.shape[-1], n_new, top_k, _p(pool_idx), _p(topk_idx), _p(ws),
                                        ws.numel() * ws.element_size(), _stream(stream)), "index_pool_update")


def sparse_swa_attn(cache, q, topk_idx, window, out, lse=None, ws=None, sm_scale=0.0, stream=None):
    """q bf16 [B, T, H, dim]; topk_idx int32 [B, T, top_k]; out fp32 [B, T, H, dim]; lse fp32 [B, T, H]."""
    B, T, H, _ = q.shape
    top_k = topk_idx.shape[-1] if topk_idx is not None else 0
    _check(lib().csa2_sparse_swa_attn(cache.ref, _p(q), T, H, _p(topk_idx), top_k, window, sm_scale, _p(out), _p(lse),
                                      _p(ws), ws.numel() * ws.element_size(), _stream(stream)), "sparse_swa_attn")


def ring_append(cache, ring, x, start_pos, stream=None):
    """Rows x bf16 [B, n_new, dim] of positions start_pos[b] + i into the
    layer's ring bf16 [B, ring_len, dim] (row t mod ring_len)."""
    _check(lib().csa2_ring_append(cache.ref, _p(ring), ring.shape[1], _p(x), _p(start_pos), x.shape[1],
                                  _stream(stream)), "ring_append")


def sparse_swa_attn_local(cache, ring, q, topk_idx, window, out, lse=None, ws=None, sm_scale=0.0, stream=None):
    """sparse_swa_attn with the window rows from the layer's bf16 ring [B, ring_len, dim]."""
    B, T, H, _ = q.shape
    top_k = topk_idx.shape[-1] if topk_idx is not None else 0
    _check(lib().csa2_sparse_swa_attn_local(cache.ref, _p(ring), ring.shape[1], _p(q), T, H, _p(topk_idx), top_k,
                                            window, sm_scale, _p(out), _p(lse), _p(ws),
                                            ws.numel() * ws.element_size(), _stream(stream)),
           "sparse_swa_attn_local")


def layer_step(cache, mode, q, topk_idx, out, ws, window, q_idx=None, head_w=None, pool_idx=None, lse=None,
               pool_k=0, sm_scale=0.0, ring=None, stream=None):
    B, T, H, _ = q.shape
    H_I = q_idx.shape[2] if q_idx is not None else 0
    a = csa2_layer_args(mode, _addr(q), _addr(q_idx), _qdt(q_idx) if q_idx is not None else BF16, _addr(head_w),
                        T, H, H_I, pool_k or (pool_idx.shape[-1] if pool_idx is not None else 0), topk_idx.shape[-1],
                        window, sm_scale, _addr(pool_idx), _addr(topk_idx), _addr(out), _addr(lse), _addr(ring),
                        0 if ring is None else ring.shape[1])
    _check(lib().csa2_layer_step(cache.ref, ctypes.byref(a), _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "layer_step")


def prefill_workspace_bytes(cache, T, H, H_I, pool_k, top_k, window):
    n = lib().csa2_prefill_workspace_bytes(cache.ref, T, H, H_I, pool_k, top_k, window)
    if n == 0:
        raise CSA2Error(ERR_INVALID_ARG, "prefill_workspace_bytes")
    return n


def prefill_layer(cache, mode, q, topk_idx, out, ws, window, q_idx=None, head_w=None, pool_idx=None, lse=None,
                  pool_k=0, sm_scale=0.0, ring=None, H_I=None, stream=None):
    """One layer for all T query tokens of q [B, T, H, dim] (any T), in
    chunks; arguments as layer_step, plus the stack's indexer head count H_I
    (taken from q_idx when given; required for Reuse layers)."""
    B, T, H, _ = q.shape
    H_I = q_idx.shape[2] if q_idx is not None else H_I
    a = csa2_layer_args(mode, _addr(q), _addr(q_idx), _qdt(q_idx) if q_idx is not None else BF16, _addr(head_w),
                        T, H, H_I, pool_k or (pool_idx.shape[-1] if pool_idx is not None else 0), topk_idx.shape[-1],
                        window, sm_scale, _addr(pool_idx), _addr(topk_idx), _addr(out), _addr(lse), _addr(ring),
                        0 if ring is None else ring.shape[1])
    _check(lib().csa2_prefill_layer(cache.ref, ctypes.byref(a), _p(ws), ws.numel() * ws.element_size(),
                                    _stream(stream)), "prefill_layer")


# ---------------------------------------------------------------- context-parallel decode
# A candidate (csa2_cand) is held as int32 [..., 2]: the global position and
# the bits of its fp32 score.

def cand_buffer(batch, n, device="cuda"):
    """Candidates [batch, n] (int32 pairs: position, score bits)."""
    return torch.empty((batch, n, 2), dtype=torch.int32, device=device)


def cand_scores(cand):
    """The fp32 scores of a candidate buffer."""
    return cand.view(torch.float32)[..., 1]


def cp_index_local(shard, pos0, q_idx, head_w, pool_k, cand, ws, stream=None):
    """A Full layer's share on a shard: its pool_k best positions (global,
    pos0 [B] int32 added) with their scores into cand [B, pool_k, 2].  q_idx
    [B, 1, H_I, idx_dim]; head_w [B, 1, H_I]."""
    B, T, H_I, _ = q_idx.shape
    if T != 1:
        raise ValueError("context-parallel calls take one query token per sequence")
    _check(lib().csa2_cp_index_local(shard.ref, _p(pos0), _p(q_idx), _qdt(q_idx), _p(head_w), H_I, pool_k, _p(cand),
                                     _p(ws), ws.numel() * ws.element_size(), _stream(stream)), "cp_index_local")


def cp_reindex_local(shard, pos0, q_idx, head_w, pool_idx, pool_scores, ws, stream=None):
    """A Reindex layer's share on a shard: pool_scores fp32 [B, pool_k] <- the
    scores of the global pool entries it holds, 0 for the others (summed over
    the ranks, every entry carries its owner's score)."""
    B, T, H_I, _ = q_idx.shape
    if T != 1:
        raise ValueError("context-parallel calls take one query token per sequence")
    _check(lib().csa2_cp_reindex_local(shard.ref, _p(pos0), _p(q_idx), _qdt(q_idx), _p(head_w), H_I, _p(pool_idx),
                                       pool_idx.shape[-1], _p(pool_scores), _p(ws), ws.numel() * ws.element_size(),
                                       _stream(stream)), "cp_reindex_local")


def cp_reindex_select(pool_idx, pool_scores, seq_lens_global, top_k, topk_idx, stream=None):
    """The top_k best entries of pool_idx [B, pool_k] by the summed
    pool_scores into topk_idx [B, top_k]."""
    B, pool_k = pool_idx.shape[0], pool_idx.shape[-1]
    _check(lib().csa2_cp_reindex_select(_p(pool_idx), _p(pool_scores), B, pool_k, _p(seq_lens_global), top_k,
                                        _p(topk_idx), _stream(stream)), "cp_reindex_select")


def cp_merge_workspace_bytes(R, batch, n_cand):
    n = lib().csa2_cp_merge_workspace_bytes(R, batch, n_cand)
    if n == 0:
        raise CSA2Error(ERR_INVALID_ARG, "cp_merge_workspace_bytes")
    return n


def cp_merge_select(cand, seq_lens_global, n_a, out_a, ws, n_b=0, out_b=None, stream=None):
    """The selection after the all-gather: cand [R, B, n_cand, 2]; the n_a best
    positions into out_a [B, n_a] and the n_b best into out_b [B, n_b]."""
    R, B, n_cand, _ = cand.shape
    _check(lib().csa2_cp_merge_select(_p(cand), R, B, n_cand, _p(seq_lens_global), n_a, _p(out_a), n_b, _p(out_b),
                                      _p(ws), ws.numel() * ws.element_size(), _stream(stream)), "cp_merge_select")


def cp_sparse_swa_attn(shard, pos0, seq_lens_global, q, topk_idx, window, out, lse, ws, sm_scale=0.0, stream=None):
    """A layer's attention on a shard: its part of window ∪ top-k (topk_idx
    global [B, top_k]); out fp32 [B, H, dim], lse fp32 [B, H] of that part."""
    B, H = q.shape[0], q.shape[-2]
    top_k = topk_idx.shape[-1] if topk_idx is not None else 0
    _check(lib().csa2_cp_sparse_swa_attn(shard.ref, _p(pos0), _p(seq_lens_global), _p(q), H, _p(topk_idx), top_k,
                                         window, sm_scale, _p(out), _p(lse), _p(ws), ws.numel() * ws.element_size(),
                                         _stream(stream)), "cp_sparse_swa_attn")


def lse_merge(outs, lses, out, lse=None, stream=None):
    """Merge R attention parts: outs [R, B, H, dim] and lses [R, B, H] (views
    of one buffer allowed: any rank stride) into out [B, H, dim], lse [B, H]."""
    R, B, H, D = outs.shape
    for t in (outs, lses):
        if not t.is_cuda:
            raise ValueError("libcsa2 takes CUDA tensors; got one on %s" % t.device)
        if not t[0].is_contiguous():
            raise ValueError("each part must be contiguous")
    _check(lib().csa2_lse_merge(R, B, H, D, ctypes.c_void_p(outs.data_ptr()), outs.stride(0),
                                ctypes.c_void_p(lses.data_ptr()), lses.stride(0), _p(out), _p(lse), _stream(stream)),
           "lse_merge")


def debug_encode(x, codes, fmt, stream=None):
    """Diagnostic: the quantiser's E2M1 (fmt 0) or E4M3 (fmt 1) conversion of
    every fp32 value of x into codes (uint8, same length)."""
    _check(lib().csa2_debug_encode(fmt, _p(x), x.numel(), _p(codes), _stream(stream)), "debug_encode")


def read_device_status(ws, stream=None):
    """Synchronise and return (then clear) the sticky device status code."""
    return lib().csa2_read_device_status(_p(ws), _stream(stream))


def debug_set_wait_limit(tries=None):
    """Diagnostic: tries of the bounded waits that guard work in the tensor-core
    kernels launched from now on (None restores the default; 0 makes them give
    up at once and record TIMEOUT).  Returns the default."""
    L = lib()
    default = int(L.csa2_debug_default_wait_limit())
    _check(L.csa2_debug_set_wait_limit(default if tries is None else int(tries)), "debug_set_wait_limit")
    return default

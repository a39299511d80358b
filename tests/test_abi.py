"""The C-ABI library loads on a host without a GPU, exports every function
include/csa2.h declares, and rejects bad arguments on the host before it
launches anything (these calls never reach the device)."""
import ctypes
import os
import re

import pytest
import torch

import fp4_sparse_attention_csa2_b200 as csa2
from fp4_sparse_attention_csa2_b200 import build as _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "csa2.h")).read()
    return re.findall(r"CSA2_API\s+[\w\s\*]+?\b(csa2_\w+)\s*\(", src)


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return csa2.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 9
    assert set(names) == set(csa2.ABI_FUNCTIONS)
    handle = ctypes.CDLL(csa2.LIB_PATH)
    for n in names:
        assert hasattr(handle, n), n


def test_debug_build_exports_every_symbol():
    # the debug variant (NVTX ranges, device-side bounds checks) has the same ABI
    path = _build.build(debug=True)
    handle = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(handle, n), n


def test_status_strings(lib):
    for code, name in enumerate(["CSA2_OK", "CSA2_ERR_INVALID_ARG", "CSA2_ERR_UNSUPPORTED", "CSA2_ERR_CUDA",
                                 "CSA2_ERR_TIMEOUT", "CSA2_ERR_DEVICE_BOUNDS"]):
        assert csa2.status_string(code) == name


def fake_cache(**kw):
    d = dict(kv_rows=0x10000, idx_keys=0x20000, page_table=None, seq_lens=0x30000, batch=1, max_pages=0,
             page_size=64, dim=512, idx_dim=64, row_stride=288, seq_stride_slots=1 << 20, n_slots=1 << 20,
             idx_key_dtype=csa2.E4M3)
    d.update(kw)
    return csa2.csa2_cache(**d)


def test_workspace_bytes_layout(lib):
    c = fake_cache()
    n = lib.csa2_workspace_bytes(ctypes.byref(c), 1, 64, 16384, 2048, 128)
    # scores (4 MiB) + two candidate lists (8 MiB) + partials of 68 chunks x 64 x 512 fp32
    assert n >= 4 * (1 << 20) * 3 + 68 * 64 * 512 * 4
    assert n % 256 == 0
    assert lib.csa2_workspace_bytes(ctypes.byref(fake_cache(dim=100)), 1, 64, 16384, 2048, 128) == 0
    assert lib.csa2_workspace_bytes(ctypes.byref(fake_cache(row_stride=280)), 1, 64, 16384, 2048, 128) == 0
    assert lib.csa2_workspace_bytes(None, 1, 64, 16384, 2048, 128) == 0


@pytest.mark.parametrize("pool_k,top_k,H_I,T", [(16385, 128, 32, 1), (100, 200, 32, 1), (512, 0, 32, 1),
                                                (512, 128, 65, 1), (512, 128, 32, 9)])
def test_index_bounds_rejected_on_host(lib, pool_k, top_k, H_I, T):
    c = fake_cache()
    rc = lib.csa2_index_full(ctypes.byref(c), 0x40000, csa2.BF16, 0x50000, T, H_I, pool_k, top_k, 0x60000, 0x70000,
                             0x80000, 1 << 40, None)
    assert rc == csa2.ERR_INVALID_ARG


def test_bad_pointers_rejected_on_host(lib):
    c = fake_cache()
    assert lib.csa2_index_full(ctypes.byref(c), None, csa2.BF16, 0x50000, 1, 32, 512, 128, 0x60000, 0x70000,
                               0x80000, 1 << 40, None) == csa2.ERR_INVALID_ARG
    assert lib.csa2_index_full(ctypes.byref(c), 0x40008, csa2.BF16, 0x50000, 1, 32, 512, 128, 0x60000, 0x70000,
                               0x80000, 1 << 40, None) == csa2.ERR_INVALID_ARG
    # wrong query dtype for an E4M3 cache
    assert lib.csa2_index_full(ctypes.byref(c), 0x40000, csa2.F32, 0x50000, 1, 32, 512, 128, 0x60000, 0x70000,
                               0x80000, 1 << 40, None) == csa2.ERR_INVALID_ARG
    # workspace too small
    assert lib.csa2_index_full(ctypes.byref(c), 0x40000, csa2.BF16, 0x50000, 1, 32, 512, 128, 0x60000, 0x70000,
                               0x80000, 1024, None) == csa2.ERR_INVALID_ARG
    assert lib.csa2_sparse_swa_attn(ctypes.byref(c), 0x40000, 1, 128, 0x60000, 2048, 128, 0.0, 0x70000, None,
                                    0x80000, 1 << 40, None) == csa2.ERR_UNSUPPORTED
    assert lib.csa2_kv_append_quant(ctypes.byref(fake_cache(dim=1024)), 0x40000, None, csa2.BF16, 0x50000, 8,
                                    None, None) == csa2.ERR_UNSUPPORTED
    bad_mode = csa2.csa2_layer_args(mode=7)
    assert lib.csa2_layer_step(ctypes.byref(c), ctypes.byref(bad_mode), 0x80000, 1 << 40, None) == \
        csa2.ERR_INVALID_ARG


def test_host_tensors_are_refused_before_any_launch(lib):
    # no CPU fallback: a host tensor never reaches the library as a pointer
    with pytest.raises(ValueError):
        csa2.workspace_init(torch.empty(4096, dtype=torch.uint8))
    with pytest.raises(ValueError):
        csa2.Cache(1, 64, 128, 64, 80, csa2.E4M3, [64], seq_stride_slots=64, device="cpu")


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(csa2, "_lib", None)
    monkeypatch.setattr(csa2, "LIB_PATH", str(tmp_path / "libcsa2.so"))
    with pytest.raises(RuntimeError):
        csa2.lib()


def test_attention_bounds_rejected_on_host(lib):
    # window or top-k beyond the 16,384 bound: invalid on any path
    c = fake_cache()
    assert lib.csa2_sparse_swa_attn(ctypes.byref(c), 0x40000, 1, 64, 0x60000, 2048, 16385, 0.0, 0x70000, None,
                                    0x80000, 1 << 40, None) == csa2.ERR_INVALID_ARG
    assert lib.csa2_sparse_swa_attn(ctypes.byref(c), 0x40000, 1, 64, 0x60000, 16385, 128, 0.0, 0x70000, None,
                                    0x80000, 1 << 40, None) == csa2.ERR_INVALID_ARG


def test_noalloc_reindex_refuses_like_the_workspace_entry_point(lib):
    # the workspace-free Reindex checks the same arguments as csa2_index_reindex,
    # in the same order and with the same statuses, before its scratch bound
    c = fake_cache()
    args = dict(q=0x40000, dt=csa2.BF16, w=0x50000, T=1, H_I=32, pool=0x60000, pool_k=512, top_k=128, out=0x70000)

    def both(cache=c, **kw):
        a = dict(args)
        a.update(kw)
        r1 = lib.csa2_index_reindex(ctypes.byref(cache), a["q"], a["dt"], a["w"], a["T"], a["H_I"], a["pool"],
                                    a["pool_k"], a["top_k"], a["out"], 0x80000, 1 << 40, None)
        r2 = lib.csa2_index_reindex_noalloc(ctypes.byref(cache), a["q"], a["dt"], a["w"], a["T"], a["H_I"],
                                            a["pool"], a["pool_k"], a["top_k"], a["out"], None)
        return r1, r2

    for kw, want in [(dict(q=0x40008), csa2.ERR_INVALID_ARG), (dict(w=0x50004), csa2.ERR_INVALID_ARG),
                     (dict(pool=0x60004), csa2.ERR_INVALID_ARG), (dict(out=0x70008), csa2.ERR_INVALID_ARG),
                     (dict(pool=None), csa2.ERR_INVALID_ARG), (dict(dt=csa2.F32), csa2.ERR_INVALID_ARG),
                     (dict(pool_k=16385), csa2.ERR_INVALID_ARG), (dict(top_k=600), csa2.ERR_INVALID_ARG),
                     (dict(H_I=65), csa2.ERR_INVALID_ARG), (dict(T=9), csa2.ERR_INVALID_ARG)]:
        assert both(**kw) == (want, want), kw
    # a malformed cache: the cache's own status, not the scratch bound's
    for cache, want in [(fake_cache(dim=1024), csa2.ERR_UNSUPPORTED), (fake_cache(idx_dim=32), csa2.ERR_UNSUPPORTED),
                        (fake_cache(row_stride=280), csa2.ERR_INVALID_ARG)]:
        assert both(cache=cache, T=8, pool_k=16384, top_k=16) == (want, want)
    # beyond the fixed scratch (80 x 16,384 pool scores > 4 MiB) once everything else is valid
    big = fake_cache(batch=80, seq_stride_slots=1 << 14, n_slots=80 << 14)
    assert lib.csa2_index_reindex_noalloc(ctypes.byref(big), 0x40000, csa2.BF16, 0x50000, 1, 32, 0x60000, 16384, 16,
                                          0x70000, None) == csa2.ERR_UNSUPPORTED


def test_ring_arguments_rejected_on_host(lib):
    # the layer-local ring: a ring shorter than window + T - 1, a misaligned or
    # missing ring, and an append of more rows than the ring holds are refused
    c = fake_cache()
    i64 = ctypes.c_int64

    def attn(ring=0x90000, ring_len=128, T=1, window=128):
        return lib.csa2_sparse_swa_attn_local(ctypes.byref(c), ring, i64(ring_len), 0x40000, T, 64, 0x60000, 2048,
                                              window, 0.0, 0x70000, None, 0x80000, 1 << 40, None)

    assert attn(ring_len=127) == csa2.ERR_INVALID_ARG
    assert attn(ring_len=128, T=2) == csa2.ERR_INVALID_ARG
    assert attn(ring=0x90008) == csa2.ERR_INVALID_ARG
    assert attn(ring=None) == csa2.ERR_INVALID_ARG
    assert attn(ring_len=0, window=0) == csa2.ERR_INVALID_ARG
    # a ring long enough: the call goes on to the attention's own checks (window too large here)
    assert attn(ring_len=20000, window=16385) == csa2.ERR_INVALID_ARG

    def append(ring=0x90000, ring_len=128, x=0xA0000, sp=0xB0000, n_new=4):
        return lib.csa2_ring_append(ctypes.byref(c), ring, i64(ring_len), x, sp, n_new, None)

    assert append(n_new=129) == csa2.ERR_INVALID_ARG
    assert append(x=0xA0002) == csa2.ERR_INVALID_ARG
    assert append(sp=None) == csa2.ERR_INVALID_ARG
    assert append(sp=0xB0002) == csa2.ERR_INVALID_ARG
    assert append(n_new=-1) == csa2.ERR_INVALID_ARG
    assert append(n_new=0) == csa2.OK                      # nothing to write: nothing launched
    assert lib.csa2_ring_append(ctypes.byref(fake_cache(dim=100)), 0x90000, i64(128), 0xA0000, 0xB0000, 4,
                                None) == csa2.ERR_INVALID_ARG


def test_pool_update_arguments_rejected_on_host(lib):
    c = fake_cache()

    def call(n_new=8, pool_k=512, top_k=64, out=0x90000, prev=0x60000):
        return lib.csa2_index_pool_update(ctypes.byref(c), 0x40000, csa2.BF16, 0x50000, 1, 32, prev, pool_k, n_new,
                                          top_k, out, 0x70000, 0x80000, 1 << 40, None)

    assert call(n_new=-1) == csa2.ERR_INVALID_ARG
    assert call(n_new=16385) == csa2.ERR_INVALID_ARG
    assert call(out=None) == csa2.ERR_INVALID_ARG
    assert call(out=0x90008) == csa2.ERR_INVALID_ARG
    assert call(prev=None) == csa2.ERR_INVALID_ARG
    assert call(top_k=600) == csa2.ERR_INVALID_ARG
    assert call(pool_k=16385) == csa2.ERR_INVALID_ARG


def test_prefill_workspace_and_arguments(lib):
    c = fake_cache()
    n1 = lib.csa2_prefill_workspace_bytes(ctypes.byref(c), 4, 64, 32, 16384, 2048, 128)
    n2 = lib.csa2_prefill_workspace_bytes(ctypes.byref(c), 8192, 64, 32, 16384, 2048, 128)
    # the workspace holds one chunk of four tokens of one sequence, whatever T is
    assert n1 == n2 > 0
    assert lib.csa2_prefill_workspace_bytes(ctypes.byref(c), 0, 64, 32, 16384, 2048, 128) == 0
    assert lib.csa2_prefill_workspace_bytes(ctypes.byref(c), 4, 64, 65, 16384, 2048, 128) == 0
    a = csa2.csa2_layer_args(mode=csa2.REUSE, q=0x40000, T=0, H=64, H_I=32, top_k=2048, window=128,
                             topk_idx=0x60000, out=0x70000)
    assert lib.csa2_prefill_layer(ctypes.byref(c), ctypes.byref(a), 0x80000, n1, None) == csa2.ERR_INVALID_ARG
    a.T = 16
    assert lib.csa2_prefill_layer(ctypes.byref(c), ctypes.byref(a), 0x80000, 1024, None) == csa2.ERR_INVALID_ARG
    a.H_I = 0                                  # the chunk size needs the stack's indexer heads
    assert lib.csa2_prefill_layer(ctypes.byref(c), ctypes.byref(a), 0x80000, n1, None) == csa2.ERR_INVALID_ARG
    a.H_I = 32
    a.mode = 7
    assert lib.csa2_prefill_layer(ctypes.byref(c), ctypes.byref(a), 0x80000, n1, None) == csa2.ERR_INVALID_ARG


def test_export_import_arguments_rejected_on_host(lib):
    c = fake_cache()
    for fn in (lib.csa2_kv_export_rows, lib.csa2_kv_import_rows):
        assert fn(ctypes.byref(c), None, 4, 0x40000, 0x50000, None, None) == csa2.ERR_INVALID_ARG
        assert fn(ctypes.byref(c), 0x30002, 4, 0x40000, 0x50000, None, None) == csa2.ERR_INVALID_ARG
        assert fn(ctypes.byref(c), 0x30000, -1, 0x40000, 0x50000, None, None) == csa2.ERR_INVALID_ARG
        assert fn(ctypes.byref(c), 0x30000, 4, None, 0x50000, None, None) == csa2.ERR_INVALID_ARG
        assert fn(ctypes.byref(c), 0x30000, 4, 0x40002, 0x50000, None, None) == csa2.ERR_INVALID_ARG
        assert fn(ctypes.byref(c), 0x30000, 0, 0x40000, 0x50000, None, None) == csa2.OK   # nothing to copy


def test_context_parallel_arguments_rejected_on_host(lib):
    c = fake_cache()
    big = 1 << 40

    def local(pos0=0x30100, cand=0x90000, pool_k=16384, H_I=32):
        return lib.csa2_cp_index_local(ctypes.byref(c), pos0, 0x40000, csa2.BF16, 0x50000, H_I, pool_k, cand, 0x80000,
                                       big, None)

    assert local(pos0=None) == csa2.ERR_INVALID_ARG
    assert local(pos0=0x30102) == csa2.ERR_INVALID_ARG
    assert local(cand=None) == csa2.ERR_INVALID_ARG
    assert local(cand=0x90004) == csa2.ERR_INVALID_ARG          # candidates are 8-byte pairs
    assert local(pool_k=16385) == csa2.ERR_INVALID_ARG
    assert local(H_I=65) == csa2.ERR_INVALID_ARG

    def reindex(pool=0x60000, pool_k=16384, scores=0x90000):
        return lib.csa2_cp_reindex_local(ctypes.byref(c), 0x30100, 0x40000, csa2.BF16, 0x50000, 32, pool, pool_k,
                                         scores, 0x80000, big, None)

    assert reindex(pool=None) == csa2.ERR_INVALID_ARG
    assert reindex(pool=0x60004) == csa2.ERR_INVALID_ARG
    assert reindex(pool_k=16385) == csa2.ERR_INVALID_ARG
    assert reindex(scores=None) == csa2.ERR_INVALID_ARG
    assert reindex(scores=0x90004) == csa2.ERR_INVALID_ARG

    def rselect(pool_k=16384, top_k=2048, topk=0xA0000, lens=0x30000, batch=1):
        return lib.csa2_cp_reindex_select(0x60000, 0x90000, batch, pool_k, lens, top_k, topk, None)

    assert rselect(top_k=0) == csa2.ERR_INVALID_ARG
    assert rselect(top_k=16385, pool_k=16385) == csa2.ERR_INVALID_ARG
    assert rselect(top_k=4096, pool_k=2048) == csa2.ERR_INVALID_ARG
    assert rselect(topk=None) == csa2.ERR_INVALID_ARG
    assert rselect(topk=0xA0004) == csa2.ERR_INVALID_ARG
    assert rselect(lens=None) == csa2.ERR_INVALID_ARG
    assert rselect(batch=0) == csa2.ERR_INVALID_ARG

    # the merge workspace: histograms, four candidate buffers and the per-sequence candidates
    n = lib.csa2_cp_merge_workspace_bytes(8, 1, 16384)
    assert n >= 8 * 16384 * (4 * 8 + 8) and n % 256 == 0
    assert lib.csa2_cp_merge_workspace_bytes(0, 1, 16384) == 0
    assert lib.csa2_cp_merge_workspace_bytes(8, 1, 0) == 0
    assert lib.csa2_cp_merge_workspace_bytes(1025, 1, 16384) == 0     # more than 2^24 candidates

    def merge(cand=0x90000, n_a=16384, out_a=0xA0000, n_b=2048, out_b=0xB0000, ws_bytes=n, lens=0x30000):
        return lib.csa2_cp_merge_select(cand, 8, 1, 16384, lens, n_a, out_a, n_b, out_b, 0x80000, ws_bytes, None)

    assert merge(cand=0x90004) == csa2.ERR_INVALID_ARG
    assert merge(lens=None) == csa2.ERR_INVALID_ARG
    assert merge(n_a=0) == csa2.ERR_INVALID_ARG
    assert merge(n_a=16385) == csa2.ERR_INVALID_ARG
    assert merge(n_b=16384 + 1) == csa2.ERR_INVALID_ARG
    assert merge(out_b=None) == csa2.ERR_INVALID_ARG
    assert merge(out_a=0xA0004) == csa2.ERR_INVALID_ARG
    assert merge(ws_bytes=n - 1) == csa2.ERR_INVALID_ARG

    def attn(lse=0x70000, H=64, top_k=2048, window=128, topk=0x60000, glens=0x30000):
        return lib.csa2_cp_sparse_swa_attn(ctypes.byref(c), 0x30100, glens, 0x40000, H, topk, top_k, window, 0.0,
                                           0xA0000, lse, 0x80000, big, None)

    assert attn(lse=None) == csa2.ERR_INVALID_ARG                  # the merge needs every part's lse
    assert attn(glens=None) == csa2.ERR_INVALID_ARG
    assert attn(topk=None) == csa2.ERR_INVALID_ARG
    assert attn(window=16385) == csa2.ERR_INVALID_ARG
    assert attn(H=24) == csa2.ERR_UNSUPPORTED

    def merge_attn(R=2, out_stride=64 * 512, lse_stride=64):
        return lib.csa2_lse_merge(R, 1, 64, 512, 0x90000, out_stride, 0xA0000, lse_stride, 0xB0000, None, None)

    assert merge_attn(R=0) == csa2.ERR_INVALID_ARG
    assert merge_attn(out_stride=64 * 512 - 1) == csa2.ERR_INVALID_ARG
    assert merge_attn(lse_stride=63) == csa2.ERR_INVALID_ARG


def test_debug_encode_arguments_rejected_on_host(lib):
    assert lib.csa2_debug_encode(2, 0x10000, 8, 0x20000, None) == csa2.ERR_INVALID_ARG
    assert lib.csa2_debug_encode(0, 0x10000, -1, 0x20000, None) == csa2.ERR_INVALID_ARG
    assert lib.csa2_debug_encode(1, 0x10002, 8, 0x20000, None) == csa2.ERR_INVALID_ARG
    assert lib.csa2_debug_encode(0, None, 8, 0x20000, None) == csa2.ERR_INVALID_ARG
    assert lib.csa2_debug_encode(0, None, 0, None, None) == csa2.OK      # nothing to convert

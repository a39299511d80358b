"""The stored form of cached positions: csa2_kv_export_rows copies FP4 rows
and index keys out of the cache exactly as stored (rows bit-exact against the
oracle's quantisation of the same bf16 latents), and csa2_kv_import_rows puts
them back (tldrocket.com "DeepSeek AI Released DeepSeek-V4.1-Flash ...",
paragraph 4: E2M1 values with one E4M3 scale per 16 channels; Hugging Face
paper page 2609.19969, abstract: the compressed KV as persistent state)."""
import numpy as np
import pytest
import torch

import fp4_sparse_attention_csa2_b200 as csa2
import oracle
from fp4_sparse_attention_csa2_b200 import workloads as wl
from gpu_harness import build_gpu_cache

pytestmark = pytest.mark.gpu


def _slots(dev, w, b, ts):
    if dev.page_table is None:
        return [b * dev.seq_stride_slots + int(t) for t in ts]
    table = dev.page_table.cpu().numpy()
    return [int(table[b, int(t) // w.page_size]) * w.page_size + int(t) % w.page_size for t in ts]


@pytest.mark.parametrize("name,L,kw,starts", [
    ("long64k", 5000, {}, [1234]),
    ("batch32_paged", 9000, {"batch": 2}, [100, 200]),      # paged: runs cross page boundaries
    ("tiny4k", 3000, {}, [0]),                              # fp32 index keys
])
def test_export_import_round_trip(name, L, kw, starts):
    w = wl.scaled(wl.WORKLOADS[name], L, **kw)
    dev = build_gpu_cache(w)
    n = 96
    row_bytes = w.D // 2 + w.D // 16
    key_bytes = dev.idx_keys.shape[1] * dev.idx_keys.element_size()
    sp = torch.tensor(starts, dtype=torch.int32, device="cuda")
    rows = torch.full((w.batch, n, row_bytes), 0xAB, dtype=torch.uint8, device="cuda")
    keys = torch.full((w.batch, n, key_bytes), 0xAB, dtype=torch.uint8, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    csa2.kv_export_rows(dev, sp, n, rows, keys, ws)
    assert csa2.read_device_status(ws) == csa2.OK
    rows_h, keys_h = rows.cpu().numpy(), keys.cpu().numpy()
    lens = wl.seq_lens(w)
    for b, t0 in enumerate(starts):
        ts = np.arange(t0, t0 + n)
        # the rows are the oracle's quantisation of the same bf16 latents
        x = wl.latent(w, b, int(lens[b]))[t0:t0 + n]
        want = oracle.quantize_rows(wl.bf16_bits(x), w.row_stride)[:, :row_bytes]
        assert np.array_equal(rows_h[b], want), b
        # the keys are the cache's, as stored
        kslots = torch.tensor(_slots(dev, w, b, ts), device="cuda")
        assert np.array_equal(keys_h[b], dev.idx_keys[kslots].view(torch.uint8).cpu().numpy().reshape(n, key_bytes))
    # back into an empty cache of the same geometry: the same bytes at the same slots
    fresh = csa2.Cache(w.batch, dev.n_slots, w.D, w.D_I, w.row_stride, w.idx_key_dtype, lens,
                       None if dev.page_table is None else dev.page_table.cpu().numpy(), w.page_size,
                       dev.seq_stride_slots)
    csa2.kv_import_rows(fresh, sp, n, rows, keys, ws)
    assert csa2.read_device_status(ws) == csa2.OK
    for b, t0 in enumerate(starts):
        sl = torch.tensor(_slots(dev, w, b, np.arange(t0, t0 + n)), device="cuda")
        assert torch.equal(fresh.rows[sl], dev.rows[sl])
        assert torch.equal(fresh.idx_keys[sl], dev.idx_keys[sl])


def test_export_outside_the_cache_is_zero_and_flagged():
    w = wl.scaled(wl.WORKLOADS["long64k"], 2000)
    dev = build_gpu_cache(w)
    cap = dev.capacity
    n = 16
    row_bytes = w.D // 2 + w.D // 16
    sp = torch.tensor([cap - 4], dtype=torch.int32, device="cuda")
    rows = torch.full((1, n, row_bytes), 0xAB, dtype=torch.uint8, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    csa2.kv_export_rows(dev, sp, n, rows, None, ws)
    assert csa2.read_device_status(ws) == csa2.ERR_DEVICE_BOUNDS
    r = rows.cpu().numpy()[0]
    assert np.all(r[4:] == 0)                    # positions cap .. cap + 11 do not exist

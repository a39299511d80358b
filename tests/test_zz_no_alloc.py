"""The workspace-free Reindex entry point.

Some callers cannot hand the library a workspace (no allocator during a
no-allocation graph capture, plugins given tensors but no allocator, real-time
paths that cannot afford cudaMalloc's synchronisation).  For them,
csa2_index_reindex_noalloc keeps its scratch in a fixed array inside the
library.  This test checks, through the C ABI, that two calls in a row give the
same top-k sets as the workspace-based csa2_index_reindex on the same inputs.
It builds all of its own inputs, so it passes alone in a fresh process and
after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import fp4_sparse_attention_csa2_b200 as csa2
from fp4_sparse_attention_csa2_b200 import workloads as wl
from gpu_harness import build_gpu_cache, device_layer, new_ws

pytestmark = pytest.mark.gpu


def test_noalloc_reindex_matches_workspace_reindex_twice():
    w = wl.scaled(wl.WORKLOADS["batch32_paged"], 24000, batch=3, T=2)
    l0 = wl.layer_queries(w, 0)
    dev = build_gpu_cache(w, q_idx0=l0["q_idx"])
    ws = new_ws(dev, w)
    L0 = device_layer(l0)
    pool = torch.empty((w.batch, w.T, w.pool_k), dtype=torch.int32, device="cuda")
    topk0 = torch.empty((w.batch, w.T, w.top_k), dtype=torch.int32, device="cuda")
    csa2.index_full(dev, L0["q_idx"], L0["w"], w.pool_k, w.top_k, pool, topk0, ws)
    for layer in (1, 2):                                # two calls in a row share the scratch
        Ll = device_layer(wl.layer_queries(w, layer))
        want = torch.full((w.batch, w.T, w.top_k), -7, dtype=torch.int32, device="cuda")
        got = torch.full((w.batch, w.T, w.top_k), -7, dtype=torch.int32, device="cuda")
        csa2.index_reindex(dev, Ll["q_idx"], Ll["w"], pool, w.top_k, want, ws)
        csa2.index_reindex_noalloc(dev, Ll["q_idx"], Ll["w"], pool, w.top_k, got)
        torch.cuda.synchronize()
        assert csa2.read_device_status(ws) == csa2.OK
        a, b = want.cpu().numpy(), got.cpu().numpy()
        for bb in range(w.batch):
            for j in range(w.T):
                assert np.array_equal(np.sort(a[bb, j]), np.sort(b[bb, j])), (layer, bb, j)
                assert np.all(b[bb, j] >= 0)        # the pools hold more than top_k positions


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

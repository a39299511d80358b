"""The bounded waits of the tensor-core kernels run out under test: with the
wait budget set to 0 (csa2_debug_set_wait_limit) the scorer, the Reindex kernel
and the attention kernel give up at their first guarded wait, record
CSA2_ERR_TIMEOUT in the workspace status, drain what they issued and return;
the context stays usable and, with the default budget back, the same calls
return the results they returned before."""
import numpy as np
import pytest
import torch

import fp4_sparse_attention_csa2_b200 as csa2
from fp4_sparse_attention_csa2_b200 import workloads as wl
from gpu_harness import build_gpu_cache, device_layer, new_ws

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def setup():
    w = wl.scaled(wl.WORKLOADS["long64k"], 20000)   # > 16,384: the Full selection takes its histogram from the scorer
    l0, l1, l2 = (wl.layer_queries(w, i) for i in range(3))
    dev = build_gpu_cache(w, q_idx0=l0["q_idx"])
    return w, dev, device_layer(l0), device_layer(l1), l2["q"].cuda()


def _calls(w, dev, ws, L0, L1, q):
    """Full, Reindex and attention in a row; the device results."""
    pool = torch.full((w.batch, w.T, w.pool_k), -7, dtype=torch.int32, device="cuda")
    topk = torch.full((w.batch, w.T, w.top_k), -7, dtype=torch.int32, device="cuda")
    csa2.index_full(dev, L0["q_idx"], L0["w"], w.pool_k, w.top_k, pool, topk, ws)
    st_full = csa2.read_device_status(ws)
    topk2 = torch.full((w.batch, w.T, w.top_k), -7, dtype=torch.int32, device="cuda")
    csa2.index_reindex(dev, L1["q_idx"], L1["w"], pool, w.top_k, topk2, ws)
    st_re = csa2.read_device_status(ws)
    out = torch.full((w.batch, w.T, w.H, w.D), 7.0, dtype=torch.float32, device="cuda")
    lse = torch.full((w.batch, w.T, w.H), 7.0, dtype=torch.float32, device="cuda")
    # the top-k order is unspecified (ties and slots are claimed): sorted, the
    # attention sees the same input in every call and its result is reproducible
    topk = torch.sort(topk, dim=-1).values.contiguous()
    csa2.sparse_swa_attn(dev, q, topk, w.window, out, lse, ws)
    st_at = csa2.read_device_status(ws)
    return (st_full, st_re, st_at), pool.cpu().numpy(), topk2.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()


def _same_sets(a, b):
    assert np.array_equal(np.sort(a, axis=-1), np.sort(b, axis=-1))


def test_waits_run_out_and_the_context_survives(setup):
    w, dev, L0, L1, q = setup
    ws = new_ws(dev, w)
    default = csa2.debug_set_wait_limit(None)
    assert default > 0
    st, pool, topk2, out, lse = _calls(w, dev, ws, L0, L1, q)
    assert st == (csa2.OK, csa2.OK, csa2.OK)
    try:
        csa2.debug_set_wait_limit(0)
        st0 = _calls(w, dev, ws, L0, L1, q)[0]
    finally:
        csa2.debug_set_wait_limit(None)
    # every one of the three tensor-core kernels gave up and said so
    assert st0 == (csa2.ERR_TIMEOUT, csa2.ERR_TIMEOUT, csa2.ERR_TIMEOUT), st0
    # the context is usable and the default budget gives the earlier results
    torch.cuda.synchronize()
    st1, pool1, topk21, out1, lse1 = _calls(w, dev, ws, L0, L1, q)
    assert st1 == (csa2.OK, csa2.OK, csa2.OK)
    _same_sets(pool1, pool)
    _same_sets(topk21, topk2)
    assert np.array_equal(out1, out) and np.array_equal(lse1, lse)


def test_graph_keeps_the_budget_it_was_captured_with(setup):
    """The budget is a launch parameter: a replay of a graph captured with the
    default budget still succeeds after the budget is set to 0."""
    w, dev, L0, L1, q = setup
    ws = new_ws(dev, w)
    out = torch.zeros((w.batch, w.T, w.H, w.D), dtype=torch.float32, device="cuda")
    topk = torch.full((w.batch, w.T, w.top_k), -1, dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        csa2.sparse_swa_attn(dev, q, topk, w.window, out, None, ws, stream=s)   # warm-up outside capture
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        csa2.sparse_swa_attn(dev, q, topk, w.window, out, None, ws, stream=s)
    assert csa2.read_device_status(ws) == csa2.OK
    try:
        csa2.debug_set_wait_limit(0)
        g.replay()
        assert csa2.read_device_status(ws, s) == csa2.OK
    finally:
        csa2.debug_set_wait_limit(None)

"""Attention parity: csa2_sparse_swa_attn against the fp64 oracle on the same
cache and the oracle's own top-k (so this step is checked in isolation):
max-abs <= 2e-3 and mean-abs <= 2e-4 on the fp32 output (hackernews.kjhq.dev
post 49735410, key point 2; tldrocket.com "DeepSeek AI Released
DeepSeek-V4.1-Flash ...", paragraphs 2-4)."""
import numpy as np
import pytest
import torch

import fp4_sparse_attention_csa2_b200 as csa2
import oracle
from fp4_sparse_attention_csa2_b200 import workloads as wl
from gpu_harness import attn_errors, build_gpu_cache, new_ws
from harness import build_ref_cache, host_layer

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-3, 2e-4


def _oracle_topk(ref, w, layer):
    h = host_layer(layer)
    tk = np.zeros((w.batch, w.T, w.top_k), dtype=np.int32)
    for b in range(w.batch):
        for j in range(w.T):
            _, tk[b, j], _ = oracle.index_full(ref, b, w.T, j, h["q_idx"][b, j], w.q_idx_dtype, h["w"][b, j],
                                               w.pool_k, w.top_k)
    return tk


def _check(w, ref, dev, q, topk, window=None, sm_scale=0.0):
    window = w.window if window is None else window
    ws = new_ws(dev, w)
    out = torch.full((w.batch, w.T, w.H, w.D), 7.0, dtype=torch.float32, device="cuda")
    lse = torch.full((w.batch, w.T, w.H), 7.0, dtype=torch.float32, device="cuda")
    csa2.sparse_swa_attn(dev, q.cuda(), torch.from_numpy(topk).cuda(), window, out, lse, ws, sm_scale)
    assert csa2.read_device_status(ws) == csa2.OK
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    qb = wl.bf16_bits(q)
    worst = 0.0
    for b in range(w.batch):
        for j in range(w.T):
            ro, rl = oracle.sparse_swa_attn(ref, b, w.T, j, qb[b, j], topk[b, j], window, sm_scale)
            mx, mean = attn_errors(out[b, j], ro)
            assert mx <= MAX_ABS and mean <= MEAN_ABS, (b, j, mx, mean)
            assert np.allclose(lse[b, j], rl, atol=MAX_ABS, rtol=0), (b, j)
            worst = max(worst, mx)
    return worst


@pytest.mark.parametrize("name,L,kw", [
    ("tiny4k", 4096, {}),
    ("long64k", 9000, {}),
    ("long64k", 3000, {"T": 4}),
    ("batch32_paged", 20000, {"batch": 4}),
    ("append_mq", 5000, {"batch": 2}),
    ("long64k", 4000, {"H": 32}),               # tensor-core path with 32 heads
    ("long64k", 3000, {"H": 48}),               # CUDA-core path; the merge with a head count that does not divide 256
])
def test_attention_on_oracle_topk(name, L, kw):
    w = wl.scaled(wl.WORKLOADS[name], L, **kw)
    l0, l2 = wl.layer_queries(w, 0), wl.layer_queries(w, 2)
    ref = build_ref_cache(w, layers=[l0])
    dev = build_gpu_cache(w, q_idx0=l0["q_idx"])
    _check(w, ref, dev, l2["q"], _oracle_topk(ref, w, l0))


@pytest.fixture(scope="module")
def small():
    w = wl.scaled(wl.WORKLOADS["long64k"], 2500)
    l0 = wl.layer_queries(w, 0)
    return w, build_ref_cache(w, layers=[l0]), build_gpu_cache(w, q_idx0=l0["q_idx"]), l0


def test_empty_topk_is_window_only(small):
    w, ref, dev, l0 = small
    topk = np.full((1, 1, w.top_k), -1, dtype=np.int32)
    _check(w, ref, dev, wl.layer_queries(w, 4)["q"], topk)


def test_topk_with_window_duplicates_padding_and_future(small):
    w, ref, dev, l0 = small
    rng = np.random.default_rng(5)
    topk = rng.choice(2500, (1, 1, w.top_k), replace=False).astype(np.int32)
    topk[0, 0, :40] = np.arange(2460, 2500)    # window positions again
    topk[0, 0, 40:60] = -1                      # padding in the middle
    _check(w, ref, dev, wl.layer_queries(w, 4)["q"], topk)


def test_context_shorter_than_window():
    w = wl.scaled(wl.WORKLOADS["long64k"], 64, T=2)
    l0 = wl.layer_queries(w, 0)
    ref = build_ref_cache(w, layers=[l0])
    dev = build_gpu_cache(w, q_idx0=l0["q_idx"])
    topk = np.full((1, 2, w.top_k), -1, dtype=np.int32)
    topk[0, :, :10] = np.arange(10)
    _check(w, ref, dev, wl.layer_queries(w, 4)["q"], topk)


def test_zero_window_and_custom_scale(small):
    w, ref, dev, l0 = small
    topk = _oracle_topk(ref, w, l0)
    _check(w, ref, dev, wl.layer_queries(w, 5)["q"], topk, window=0, sm_scale=0.02)


def test_topk_covering_context_matches_dense(small):
    # k >= L: the sparse path equals dense softmax attention over every position
    w, ref, dev, l0 = small
    w2 = wl.Workload(**{**w.__dict__, "top_k": 2500})
    topk = np.arange(2500, dtype=np.int32)[::-1].copy().reshape(1, 1, -1)
    q = wl.layer_queries(w, 6)["q"]
    ws = new_ws(dev, w2)
    out = torch.empty((1, 1, w.H, w.D), dtype=torch.float32, device="cuda")
    csa2.sparse_swa_attn(dev, q.cuda(), torch.from_numpy(topk).cuda(), w.window, out, None, ws)
    do, _ = oracle.dense_attn(ref, 0, 1, 0, wl.bf16_bits(q)[0, 0])
    mx, mean = attn_errors(out.cpu().numpy()[0, 0], do)
    assert mx <= MAX_ABS and mean <= MEAN_ABS


def test_out_of_range_topk_flags_status(small):
    w, ref, dev, l0 = small
    topk = np.zeros((1, 1, w.top_k), dtype=np.int32)
    topk[0, 0, 3] = 2500                        # == L: outside the sequence
    topk[0, 0, 4] = -9
    ws = new_ws(dev, w)
    out = torch.empty((1, 1, w.H, w.D), dtype=torch.float32, device="cuda")
    csa2.sparse_swa_attn(dev, wl.layer_queries(w, 4)["q"].cuda(), torch.from_numpy(topk).cuda(), w.window, out,
                         None, ws)
    assert csa2.read_device_status(ws) == csa2.ERR_DEVICE_BOUNDS
    assert np.all(np.isfinite(out.cpu().numpy()))


def test_largest_topk_and_window():
    # the largest attended set the boundary accepts: top-k 16,384 and window
    # 16,384 (the pool bound), 257 chunks of 128 entries to merge
    L = 40000
    w = wl.scaled(wl.WORKLOADS["long64k"], L, pool_k=16384, top_k=16384, window=16384)
    l0 = wl.layer_queries(w, 0)
    ref = build_ref_cache(w, layers=[l0])
    dev = build_gpu_cache(w, q_idx0=l0["q_idx"])
    rng = np.random.default_rng(11)
    topk = rng.choice(L, (1, 1, w.top_k), replace=False).astype(np.int32)   # partly inside the window
    _check(w, ref, dev, wl.layer_queries(w, 3)["q"], topk)

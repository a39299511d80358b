"""Prefill / verification through csa2_prefill_layer: a whole CSA2 stack run
for T query tokens (more than one decode step takes), each token at its own
causal position, checked like a decode stack against the oracle: index sets
exact outside the 1e-5 band, attention within 2e-3 / 2e-4 (tldrocket.com
"DeepSeek AI Released DeepSeek-V4.1-Flash ...", paragraphs 2-3;
hackernews.kjhq.dev post 49735410, summary)."""
import pytest
import torch

import fp4_sparse_attention_csa2_b200 as csa2
from fp4_sparse_attention_csa2_b200 import workloads as wl
from gpu_harness import build_gpu_cache, device_layer
from harness import build_ref_cache
from test_gpu_stack import compare_stack

pytestmark = pytest.mark.gpu


def run_gpu_prefill(cache, w, layers):
    B, T = w.batch, w.T
    n = csa2.prefill_workspace_bytes(cache, T, w.H, w.H_I, w.pool_k, w.top_k, w.window)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    csa2.workspace_init(ws)
    pool = torch.full((B, T, w.pool_k), -7, dtype=torch.int32, device="cuda")
    topk = torch.full((B, T, w.top_k), -7, dtype=torch.int32, device="cuda")
    res = []
    for l, mode in enumerate(w.pattern):
        L = device_layer(layers[l])
        out = torch.empty((B, T, w.H, w.D), dtype=torch.float32, device="cuda")
        lse = torch.empty((B, T, w.H), dtype=torch.float32, device="cuda")
        m = {"F": csa2.FULL, "R": csa2.REINDEX, "U": csa2.REUSE}[mode]
        csa2.prefill_layer(cache, m, L["q"], topk, out, ws, w.window, q_idx=L["q_idx"] if mode != "U" else None,
                           head_w=L["w"] if mode != "U" else None, pool_idx=pool, lse=lse, pool_k=w.pool_k,
                           H_I=w.H_I)
        res.append((pool.cpu().numpy().copy() if mode == "F" else None, topk.cpu().numpy().copy(),
                    out.cpu().numpy(), lse.cpu().numpy()))
    return res, csa2.read_device_status(ws)


@pytest.mark.parametrize("name,L,T,kw", [
    ("long64k", 6000, 16, {}),                  # four chunks of four tokens
    ("tiny4k", 3000, 20, {}),                   # fp32 keys, chunks of eight: the last one moved back
    ("batch32_paged", 8000, 9, {"batch": 2}),   # paged, ragged, two sequences
    ("long64k", 300, 40, {"pool_k": 512, "top_k": 64}),   # tokens near the start: short visible prefixes
])
def test_prefill_stack(name, L, T, kw):
    w = wl.scaled(wl.WORKLOADS[name], L, T=T, **kw)
    layers = [wl.layer_queries(w, l) for l in range(len(w.pattern))]
    ref = build_ref_cache(w, layers=layers)
    dev = build_gpu_cache(w, q_idx0=layers[0]["q_idx"])
    got, status = run_gpu_prefill(dev, w, layers)
    assert status == csa2.OK
    pairs = [(b, j) for b in range(w.batch) for j in range(w.T)]
    compare_stack(w, ref, got, layers, pairs)

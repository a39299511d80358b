"""Layer-local window state on the GPU: csa2_ring_append writes each layer's
bf16 rows into its ring (bit-exact), and csa2_sparse_swa_attn_local attends
over the window rows of that ring and the FP4 rows of the shared top-k,
against the oracle's ref_sparse_swa_attn_local: max-abs <= 2e-3 and mean-abs
<= 2e-4 on the fp32 output ([FANOUT] item 2: the layers share the global KV
and the sparse selections and keep their own queries and sliding-window
state; tldrocket.com "DeepSeek AI Released DeepSeek-V4.1-Flash ...",
paragraph 2: the window runs in every layer)."""
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


def _ring_inputs(w, lens, ring_len, l=3, scale=1.0):
    """The rows a step appends: for every sequence the last ring_len positions
    (x [B, ring_len, D] bf16, start_pos = L_b - ring_len; positions below 0
    are skipped by the append), and the ring they must produce."""
    x = torch.zeros((w.batch, ring_len, w.D), dtype=torch.bfloat16)
    ring = torch.zeros((w.batch, ring_len, w.D), dtype=torch.bfloat16)
    start = np.asarray(lens, dtype=np.int64) - ring_len
    for b in range(w.batch):
        rows = wl.window_rows(w, l, b, int(start[b]), ring_len, scale=scale)
        x[b] = rows
        for i in range(ring_len):
            t = int(start[b]) + i
            if t >= 0:
                ring[b, t % ring_len] = rows[i]
    return x, torch.from_numpy(start.astype(np.int32)), ring


def _oracle_topk(ref, w, layer):
    h = host_layer(layer)
    tk = np.zeros((w.batch, w.T, w.top_k), dtype=np.int32)
    for b in range(w.batch):
        for j in range(w.T):
            _, tk[b, j], _ = oracle.index_full(ref, b, w.T, j, h["q_idx"][b, j], w.q_idx_dtype, h["w"][b, j],
                                               w.pool_k, w.top_k)
    return tk


def _run(w, ring_len, topk=None, scale=1.0, q_scale=1.0, window=None, sm_scale=0.0, via_layer_step=False):
    window = w.window if window is None else window
    lens = wl.seq_lens(w)
    l0, l2 = wl.layer_queries(w, 0), wl.layer_queries(w, 2)
    ref = build_ref_cache(w, layers=[l0])
    dev = build_gpu_cache(w, q_idx0=l0["q_idx"])
    if topk is None:
        topk = _oracle_topk(ref, w, l0)
    x, start, ring_host = _ring_inputs(w, lens, ring_len, scale=scale)
    ring = torch.zeros((w.batch, ring_len, w.D), dtype=torch.bfloat16, device="cuda")
    csa2.ring_append(dev, ring, x.cuda(), start.cuda())
    # the append is a copy: bit-exact
    assert torch.equal(ring.cpu().view(torch.int16), ring_host.view(torch.int16))
    q = (l2["q"].float() * q_scale).to(torch.bfloat16)
    ws = new_ws(dev, w)
    out = torch.full((w.batch, w.T, w.H, w.D), 7.0, dtype=torch.float32, device="cuda")
    lse = torch.full((w.batch, w.T, w.H), 7.0, dtype=torch.float32, device="cuda")
    tk = torch.from_numpy(topk).cuda()
    if via_layer_step:
        csa2.layer_step(dev, csa2.REUSE, q.cuda(), tk, out, ws, window, lse=lse, sm_scale=sm_scale, ring=ring)
    else:
        csa2.sparse_swa_attn_local(dev, ring, q.cuda(), tk, window, out, lse, ws, sm_scale)
    assert csa2.read_device_status(ws) == csa2.OK
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    qb, rb = wl.bf16_bits(q), wl.bf16_bits(ring_host)
    worst = 0.0
    for b in range(w.batch):
        for j in range(w.T):
            ro, rl = oracle.sparse_swa_attn_local(ref, rb, b, w.T, j, qb[b, j], topk[b, j], window, sm_scale)
            # rows far outside the unit range: compare in units of the row scale
            mx, mean = attn_errors(out[b, j] / scale, ro / scale)
            assert mx <= MAX_ABS and mean <= MEAN_ABS, (b, j, mx, mean)
            assert np.allclose(lse[b, j], rl, atol=MAX_ABS, rtol=0), (b, j)
            worst = max(worst, mx)
    return worst


@pytest.mark.parametrize("name,L,ring_len,kw", [
    ("tiny4k", 4096, 128, {}),                     # ring_len = window, 4096 % 128 == 0
    ("long64k", 9000, 160, {}),                    # wraps: 9000 % 160 != 0
    ("long64k", 3000, 131, {"T": 4}),              # T = 4: ring_len = window + T - 1
    ("batch32_paged", 20000, 200, {"batch": 4}),   # paged cache, ragged lengths
    ("long64k", 100, 128, {}),                     # window longer than the context
    ("long64k", 4000, 128, {"H": 32}),             # tensor-core path with 32 heads
    ("long64k", 3000, 128, {"H": 48}),             # CUDA-core path
])
def test_local_attention_on_oracle_topk(name, L, ring_len, kw):
    _run(wl.scaled(wl.WORKLOADS[name], L, **kw), ring_len)


def test_window_not_a_multiple_of_the_chunk():
    # window 100: the second chunk holds ring rows and FP4 top-k rows together
    w = wl.scaled(wl.WORKLOADS["long64k"], 5000, window=100)
    _run(w, 100)


def test_rows_above_the_fp16_range():
    # ring rows of magnitude ~2^20 (fp16 overflows at 65504) with queries 2^-20
    # smaller: moderate logits, outputs of order 2^20
    w = wl.scaled(wl.WORKLOADS["long64k"], 6000)
    _run(w, 128, scale=2.0 ** 20, q_scale=2.0 ** -20)


def test_rows_below_the_fp16_range_window_only():
    # ring rows of magnitude ~2^-20 (fp16 subnormal) and queries 2^20 larger;
    # window only, so the output is made of those rows alone
    w = wl.scaled(wl.WORKLOADS["long64k"], 6000)
    topk = np.full((w.batch, w.T, w.top_k), -1, dtype=np.int32)
    _run(w, 128, topk=topk, scale=2.0 ** -20, q_scale=2.0 ** 20)


def test_through_layer_step():
    _run(wl.scaled(wl.WORKLOADS["long64k"], 7000), 160, via_layer_step=True)


def test_ring_arguments_rejected_on_host():
    w = wl.scaled(wl.WORKLOADS["long64k"], 500, T=2)
    dev = build_gpu_cache(w)
    ws = new_ws(dev, w)
    q = torch.zeros((w.batch, w.T, w.H, w.D), dtype=torch.bfloat16, device="cuda")
    tk = torch.full((w.batch, w.T, w.top_k), -1, dtype=torch.int32, device="cuda")
    out = torch.zeros((w.batch, w.T, w.H, w.D), dtype=torch.float32, device="cuda")
    short = torch.zeros((w.batch, w.window, w.D), dtype=torch.bfloat16, device="cuda")   # T = 2 needs window + 1
    with pytest.raises(csa2.CSA2Error) as e:
        csa2.sparse_swa_attn_local(dev, short, q, tk, w.window, out, None, ws)
    assert e.value.code == csa2.ERR_INVALID_ARG
    x = torch.zeros((w.batch, 3, w.D), dtype=torch.bfloat16, device="cuda")
    sp = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
    tiny = torch.zeros((w.batch, 2, w.D), dtype=torch.bfloat16, device="cuda")         # n_new > ring_len
    with pytest.raises(csa2.CSA2Error) as e:
        csa2.ring_append(dev, tiny, x, sp)
    assert e.value.code == csa2.ERR_INVALID_ARG

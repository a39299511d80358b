"""Quantise-on-append parity: FP4 codes, scales and E4M3 index keys written by
csa2_kv_append_quant are bit-exact with the oracle on the same seeded inputs
(format: tldrocket.com "DeepSeek AI Released DeepSeek-V4.1-Flash ...",
paragraph 4)."""
import json
import os

import numpy as np
import pytest
import torch

import fp4_sparse_attention_csa2_b200 as csa2
import oracle
from conftest import read_golden
from fp4_sparse_attention_csa2_b200 import workloads as wl
from gpu_harness import build_gpu_cache, new_ws
from harness import build_ref_cache

pytestmark = pytest.mark.gpu


def _payload(rows, D):
    return rows[:, :D // 2 + D // 16]


@pytest.mark.parametrize("name,L", [("tiny4k", 4096), ("long64k", 20000), ("batch32_paged", 3000)])
def test_append_bitexact(name, L):
    w = wl.scaled(wl.WORKLOADS[name], L, batch=min(4, wl.WORKLOADS[name].batch))
    ref = build_ref_cache(w)
    dev = build_gpu_cache(w)
    assert np.array_equal(_payload(dev.rows.cpu().numpy(), w.D), _payload(ref.rows, w.D))
    got = dev.idx_keys.cpu().numpy()
    assert np.array_equal(got.view(np.uint8), ref.idx_keys.view(np.uint8))


def _append_blocks(xs, D=16 * 32):
    """Append rows made of the given 16-value blocks; return device and oracle rows."""
    xs = np.asarray(xs, dtype=np.float32).reshape(-1)
    n_rows = (xs.size + D - 1) // D
    buf = np.zeros(n_rows * D, dtype=np.float32)
    buf[:xs.size] = xs
    xb = torch.from_numpy(buf.reshape(n_rows, D)).to(torch.bfloat16)
    assert torch.equal(xb.float(), torch.from_numpy(buf.reshape(n_rows, D))), "inputs must be exact in bf16"
    stride = (n_rows + 63) // 64 * 64
    row_stride = (D // 2 + D // 16 + 15) // 16 * 16
    cache = csa2.Cache(1, stride, D, 64, row_stride, csa2.E4M3, [n_rows], seq_stride_slots=stride)
    sp = torch.zeros(1, dtype=torch.int32, device="cuda")
    csa2.kv_append_quant(cache, xb[None].cuda(), sp)
    torch.cuda.synchronize()
    want = oracle.quantize_rows(wl.bf16_bits(xb), row_stride)
    return _payload(cache.rows.cpu().numpy()[:n_rows], D), _payload(want, D)


def test_golden_blocks():
    blocks = {}
    cur = None
    for r in read_golden("quant_blocks.txt"):
        if r[0] == "block":
            cur = blocks.setdefault(r[1], {})
        else:
            cur[r[0]] = r[1:]
    xs = np.concatenate([np.array([float(v) for v in b["x"]]) for b in blocks.values()])
    got, want = _append_blocks(xs)
    assert np.array_equal(got, want)
    # and the hand-worked bytes themselves
    D = 512
    for i, b in enumerate(blocks.values()):
        assert list(got[0, 8 * i:8 * i + 8]) == [int(v, 16) for v in b["packed"]]
        assert got[0, D // 2 + i] == int(b["scale"][0], 16)


def test_ties_zeros_saturation_underflow():
    rng = np.random.default_rng(11)
    e2m1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    mids = (e2m1[1:] + e2m1[:-1]) / 2                        # the E2M1 rounding ties
    blocks = []
    for sc in [0x38, 0x3C, 0x30, 0x48, 0x01, 0x05, 0x7E, 0x52]:
        s = oracle.e4m3_value(sc)
        for sign in (1, -1):
            blk = np.zeros(16)
            blk[0] = 6 * s
            blk[1:8] = sign * mids * s
            blk[8:15] = sign * e2m1[1:] * s
            blk[15] = -0.0
            blocks.append(blk)
    blocks.append(np.zeros(16))                              # amax = 0
    blocks.append(np.full(16, -0.0))
    blocks.append(np.array([2.0 ** -13, -2.0 ** -14] + [0.0] * 14))   # scale underflows to 0
    blocks.append(np.array([3e4, -3e4, 1e4] + [1.0] * 13))  # scale saturates at 448
    for _ in range(200):
        blocks.append(rng.standard_normal(16) * 10.0 ** rng.uniform(-4, 3))
    xs = torch.tensor(np.concatenate(blocks)).to(torch.bfloat16).float().numpy()
    got, want = _append_blocks(xs)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("sc", [0x38, 0x3C, 0x2B, 0x01, 0x6D])
def test_e2m1_sweep_every_bf16_input(sc):
    # channel 0 of each block fixes amax = 6 s (so the scale is s exactly);
    # channels 1..15 sweep every finite bf16 value in [-7 s, 7 s]
    s = oracle.e4m3_value(sc)
    allb = torch.arange(-32768, 32768, dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float()
    v = allb[torch.isfinite(allb) & (allb.abs() <= 7 * s)].numpy()
    n = (v.size + 14) // 15
    blk = np.zeros((n, 16), dtype=np.float32)
    blk[:, 0] = 6 * s
    flat = np.zeros(n * 15, dtype=np.float32)
    flat[:v.size] = v
    blk[:, 1:] = flat.reshape(n, 15)
    got, want = _append_blocks(blk)
    assert np.array_equal(got, want)


def test_e4m3_keys_every_bf16_input():
    allb = torch.arange(-32768, 32768, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    keys = allb[torch.isfinite(allb.float())]
    n = (keys.numel() + 63) // 64
    buf = torch.zeros(n * 64, dtype=torch.bfloat16)
    buf[:keys.numel()] = keys
    stride = (n + 63) // 64 * 64
    cache = csa2.Cache(1, stride, 128, 64, 80, csa2.E4M3, [n], seq_stride_slots=stride)
    sp = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = torch.zeros((1, n, 128), dtype=torch.bfloat16, device="cuda")
    csa2.kv_append_quant(cache, x, sp, buf.view(1, n, 64).cuda())
    got = cache.idx_keys.cpu().numpy()[:n].reshape(-1)
    want = oracle.e4m3_encode(buf.float().numpy())
    assert np.array_equal(got, want)


def test_f32_keys_are_stored_as_given():
    w = wl.scaled(wl.WORKLOADS["tiny4k"], 1000)
    dev = build_gpu_cache(w)
    keys, _ = wl.index_keys(w, 0, 1000, wl.layer_queries(w, 0)["q_idx"][0, 0])
    assert np.array_equal(dev.idx_keys.cpu().numpy()[:1000], keys.numpy())


def test_out_of_range_append_flags_status():
    cache = csa2.Cache(1, 64, 128, 64, 80, csa2.E4M3, [64], seq_stride_slots=64)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    sp = torch.tensor([60], dtype=torch.int32, device="cuda")
    x = torch.ones((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    csa2.kv_append_quant(cache, x, sp, ws=ws)
    assert csa2.read_device_status(ws) == csa2.ERR_DEVICE_BOUNDS
    rows = cache.rows.cpu().numpy()
    assert np.all(rows[60:64, :72] != 0) and csa2.read_device_status(ws) == csa2.OK


def _sums_on_device(codes, bits, fin):
    """Per block: the two position-weighted sums of tests/golden/make_encoder_sweep.py."""
    c = codes.to(torch.int64) * fin
    w1 = (((bits * 2654435761) & 0xFFFFFFFF) >> 12) + 1      # int64 products wrap: the low 32 bits are exact
    w2 = (((bits * 40503) & 0xFFFFFFFF) >> 12) + 1
    return [int((c * w1).sum()), int((c * w2).sum()), int(fin.sum())]


@pytest.mark.parametrize("fmt,name", [(0, "e2m1"), (1, "e4m3")])
def test_encoders_every_fp32_input(fmt, name):
    # the quantiser's conversions on all 2^32 fp32 bit patterns against the
    # oracle's encoders (tests/golden/encoder_sweep.json, written by
    # tests/golden/make_encoder_sweep.py from the oracle alone), block by block
    with open(os.path.join(os.path.dirname(__file__), "golden", "encoder_sweep.json")) as f:
        golden = json.load(f)
    nb = 1 << golden["block_bits"]
    codes = torch.empty(nb, dtype=torch.uint8, device="cuda")
    for blk, want in enumerate(golden[name]):
        bits = torch.arange(blk * nb, (blk + 1) * nb, dtype=torch.int64, device="cuda")
        x = torch.where(bits >= (1 << 31), bits - (1 << 32), bits).to(torch.int32).view(torch.float32)
        csa2.debug_encode(x, codes, fmt)
        fin = torch.isfinite(x).to(torch.int64)
        assert _sums_on_device(codes, bits, fin) == list(want), (name, blk)

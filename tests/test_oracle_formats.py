"""Pins of the oracle's number formats and block quantisation against what the
format definitions fix (E2M1 / E4M3, named on the tldrocket.com page "DeepSeek
AI Released DeepSeek-V4.1-Flash with 1M Context, FP4 KV Cache, and Cross-Layer
Attention Reuse", paragraph 4) and against an independent library encoder
(torch.float8_e4m3fn)."""
import math

import numpy as np
import torch

import oracle
from conftest import read_golden


def test_e2m1_table_matches_definition():
    for code, val in read_golden("e2m1_values.txt"):
        c = int(code, 16)
        v = oracle.e2m1_value(c)
        assert v == float(val) and math.copysign(1, v) == math.copysign(1, float(val)), code


def test_e4m3_points_match_definition():
    for code, val in read_golden("e4m3_points.txt"):
        v = oracle.e4m3_value(int(code, 16))
        if val == "nan":
            assert math.isnan(v)
        else:
            assert v == float(val) and math.copysign(1, v) == math.copysign(1, float(val)), code


def test_e4m3_decode_matches_torch_for_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib_vals = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = oracle.e4m3_value(c)
        if math.isnan(lib_vals[c]):
            assert math.isnan(v)
        else:
            assert v == lib_vals[c], hex(c)


def test_roundtrip_every_code():
    # decode(encode(v)) == v for all 16 E2M1 and all 254 finite E4M3 codes
    for c in range(16):
        v = np.float32(oracle.e2m1_value(c))
        e = int(oracle.e2m1_encode(np.array([v]))[0])
        assert oracle.e2m1_value(e) == v and (e == c or v == 0)
        assert math.copysign(1, oracle.e2m1_value(e)) == math.copysign(1, v)
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        v = np.float32(oracle.e4m3_value(c))
        assert int(oracle.e4m3_encode(np.array([v]))[0]) == c


def test_e2m1_ties_and_saturation_by_hand():
    # round half to the even code; saturate at +-6; sign kept on zero
    x = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 1e30, -0.1, -0.0, 0.2500001, -5.0],
                 dtype=np.float32)
    want = [0x0, 0x2, 0x2, 0x4, 0x4, 0x6, 0x6, 0x7, 0x7, 0x8, 0x8, 0x1, 0xE]
    assert list(oracle.e2m1_encode(x)) == want


def test_e4m3_encode_matches_torch_rne():
    # torch's float8_e4m3fn conversion is round-to-nearest-even; it maps values
    # at or beyond the 464 midpoint to NaN instead of saturating, so compare below it.
    g = torch.Generator().manual_seed(1234)
    parts = [
        torch.randn(200000, generator=g) * 30,
        torch.randn(200000, generator=g) * 1e-3,
        (torch.rand(200000, generator=g) - 0.5) * 900,
    ]
    # every midpoint between neighbouring codes, and its fp32 neighbours
    vals = np.array([oracle.e4m3_value(c) for c in range(0x7F)], dtype=np.float64)
    mids = torch.tensor((vals[1:] + vals[:-1]) / 2, dtype=torch.float32)
    parts += [mids, torch.nextafter(mids, torch.full_like(mids, 1e9)),
              torch.nextafter(mids, torch.full_like(mids, -1e9))]
    x = torch.cat(parts)
    x = torch.cat([x, -x])
    x = x[x.abs() < 464]
    lib = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = oracle.e4m3_encode(x.numpy())
    assert np.array_equal(lib, ours)


def test_e4m3_saturates():
    x = np.array([448, 463.99, 464, 500, 1e6, 3e38, -464, -1e9], dtype=np.float32)
    assert list(oracle.e4m3_encode(x)) == [0x7E] * 6 + [0xFE] * 2


def test_quant_blocks_worked_by_hand():
    rows = read_golden("quant_blocks.txt")
    blocks = {}
    cur = None
    for r in rows:
        if r[0] == "block":
            cur = blocks.setdefault(r[1], {})
        else:
            cur[r[0]] = r[1:]
    assert len(blocks) == 5
    for name, b in blocks.items():
        x = np.array([float(v) for v in b["x"]], dtype=np.float32)
        # every fixture value is exact in bf16
        assert np.array_equal(torch.from_numpy(x).to(torch.bfloat16).float().numpy(), x)
        codes, sc = oracle.quantize_block16(x)
        assert list(codes) == [int(v) for v in b["codes"]], name
        assert sc == int(b["scale"][0], 16), name
        xb = torch.from_numpy(x).to(torch.bfloat16)
        row = oracle.quantize_rows(xb.view(torch.int16).numpy().view(np.uint16)[None, :], 16)[0]
        assert list(row[:8]) == [int(v, 16) for v in b["packed"]], name
        assert row[8] == sc


def test_block_roundtrip_exact():
    # a block built as c_i * s with s an E4M3 value and some |c_i| = 6 gives
    # back exactly the same codes and scale
    rng = np.random.default_rng(7)
    e2m1_vals = np.array([oracle.e2m1_value(c) for c in range(16)])
    tried = 0
    for sc in range(1, 0x7F):
        s = oracle.e4m3_value(sc)
        for _ in range(3):
            codes = rng.integers(0, 16, 16).astype(np.uint8)
            codes[rng.integers(0, 16)] = 0x7 | (rng.integers(0, 2) << 3)
            x = (e2m1_vals[codes] * s).astype(np.float32)
            got, gsc = oracle.quantize_block16(x)
            assert gsc == sc
            assert np.array_equal(got, codes), (sc, codes, got)
            tried += 1
    assert tried == 3 * 126


def test_row_bytes_and_storage_ratio():
    # D = 512: 256 code bytes + 32 scale bytes = 288 B per position; an FP8
    # row with the same 16-channel scales would take 512 + 32 B, so FP4
    # "nearly halves" the row (tldrocket.com, paragraph 4).
    D = 512
    fp4 = D // 2 + D // 16
    assert fp4 == 288
    assert 0.5 < fp4 / (D + D // 16) < 0.56
    x = torch.randn(3, D).to(torch.bfloat16)
    rows = oracle.quantize_rows(x.view(torch.int16).numpy().view(np.uint16), 288)
    assert rows.shape == (3, 288)


def test_dequant_is_code_times_scale():
    x = torch.randn(4, 64, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    rows = oracle.quantize_rows(x.view(torch.int16).numpy().view(np.uint16), 48)
    tbl = {int(c, 16): float(v) for c, v in read_golden("e2m1_values.txt")}
    for r in range(4):
        deq = oracle.dequant_row(rows[r], 64)
        for d in range(64):
            byte = rows[r][d // 2]
            code = (byte >> 4) if d & 1 else (byte & 0xF)
            s = torch.tensor([rows[r][32 + d // 16]], dtype=torch.uint8).view(torch.float8_e4m3fn).double().item()
            assert deq[d] == tbl[code] * s
        # quantisation error stays within half a code step of each block's grid
        xd = x[r].double().numpy()
        for blk in range(4):
            s = torch.tensor([rows[r][32 + blk]], dtype=torch.uint8).view(torch.float8_e4m3fn).double().item()
            err = np.abs(deq[blk * 16:(blk + 1) * 16] - xd[blk * 16:(blk + 1) * 16])
            assert np.all(err <= 1.0 * s + 1e-12)


def test_encoder_sweep_golden_is_the_oracles():
    # the stored per-block sums of the exhaustive encoder sweep are the oracle's
    # own (recomputed here for one block of values in [2^-7, 2) and one of
    # negative values), and every block counts its finite patterns
    import json
    import os
    import sys
    here = os.path.join(os.path.dirname(__file__), "golden")
    sys.path.insert(0, here)
    import make_encoder_sweep as mk
    with open(os.path.join(here, "encoder_sweep.json")) as f:
        g = json.load(f)
    assert g["block_bits"] == mk.BLOCK_BITS and len(g["e2m1"]) == len(g["e4m3"]) == mk.N_BLOCKS
    for blk in (15, 48):
        _, sums = mk._work(blk)
        assert [list(sums["e2m1"]), list(sums["e4m3"])] == [g["e2m1"][blk], g["e4m3"][blk]]
    # the 2 x 2^23 patterns with exponent 255 (Inf / NaN) are the only ones left out
    n_fin = [g["e4m3"][b][2] for b in range(mk.N_BLOCKS)]
    assert sum(n_fin) == (1 << 32) - 2 * (1 << 23)

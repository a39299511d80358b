"""Write tests/golden/encoder_sweep.json: the oracle's E2M1 and E4M3 codes of
every finite fp32 value, summarised per block of 2^26 bit patterns as two
position-weighted sums (tldrocket.com "DeepSeek AI Released DeepSeek-V4.1-Flash
...", paragraph 4: E2M1 values with one E4M3 scale per 16 channels; both
encoders round to nearest, ties to even, saturating).

    python tests/golden/make_encoder_sweep.py        (about a minute on 8 cores)

Only the oracle computes codes here.  The GPU test computes the same sums
from the library's conversions and compares block by block; a single wrong
code changes both sums of its block.
"""
import json
import multiprocessing as mp
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
BLOCK_BITS = 26
N_BLOCKS = 1 << (32 - BLOCK_BITS)


def block_patterns(blk):
    """The fp32 bit patterns of block blk as uint32."""
    return np.arange(blk << BLOCK_BITS, (blk + 1) << BLOCK_BITS, dtype=np.uint64).astype(np.uint32)


def weights(bits):
    """Two 20-bit position weights (>= 1) of each bit pattern."""
    b = bits.astype(np.uint64)
    w1 = (((b * np.uint64(2654435761)) & np.uint64(0xFFFFFFFF)) >> np.uint64(12)) + np.uint64(1)
    w2 = (((b * np.uint64(40503)) & np.uint64(0xFFFFFFFF)) >> np.uint64(12)) + np.uint64(1)
    return w1.astype(np.int64), w2.astype(np.int64)


def block_sums(codes, bits):
    w1, w2 = weights(bits)
    c = codes.astype(np.int64)
    return int(np.sum(c * w1)), int(np.sum(c * w2)), int(bits.size)


def _work(blk):
    sys.path.insert(0, ROOT)
    import oracle
    bits = block_patterns(blk)
    x = bits.view(np.float32)
    fin = np.isfinite(x)
    out = {}
    for name, enc in (("e2m1", oracle.e2m1_encode), ("e4m3", oracle.e4m3_encode)):
        out[name] = block_sums(enc(x[fin]), bits[fin])
    return blk, out


def main():
    with mp.get_context("spawn").Pool(os.cpu_count()) as pool:
        res = dict(pool.map(_work, range(N_BLOCKS)))
    doc = {"source": "oracle/ (ref_e2m1_encode, ref_e4m3_encode) over every finite fp32 bit pattern",
           "block_bits": BLOCK_BITS,
           "weights": "w1 = ((b * 2654435761) mod 2^32) >> 12 + 1, w2 = ((b * 40503) mod 2^32) >> 12 + 1, "
                      "b = the bit pattern; per block: (sum code * w1, sum code * w2, finite count)",
           "e2m1": [res[b]["e2m1"] for b in range(N_BLOCKS)],
           "e4m3": [res[b]["e4m3"] for b in range(N_BLOCKS)]}
    with open(os.path.join(HERE, "encoder_sweep.json"), "w") as f:
        json.dump(doc, f, indent=0)


if __name__ == "__main__":
    main()

"""Seeded synthetic inputs for the CSA2 decode workloads.

This module only draws inputs: it holds none of the method's arithmetic (no
quantisation, scoring, selection or attention).  Tests, the smoke check and the
benchmark take their inputs from here; both the CUDA library and the CPU oracle
then consume the same tensors.

Every tensor is drawn on the CPU with its own ``torch.Generator`` so that any
one sequence can be regenerated alone:  seed(tensor, b) = (seed*1000 + id)
* 65536 + b, with ids q=1, latent=2, q_idx=3, idx_key=4, plant=5, lens=6,
pages=7, and layer l's queries 10+l (q) / 40+l (q_idx).

The shapes follow the workloads the pages imply: a 1M-token context
("DeepSeek AI Released DeepSeek-V4.1-Flash with 1M Context, FP4 KV Cache, and
Cross-Layer Attention Reuse", tldrocket.com, paragraph 1), a candidate pool of
16,384 positions (paragraph 3) and a 128-token window (paragraph 2).
"""
from dataclasses import dataclass, field
import math

import numpy as np
import torch

F32, BF16, E4M3 = 0, 1, 2  # dtype codes shared with the C ABI's csa2_dtype


@dataclass
class Workload:
    name: str
    batch: int
    T: int                      # query tokens per sequence
    H: int                      # attention heads
    D: int                      # latent dim
    H_I: int                    # indexer heads
    D_I: int                    # indexer dim
    idx_key_dtype: int          # F32 or E4M3
    q_idx_dtype: int            # F32 or BF16
    pool_k: int
    top_k: int
    window: int
    pattern: str                # e.g. "FRUU"
    lens: tuple                 # ("fixed", L) or ("uniform", lo, hi)
    paged: bool = False
    page_size: int = 64
    plant: tuple = ()           # ("spread", n) | ("random", n) | ("frac", f) | ()
    row_stride: int = 0         # bytes per FP4 row (>= D/2 + D/16, multiple of 16)
    append_n: int = 0           # positions appended per sequence just before decode
    note: str = ""

    def __post_init__(self):
        if not self.row_stride:
            r = self.D // 2 + self.D // 16
            self.row_stride = (r + 15) // 16 * 16


WORKLOADS = {
    # 3-layer stack at 4K context; fp32 index keys / queries, 16 x 128 attention.
    "tiny4k": Workload("tiny4k", 1, 1, 16, 128, 4, 64, F32, F32, 512, 128, 128, "FRU",
                       ("fixed", 4096), plant=("random", 8)),
    # One long sequence, 64K context, 64 x 512 attention, 32 x 64 indexer, E4M3 keys.
    "long64k": Workload("long64k", 1, 1, 64, 512, 32, 64, E4M3, BF16, 16384, 2048, 128, "FRUU",
                        ("fixed", 65536), plant=("spread", 64)),
    # 32 sequences of 16K..128K context in 64-token pages scattered over HBM.
    "batch32_paged": Workload("batch32_paged", 32, 1, 64, 512, 32, 64, E4M3, BF16, 16384, 2048, 128,
                              "FRUU", ("uniform", 16384, 131072), paged=True, plant=("frac", 0.01)),
    # One 1,048,576-token sequence: Full, Reindex, 6 x Reuse.
    "ctx1m": Workload("ctx1m", 1, 1, 64, 512, 32, 64, E4M3, BF16, 16384, 2048, 128, "FRUUUUUU",
                      ("fixed", 1048576), plant=("random", 256)),
    # 8 sequences: 262,144 cached + 8,192 appended positions, 4 query tokens each.
    "append_mq": Workload("append_mq", 8, 4, 64, 512, 32, 64, E4M3, BF16, 16384, 2048, 128, "FRUU",
                          ("fixed", 262144 + 8192), append_n=8192),
}


def scaled(w: Workload, L: int, name=None, **kw) -> Workload:
    """The same workload at a smaller context (parity cases the oracle finishes quickly)."""
    d = dict(w.__dict__)
    d.update(kw)
    d["name"] = name or "%s@%d" % (w.name, L)
    if d["lens"][0] == "fixed":
        d["lens"] = ("fixed", L)
    else:
        lo, hi = d["lens"][1], d["lens"][2]
        d["lens"] = ("uniform", max(1, lo * L // hi), L)
    if d.get("plant") and d["plant"][0] in ("spread", "random"):
        d["plant"] = (d["plant"][0], min(d["plant"][1], max(1, L // 64)))
    return Workload(**d)


def _gen(seed, tid, b=0):
    g = torch.Generator(device="cpu")
    g.manual_seed(((seed * 1000 + tid) * 65536 + b) & 0x7FFFFFFFFFFFFFFF)
    return g


def seq_lens(w: Workload, seed=0) -> np.ndarray:
    if w.lens[0] == "fixed":
        return np.full(w.batch, w.lens[1], dtype=np.int32)
    lo, hi = w.lens[1], w.lens[2]
    g = _gen(seed, 6)
    return torch.randint(lo, hi + 1, (w.batch,), generator=g).numpy().astype(np.int32)


def capacity(w: Workload, lens=None) -> int:
    """Positions per sequence the cache must hold (a multiple of the page size)."""
    L = int(np.max(lens)) if lens is not None else (w.lens[1] if w.lens[0] == "fixed" else w.lens[2])
    return (L + w.page_size - 1) // w.page_size * w.page_size


def page_table(w: Workload, lens, seed=0):
    """[B, max_pages] int32 physical page ids: a seeded permutation of one pool of
    sum_b ceil(L_b / page) pages; unused entries are -1.  Returns (table, n_pages)."""
    pages = [(int(L) + w.page_size - 1) // w.page_size for L in lens]
    n_pages = int(sum(pages))
    maxp = capacity(w, lens) // w.page_size
    perm = torch.randperm(n_pages, generator=_gen(seed, 7)).numpy().astype(np.int32)
    table = np.full((w.batch, maxp), -1, dtype=np.int32)
    k = 0
    for b, n in enumerate(pages):
        table[b, :n] = perm[k:k + n]
        k += n
    return table, n_pages


def cache_geometry(w: Workload, lens, seed=0):
    """(n_slots, page_table | None, seq_stride_slots) of the cache that holds
    sequences of these lengths."""
    if w.paged:
        table, n_pages = page_table(w, lens, seed)
        return n_pages * w.page_size, table, 0
    cap = capacity(w, lens)
    return w.batch * cap, None, cap


def latent(w: Workload, b, L, seed=0, t0=0):
    """bf16 N(0,1) latent rows [L - t0, D] for positions t0..L-1 of sequence b."""
    g = _gen(seed, 2, b)
    out = torch.empty((L - t0, w.D), dtype=torch.bfloat16)
    step = 1 << 16
    # positions are drawn in fixed blocks so that any suffix is reproducible
    for s in range(0, L, step):
        e = min(L, s + step)
        blk = torch.randn((e - s, w.D), generator=g, dtype=torch.float32)
        if e <= t0:
            continue
        a = max(s, t0)
        out[a - t0:e - t0] = blk[a - s:].to(torch.bfloat16)
    return out


def window_rows(w: Workload, l, b, t0, n, seed=0, scale=1.0):
    """Layer l's own bf16 rows (its layer-local sliding-window state) of
    positions t0 .. t0 + n - 1 of sequence b: N(0, 1) x scale, rounded to bf16,
    [n, D].  Drawn per (layer, sequence, t0)."""
    g = _gen(seed, 70 + l, (b * 131071 + t0) & 0xFFFF)
    return (torch.randn((n, w.D), generator=g, dtype=torch.float32) * scale).to(torch.bfloat16)


def layer_queries(w: Workload, l, seed=0):
    """Layer l's inputs: q bf16 [B, T, H, D], q_idx [B, T, H_I, D_I] (bf16 or
    fp32), head weights w fp32 [B, T, H_I] = 1/H_I."""
    q = torch.randn((w.batch, w.T, w.H, w.D), generator=_gen(seed, 10 + l), dtype=torch.float32)
    qi = torch.randn((w.batch, w.T, w.H_I, w.D_I), generator=_gen(seed, 40 + l), dtype=torch.float32)
    qi = qi if w.q_idx_dtype == F32 else qi.to(torch.bfloat16)
    hw = torch.full((w.batch, w.T, w.H_I), 1.0 / w.H_I, dtype=torch.float32)
    return {"q": q.to(torch.bfloat16), "q_idx": qi, "w": hw}


def _unit(v):
    return v / v.norm()


def index_keys(w: Workload, b, L, q_idx0, seed=0, t0=0):
    """Index-key inputs [L - t0, D_I] for sequence b (fp32 for F32 caches, else bf16):
    N(0,1) background plus planted positions aligned with the layer-0 indexer
    query direction u = normalize(sum_h w_h q_h) of the last query token.
      spread n : t_i = floor((i + 1/2) L / n), cosine 0.9
      random n : n seeded distinct positions, cosine 0.9
      frac f   : a seeded fraction f of positions, cosine 0.9 + N(0, 0.02^2)
    A planted key is sqrt(D_I) * (c u + sqrt(1 - c^2) xi), xi a random unit
    vector orthogonal to u."""
    g = _gen(seed, 4, b)
    keys = torch.randn((L, w.D_I), generator=g, dtype=torch.float32)
    planted = np.zeros(0, dtype=np.int64)
    cos = None
    gp = _gen(seed, 5, b)
    if w.plant:
        kind, arg = w.plant
        if kind == "spread":
            planted = np.array([int(math.floor((i + 0.5) * L / arg)) for i in range(arg)], dtype=np.int64)
        elif kind == "random":
            planted = torch.randperm(L, generator=gp)[:arg].numpy().astype(np.int64)
        elif kind == "frac":
            n = max(1, int(round(arg * L)))
            planted = torch.randperm(L, generator=gp)[:n].numpy().astype(np.int64)
            cos = (0.9 + 0.02 * torch.randn(n, generator=gp, dtype=torch.float32)).clamp(-1, 1)
    if planted.size:
        qv = q_idx0.float()                       # [H_I, D_I]
        u = _unit(qv.mean(dim=0))                 # equal head weights: mean direction
        n = planted.size
        xi = torch.randn((n, w.D_I), generator=gp, dtype=torch.float32)
        xi = xi - (xi @ u)[:, None] * u[None, :]
        xi = xi / xi.norm(dim=1, keepdim=True)
        c = torch.full((n,), 0.9) if cos is None else cos
        pk = math.sqrt(w.D_I) * (c[:, None] * u[None, :] + torch.sqrt(1 - c * c)[:, None] * xi)
        keys[torch.from_numpy(planted)] = pk
    keys = keys[t0:]
    return (keys if w.idx_key_dtype == F32 else keys.to(torch.bfloat16)), planted


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of a bf16 tensor (for the oracle's C interface)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def host_array(t: torch.Tensor) -> np.ndarray:
    """bf16 -> uint16 bits, fp32 -> float32 (no conversion of values)."""
    return bf16_bits(t) if t.dtype == torch.bfloat16 else t.contiguous().numpy()


def shard_bounds(L, R):
    """Context-parallel split of one sequence of L positions over R ranks:
    rank r holds [L r / R, L (r + 1) / R) (floors; ragged when R does not
    divide L)."""
    return [(L * r // R, L * (r + 1) // R - L * r // R) for r in range(R)]

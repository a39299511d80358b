"""The context-parallel driver (fp4_sparse_attention_csa2_b200.cp) on CPU
processes: two or three ranks over gloo, each holding a shard of every sequence, run a
Full, Reindex, Reuse stack through ContextParallelStack with the library's
shard calls replaced by oracle stand-ins of the same names.  This covers the
exchange plumbing with no GPU: the order of the all-gathers, the candidate and
(out, lse) buffer layouts, and the merges.  Every rank must end with the same
pool, top-k and outputs, equal to the oracle run on the whole sequence
(tldrocket.com "DeepSeek AI Released DeepSeek-V4.1-Flash ...", paragraphs 1
and 3; zerohour.day: a context of one million tokens)."""
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

WORKLOAD = ("long64k", 3000, dict(batch=2, pool_k=1024, top_k=128, T=1, lens=("uniform", 2000, 3000),
                                  pattern="FRUU"))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _setup():
    sys.path.insert(0, ROOT)
    sys.path.insert(0, HERE)
    from fp4_sparse_attention_csa2_b200 import workloads as wl
    name, L, kw = WORKLOAD
    w = wl.Workload(**{**wl.WORKLOADS[name].__dict__, **kw, "name": "cp-cpu"})
    layers = [wl.layer_queries(w, l) for l in range(len(w.pattern))]
    return w, layers, wl.seq_lens(w)


class ShardRef:
    """A rank's shard for the stand-ins: the oracle's cache of its positions."""

    def __init__(self, w, layers, lens, r, R):
        import oracle
        from fp4_sparse_attention_csa2_b200 import workloads as wl
        self.bounds = [wl.shard_bounds(int(lens[b]), R)[r] for b in range(w.batch)]
        n = [nb for _, nb in self.bounds]
        cap = max(64, (max(n) + 63) // 64 * 64)
        self.ref = oracle.RefCache(w.batch, w.batch * cap, w.D, w.D_I, w.row_stride, w.idx_key_dtype, n,
                                   seq_stride_slots=cap)
        for b in range(w.batch):
            L = int(lens[b])
            p0, nb = self.bounds[b]
            keys, _ = wl.index_keys(w, b, L, layers[0]["q_idx"][b, w.T - 1])
            x = wl.bf16_bits(wl.latent(w, b, L))
            self.ref.write(b, 0, x[p0:p0 + nb], wl.host_array(keys)[p0:p0 + nb],
                           wl.F32 if w.idx_key_dtype == wl.F32 else wl.BF16)
        self.batch, self.dim = w.batch, w.D


class OracleOps:
    """The shard calls of the binding, computed by the oracle on host tensors
    (same names and arguments as fp4_sparse_attention_csa2_b200's)."""

    def __init__(self, w):
        self.w = w

    def workspace_bytes(self, *a):
        return 16

    def cp_merge_workspace_bytes(self, *a):
        return 16

    def workspace_init(self, ws):
        pass

    @staticmethod
    def _put(cand, b, pos, scores):
        cand[b, :, 0] = -1
        cand[b].view(torch.float32)[:, 1] = 0.0
        cand[b, :len(pos), 0] = torch.as_tensor(pos, dtype=torch.int32)
        cand[b].view(torch.float32)[:len(pos), 1] = torch.as_tensor(scores, dtype=torch.float32)

    def cp_index_local(self, shard, pos0, q_idx, head_w, pool_k, cand, ws):
        import oracle
        from fp4_sparse_attention_csa2_b200 import workloads as wl
        for b in range(shard.batch):
            pool, _, s = oracle.index_full(shard.ref, b, 1, 0, wl.host_array(q_idx)[b, 0], self.w.q_idx_dtype,
                                           head_w[b, 0].numpy(), pool_k, 1, want_scores=True)
            pool = pool[pool >= 0]
            self._put(cand, b, pool + int(pos0[b]), s[pool])

    def cp_reindex_local(self, shard, pos0, q_idx, head_w, pool, pool_scores, ws):
        import oracle
        from fp4_sparse_attention_csa2_b200 import workloads as wl
        for b in range(shard.batch):
            p0, nb = shard.bounds[b]
            g = pool[b].numpy()
            local = np.where((g >= p0) & (g < p0 + nb), g - p0, -1).astype(np.int32)
            _, s = oracle.index_reindex(shard.ref, b, 1, 0, wl.host_array(q_idx)[b, 0], self.w.q_idx_dtype,
                                        head_w[b, 0].numpy(), local, 1, want_scores=True)
            pool_scores[b] = torch.from_numpy(np.where(local >= 0, s, 0.0).astype(np.float32))

    def cp_reindex_select(self, pool, pool_scores, lens_global, top_k, topk):
        import oracle
        for b in range(pool.shape[0]):
            pos = pool[b].numpy()
            sc = pool_scores[b].numpy().astype(np.float64)
            ok = (pos >= 0) & (pos < int(lens_global[b])) & ~np.isnan(sc)
            topk[b] = torch.from_numpy(oracle.select_top(sc[ok], pos[ok], top_k))

    def cp_merge_select(self, cand, lens_global, n_a, out_a, ws, n_b=0, out_b=None):
        import oracle
        Rr, B = cand.shape[:2]
        for b in range(B):
            pos = cand[:, b, :, 0].reshape(-1).numpy()
            sc = cand[:, b].view(torch.float32)[..., 1].reshape(-1).numpy().astype(np.float64)
            ok = (pos >= 0) & (pos < int(lens_global[b]))
            out_a[b] = torch.from_numpy(oracle.select_top(sc[ok], pos[ok], n_a))
            if n_b:
                out_b[b] = torch.from_numpy(oracle.select_top(sc[ok], pos[ok], n_b))

    def cp_sparse_swa_attn(self, shard, pos0, lens_global, q, topk, window, out, lse, ws, sm_scale=0.0):
        import oracle
        from fp4_sparse_attention_csa2_b200 import workloads as wl
        from harness import attended_positions
        for b in range(shard.batch):
            p0, nb = shard.bounds[b]
            S = attended_positions(topk[b].numpy(), int(lens_global[b]) - 1, window)
            part = np.array(sorted(t - p0 for t in S if p0 <= t < p0 + nb), dtype=np.int32)
            if part.size == 0:
                out[b] = 0.0
                lse[b] = -float("inf")
                continue
            o, l = oracle.sparse_swa_attn(shard.ref, b, 1, 0, wl.bf16_bits(q)[b, 0], part, 0, sm_scale)
            out[b] = torch.from_numpy(o)
            lse[b] = torch.from_numpy(l)

    def lse_merge(self, outs, lses, out, lse=None):
        import oracle
        for b in range(outs.shape[1]):
            o, l = oracle.lse_merge(outs[:, b].numpy(), lses[:, b].numpy())
            out[b] = torch.from_numpy(o)
            if lse is not None:
                lse[b] = torch.from_numpy(l)


def _worker(rank, R, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import traceback
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=R, timeout=datetime.timedelta(seconds=60))
    try:
        _run(rank, R, q)
    except Exception:
        q.put((rank, traceback.format_exc()))
    finally:
        dist.destroy_process_group()


def _run(rank, R, q):
    if True:
        w, layers, lens = _setup()
        import fp4_sparse_attention_csa2_b200 as csa2
        from fp4_sparse_attention_csa2_b200.cp import ContextParallelStack
        shard = ShardRef(w, layers, lens, rank, R)
        pos0 = torch.tensor([p0 for p0, _ in shard.bounds], dtype=torch.int32)
        st = ContextParallelStack(shard, pos0, torch.as_tensor(lens), w.H, w.pool_k, w.top_k, w.window,
                                  ops=OracleOps(w), device="cpu")
        assert st.R == R
        B = w.batch
        pool = torch.full((B, w.pool_k), -7, dtype=torch.int32)
        topk = torch.full((B, w.top_k), -7, dtype=torch.int32)
        res = []
        for l, mode in enumerate(w.pattern):
            out = torch.empty((B, w.H, w.D), dtype=torch.float32)
            lse = torch.empty((B, w.H), dtype=torch.float32)
            m = {"F": csa2.FULL, "R": csa2.REINDEX, "U": csa2.REUSE}[mode]
            L = layers[l]
            st.layer(m, L["q"], topk, out, lse, q_idx=L["q_idx"], head_w=L["w"], pool=pool)
            res.append((pool.numpy().copy(), topk.numpy().copy(), out.numpy().copy(), lse.numpy().copy()))
        q.put((rank, res))


@pytest.mark.parametrize("R", [2, 3])
def test_ranks_match_the_whole_sequence(R):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, R, port, q)) for r in range(R)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    for r in range(R):
        assert not isinstance(got[r], str), got[r]
    for p in procs:
        assert p.exitcode == 0
    # every rank holds the same results
    for r in range(1, R):
        for a, b in zip(got[0], got[r]):
            for x, y in zip(a, b):
                assert np.array_equal(x, y)
    sys.path.insert(0, HERE)
    import oracle
    from harness import band_set_check, build_ref_cache, host_layer
    from fp4_sparse_attention_csa2_b200 import workloads as wl
    w, layers, lens = _setup()
    ref = build_ref_cache(w, layers=layers)
    hl = [host_layer(L) for L in layers]
    res = got[0]
    for b in range(w.batch):
        pool_cur = None
        for l, mode in enumerate(w.pattern):
            gpool, gtopk, gout, glse = res[l]
            if mode == "F":
                pool, topk, s = oracle.index_full(ref, b, 1, 0, hl[l]["q_idx"][b, 0], w.q_idx_dtype, hl[l]["w"][b, 0],
                                                  w.pool_k, w.top_k, want_scores=True)
                # the same oracle scores on both sides: the sets agree exactly
                # outside ties at the cutoff
                band_set_check(gpool[b], pool, lambda t: s[t], s.size, rel=1e-6)
                band_set_check(gtopk[b], topk, lambda t: s[t], s.size, rel=1e-6)
                pool_cur = gpool[b]
            elif mode == "R":
                topk, s = oracle.index_reindex(ref, b, 1, 0, hl[l]["q_idx"][b, 0], w.q_idx_dtype, hl[l]["w"][b, 0],
                                               pool_cur, w.top_k, want_scores=True)
                by_pos = {int(t): float(v) for t, v in zip(pool_cur, s) if t >= 0}
                band_set_check(gtopk[b], topk, lambda t: by_pos[t], len(by_pos), rel=1e-6)
            else:
                assert np.array_equal(gtopk[b], res[l - 1][1][b])
            ro, rl = oracle.sparse_swa_attn(ref, b, 1, 0, wl.bf16_bits(layers[l]["q"])[b, 0], gtopk[b], w.window)
            assert np.max(np.abs(gout[b] - ro)) <= 1e-5
            assert np.max(np.abs(glse[b] - rl)) <= 1e-5

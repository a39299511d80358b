"""Context-parallel decode of a CSA2 stack: one sequence's positions spread
over the ranks of a process group, one rank per GPU (tldrocket.com, "DeepSeek
AI Released DeepSeek-V4.1-Flash with 1M Context, FP4 KV Cache, and
Cross-Layer Attention Reuse", paragraphs 1 and 3; zerohour.day: a context of
one million tokens).

Each rank holds a shard of the cache (positions [pos0[b], pos0[b] + n_r[b]) of
sequence b, as its own positions 0 .. n_r[b] - 1) and runs the library's shard
calls; the exchanges between them are all-gathers over the process group
(NCCL over NVLink on GPUs):

    Full     cp_index_local -> all-gather (pool_k candidates a rank) ->
             cp_merge_select (pool and top-k, the same on every rank)
    Reindex  cp_reindex_local -> all-reduce (sum) of the pool's scores (each
             entry is scored by its one owner, the other ranks add zeros) ->
             cp_reindex_select (top-k)
    every    cp_sparse_swa_attn -> all-gather of (out, lse) -> lse_merge

Per layer and sequence that is pool_k * 8 B of candidates a rank (Full),
pool_k * 4 B of scores (Reindex) and H * (dim + 1) * 4 B of attention part a
rank; every rank then holds the whole layer's output.  The library's calls are the only
compute; this module only sequences them and the collectives.
"""
import torch
import torch.distributed as dist

import fp4_sparse_attention_csa2_b200 as csa2


class ContextParallelStack:
    """One rank's side of a context-parallel stack.

    shard        this rank's cache (a csa2.Cache, or anything with .ref for
                 the library and .batch / .dim)
    pos0         int32 [B]: the global position of the shard's position 0
    lens_global  int32 [B]: the sequences' global lengths (the query token
                 sits at Lg - 1)
    ops          the module whose functions run the steps (default: the
                 library binding); tests hand in a stand-in with the same
                 function names
    """

    def __init__(self, shard, pos0, lens_global, H, pool_k, top_k, window, group=None, ops=None, device="cuda"):
        self.ops = csa2 if ops is None else ops
        self.group = group
        self.R = dist.get_world_size(group)
        self.shard, self.pos0, self.lens_global = shard, pos0, lens_global
        self.B, self.D = shard.batch, shard.dim
        self.H, self.pool_k, self.top_k, self.window = H, pool_k, top_k, window
        o = self.ops
        self.ws = torch.empty(o.workspace_bytes(shard, 1, H, pool_k, top_k, window), dtype=torch.uint8, device=device)
        o.workspace_init(self.ws)
        self.mws = torch.empty(o.cp_merge_workspace_bytes(self.R, self.B, pool_k), dtype=torch.uint8, device=device)
        o.workspace_init(self.mws)
        B, R = self.B, self.R
        self.cand_pool = torch.empty((B, pool_k, 2), dtype=torch.int32, device=device)
        self.pool_scores = torch.empty((B, pool_k), dtype=torch.float32, device=device)
        self.gath_pool = torch.empty((R, B, pool_k, 2), dtype=torch.int32, device=device)
        # a rank's attention part as one buffer: out [B][H][D] then lse [B][H]
        self.n_out = B * H * self.D
        self.part = torch.empty(self.n_out + B * H, dtype=torch.float32, device=device)
        self.gath_part = torch.empty((R, self.n_out + B * H), dtype=torch.float32, device=device)

    def _gather(self, out, inp):
        # flat views: rank r's buffer lands at out[r]
        dist.all_gather_into_tensor(out.view(-1), inp.view(-1), group=self.group)

    def layer(self, mode, q, topk, out, lse=None, q_idx=None, head_w=None, pool=None, sm_scale=0.0):
        """One layer on every rank (all ranks call it with the same mode):
        q bf16 [B, 1, H, dim]; topk int32 [B, top_k] (written by FULL and
        REINDEX, read by every mode); pool int32 [B, pool_k] (written by FULL,
        read by REINDEX); out fp32 [B, H, dim] and lse fp32 [B, H] (nullable)
        receive the layer's attention over the whole sequence."""
        o, B = self.ops, self.B
        if mode == csa2.FULL:
            o.cp_index_local(self.shard, self.pos0, q_idx, head_w, self.pool_k, self.cand_pool, self.ws)
            self._gather(self.gath_pool, self.cand_pool)
            o.cp_merge_select(self.gath_pool, self.lens_global, self.pool_k, pool, self.mws, n_b=self.top_k,
                              out_b=topk)
        elif mode == csa2.REINDEX:
            o.cp_reindex_local(self.shard, self.pos0, q_idx, head_w, pool, self.pool_scores, self.ws)
            dist.all_reduce(self.pool_scores, op=dist.ReduceOp.SUM, group=self.group)
            o.cp_reindex_select(pool, self.pool_scores, self.lens_global, self.top_k, topk)
        elif mode != csa2.REUSE:
            raise ValueError("mode must be FULL, REINDEX or REUSE")
        part_out = self.part[:self.n_out].view(B, self.H, self.D)
        part_lse = self.part[self.n_out:].view(B, self.H)
        o.cp_sparse_swa_attn(self.shard, self.pos0, self.lens_global, q, topk, self.window, part_out, part_lse,
                             self.ws, sm_scale=sm_scale)
        self._gather(self.gath_part, self.part)
        outs = self.gath_part[:, :self.n_out].view(self.R, B, self.H, self.D)
        lses = self.gath_part[:, self.n_out:].view(self.R, B, self.H)
        o.lse_merge(outs, lses, out, lse)

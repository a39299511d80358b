// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"

namespace csa2 {

// Tries of the bounded mbarrier waits that guard work (not the drains that
// wait for copies and MMAs already in flight) in the kernels launched from now
// on; csa2_debug_set_wait_limit sets it (a diagnostic: 0 makes those waits
// give up at once), the default is tc::kWaitLimit (about two seconds).
uint32_t wait_limit();

// Radix-select state of one workspace (see topk.cu).  Counts and histograms
// are per segment (one segment = one (sequence, query token)).
constexpr int kRadixBins = 2048;
constexpr int kSelCounters = 32;  // per segment: counters of two targets, an arrival count, the plan
struct SelWork {
    uint32_t* hist;   // [nseg][3][kRadixBins]
    uint32_t* cnt;    // [nseg][kSelCounters]: a outputs, a candidates, b outputs, b candidates, a / b survivors,
                      // -, -, pass-1 arrivals, then the published plan
    uint32_t* cand1;  // [nseg][cand_stride] (key, id) pairs: level-1 candidates of target a
    uint32_t* cand2;  // [nseg][cand_stride]: of target b
    uint32_t* surv1;  // [nseg][cand_stride]: level-2 survivors of target a
    uint32_t* surv2;  // [nseg][cand_stride]: of target b
    int64_t cand_stride;
    uint32_t* hist3 = nullptr;   // [nseg][2][kRadixBins]: digit 3 of both targets (one-grid selection; nullable)
    uint32_t* status = nullptr;  // sticky device status word
};

// Where the elements of one selection come from.
//   ids == nullptr: element i is position i, valid for i <= p_j (Full scores).
//   ids != nullptr: element i is position ids[seg*ids_stride + i], valid when
//                   0 <= id <= p_j; its value is vals[seg*vals_stride + (gather ? id : i)].
struct SelSrc {
    const float* vals;
    int64_t vals_stride;
    const int32_t* ids;
    int64_t ids_stride;
    int gather;
    int64_t n;                // elements per segment (upper bound)
    const int32_t* seq_lens;  // for ids == nullptr
    int T;
    int64_t cap;
};

cudaError_t launch_append_quant(const DevCache& c, const void* x, const void* idx_new, int idx_new_f32,
                                const int32_t* start_pos, int n_new, uint32_t* status, cudaStream_t st,
                                int num_sms);

// Diagnostic: the quantiser's conversions on arbitrary fp32 values (format 0:
// E2M1 codes, 1: E4M3 codes), one code per byte.
cudaError_t launch_debug_encode(int format, const float* x, int64_t n, uint8_t* out, cudaStream_t st, int num_sms);

// Stored rows and keys of positions start_pos[b] + i between the cache and
// packed buffers [batch][n][dim / 2 + dim / 16] and [batch][n][key bytes].
cudaError_t launch_rows_io(const DevCache& c, bool to_buffers, const int32_t* start_pos, int n, void* rows, void* keys,
                           uint32_t* status, cudaStream_t st);

// Full scoring: scores[(b*T + j) * cap + t] for t <= p_j.
cudaError_t launch_score_full(const DevCache& c, const void* q, int q_f32, const float* hw, int T, int H_I,
                              float* scores, uint32_t* status, cudaStream_t st, int num_sms);

// Full scoring on tensor cores (E4M3 keys); also accumulates the level-1 radix
// histogram of every (sequence, token) into hist when it is not null.
bool score_full_tc_supported(const DevCache& c, int T, int H_I);
cudaError_t launch_score_full_tc(const DevCache& c, const void* q, const float* hw, int T, int H_I, float* scores,
                                 uint32_t* hist, uint32_t* status, cudaStream_t st, int num_sms);

// Reindex on the tensor cores (E4M3 keys, bf16 queries): pool rescoring into
// scores[seg * pool_k + i] (NaN for entries that are not candidates) and the
// top_k of each segment's pool, in one kernel; counters[seg] are zero on entry
// and on exit.
bool reindex_tc_supported(const DevCache& c, int H_I);
// The same kernel's scores alone: scores[seg][i] for the pool entries (NaN
// for entries that are not candidates), no selection.
cudaError_t launch_reindex_tc_scores(const DevCache& c, const void* q, const float* hw, int T, int H_I,
                                     const int32_t* pool, int pool_k, float* scores, uint32_t* status, cudaStream_t st);
// grid_hist / grid_cnt (nullable): the segment histograms [nseg][3][2048] and
// counters [nseg][kSelCounters] (zero between calls) of the grid-mode select.
cudaError_t launch_reindex_tc(const DevCache& c, const void* q, const float* hw, int T, int H_I,
                              const int32_t* pool, int pool_k, int top_k, int32_t* topk, float* scores,
                              uint32_t* counters, uint32_t* grid_hist, uint32_t* grid_cnt, uint32_t* status,
                              cudaStream_t st);

// Pool rescoring: scores[seg * pool_k + i] for pool entry i of segment seg.
cudaError_t launch_score_pool(const DevCache& c, const void* q, int q_f32, const float* hw, int T, int H_I,
                              const int32_t* pool, int pool_k, float* scores, uint32_t* status, cudaStream_t st);
// Candidate list of a pool update, ids[seg][0 .. pool_k + n_new): the previous
// pool's entries (-1 kept; an entry at or beyond the first appended position
// L - n_new, or beyond the token's position, is flagged and dropped), then the
// appended positions L - n_new .. L - 1 (those beyond the token's position -1).
// *len = max(0, *seq_len - drop): the length of a sequence cut back by `drop` positions.
cudaError_t launch_chunk_len(const int32_t* seq_len, int drop, int32_t* len, cudaStream_t st);
cudaError_t launch_pool_candidates(const DevCache& c, int T, const int32_t* pool_prev, int pool_k, int n_new,
                                   int32_t* ids, uint32_t* status, cudaStream_t st);

// Top-n selection per segment into out[seg * out_stride + 0..n_out) (-1 padded).
// hist_ready: the level-1 histogram was zeroed and accumulated by the scoring
// kernel already (the counters are still cleared here).  out_vals (nullable)
// receives the score of every selected element at the same index.
cudaError_t launch_select(const SelSrc& src, const SelWork& wk, int nseg, int n_out, int32_t* out,
                          int64_t out_stride, cudaStream_t st, bool hist_ready = false, float* out_vals = nullptr);
// One CTA per segment of at most 16,384 elements: the n_a best into out_a
// (scores into vals_a, nullable) and, with n_b > 0, the n_b best of those
// into out_b (a subset of out_a).
cudaError_t launch_select_local(const SelSrc& src, int nseg, int n_a, int32_t* out_a, float* vals_a, int64_t stride_a,
                                int n_b, int32_t* out_b, int64_t stride_b, cudaStream_t st);
// Two selections of the same segments (more than 16,384 elements each): the
// n_a best into out_a (scores into vals_a, nullable) and the n_b <= n_a best
// into out_b (n_b == 0: none), out_b a subset of out_a.
cudaError_t launch_select_dual(const SelSrc& src, const SelWork& wk, int nseg, int n_a, int32_t* out_a, float* vals_a,
                               int64_t stride_a, int n_b, int32_t* out_b, int64_t stride_b, cudaStream_t st,
                               bool hist_ready);

// A layer's own window state: bf16 rows [batch][len][dim], position t of
// sequence b at row t mod len (rows == nullptr: the window comes from the
// shared FP4 cache).
struct Ring {
    __nv_bfloat16* rows = nullptr;
    int64_t len = 0;
};
cudaError_t launch_ring_append(const Ring& ring, int batch, int dim, const void* x, const int32_t* start_pos,
                               int n_new, cudaStream_t st);

// Attention partials + combine.
struct AttnWork {
    float* part_o;    // [nseg][nchunk][D][H]
    float* part_ml;   // [nseg][nchunk][H][2]
    int nchunk;
};
int attn_rows_per_chunk();       // smallest chunk of any attention kernel (sizes the workspace)
bool attn_tc_supported(const DevCache& c, int H);
int attn_tc_rows_per_chunk();
// heads per CTA: H, halved (down to 16) while the grid would leave SMs idle
int attn_tc_heads_per_cta(int H, int nchunk, int nseg, int num_sms);
// A context-parallel shard's place in its sequence (pos0 == nullptr: not a shard).
struct CpShard {
    const int32_t* pos0 = nullptr;   // [batch] the sequence position of the shard's position 0
    const int32_t* glens = nullptr;  // [batch] the sequences' lengths
};
cudaError_t launch_attention_tc(const DevCache& c, const void* q, int T, int H, const int32_t* topk, int top_k,
                                int window, float sm_scale, const Ring& ring, const AttnWork& aw, uint32_t* status,
                                cudaStream_t st, int num_sms, const CpShard& cp = CpShard{});
cudaError_t launch_attn_combine(const DevCache& c, int T, int H, const AttnWork& aw, float* out, float* lse,
                                cudaStream_t st);
cudaError_t launch_attention(const DevCache& c, const void* q, int T, int H, const int32_t* topk, int top_k,
                             int window, float sm_scale, const Ring& ring, float* out, float* lse,
                             const AttnWork& aw, uint32_t* status, cudaStream_t st, int num_sms);

// Context-parallel decode (cp.cu): a candidate is a global position and its
// score, laid out as csa2_cand.
struct CpCand {
    int32_t pos;
    float score;
};
// cand[b][i] <- (ids[b][i] + pos0[b], vals[b][i]), or (-1, 0) for ids < 0.
cudaError_t launch_cp_pack(const int32_t* ids, const float* vals, int64_t in_stride, const int32_t* pos0, int batch,
                           int n, CpCand* cand, cudaStream_t st);
// local[b][i] <- pool[b][i] - pos0[b] when in [0, shard_lens[b]), else -1.
cudaError_t launch_cp_localize(const int32_t* pool, const int32_t* pos0, const int32_t* shard_lens, int batch, int n,
                               int32_t* local, cudaStream_t st);
// out[e] <- sc[e] where local[e] >= 0 (this shard's pool entries), else 0.
cudaError_t launch_cp_owned_scores(const int32_t* local, const float* sc, int64_t n, float* out, cudaStream_t st);
// [R][batch][n] candidates -> ids / vals [batch][R * n].
cudaError_t launch_cp_unpack(const CpCand* cand, int R, int batch, int n, int32_t* ids, float* vals,
                             cudaStream_t st);
// The shard's part of window ∪ top-k as a list [batch][window + top_k] of shard positions (-1: none).
cudaError_t launch_cp_attn_list(const int32_t* topk, int top_k, int window, const int32_t* pos0,
                                const int32_t* shard_lens, const int32_t* lens_global, int batch, int32_t* list,
                                uint32_t* status, cudaStream_t st);
cudaError_t launch_lse_merge(int R, int batch, int H, int D, const float* outs, int64_t out_stride, const float* lses,
                             int64_t lse_stride, float* out, float* lse, cudaStream_t st);

}  // namespace csa2

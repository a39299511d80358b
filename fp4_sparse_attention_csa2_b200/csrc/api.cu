// Host side of the libcsa2 C ABI: argument validation, workspace layout and
// kernel dispatch.  Every entry point validates on the host, then only
// enqueues work on the caller's stream.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>

#include "../../include/csa2.h"
#include "abi_checks.h"
#include "kernels.h"
#include "tc.cuh"

using namespace csa2;

namespace {
std::atomic<uint32_t> g_wait_limit{tc::kWaitLimit};
}  // namespace

uint32_t csa2::wait_limit() { return g_wait_limit.load(std::memory_order_relaxed); }

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxPool = 16384;  // candidate pool bound, tldrocket.com page, paragraph 3
constexpr int64_t kSmallSelect = 16384;  // selections over at most this many elements run in one CTA

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int64_t capacity(const csa2_cache* c) {
    return c->page_table ? (int64_t)c->max_pages * c->page_size : c->seq_stride_slots;
}

csa2_status check_cache(const csa2_cache* c) {
    if (!c || !c->kv_rows || !c->idx_keys || !c->seq_lens) return CSA2_ERR_INVALID_ARG;
    if (!aligned16(c->kv_rows) || !aligned16(c->idx_keys) || !aligned4(c->seq_lens)) return CSA2_ERR_INVALID_ARG;
    if (c->page_table && !aligned4(c->page_table)) return CSA2_ERR_INVALID_ARG;
    if (c->batch < 1 || c->batch > 65535 || c->n_slots < 1) return CSA2_ERR_INVALID_ARG;
    if (c->dim < 32 || c->dim % 32) return CSA2_ERR_INVALID_ARG;
    if (c->dim > 512) return CSA2_ERR_UNSUPPORTED;
    if (c->idx_dim != 64) return CSA2_ERR_UNSUPPORTED;
    if (c->row_stride < c->dim / 2 + c->dim / 16 || c->row_stride % 16) return CSA2_ERR_INVALID_ARG;
    if (c->idx_key_dtype != CSA2_E4M3 && c->idx_key_dtype != CSA2_F32) return CSA2_ERR_INVALID_ARG;
    if (c->page_table) {
        if (c->max_pages < 1 || c->page_size < 64 || c->page_size % 64) return CSA2_ERR_INVALID_ARG;
        if (c->n_slots % c->page_size) return CSA2_ERR_INVALID_ARG;
    } else {
        if (c->seq_stride_slots < 64 || c->seq_stride_slots % 64) return CSA2_ERR_INVALID_ARG;
        if (c->seq_stride_slots * (int64_t)c->batch > c->n_slots) return CSA2_ERR_INVALID_ARG;
    }
    if (capacity(c) > (int64_t)1 << 30) return CSA2_ERR_UNSUPPORTED;
    return CSA2_OK;
}

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

// Workspace layout (byte offsets, each section 256-byte aligned):
//   status word | full-layer scores | radix histograms | digit-3 histograms | scratch histogram |
//   radix counters | Reindex arrival counters | candidates 1, 2 | survivors 1, 2 |
//   pool scores | pool-update candidates and their scores | attention partials
// The radix histograms and counters are zero between calls: the workspace
// starts zeroed and every large selection clears what it used.
struct Layout {
    size_t status, scores, hist, hist3, hist_scratch, cnt, rx_cnt, cand1, cand2, surv1, surv2, pscores, upd_ids,
        upd_scores, part_o, part_ml, total;
    int64_t nseg, cap, cand_stride;
    int nchunk;
};

bool make_layout(const csa2_cache* c, int T, int H, int pool_k, int top_k, int window, Layout* L) {
    if (check_cache(c) != CSA2_OK || T < 1 || H < 1 || pool_k < 1 || top_k < 0 || window < 0) return false;
    L->cap = capacity(c);
    L->nseg = (int64_t)c->batch * T;
    L->cand_stride = L->cap > pool_k ? L->cap : pool_k;
    L->nchunk = (int)((window + top_k + attn_rows_per_chunk() - 1) / attn_rows_per_chunk());
    if (L->nchunk < 1) L->nchunk = 1;
    size_t off = 0;
    L->status = off; off = align_up(off + 16);
    L->scores = off; off = align_up(off + sizeof(float) * (size_t)(L->nseg * L->cap));
    L->hist = off; off = align_up(off + sizeof(uint32_t) * (size_t)L->nseg * 3 * kRadixBins);
    L->hist3 = off; off = align_up(off + sizeof(uint32_t) * (size_t)L->nseg * 2 * kRadixBins);
    L->hist_scratch = off; off = align_up(off + sizeof(uint32_t) * (size_t)L->nseg * kRadixBins);
    L->cnt = off; off = align_up(off + sizeof(uint32_t) * (size_t)L->nseg * kSelCounters);
    L->rx_cnt = off; off = align_up(off + sizeof(uint32_t) * (size_t)L->nseg);
    L->cand1 = off; off = align_up(off + 2 * sizeof(uint32_t) * (size_t)(L->nseg * L->cand_stride));
    L->cand2 = off; off = align_up(off + 2 * sizeof(uint32_t) * (size_t)(L->nseg * L->cand_stride));
    L->surv1 = off; off = align_up(off + 2 * sizeof(uint32_t) * (size_t)(L->nseg * L->cand_stride));
    L->surv2 = off; off = align_up(off + 2 * sizeof(uint32_t) * (size_t)(L->nseg * L->cand_stride));
    L->pscores = off; off = align_up(off + sizeof(float) * (size_t)L->nseg * pool_k);
    // the candidate list of a pool update: the previous pool and up to kMaxPool appended positions
    L->upd_ids = off; off = align_up(off + sizeof(int32_t) * (size_t)L->nseg * (pool_k + kMaxPool));
    L->upd_scores = off; off = align_up(off + sizeof(float) * (size_t)L->nseg * (pool_k + kMaxPool));
    L->part_o = off; off = align_up(off + sizeof(float) * (size_t)L->nseg * L->nchunk * H * c->dim);
    L->part_ml = off; off = align_up(off + sizeof(float) * (size_t)L->nseg * L->nchunk * H * 2);
    L->total = off;
    return true;
}

template <typename T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }

SelWork sel_work(void* ws, const Layout& L) {
    SelWork w;
    w.hist = at<uint32_t>(ws, L.hist);
    w.cnt = at<uint32_t>(ws, L.cnt);
    w.cand1 = at<uint32_t>(ws, L.cand1);
    w.cand2 = at<uint32_t>(ws, L.cand2);
    w.surv1 = at<uint32_t>(ws, L.surv1);
    w.surv2 = at<uint32_t>(ws, L.surv2);
    w.cand_stride = L.cand_stride;
    w.hist3 = at<uint32_t>(ws, L.hist3);
    w.status = at<uint32_t>(ws, L.status);
    return w;
}

csa2_status cuda_status(cudaError_t e) { return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA; }

csa2_status check_ws(const csa2_cache* c, int T, int H, int pool_k, int top_k, int window, void* ws,
                     size_t ws_bytes, Layout* L) {
    if (!make_layout(c, T, H, pool_k, top_k, window, L)) return CSA2_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws) || ws_bytes < L->total) return CSA2_ERR_INVALID_ARG;
    return CSA2_OK;
}

csa2_status check_index_args(const csa2_cache* c, const void* q_idx, csa2_dtype q_dtype, const float* head_w, int T,
                             int H_I, int pool_k, int top_k) {
    csa2_status s = check_cache(c);
    if (s != CSA2_OK) return s;
    if (!q_idx || !head_w || !aligned16(q_idx) || !aligned16(head_w)) return CSA2_ERR_INVALID_ARG;
    if (T < 1 || H_I < 1 || H_I > 64 || T * H_I > 256) return CSA2_ERR_INVALID_ARG;
    if (top_k < 1 || top_k > pool_k || pool_k > kMaxPool) return CSA2_ERR_INVALID_ARG;
    if (c->idx_key_dtype == CSA2_E4M3 && q_dtype != CSA2_BF16) return CSA2_ERR_INVALID_ARG;
    if (c->idx_key_dtype == CSA2_F32 && q_dtype != CSA2_F32) return CSA2_ERR_INVALID_ARG;
    return CSA2_OK;
}

csa2_status topk_from_pool(const csa2_cache* c, const Layout& L, void* ws, const float* vals, int64_t vals_stride,
                           int gather, const int32_t* pool_idx, int pool_k, int top_k, int32_t* topk_idx, int T,
                           cudaStream_t st) {
    SelSrc src;
    src.vals = vals;
    src.vals_stride = vals_stride;
    src.ids = pool_idx;
    src.ids_stride = pool_k;
    src.gather = gather;
    src.n = pool_k;
    src.seq_lens = c->seq_lens;
    src.T = T;
    src.cap = L.cap;
    return cuda_status(launch_select(src, sel_work(ws, L), (int)L.nseg, top_k, topk_idx, top_k, st));
}

// Scoring launch shared by csa2_index_scores and csa2_index_full: tensor cores
// for E4M3 keys, CUDA cores for fp32 keys.  hist (nullable) receives the
// level-1 radix histogram when the tensor-core kernel runs; returns whether it did.
csa2_status launch_scores(const csa2_cache* cache, const void* q_idx, csa2_dtype q_dtype, const float* head_w, int T,
                          int H_I, float* scores, uint32_t* hist, uint32_t* status, cudaStream_t st, bool* fused) {
    DevCache d = dev_cache(cache);
    *fused = false;
    cudaError_t e;
    if (score_full_tc_supported(d, T, H_I)) {
        e = launch_score_full_tc(d, q_idx, head_w, T, H_I, scores, hist, status, st, num_sms());
        *fused = hist != nullptr;
    } else {
        e = launch_score_full(d, q_idx, q_dtype == CSA2_F32, head_w, T, H_I, scores, status, st, num_sms());
    }
    return cuda_status(e);
}

}  // namespace

DevCache csa2::dev_cache(const csa2_cache* c) {
    DevCache d;
    d.rows = c->kv_rows;
    d.keys = c->idx_keys;
    d.page_table = c->page_table;
    d.seq_lens = c->seq_lens;
    d.batch = c->batch;
    d.max_pages = c->max_pages;
    d.page_size = c->page_size;
    d.dim = c->dim;
    d.idx_dim = c->idx_dim;
    d.row_stride = c->row_stride;
    d.seq_stride = c->seq_stride_slots;
    d.n_slots = c->n_slots;
    d.cap = capacity(c);
    d.key_dtype = c->idx_key_dtype == CSA2_E4M3 ? 2 : 0;
    return d;
}

csa2_status csa2::check_reindex_args(const csa2_cache* c, const void* q_idx, csa2_dtype q_dtype,
                                     const float* head_w, int T, int H_I, const int32_t* pool_idx, int pool_k,
                                     int top_k, const int32_t* topk_idx) {
    csa2_status s = check_index_args(c, q_idx, q_dtype, head_w, T, H_I, pool_k, top_k);
    if (s != CSA2_OK) return s;
    if (!pool_idx || !topk_idx || !aligned16(pool_idx) || !aligned16(topk_idx)) return CSA2_ERR_INVALID_ARG;
    return CSA2_OK;
}

namespace {

// Attention with the window rows from the FP4 cache (ring.rows == nullptr) or
// from a layer-local bf16 ring.
csa2_status attention(const csa2_cache* cache, const Ring& ring, const void* q_bf16, int T, int H,
                      const int32_t* topk_idx, int top_k, int window, float sm_scale, float* out, float* lse,
                      void* ws, size_t ws_bytes, void* stream) {
    csa2_status s = check_cache(cache);
    if (s != CSA2_OK) return s;
    if (!q_bf16 || !out || !aligned16(q_bf16) || !aligned16(out) || (lse && !aligned16(lse))) return CSA2_ERR_INVALID_ARG;
    if (T < 1 || H < 1 || top_k < 0 || window < 0 || window > kMaxPool || top_k > kMaxPool) return CSA2_ERR_INVALID_ARG;
    if (top_k > 0 && (!topk_idx || !aligned16(topk_idx))) return CSA2_ERR_INVALID_ARG;
    if (H > 64 || H % 16) return CSA2_ERR_UNSUPPORTED;
    if (!std::isfinite(sm_scale)) return CSA2_ERR_INVALID_ARG;
    Layout L;
    s = check_ws(cache, T, H, top_k > 0 ? top_k : 1, top_k, window, ws, ws_bytes, &L);
    if (s != CSA2_OK) return s;
    if (sm_scale <= 0.0f) sm_scale = 1.0f / std::sqrt((float)cache->dim);
    AttnWork aw;
    aw.part_o = at<float>(ws, L.part_o);
    aw.part_ml = at<float>(ws, L.part_ml);
    aw.nchunk = L.nchunk;
    return cuda_status(launch_attention(dev_cache(cache), q_bf16, T, H, topk_idx, top_k, window, sm_scale, ring, out,
                                        lse, aw, at<uint32_t>(ws, L.status), static_cast<cudaStream_t>(stream),
                                        num_sms()));
}

// A ring of ring_len rows for T new tokens a step and a window of `window`:
// the window of the step's first token reaches back T - 1 positions further.
bool ring_ok(const void* ring, int64_t ring_len, int T, int window) {
    return ring && aligned16(ring) && ring_len >= 1 && ring_len >= (int64_t)window + T - 1 && ring_len <= ((int64_t)1 << 30);
}

// Prefill: tokens per chunk, so that every chunk fits the single-step limits
// (T * H_I <= 256 and the tensor-core scorer's 2 T HP <= 256 columns).
int prefill_chunk(int T, int H_I) {
    const int HP = (H_I + 15) / 16 * 16;
    int c = 128 / (HP > 0 ? HP : 16);
    if (c * H_I > 256) c = 256 / H_I;
    if (c < 1) c = 1;
    return c < T ? c : T;
}

// A cache view of sequence b whose length is the device int32 at `len`.
csa2_cache seq_view(const csa2_cache* c, int b, const int32_t* len) {
    csa2_cache v = *c;
    v.batch = 1;
    v.seq_lens = len;
    if (c->page_table) {
        v.page_table = c->page_table + (int64_t)b * c->max_pages;
    } else {
        const int64_t key_bytes = c->idx_key_dtype == CSA2_E4M3 ? c->idx_dim : 4 * c->idx_dim;
        v.kv_rows = static_cast<uint8_t*>(c->kv_rows) + (int64_t)b * c->seq_stride_slots * c->row_stride;
        v.idx_keys = static_cast<uint8_t*>(c->idx_keys) + (int64_t)b * c->seq_stride_slots * key_bytes;
        v.n_slots = c->seq_stride_slots;
    }
    return v;
}

}  // namespace

extern "C" {

size_t csa2_workspace_bytes(const csa2_cache* cache, int T, int H, int pool_k, int top_k, int window) {
    CSA2_RANGE("csa2_workspace_bytes");
    Layout L;
    if (!make_layout(cache, T, H, pool_k, top_k, window, &L)) return 0;
    return L.total;
}

csa2_status csa2_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    CSA2_RANGE("csa2_workspace_init");
    if (!ws || !aligned16(ws) || ws_bytes < 16) return CSA2_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

csa2_status csa2_kv_append_quant(const csa2_cache* cache, const void* x_bf16, const void* idx_new,
                                 csa2_dtype idx_new_dtype, const int32_t* start_pos, int n_new, void* ws,
                                 void* stream) {
    CSA2_RANGE("csa2_kv_append_quant");
    csa2_status s = check_cache(cache);
    if (s != CSA2_OK) return s;
    if (!x_bf16 || !start_pos || !aligned16(x_bf16) || !aligned4(start_pos) || n_new < 0) return CSA2_ERR_INVALID_ARG;
    if (idx_new && (!aligned16(idx_new) || (idx_new_dtype != CSA2_BF16 && idx_new_dtype != CSA2_F32)))
        return CSA2_ERR_INVALID_ARG;
    if (ws && !aligned16(ws)) return CSA2_ERR_INVALID_ARG;
    if (n_new == 0) return CSA2_OK;
    return cuda_status(launch_append_quant(dev_cache(cache), x_bf16, idx_new, idx_new_dtype == CSA2_F32 ? 1 : 0,
                                           start_pos, n_new, static_cast<uint32_t*>(ws),
                                           static_cast<cudaStream_t>(stream), num_sms()));
}

csa2_status csa2_kv_export_rows(const csa2_cache* cache, const int32_t* start_pos, int n, void* rows, void* keys,
                                void* ws, void* stream) {
    CSA2_RANGE("csa2_kv_export_rows");
    csa2_status s = check_cache(cache);
    if (s != CSA2_OK) return s;
    if (!start_pos || !aligned4(start_pos) || n < 0 || !rows || !aligned4(rows) || (keys && !aligned4(keys)) ||
        (ws && !aligned16(ws)))
        return CSA2_ERR_INVALID_ARG;
    if (n == 0) return CSA2_OK;
    return cuda_status(launch_rows_io(dev_cache(cache), true, start_pos, n, rows, keys, static_cast<uint32_t*>(ws),
                                      static_cast<cudaStream_t>(stream)));
}

csa2_status csa2_kv_import_rows(const csa2_cache* cache, const int32_t* start_pos, int n, const void* rows,
                                const void* keys, void* ws, void* stream) {
    CSA2_RANGE("csa2_kv_import_rows");
    csa2_status s = check_cache(cache);
    if (s != CSA2_OK) return s;
    if (!start_pos || !aligned4(start_pos) || n < 0 || !rows || !aligned4(rows) || (keys && !aligned4(keys)) ||
        (ws && !aligned16(ws)))
        return CSA2_ERR_INVALID_ARG;
    if (n == 0) return CSA2_OK;
    return cuda_status(launch_rows_io(dev_cache(cache), false, start_pos, n, const_cast<void*>(rows),
                                      const_cast<void*>(keys), static_cast<uint32_t*>(ws),
                                      static_cast<cudaStream_t>(stream)));
}

csa2_status csa2_index_scores(const csa2_cache* cache, const void* q_idx, csa2_dtype q_dtype, const float* head_w,
                              int T, int H_I, float* scores, void* ws, size_t ws_bytes, void* stream) {
    CSA2_RANGE("csa2_index_scores");
    csa2_status s = check_index_args(cache, q_idx, q_dtype, head_w, T, H_I, 1, 1);
    if (s != CSA2_OK) return s;
    if (scores && !aligned16(scores)) return CSA2_ERR_INVALID_ARG;
    Layout L;
    s = check_ws(cache, T, 1, 1, 1, 0, ws, ws_bytes, &L);
    if (s != CSA2_OK) return s;
    bool fused;
    // the same kernel as in csa2_index_full; its histogram goes to a scratch
    // section that no selection reads
    return launch_scores(cache, q_idx, q_dtype, head_w, T, H_I, scores ? scores : at<float>(ws, L.scores),
                         L.cap > kSmallSelect ? at<uint32_t>(ws, L.hist_scratch) : nullptr,
                         at<uint32_t>(ws, L.status), static_cast<cudaStream_t>(stream), &fused);
}

csa2_status csa2_index_full(const csa2_cache* cache, const void* q_idx, csa2_dtype q_dtype, const float* head_w,
                            int T, int H_I, int pool_k, int top_k, int32_t* pool_idx, int32_t* topk_idx, void* ws,
                            size_t ws_bytes, void* stream) {
    CSA2_RANGE("csa2_index_full");
    csa2_status s = check_index_args(cache, q_idx, q_dtype, head_w, T, H_I, pool_k, top_k);
    if (s != CSA2_OK) return s;
    if (!pool_idx || !topk_idx || !aligned16(pool_idx) || !aligned16(topk_idx)) return CSA2_ERR_INVALID_ARG;
    Layout L;
    s = check_ws(cache, T, 1, pool_k, top_k, 0, ws, ws_bytes, &L);
    if (s != CSA2_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // a large selection takes its level-1 histogram from the scoring kernel
    // (the histograms are zero on entry); a small one builds its own
    uint32_t* hist = L.cap > kSmallSelect ? at<uint32_t>(ws, L.hist) : nullptr;
    // every visible position scored into the workspace
    float* scores = at<float>(ws, L.scores);
    bool fused = false;
    s = launch_scores(cache, q_idx, q_dtype, head_w, T, H_I, scores, hist, at<uint32_t>(ws, L.status), st, &fused);
    if (s != CSA2_OK) return s;
    // the candidate pool: the pool_k best of all visible scores
    SelSrc src;
    src.vals = scores;
    src.vals_stride = L.cap;
    src.ids = nullptr;
    src.ids_stride = 0;
    src.gather = 0;
    src.n = L.cap;
    src.seq_lens = cache->seq_lens;
    src.T = T;
    src.cap = L.cap;
    float* ps = at<float>(ws, L.pscores);
    if (L.cap > kSmallSelect) {
        // long contexts: the pool and this layer's top-k (the top_k best of the
        // same scores, a subset of the pool) come out of one selection
        return cuda_status(launch_select_dual(src, sel_work(ws, L), (int)L.nseg, pool_k, pool_idx, ps, pool_k, top_k,
                                              topk_idx, top_k, st, fused));
    }
    // short contexts: the pool and, from it, the top-k, by one CTA per (sequence, token)
    (void)ps;
    return cuda_status(launch_select_local(src, (int)L.nseg, pool_k, pool_idx, nullptr, pool_k, top_k, topk_idx, top_k,
                                           st));
}

csa2_status csa2_index_reindex(const csa2_cache* cache, const void* q_idx, csa2_dtype q_dtype, const float* head_w,
                               int T, int H_I, const int32_t* pool_idx, int pool_k, int top_k, int32_t* topk_idx,
                               void* ws, size_t ws_bytes, void* stream) {
    CSA2_RANGE("csa2_index_reindex");
    csa2_status s = check_reindex_args(cache, q_idx, q_dtype, head_w, T, H_I, pool_idx, pool_k, top_k, topk_idx);
    if (s != CSA2_OK) return s;
    Layout L;
    s = check_ws(cache, T, 1, pool_k, top_k, 0, ws, ws_bytes, &L);
    if (s != CSA2_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DevCache d = dev_cache(cache);
    uint32_t* status = at<uint32_t>(ws, L.status);
    float* ps = at<float>(ws, L.pscores);
    if (reindex_tc_supported(d, H_I))
        return cuda_status(launch_reindex_tc(d, q_idx, head_w, T, H_I, pool_idx, pool_k, top_k, topk_idx, ps,
                                             at<uint32_t>(ws, L.rx_cnt), at<uint32_t>(ws, L.hist),
                                             at<uint32_t>(ws, L.cnt), status, st));
    cudaError_t e = launch_score_pool(d, q_idx, q_dtype == CSA2_F32, head_w, T, H_I, pool_idx, pool_k, ps, status, st);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;
    return topk_from_pool(cache, L, ws, ps, pool_k, 0, pool_idx, pool_k, top_k, topk_idx, T, st);
}

csa2_status csa2_index_pool_update(const csa2_cache* cache, const void* q_idx, csa2_dtype q_dtype,
                                   const float* head_w, int T, int H_I, const int32_t* pool_prev, int pool_k, int n_new,
                                   int top_k, int32_t* pool_idx, int32_t* topk_idx, void* ws, size_t ws_bytes,
                                   void* stream) {
    CSA2_RANGE("csa2_index_pool_update");
    csa2_status s = check_reindex_args(cache, q_idx, q_dtype, head_w, T, H_I, pool_prev, pool_k, top_k, topk_idx);
    if (s != CSA2_OK) return s;
    if (!pool_idx || !aligned16(pool_idx) || n_new < 0 || n_new > kMaxPool) return CSA2_ERR_INVALID_ARG;
    Layout L;
    s = check_ws(cache, T, 1, pool_k, top_k, 0, ws, ws_bytes, &L);
    if (s != CSA2_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DevCache d = dev_cache(cache);
    uint32_t* status = at<uint32_t>(ws, L.status);
    const int m = pool_k + n_new;                      // candidates per (sequence, token)
    int32_t* ids = at<int32_t>(ws, L.upd_ids);
    float* sc = at<float>(ws, L.upd_scores);
    cudaError_t e = launch_pool_candidates(d, T, pool_prev, pool_k, n_new, ids, status, st);
    if (e == cudaSuccess)
        e = reindex_tc_supported(d, H_I) ? launch_reindex_tc_scores(d, q_idx, head_w, T, H_I, ids, m, sc, status, st)
                                         : launch_score_pool(d, q_idx, q_dtype == CSA2_F32, head_w, T, H_I, ids, m, sc,
                                                             status, st);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;
    SelSrc src;
    src.vals = sc;
    src.vals_stride = m;
    src.ids = ids;
    src.ids_stride = m;
    src.gather = 0;
    src.n = m;
    src.seq_lens = cache->seq_lens;
    src.T = T;
    src.cap = L.cap;
    // the new pool and this token's top-k (a subset of it) from the same scores
    if (m <= kSmallSelect)
        return cuda_status(launch_select_local(src, (int)L.nseg, pool_k, pool_idx, nullptr, pool_k, top_k, topk_idx,
                                               top_k, st));
    return cuda_status(launch_select_dual(src, sel_work(ws, L), (int)L.nseg, pool_k, pool_idx, nullptr, pool_k, top_k,
                                          topk_idx, top_k, st, false));
}

csa2_status csa2_sparse_swa_attn(const csa2_cache* cache, const void* q_bf16, int T, int H, const int32_t* topk_idx,
                                 int top_k, int window, float sm_scale, float* out, float* lse, void* ws,
                                 size_t ws_bytes, void* stream) {
    CSA2_RANGE("csa2_sparse_swa_attn");
    return attention(cache, Ring{}, q_bf16, T, H, topk_idx, top_k, window, sm_scale, out, lse, ws, ws_bytes, stream);
}

csa2_status csa2_sparse_swa_attn_local(const csa2_cache* cache, const void* ring, int64_t ring_len, const void* q_bf16,
                                       int T, int H, const int32_t* topk_idx, int top_k, int window, float sm_scale,
                                       float* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
    CSA2_RANGE("csa2_sparse_swa_attn_local");
    if (!ring_ok(ring, ring_len, T, window)) return CSA2_ERR_INVALID_ARG;
    Ring r;
    r.rows = static_cast<__nv_bfloat16*>(const_cast<void*>(ring));
    r.len = ring_len;
    return attention(cache, r, q_bf16, T, H, topk_idx, top_k, window, sm_scale, out, lse, ws, ws_bytes, stream);
}

csa2_status csa2_ring_append(const csa2_cache* cache, void* ring, int64_t ring_len, const void* x_bf16,
                             const int32_t* start_pos, int n_new, void* stream) {
    CSA2_RANGE("csa2_ring_append");
    csa2_status s = check_cache(cache);
    if (s != CSA2_OK) return s;
    if (!ring_ok(ring, ring_len, 1, 0) || !x_bf16 || !aligned16(x_bf16) || !start_pos || !aligned4(start_pos) ||
        n_new < 0 || (int64_t)n_new > ring_len)
        return CSA2_ERR_INVALID_ARG;
    if (n_new == 0) return CSA2_OK;
    Ring r;
    r.rows = static_cast<__nv_bfloat16*>(ring);
    r.len = ring_len;
    return cuda_status(launch_ring_append(r, cache->batch, cache->dim, x_bf16, start_pos, n_new,
                                          static_cast<cudaStream_t>(stream)));
}

csa2_status csa2_layer_step(const csa2_cache* cache, const csa2_layer_args* a, void* ws, size_t ws_bytes,
                            void* stream) {
    CSA2_RANGE("csa2_layer_step");
    if (!a) return CSA2_ERR_INVALID_ARG;
    csa2_status s = CSA2_OK;
    if (a->mode == CSA2_FULL) {
        s = csa2_index_full(cache, a->q_idx, a->q_idx_dtype, a->head_w, a->T, a->H_I, a->pool_k, a->top_k,
                            a->pool_idx, a->topk_idx, ws, ws_bytes, stream);
    } else if (a->mode == CSA2_REINDEX) {
        s = csa2_index_reindex(cache, a->q_idx, a->q_idx_dtype, a->head_w, a->T, a->H_I, a->pool_idx, a->pool_k,
                               a->top_k, a->topk_idx, ws, ws_bytes, stream);
    } else if (a->mode != CSA2_REUSE) {
        return CSA2_ERR_INVALID_ARG;
    }
    if (s != CSA2_OK) return s;
    if (a->ring)
        return csa2_sparse_swa_attn_local(cache, a->ring, a->ring_len, a->q, a->T, a->H, a->topk_idx, a->top_k,
                                          a->window, a->sm_scale, a->out, a->lse, ws, ws_bytes, stream);
    return csa2_sparse_swa_attn(cache, a->q, a->T, a->H, a->topk_idx, a->top_k, a->window, a->sm_scale, a->out, a->lse,
                                ws, ws_bytes, stream);
}

size_t csa2_prefill_workspace_bytes(const csa2_cache* cache, int T, int H, int H_I, int pool_k, int top_k,
                                    int window) {
    CSA2_RANGE("csa2_prefill_workspace_bytes");
    if (check_cache(cache) != CSA2_OK || T < 1 || H_I < 1 || H_I > 64) return 0;
    const csa2_cache v = seq_view(cache, 0, cache->seq_lens);
    Layout L;
    if (!make_layout(&v, prefill_chunk(T, H_I), H, pool_k, top_k, window, &L)) return 0;
    return L.total + 256;                               // + the chunk's sequence length
}

csa2_status csa2_prefill_layer(const csa2_cache* cache, const csa2_layer_args* a, void* ws, size_t ws_bytes,
                               void* stream) {
    CSA2_RANGE("csa2_prefill_layer");
    csa2_status s = check_cache(cache);
    if (s != CSA2_OK) return s;
    if (!a || a->T < 1 || !ws || !aligned16(ws)) return CSA2_ERR_INVALID_ARG;
    const bool idx = a->mode == CSA2_FULL || a->mode == CSA2_REINDEX;
    if (!idx && a->mode != CSA2_REUSE) return CSA2_ERR_INVALID_ARG;
    // the stack's indexer heads set the chunk size, in every mode (a Reuse
    // layer runs in the same chunks as the index layers, on the same workspace)
    const int H_I = a->H_I;
    if (H_I < 1 || H_I > 64 || a->H < 1) return CSA2_ERR_INVALID_ARG;
    const int T = a->T, tc = prefill_chunk(T, H_I);
    const csa2_cache v0 = seq_view(cache, 0, cache->seq_lens);
    Layout L;
    if (!make_layout(&v0, tc, a->H, idx ? a->pool_k : (a->top_k > 0 ? a->top_k : 1), a->top_k, a->window, &L))
        return CSA2_ERR_INVALID_ARG;
    const size_t need = csa2_prefill_workspace_bytes(cache, T, a->H, H_I, idx ? a->pool_k : (a->top_k > 0 ? a->top_k : 1),
                                                     a->top_k, a->window);
    if (need == 0 || ws_bytes < need) return CSA2_ERR_INVALID_ARG;
    int32_t* len = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + need - 256);
    const size_t chunk_ws = need - 256;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int D = cache->dim;
    const size_t qi_elem = a->q_idx_dtype == CSA2_F32 ? 4 : 2;
    for (int b = 0; b < cache->batch; ++b) {
        for (int k0 = 0; k0 < T; k0 += tc) {
            // every chunk has tc tokens, so that the workspace layout (and its
            // sections that stay zero between calls) is the same for all; the
            // last one is moved back to end at token T - 1 and recomputes a few
            // tokens with the same inputs
            const int c = tc;
            const int j0 = k0 + tc <= T ? k0 : T - tc;
            // the chunk's tokens are the last c positions of a sequence of length L_b - (T - j0 - c)
            if (launch_chunk_len(cache->seq_lens + b, T - j0 - c, len, st) != cudaSuccess) return CSA2_ERR_CUDA;
            const csa2_cache v = seq_view(cache, b, len);
            const int64_t tok = (int64_t)b * T + j0;     // first (sequence, token) row of the chunk
            csa2_layer_args ca = *a;
            ca.T = c;
            ca.q = static_cast<const uint16_t*>(a->q) + tok * a->H * D;
            if (a->q_idx) ca.q_idx = static_cast<const char*>(a->q_idx) + tok * H_I * cache->idx_dim * qi_elem;
            if (a->head_w) ca.head_w = a->head_w + tok * H_I;
            if (a->pool_idx) ca.pool_idx = a->pool_idx + tok * a->pool_k;
            ca.topk_idx = a->topk_idx ? a->topk_idx + tok * a->top_k : nullptr;
            ca.out = a->out + tok * a->H * D;
            ca.lse = a->lse ? a->lse + tok * a->H : nullptr;
            if (a->ring) ca.ring = static_cast<const uint16_t*>(a->ring) + (int64_t)b * a->ring_len * D;
            s = csa2_layer_step(&v, &ca, ws, chunk_ws, stream);
            if (s != CSA2_OK) return s;
        }
    }
    return CSA2_OK;
}

// ---------------------------------------------------------------- context-parallel decode
// The shard calls run the single-device kernels on the shard's cache (T = 1:
// every shard position is visible) and use the shard workspace's sections as
// follows: scores / selection state as csa2_index_full; the shard's pool or
// top-k ids in upd_ids or upd_scores, their scores in pscores or upd_scores;
// the attention list in upd_ids.

static_assert(sizeof(csa2_cand) == sizeof(CpCand), "csa2_cand and CpCand must have one layout");

csa2_status csa2_cp_index_local(const csa2_cache* shard, const int32_t* pos0, const void* q_idx, csa2_dtype q_dtype,
                                const float* head_w, int H_I, int pool_k, csa2_cand* cand, void* ws, size_t ws_bytes,
                                void* stream) {
    CSA2_RANGE("csa2_cp_index_local");
    csa2_status s = check_index_args(shard, q_idx, q_dtype, head_w, 1, H_I, pool_k, 1);
    if (s != CSA2_OK) return s;
    if (!pos0 || !aligned4(pos0) || !cand || (reinterpret_cast<uintptr_t>(cand) & 7u)) return CSA2_ERR_INVALID_ARG;
    Layout L;
    s = check_ws(shard, 1, 1, pool_k, 1, 0, ws, ws_bytes, &L);
    if (s != CSA2_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t* hist = L.cap > kSmallSelect ? at<uint32_t>(ws, L.hist) : nullptr;
    float* scores = at<float>(ws, L.scores);
    bool fused = false;
    s = launch_scores(shard, q_idx, q_dtype, head_w, 1, H_I, scores, hist, at<uint32_t>(ws, L.status), st, &fused);
    if (s != CSA2_OK) return s;
    SelSrc src;
    src.vals = scores;
    src.vals_stride = L.cap;
    src.ids = nullptr;
    src.ids_stride = 0;
    src.gather = 0;
    src.n = L.cap;
    src.seq_lens = shard->seq_lens;
    src.T = 1;
    src.cap = L.cap;
    int32_t* ids = at<int32_t>(ws, L.upd_ids);
    float* vals = at<float>(ws, L.pscores);
    cudaError_t e = L.cap > kSmallSelect
                        ? launch_select_dual(src, sel_work(ws, L), (int)L.nseg, pool_k, ids, vals, pool_k, 0, nullptr,
                                             0, st, fused)
                        : launch_select_local(src, (int)L.nseg, pool_k, ids, vals, pool_k, 0, nullptr, 0, st);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;
    return cuda_status(launch_cp_pack(ids, vals, pool_k, pos0, shard->batch, pool_k, reinterpret_cast<CpCand*>(cand),
                                      st));
}

csa2_status csa2_cp_reindex_local(const csa2_cache* shard, const int32_t* pos0, const void* q_idx,
                                  csa2_dtype q_dtype, const float* head_w, int H_I, const int32_t* pool_idx,
                                  int pool_k, float* pool_scores, void* ws, size_t ws_bytes, void* stream) {
    CSA2_RANGE("csa2_cp_reindex_local");
    csa2_status s = check_index_args(shard, q_idx, q_dtype, head_w, 1, H_I, pool_k, 1);
    if (s != CSA2_OK) return s;
    if (!pos0 || !aligned4(pos0) || !pool_idx || !aligned16(pool_idx) || !pool_scores || !aligned16(pool_scores))
        return CSA2_ERR_INVALID_ARG;
    Layout L;
    s = check_ws(shard, 1, 1, pool_k, 1, 0, ws, ws_bytes, &L);
    if (s != CSA2_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DevCache d = dev_cache(shard);
    uint32_t* status = at<uint32_t>(ws, L.status);
    int32_t* local = at<int32_t>(ws, L.upd_ids);           // [batch][pool_k] shard positions or -1
    float* sc = at<float>(ws, L.pscores);                   // [batch][pool_k]
    cudaError_t e = launch_cp_localize(pool_idx, pos0, shard->seq_lens, shard->batch, pool_k, local, st);
    if (e == cudaSuccess)
        e = reindex_tc_supported(d, H_I) ? launch_reindex_tc_scores(d, q_idx, head_w, 1, H_I, local, pool_k, sc, status, st)
                                         : launch_score_pool(d, q_idx, q_dtype == CSA2_F32, head_w, 1, H_I, local, pool_k,
                                                             sc, status, st);
    if (e == cudaSuccess) e = launch_cp_owned_scores(local, sc, (int64_t)shard->batch * pool_k, pool_scores, st);
    return cuda_status(e);
}

csa2_status csa2_cp_reindex_select(const int32_t* pool_idx, const float* pool_scores, int batch, int pool_k,
                                   const int32_t* seq_lens_global, int top_k, int32_t* topk_idx, void* stream) {
    CSA2_RANGE("csa2_cp_reindex_select");
    if (batch < 1 || batch > 65535 || pool_k < 1 || pool_k > kMaxPool || top_k < 1 || top_k > pool_k)
        return CSA2_ERR_INVALID_ARG;
    if (!pool_idx || !aligned16(pool_idx) || !pool_scores || !aligned16(pool_scores) || !topk_idx ||
        !aligned16(topk_idx) || !seq_lens_global || !aligned4(seq_lens_global))
        return CSA2_ERR_INVALID_ARG;
    SelSrc src;
    src.vals = pool_scores;
    src.vals_stride = pool_k;
    src.ids = pool_idx;
    src.ids_stride = pool_k;
    src.gather = 0;
    src.n = pool_k;
    src.seq_lens = seq_lens_global;      // an entry is valid when 0 <= pos < Lg (T = 1) and its score is a number
    src.T = 1;
    src.cap = (int64_t)1 << 31;
    return cuda_status(launch_select_local(src, batch, top_k, topk_idx, nullptr, top_k, 0, nullptr, 0,
                                           static_cast<cudaStream_t>(stream)));
}

namespace {
// Workspace of csa2_cp_merge_select: status | histograms | digit-3 histograms |
// counters | candidate and survivor buffers | the candidates per sequence.
struct MergeLayout {
    size_t status, hist, hist3, cnt, cand1, cand2, surv1, surv2, ids, vals, total;
    int64_t m;
};

bool make_merge_layout(int R, int batch, int n_cand, MergeLayout* L) {
    if (R < 1 || batch < 1 || batch > 65535 || n_cand < 1) return false;
    L->m = (int64_t)R * n_cand;
    if (L->m > ((int64_t)1 << 24)) return false;
    const size_t nseg = (size_t)batch, m = (size_t)L->m;
    size_t off = 0;
    L->status = off; off = align_up(off + 16);
    L->hist = off; off = align_up(off + sizeof(uint32_t) * nseg * 3 * kRadixBins);
    L->hist3 = off; off = align_up(off + sizeof(uint32_t) * nseg * 2 * kRadixBins);
    L->cnt = off; off = align_up(off + sizeof(uint32_t) * nseg * kSelCounters);
    L->cand1 = off; off = align_up(off + 2 * sizeof(uint32_t) * nseg * m);
    L->cand2 = off; off = align_up(off + 2 * sizeof(uint32_t) * nseg * m);
    L->surv1 = off; off = align_up(off + 2 * sizeof(uint32_t) * nseg * m);
    L->surv2 = off; off = align_up(off + 2 * sizeof(uint32_t) * nseg * m);
    L->ids = off; off = align_up(off + sizeof(int32_t) * nseg * m);
    L->vals = off; off = align_up(off + sizeof(float) * nseg * m);
    L->total = off;
    return true;
}
}  // namespace

size_t csa2_cp_merge_workspace_bytes(int R, int batch, int n_cand) {
    CSA2_RANGE("csa2_cp_merge_workspace_bytes");
    MergeLayout L;
    return make_merge_layout(R, batch, n_cand, &L) ? L.total : 0;
}

csa2_status csa2_cp_merge_select(const csa2_cand* cand, int R, int batch, int n_cand, const int32_t* seq_lens_global,
                                 int n_a, int32_t* out_a, int n_b, int32_t* out_b, void* ws, size_t ws_bytes,
                                 void* stream) {
    CSA2_RANGE("csa2_cp_merge_select");
    MergeLayout L;
    if (!make_merge_layout(R, batch, n_cand, &L)) return CSA2_ERR_INVALID_ARG;
    if (!cand || (reinterpret_cast<uintptr_t>(cand) & 7u) || !seq_lens_global || !aligned4(seq_lens_global))
        return CSA2_ERR_INVALID_ARG;
    if (n_a < 1 || n_a > kMaxPool || !out_a || !aligned16(out_a)) return CSA2_ERR_INVALID_ARG;
    if (n_b < 0 || n_b > n_a || (n_b > 0 && (!out_b || !aligned16(out_b)))) return CSA2_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws) || ws_bytes < L.total) return CSA2_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* ids = at<int32_t>(ws, L.ids);
    float* vals = at<float>(ws, L.vals);
    if (launch_cp_unpack(reinterpret_cast<const CpCand*>(cand), R, batch, n_cand, ids, vals, st) != cudaSuccess)
        return CSA2_ERR_CUDA;
    SelSrc src;
    src.vals = vals;
    src.vals_stride = L.m;
    src.ids = ids;
    src.ids_stride = L.m;
    src.gather = 0;
    src.n = L.m;
    src.seq_lens = seq_lens_global;      // a candidate is valid when 0 <= pos < Lg (T = 1)
    src.T = 1;
    src.cap = (int64_t)1 << 31;
    if (L.m <= kSmallSelect)
        return cuda_status(launch_select_local(src, batch, n_a, out_a, nullptr, n_a, n_b, n_b > 0 ? out_b : nullptr,
                                               n_b, st));
    SelWork w;
    w.hist = at<uint32_t>(ws, L.hist);
    w.cnt = at<uint32_t>(ws, L.cnt);
    w.cand1 = at<uint32_t>(ws, L.cand1);
    w.cand2 = at<uint32_t>(ws, L.cand2);
    w.surv1 = at<uint32_t>(ws, L.surv1);
    w.surv2 = at<uint32_t>(ws, L.surv2);
    w.cand_stride = L.m;
    w.hist3 = at<uint32_t>(ws, L.hist3);
    w.status = at<uint32_t>(ws, L.status);
    return cuda_status(launch_select_dual(src, w, batch, n_a, out_a, nullptr, n_a, n_b, n_b > 0 ? out_b : nullptr,
                                          n_b, st, false));
}

csa2_status csa2_cp_sparse_swa_attn(const csa2_cache* shard, const int32_t* pos0, const int32_t* seq_lens_global,
                                    const void* q_bf16, int H, const int32_t* topk_idx, int top_k, int window,
                                    float sm_scale, float* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
    CSA2_RANGE("csa2_cp_sparse_swa_attn");
    csa2_status s = check_cache(shard);
    if (s != CSA2_OK) return s;
    if (!pos0 || !aligned4(pos0) || !seq_lens_global || !aligned4(seq_lens_global)) return CSA2_ERR_INVALID_ARG;
    if (!q_bf16 || !out || !lse || !aligned16(q_bf16) || !aligned16(out) || !aligned16(lse)) return CSA2_ERR_INVALID_ARG;
    if (H < 1 || top_k < 0 || window < 0 || window > kMaxPool || top_k > kMaxPool) return CSA2_ERR_INVALID_ARG;
    if (top_k > 0 && (!topk_idx || !aligned16(topk_idx))) return CSA2_ERR_INVALID_ARG;
    if (H > 64 || H % 16) return CSA2_ERR_UNSUPPORTED;
    if (!std::isfinite(sm_scale)) return CSA2_ERR_INVALID_ARG;
    Layout L;
    s = check_ws(shard, 1, H, top_k > 0 ? top_k : 1, top_k, window, ws, ws_bytes, &L);
    if (s != CSA2_OK) return s;
    if (sm_scale <= 0.0f) sm_scale = 1.0f / std::sqrt((float)shard->dim);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t* status = at<uint32_t>(ws, L.status);
    AttnWork aw;
    aw.part_o = at<float>(ws, L.part_o);
    aw.part_ml = at<float>(ws, L.part_ml);
    aw.nchunk = L.nchunk;
    DevCache d = dev_cache(shard);
    if (attn_tc_supported(d, H)) {
        // the tensor-core kernel maps the global window and top-k entries to the
        // shard's positions itself
        CpShard cp;
        cp.pos0 = pos0;
        cp.glens = seq_lens_global;
        aw.nchunk = (window + top_k + attn_tc_rows_per_chunk() - 1) / attn_tc_rows_per_chunk();
        if (aw.nchunk < 1) aw.nchunk = 1;
        cudaError_t e = launch_attention_tc(d, q_bf16, 1, H, top_k > 0 ? topk_idx : nullptr, top_k, window, sm_scale,
                                            Ring{}, aw, status, st, num_sms(), cp);
        if (e == cudaSuccess) e = launch_attn_combine(d, 1, H, aw, out, lse, st);
        return cuda_status(e);
    }
    // otherwise the shard's part of window ∪ top-k as one list of shard
    // positions, attended with no window of its own (the list's window part
    // and top-k part are disjoint)
    const int n = window + top_k;
    int32_t* list = at<int32_t>(ws, L.upd_ids);
    if (n > 0 && launch_cp_attn_list(topk_idx, top_k, window, pos0, shard->seq_lens, seq_lens_global, shard->batch,
                                     list, status, st) != cudaSuccess)
        return CSA2_ERR_CUDA;
    return cuda_status(launch_attention(d, q_bf16, 1, H, n > 0 ? list : nullptr, n, 0, sm_scale, Ring{}, out, lse, aw,
                                        status, st, num_sms()));
}

csa2_status csa2_lse_merge(int R, int batch, int H, int dim, const float* outs, int64_t out_stride,
                           const float* lses, int64_t lse_stride, float* out, float* lse, void* stream) {
    CSA2_RANGE("csa2_lse_merge");
    if (R < 1 || batch < 1 || H < 1 || dim < 1 || !outs || !lses || !out) return CSA2_ERR_INVALID_ARG;
    if (!aligned4(outs) || !aligned4(lses) || !aligned4(out) || (lse && !aligned4(lse))) return CSA2_ERR_INVALID_ARG;
    if (R > 1 && (out_stride < (int64_t)batch * H * dim || lse_stride < (int64_t)batch * H))
        return CSA2_ERR_INVALID_ARG;
    return cuda_status(launch_lse_merge(R, batch, H, dim, outs, out_stride, lses, lse_stride, out, lse,
                                        static_cast<cudaStream_t>(stream)));
}

csa2_status csa2_read_device_status(void* ws, void* stream) {
    CSA2_RANGE("csa2_read_device_status");
    if (!ws || !aligned16(ws)) return CSA2_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess) return CSA2_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return CSA2_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, sizeof(word), st) != cudaSuccess) return CSA2_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return CSA2_ERR_CUDA;
    if (word & kStatusTimeout) return CSA2_ERR_TIMEOUT;
    if (word & kStatusBounds) return CSA2_ERR_DEVICE_BOUNDS;
    return CSA2_OK;
}

csa2_status csa2_debug_set_wait_limit(uint32_t tries) {
    CSA2_RANGE("csa2_debug_set_wait_limit");
    g_wait_limit.store(tries, std::memory_order_relaxed);
    return CSA2_OK;
}

uint32_t csa2_debug_default_wait_limit(void) { return tc::kWaitLimit; }

csa2_status csa2_debug_encode(int format, const float* x, int64_t n, uint8_t* codes, void* stream) {
    CSA2_RANGE("csa2_debug_encode");
    if ((format != 0 && format != 1) || n < 0 || (n > 0 && (!x || !codes || !aligned4(x))))
        return CSA2_ERR_INVALID_ARG;
    if (n == 0) return CSA2_OK;
    return cuda_status(launch_debug_encode(format, x, n, codes, static_cast<cudaStream_t>(stream), num_sms()));
}

const char* csa2_status_string(csa2_status s) {
    CSA2_RANGE("csa2_status_string");
    switch (s) {
        case CSA2_OK: return "CSA2_OK";
        case CSA2_ERR_INVALID_ARG: return "CSA2_ERR_INVALID_ARG";
        case CSA2_ERR_UNSUPPORTED: return "CSA2_ERR_UNSUPPORTED";
        case CSA2_ERR_CUDA: return "CSA2_ERR_CUDA";
        case CSA2_ERR_TIMEOUT: return "CSA2_ERR_TIMEOUT";
        case CSA2_ERR_DEVICE_BOUNDS: return "CSA2_ERR_DEVICE_BOUNDS";
    }
    return "CSA2_UNKNOWN_STATUS";
}

}  // extern "C"

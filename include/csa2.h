/*
 * csa2.h -- C ABI of libcsa2: the CSA2 decode-time attention step over an FP4
 * global KV cache, on one NVIDIA B200 (sm_100a).
 *
 * The method is described on these pages ("DeepSeek-V4.1-Flash: Pushing the
 * Limits of KV Cache Compression"):
 *   [TLDR]   tldrocket.com, "DeepSeek AI Released DeepSeek-V4.1-Flash with 1M
 *            Context, FP4 KV Cache, and Cross-Layer Attention Reuse":
 *            paragraph 2 (sliding window of 128 tokens in every layer),
 *            paragraph 3 (Full / Reindex / Reuse layer roles; a Full layer
 *            builds a candidate pool of up to 16,384 positions),
 *            paragraph 4 (main KV as E2M1 values with one E4M3 scale per 16
 *            channels, NVFP4 without the global scale).
 *   [HN]     hackernews.kjhq.dev post 49735410, "key points" 2-3 (layers share
 *            the main KV and Top-K indices; the hierarchical sparse indexer).
 *   [FANOUT] fanout.sh daily lesson, "What you will learn" item 2 (modes share
 *            global KV and sparse selections; queries and window stay
 *            layer-local).
 *   [ZH]     zerohour.day item on the same release (a context of one million
 *            tokens).
 *
 * Conventions for every call:
 *  - All pointers inside csa2_cache and all tensor arguments are DEVICE
 *    pointers owned by the caller; the library allocates and frees nothing.
 *  - Every call only validates its arguments on the host and enqueues work on
 *    `stream` (a cudaStream_t, NULL = legacy default stream); it never
 *    synchronises, except csa2_read_device_status.
 *  - Host-side validation failures return CSA2_ERR_INVALID_ARG (or
 *    CSA2_ERR_UNSUPPORTED for legal but unimplemented shapes) before anything
 *    is launched.  A failed launch returns CSA2_ERR_CUDA.
 *  - Problems only the device can see (an index or page id out of range, a
 *    sequence longer than the cache, a bounded wait that ran out) never trap:
 *    the kernel skips the bad element and ORs a bit into a sticky status word
 *    in the workspace, read back with csa2_read_device_status.
 *  - Some kernels run as one grid whose CTAs wait for each other at bounded
 *    barriers (the Full layer's selection over more than 16,384 positions,
 *    the Reindex select and the pool update's large selections, when the
 *    grid fits on the GPU at once; they fall back to other kernels when it
 *    does not).  They assume the GPU is not shared with work that keeps its
 *    SMs busy for seconds; otherwise a barrier can run out and the call
 *    reports CSA2_ERR_TIMEOUT (results of that call unusable; re-initialise
 *    the workspace with csa2_workspace_init).
 *  - The library keeps no mutable global state, except the fixed scratch of
 *    csa2_index_reindex_noalloc (see there) and the wait budget of the
 *    diagnostic csa2_debug_set_wait_limit: calls on different streams with
 *    different workspaces may run concurrently.
 *  - Tensors are dense and row-major in the shapes given.  Pointers must be
 *    16-byte aligned, except seq_lens, page_table and start_pos (4-byte):
 *    a cache view of one sequence (page_table + b * max_pages, seq_lens + b)
 *    is a valid cache.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symbols of the shared library; everything else in it is hidden. */
#if defined(__GNUC__)
#define CSA2_API __attribute__((visibility("default")))
#else
#define CSA2_API
#endif

typedef enum {
    CSA2_OK = 0,
    CSA2_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or bound */
    CSA2_ERR_UNSUPPORTED = 2,   /* legal shape this build does not implement */
    CSA2_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    CSA2_ERR_TIMEOUT = 4,       /* device: a bounded wait gave up */
    CSA2_ERR_DEVICE_BOUNDS = 5  /* device: index / page / length out of range */
} csa2_status;

/* Layer roles, [TLDR] paragraph 3. */
typedef enum { CSA2_FULL = 0, CSA2_REINDEX = 1, CSA2_REUSE = 2 } csa2_mode;

typedef enum { CSA2_F32 = 0, CSA2_BF16 = 1, CSA2_E4M3 = 2 } csa2_dtype;

/*
 * The global cache shared by every layer of a stack ([HN] key point 2):
 * one FP4 latent row per position (key and value for all heads) and one
 * index key per position.
 *
 *   kv_rows    [n_slots][row_stride] bytes.  A row holds dim/2 code bytes (two
 *              E2M1 codes per byte, channel 2j in the low nibble of byte j)
 *              followed by dim/16 E4M3 scale bytes (one per 16 channels, no
 *              global scale: [TLDR] paragraph 4).  Padding bytes are unused.
 *   idx_keys   [n_slots][idx_dim] of idx_key_dtype (CSA2_E4M3 or CSA2_F32).
 *   page_table [batch][max_pages] int32 physical page ids, or NULL for the
 *              contiguous layout.  Position t of sequence b lives in slot
 *              page_table[b][t / page_size] * page_size + t % page_size
 *              (paged) or b * seq_stride_slots + t (contiguous).
 *   seq_lens   [batch] int32, the number of valid positions L_b of each
 *              sequence.  Read on the device, never written.
 *
 * Limits: dim % 32 == 0 and 32 <= dim <= 512; idx_dim == 64; row_stride >=
 * dim/2 + dim/16 and a multiple of 16; page_size a multiple of 64 (paged);
 * seq_stride_slots a multiple of 64 (contiguous).  The capacity of one
 * sequence is max_pages * page_size (paged) or seq_stride_slots.
 */
typedef struct {
    uint8_t* kv_rows;
    void* idx_keys;
    const int32_t* page_table;
    const int32_t* seq_lens;
    int32_t batch;
    int32_t max_pages;
    int32_t page_size;
    int32_t dim;
    int32_t idx_dim;
    int32_t row_stride;
    int64_t seq_stride_slots;
    int64_t n_slots;
    csa2_dtype idx_key_dtype;
} csa2_cache;

/*
 * Bytes of device workspace the index and attention calls need for this cache
 * with T query tokens per sequence, H attention heads, a pool of pool_k and a
 * top-k of top_k positions, and a window of `window` positions.  Returns 0 on
 * invalid arguments.  One workspace serves every call of a stack on one
 * stream; it must be cleared once with csa2_workspace_init before first use.
 */
CSA2_API size_t csa2_workspace_bytes(const csa2_cache* cache, int T, int H, int pool_k, int top_k, int window);

/* Zero the workspace (including the sticky device status word) on `stream`. */
CSA2_API csa2_status csa2_workspace_init(void* ws, size_t ws_bytes, void* stream);

/*
 * Quantise-on-append ([TLDR] paragraph 4).  For every sequence b and i <
 * n_new, the bf16 latent x_bf16[b][i][0..dim) is written as the FP4 row of
 * position start_pos[b] + i:
 *     amax = max |x| over each 16-channel block,
 *     s    = E4M3 round-to-nearest-even, saturating (fp32 amax / 6),
 *     c_j  = E2M1 round-to-nearest-even, saturating (fp32 x_j / s), sign kept,
 *            all codes 0 when s is 0.
 * The divisions are IEEE binary32 divisions.  idx_new (nullable,
 * [batch][n_new][idx_dim] of idx_new_dtype CSA2_BF16 or CSA2_F32) is stored as
 * the position's index key: E4M3 (round-to-nearest-even, saturating) for an
 * E4M3 cache, the fp32 value for an F32 cache.  start_pos is a device int32
 * [batch] array; the call does not change seq_lens.  Inputs must be finite.
 * ws (nullable) is a workspace whose sticky status word records positions
 * outside the cache (those rows are skipped); with ws == NULL they are skipped
 * silently.
 */
CSA2_API csa2_status csa2_kv_append_quant(const csa2_cache* cache, const void* x_bf16, const void* idx_new,
                                 csa2_dtype idx_new_dtype, const int32_t* start_pos, int n_new,
                                 void* ws, void* stream);

/*
 * The stored form of cached positions, for persistent storage ([TLDR]
 * paragraph 4: the FP4 rows and E4M3 keys are what the cache holds; [HF]
 * abstract: the compressed KV as persistent state).  csa2_kv_export_rows
 * copies, for every sequence b and i < n, position start_pos[b] + i of the
 * cache into packed device buffers (the caller copies them to the host):
 *     rows [batch][n][dim/2 + dim/16]  the D/2 code bytes (channel 2j in the
 *                                       low nibble) then the D/16 E4M3 scales,
 *     keys [batch][n][idx_dim or 4 * idx_dim]  the index key as stored
 *                                       (E4M3 bytes or fp32), nullable.
 * csa2_kv_import_rows writes such buffers back into the cache at the same
 * positions (seq_lens unchanged), e.g. when a request is restored.  A position
 * outside the cache is written as zeros (export) or skipped (import), and sets
 * CSA2_ERR_DEVICE_BOUNDS in ws (nullable).  start_pos is a device int32
 * [batch]; rows and keys are 4-byte aligned device buffers.
 */
CSA2_API csa2_status csa2_kv_export_rows(const csa2_cache* cache, const int32_t* start_pos, int n, void* rows,
                                         void* keys, void* ws, void* stream);
CSA2_API csa2_status csa2_kv_import_rows(const csa2_cache* cache, const int32_t* start_pos, int n,
                                         const void* rows, const void* keys, void* ws, void* stream);

/*
 * Full-layer indexing ([TLDR] paragraph 3; [HN] key point 3).  Query token j
 * of sequence b sits at p = seq_lens[b] - T + j and sees positions t <= p.
 * Every visible position gets the score
 *     s_t = sum_h head_w[b][j][h] * max(0, q_idx[b][j][h] . k_t)
 * (fp32 accumulation), and
 *     pool_idx[b][j][0..pool_k)  <- the min(pool_k, p+1) positions with the
 *                                   largest s_t (the candidate pool),
 *     topk_idx[b][j][0..top_k)   <- the min(top_k, p+1) largest of the same
 *                                   scores (a subset of the pool),
 * each as a set in unspecified order followed by -1 padding.  Ties at the
 * cutoff are broken arbitrarily.  q_idx is [batch][T][H_I][idx_dim] of q_dtype
 * (CSA2_BF16 with an E4M3 cache, CSA2_F32 with an F32 cache); head_w is fp32
 * [batch][T][H_I].  Requires 1 <= top_k <= pool_k <= 16384, 1 <= H_I <= 64,
 * T*H_I <= 256.
 */
CSA2_API csa2_status csa2_index_full(const csa2_cache* cache, const void* q_idx, csa2_dtype q_dtype,
                            const float* head_w, int T, int H_I, int pool_k, int top_k,
                            int32_t* pool_idx, int32_t* topk_idx, void* ws, size_t ws_bytes,
                            void* stream);

/*
 * The scoring half of csa2_index_full on its own: s_t for every visible
 * position t <= p of every (b, j), written to scores[(b*T + j)*capacity + t]
 * (fp32; entries beyond p are left untouched).  With scores == NULL the
 * scores go to the workspace, where csa2_index_full keeps them.  Same
 * argument rules as csa2_index_full.
 */
CSA2_API csa2_status csa2_index_scores(const csa2_cache* cache, const void* q_idx, csa2_dtype q_dtype,
                                       const float* head_w, int T, int H_I, float* scores, void* ws,
                                       size_t ws_bytes, void* stream);

/*
 * Reindex-layer indexing ([TLDR] paragraph 3, "rescore a shared candidate
 * set").  For each (b, j), the valid entries of pool_idx[b][j][0..pool_k)
 * (those >= 0; usually the pool of the last Full layer) are rescored with this
 * layer's q_idx / head_w exactly as csa2_index_full scores, and topk_idx[b][j]
 * receives the min(top_k, |pool|) best as a set followed by -1 padding.
 * Pool entries > p or >= seq_lens[b] set CSA2_ERR_DEVICE_BOUNDS.
 */
CSA2_API csa2_status csa2_index_reindex(const csa2_cache* cache, const void* q_idx, csa2_dtype q_dtype,
                               const float* head_w, int T, int H_I, const int32_t* pool_idx,
                               int pool_k, int top_k, int32_t* topk_idx, void* ws, size_t ws_bytes,
                               void* stream);

/*
 * Append-time pool update for an in-flight request ([TLDR] paragraphs 3-4:
 * the candidate pool kept current as quantised tokens are appended).  The
 * last n_new positions of every sequence (L - n_new .. L - 1, L =
 * seq_lens[b]) have just been appended (csa2_kv_append_quant).  For query
 * token j at p = L - T + j the candidates are the valid entries of
 * pool_prev[b][j][0..pool_k) (-1 entries are padding; an entry at or beyond
 * L - n_new, or beyond p, sets CSA2_ERR_DEVICE_BOUNDS and is dropped) and the
 * new positions L - n_new .. p, all scored with this token's query as in
 * csa2_index_full:
 *     pool_idx[b][j]  <- the min(pool_k, |candidates|) best (the new pool),
 *     topk_idx[b][j]  <- the min(top_k, |candidates|) best (a subset of it),
 * each a set in unspecified order followed by -1 padding.  Pool entries are
 * distinct positions.  pool_idx may be pool_prev (an in-place update).
 * 0 <= n_new <= 16384 (a longer append is a new Full layer); other limits and
 * layouts as in csa2_index_reindex.
 */
CSA2_API csa2_status csa2_index_pool_update(const csa2_cache* cache, const void* q_idx, csa2_dtype q_dtype,
                                            const float* head_w, int T, int H_I, const int32_t* pool_prev,
                                            int pool_k, int n_new, int top_k, int32_t* pool_idx,
                                            int32_t* topk_idx, void* ws, size_t ws_bytes, void* stream);

/*
 * csa2_index_reindex without a workspace, for callers that cannot allocate
 * device memory: code running while a framework captures a CUDA graph under a
 * no-allocation policy, plugins handed tensors but no allocator, or real-time
 * paths that cannot pay for cudaMalloc's implicit synchronisation.  The pages
 * describe no such call; it is a convenience of this library.
 *
 * Same arguments, argument checks and results as csa2_index_reindex, minus
 * ws / ws_bytes.  The scratch lives in a 4 MiB array inside the library's own
 * device memory (held by every GPU that loads the library until the process
 * exits): 256 bytes of status word, one 4-byte counter per (sequence, token)
 * rounded up to 256 bytes, and batch * T * pool_k floats must fit in it
 * (e.g. batch * T * pool_k <= 1,048,448 while batch * T <= 64); larger
 * problems return CSA2_ERR_UNSUPPORTED before anything is launched, after the
 * other argument checks.  The first call in a CUDA context looks up that
 * array's device address in that context (cudaGetSymbolAddress), so make the
 * first call on each device before any stream capture; a new context (e.g.
 * after cudaDeviceReset) gets a fresh lookup.  Every call on a device shares
 * the one array, and each call clears its status word and counters with an
 * asynchronous memset on `stream`: calls whose work may overlap on the GPU
 * (different streams without ordering between them) race and must not be
 * issued.  Device-detected bound violations are skipped; this variant has no
 * status word the caller can read.
 */
CSA2_API csa2_status csa2_index_reindex_noalloc(const csa2_cache* cache, const void* q_idx, csa2_dtype q_dtype,
                                                const float* head_w, int T, int H_I, const int32_t* pool_idx,
                                                int pool_k, int top_k, int32_t* topk_idx, void* stream);

/*
 * Sparse + sliding-window attention ([HN] key point 2; [TLDR] paragraphs 2-3).
 * For query token j of sequence b at p = seq_lens[b] - T + j, the attended set
 * is S = window ∪ topk without double counting, with window = [max(0, p -
 * window + 1), p]; topk entries that are -1 or > p are not attended.  With
 * v_t the dequantised row of position t (value(code) * value(scale), used as
 * both key and value for every head):
 *     z_t   = sm_scale * q[b][j][h] . v_t          (sm_scale <= 0: 1/sqrt(dim))
 *     out   = sum_{t in S} softmax(z)_t v_t        fp32 [batch][T][H][dim]
 *     lse   = log sum_{t in S} exp(z_t)            fp32 [batch][T][H], nullable
 * q is bf16 [batch][T][H][dim] with H a multiple of 16, at most 64.  An empty
 * S gives out = 0, lse = -inf.  top_k and window are each at most 16,384.
 * topk entries < -1 or >= seq_lens[b] set CSA2_ERR_DEVICE_BOUNDS.
 */
CSA2_API csa2_status csa2_sparse_swa_attn(const csa2_cache* cache, const void* q_bf16, int T, int H,
                                 const int32_t* topk_idx, int top_k, int window, float sm_scale,
                                 float* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * Layer-local window state ([FANOUT] item 2: the layers share the global KV and
 * the sparse selections but keep their own queries and sliding-window state;
 * [TLDR] paragraph 2: the window runs in every layer over the last 128
 * tokens).  A layer's ring is bf16 [batch][ring_len][dim] in device memory,
 * owned by the caller; position t of sequence b lives in row t mod ring_len.
 *
 * csa2_ring_append writes, for every sequence b and i < n_new, the bf16 row
 * x_bf16[b][i][0..dim) into ring row (start_pos[b] + i) mod ring_len
 * (start_pos: device int32 [batch]; a negative start_pos[b] + i is skipped).
 * Requires 1 <= ring_len <= 2^30, n_new <= ring_len, ring and x_bf16 16-byte
 * aligned.  Rows must be finite.  The call reads cache->batch and cache->dim
 * only.
 *
 * csa2_sparse_swa_attn_local is csa2_sparse_swa_attn with the rows of the
 * window positions (p - window < t <= p) taken from the ring, exact bf16,
 * instead of dequantised from the FP4 cache; top-k positions outside the
 * window keep their FP4 rows.  The ring must hold the window of every query
 * token of the call: ring_len >= window + T - 1 (else CSA2_ERR_INVALID_ARG).
 * Rows may take any finite bf16 value: the tensor-core kernel scales a chunk
 * of 64 entries that holds ring rows by one exact power of two (its largest
 * magnitude to [2^14, 2^15)) before its fp16 operands are formed, and takes
 * the scale off the logits and the partial output (chunks whose largest
 * magnitude is below 2^-86 keep a scale of 2^100 and lose precision).
 */
CSA2_API csa2_status csa2_ring_append(const csa2_cache* cache, void* ring, int64_t ring_len, const void* x_bf16,
                                      const int32_t* start_pos, int n_new, void* stream);

CSA2_API csa2_status csa2_sparse_swa_attn_local(const csa2_cache* cache, const void* ring, int64_t ring_len,
                                                const void* q_bf16, int T, int H, const int32_t* topk_idx,
                                                int top_k, int window, float sm_scale, float* out, float* lse,
                                                void* ws, size_t ws_bytes, void* stream);

/*
 * One layer of a CSA2 stack ([TLDR] paragraph 3; [FANOUT] item 2):
 *   CSA2_FULL    csa2_index_full (writes pool_idx and topk_idx), then attention
 *   CSA2_REINDEX csa2_index_reindex (reads pool_idx, writes topk_idx), then
 *                attention
 *   CSA2_REUSE   attention only, with topk_idx as given; no index buffer is
 *                read or written other than topk_idx, which is only read.
 * With ring != NULL the attention is csa2_sparse_swa_attn_local over that
 * ring (the layer's own window rows, appended by the caller beforehand).
 */
typedef struct {
    csa2_mode mode;
    const void* q;           /* bf16 [batch][T][H][dim] */
    const void* q_idx;       /* [batch][T][H_I][idx_dim]; FULL / REINDEX only */
    csa2_dtype q_idx_dtype;
    const float* head_w;     /* [batch][T][H_I]; FULL / REINDEX only */
    int T, H, H_I, pool_k, top_k, window;
    float sm_scale;
    int32_t* pool_idx;       /* [batch][T][pool_k] */
    int32_t* topk_idx;       /* [batch][T][top_k] */
    float* out;              /* [batch][T][H][dim] */
    float* lse;              /* [batch][T][H] or NULL */
    const void* ring;        /* bf16 [batch][ring_len][dim], this layer's window rows, or NULL */
    int64_t ring_len;
} csa2_layer_args;

CSA2_API csa2_status csa2_layer_step(const csa2_cache* cache, const csa2_layer_args* args, void* ws,
                            size_t ws_bytes, void* stream);

/*
 * Prefill and verification: one layer (as csa2_layer_step) for T query tokens
 * of every sequence, any T >= 1 ([TLDR] paragraphs 2-3: the layers run over
 * the prompt as well as over decoded tokens; [HN] summary: prefill compute).
 * Token j of sequence b sits at p = seq_lens[b] - T + j (its row appended
 * beforehand) and sees positions <= p only, exactly as in a decode step; the
 * arguments and output layouts are those of csa2_layer_step with args->T = T
 * (out [batch][T][H][dim], pool_idx [batch][T][pool_k], ...; a ring is
 * [batch][ring_len][dim] with ring_len >= window + min(T, chunk) - 1), except
 * that args->H_I is required in every mode, CSA2_REUSE included: the stack's
 * indexer heads set the chunk size.  The
 * tokens run in chunks of min(T, 128 / HP) tokens (HP = H_I rounded up to 16;
 * 4 for 32 indexer heads), one sequence at a time; the last chunk of a
 * sequence is moved back to end at token T - 1 and recomputes a few tokens.
 * ws is a workspace of csa2_prefill_workspace_bytes bytes (0 on invalid
 * arguments), cleared once with csa2_workspace_init; its status word is read
 * with csa2_read_device_status as usual.
 */
CSA2_API size_t csa2_prefill_workspace_bytes(const csa2_cache* cache, int T, int H, int H_I, int pool_k, int top_k,
                                             int window);
CSA2_API csa2_status csa2_prefill_layer(const csa2_cache* cache, const csa2_layer_args* args, void* ws,
                                        size_t ws_bytes, void* stream);

/*
 * Context-parallel decode: the positions of one sequence spread over R
 * devices ([TLDR] paragraph 1 and [ZH]: contexts of a million tokens; [TLDR]
 * paragraph 3: pool and top-k are selections by score, so they
 * split by position).  Rank r keeps positions [pos0[b], pos0[b] + n_r[b]) of
 * sequence b in a cache of its own, its "shard": there they are positions 0 ..
 * n_r[b] - 1 and the shard's seq_lens holds n_r.  The shards of a sequence are
 * disjoint and together hold 0 .. Lg[b] - 1 (Lg: the global lengths).  One
 * query token per sequence (T = 1) at p = Lg[b] - 1, so every position of every
 * shard is visible to it.  Two identities make the split exact:
 *   - the n best positions overall are among the union of every shard's n
 *     best (a position outside its shard's n best has n better ones there);
 *   - attention over S is the log-sum-exp merge of attention over the
 *     disjoint parts S ∩ shard_r.
 * One layer on every rank:
 *   FULL     csa2_cp_index_local -> all-gather of the candidates ->
 *            csa2_cp_merge_select (pool and top-k)
 *   REINDEX  csa2_cp_reindex_local -> all-reduce (sum) of the pool's scores ->
 *            csa2_cp_reindex_select
 *   any      csa2_cp_sparse_swa_attn -> all-gather of (out, lse) ->
 *            csa2_lse_merge
 * The collectives are the caller's (NCCL over NVLink, at most a few hundred KB
 * a layer); every rank ends with the same pool, top-k, output and lse.  The
 * shard calls share one workspace of csa2_workspace_bytes(shard, 1, H, pool_k,
 * top_k, window) bytes (cleared once with csa2_workspace_init; its status word
 * read with csa2_read_device_status); the merge selection has its own.
 *
 * A candidate is a global position with its score; position -1 is padding.
 */
typedef struct {
    int32_t pos;
    float score;
} csa2_cand;

/*
 * A Full layer's share on one shard: every shard position scored as
 * csa2_index_full scores it (T = 1), and cand[b][0..pool_k) <- the
 * min(pool_k, n_r[b]) best with their scores and global positions (shard
 * position + pos0[b]), in unspecified order, then (-1, 0) padding.  pos0:
 * device int32 [batch], >= 0, pos0 + n_r < 2^31; cand: 8-byte aligned device
 * array [batch][pool_k].  Other arguments and limits as csa2_index_full.
 */
CSA2_API csa2_status csa2_cp_index_local(const csa2_cache* shard, const int32_t* pos0, const void* q_idx,
                                         csa2_dtype q_dtype, const float* head_w, int H_I, int pool_k,
                                         csa2_cand* cand, void* ws, size_t ws_bytes, void* stream);

/*
 * A Reindex layer's share on one shard: the entries of the global pool
 * pool_idx[b][0..pool_k) that this shard holds (pos0[b] <= t < pos0[b] +
 * n_r[b]) are rescored as csa2_index_reindex rescores them, and
 *     pool_scores[b][i] <- that score for an entry this shard holds (NaN if it
 *                          could not be scored: CSA2_ERR_DEVICE_BOUNDS),
 *                          0 for an entry another shard holds and for -1
 *                          padding.
 * Every pool entry has exactly one owner, so the sum of the ranks'
 * pool_scores (an all-reduce, exact: the other terms are zeros) holds every
 * entry's score; csa2_cp_reindex_select then picks the top-k.  pool_scores is
 * fp32 [batch][pool_k], 16-byte aligned.  Other arguments as
 * csa2_cp_index_local and csa2_index_reindex.
 */
CSA2_API csa2_status csa2_cp_reindex_local(const csa2_cache* shard, const int32_t* pos0, const void* q_idx,
                                           csa2_dtype q_dtype, const float* head_w, int H_I,
                                           const int32_t* pool_idx, int pool_k, float* pool_scores, void* ws,
                                           size_t ws_bytes, void* stream);

/*
 * The Reindex top-k after the all-reduce: topk_idx[b][0..top_k) <- the
 * min(top_k, valid) best entries of pool_idx[b] by pool_scores[b] (summed over
 * the ranks), an entry being valid when 0 <= pos < seq_lens_global[b] and its
 * score is a number; a set in unspecified order, -1 padding last, ties at the
 * cutoff broken arbitrarily.  1 <= top_k <= pool_k <= 16384; pool_idx,
 * pool_scores and topk_idx 16-byte aligned.  Needs no workspace.
 */
CSA2_API csa2_status csa2_cp_reindex_select(const int32_t* pool_idx, const float* pool_scores, int batch,
                                            int pool_k, const int32_t* seq_lens_global, int top_k,
                                            int32_t* topk_idx, void* stream);

/*
 * The selection after the all-gather: cand is [R][batch][n_cand] (rank r's
 * candidates of sequence b at cand + (r * batch + b) * n_cand).  For each b, of
 * the candidates with 0 <= pos < seq_lens_global[b] (device int32 [batch]),
 *     out_a[b][0..n_a) <- the min(n_a, count) best positions,
 *     out_b[b][0..n_b) <- the min(n_b, count) best (a subset of out_a; n_b = 0
 *                         and out_b = NULL for none),
 * each a set in unspecified order followed by -1 padding, ties at the cutoff
 * broken arbitrarily.  Positions must be distinct.  1 <= n_b <= n_a <= 16384
 * (or n_b = 0), R * n_cand <= 2^24.  ws is a separate workspace of
 * csa2_cp_merge_workspace_bytes(R, batch, n_cand) bytes (0 on invalid
 * arguments), cleared once with csa2_workspace_init; its status word (a
 * selection's bounded barrier that ran out: CSA2_ERR_TIMEOUT) is read with
 * csa2_read_device_status.
 */
CSA2_API size_t csa2_cp_merge_workspace_bytes(int R, int batch, int n_cand);
CSA2_API csa2_status csa2_cp_merge_select(const csa2_cand* cand, int R, int batch, int n_cand,
                                          const int32_t* seq_lens_global, int n_a, int32_t* out_a, int n_b,
                                          int32_t* out_b, void* ws, size_t ws_bytes, void* stream);

/*
 * A layer's attention on one shard: with the global attended set S of
 * csa2_sparse_swa_attn (T = 1, p = seq_lens_global[b] - 1, window ∪ the
 * top-k entries topk_idx[b][0..top_k) that are global positions), this shard
 * attends over S ∩ shard and writes that part's normalised output and
 * log-sum-exp: out fp32 [batch][H][dim], lse fp32 [batch][H] (required; an
 * empty part gives out = 0, lse = -inf).  Top-k entries must be distinct;
 * entries < -1 or >= seq_lens_global[b] set CSA2_ERR_DEVICE_BOUNDS.  The
 * window rows come from the FP4 cache.  Other arguments as
 * csa2_sparse_swa_attn.
 */
CSA2_API csa2_status csa2_cp_sparse_swa_attn(const csa2_cache* shard, const int32_t* pos0,
                                             const int32_t* seq_lens_global, const void* q_bf16, int H,
                                             const int32_t* topk_idx, int top_k, int window, float sm_scale,
                                             float* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * The merge of R attention parts over disjoint parts of one attended set:
 * part r's output at outs + r * out_stride (fp32 [batch][H][dim]) and its lse
 * at lses + r * lse_stride (fp32 [batch][H]); strides in floats, so that both
 * may sit in one all-gathered buffer.  Per (b, h):
 *     lse = log sum_r exp(lse_r),   out = sum_r exp(lse_r - lse) out_r,
 * a part with lse_r = -inf contributing nothing (all empty: out = 0, lse =
 * -inf).  out fp32 [batch][H][dim]; lse nullable.  R >= 1; with R > 1,
 * out_stride >= batch * H * dim and lse_stride >= batch * H.  Pointers 4-byte
 * aligned.
 */
CSA2_API csa2_status csa2_lse_merge(int R, int batch, int H, int dim, const float* outs, int64_t out_stride,
                                    const float* lses, int64_t lse_stride, float* out, float* lse, void* stream);

/*
 * Synchronise `stream`, then return the sticky device status recorded in the
 * workspace (CSA2_OK, CSA2_ERR_DEVICE_BOUNDS or CSA2_ERR_TIMEOUT; the first
 * error class found in that order of severity: TIMEOUT, then BOUNDS) and clear
 * it.  Returns CSA2_ERR_CUDA if the synchronisation or copy fails.
 */
CSA2_API csa2_status csa2_read_device_status(void* ws, void* stream);

/* A static, human-readable name for a status code. */
CSA2_API const char* csa2_status_string(csa2_status status);

/*
 * Diagnostic: set how many times the bounded mbarrier waits that guard work in
 * the tensor-core kernels (scorer, Reindex, attention) try before they give up
 * and record CSA2_ERR_TIMEOUT, for every launch made after this call returns
 * (the value is read on the host when a launch is set up; a CUDA graph keeps
 * the value it was captured with).  A try sleeps for at most about 0.5 us, so
 * the default, csa2_debug_default_wait_limit(), is about two seconds.  0 makes
 * those waits give up at once: the kernel then writes no result, flags the
 * status, waits (bounded) for the copies and MMAs it already issued, frees its
 * tensor memory and returns, leaving the context usable.  Process-wide; not
 * meant to be changed while other threads launch.  Always returns CSA2_OK.
 */
CSA2_API csa2_status csa2_debug_set_wait_limit(uint32_t tries);

/* The default try count of those waits (the value the library starts with). */
CSA2_API uint32_t csa2_debug_default_wait_limit(void);

/*
 * Diagnostic: the conversions csa2_kv_append_quant uses, applied to n
 * arbitrary fp32 values x (device, 4-byte aligned), one code per byte into
 * codes (device): format 0 gives the E2M1 code of each value (round to
 * nearest, ties to even, saturating at 6, sign kept; the low nibble), format
 * 1 its E4M3 code (the same rules, saturating at 448), as the quantiser forms
 * FP4 codes from quotients x / s and E4M3 scales and keys ([TLDR] paragraph
 * 4).  It lets a test check those conversions on every fp32 input, not only
 * on the quotients that bf16 inputs reach.  Non-finite inputs give whatever
 * the conversion instruction gives.
 */
CSA2_API csa2_status csa2_debug_encode(int format, const float* x, int64_t n, uint8_t* codes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA2_H */

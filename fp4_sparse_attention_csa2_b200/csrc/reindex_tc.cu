// Reindex layer on the tensor cores: rescore a candidate pool and keep its
// top-k, in one kernel.
//
// Role: tldrocket.com, "DeepSeek AI Released DeepSeek-V4.1-Flash with 1M
// Context, FP4 KV Cache, and Cross-Layer Attention Reuse", paragraph 3 (a
// Reindex layer rescores the shared candidate pool, at most 16,384
// positions, with its own query); hackernews.kjhq.dev post 49735410, key
// point 3 (the indexer).  The score is the one of the Full layer,
// s_t = sum_h w_h * max(0, q_h . k_t), computed exactly as the Full scorer
// computes it (index_tc.cu): the E4M3 keys are the A operand of
// tcgen05.mma.kind::f8f6f4 as stored, the bf16 query becomes U power-of-two
// rescaled E4M3 terms stacked along N (q = t0 + t1/16 + t2/256, exact for every
// value at or above 2^-14 of its row maximum), and the epilogue adds the term
// columns with their exact weights, applies the ReLU and the head weights.
//
// grid (ceil(pool_k / 128), batch * T), 512 threads.  CTA x of segment seg:
//   threads 0..127    gather the keys of pool entries 128 x .. 128 x + 127
//                     (64 bytes each, straight into the 64-byte-swizzled A
//                     tile; an entry that is padding, beyond p, or on a page
//                     outside the cache gets zeros and, later, a NaN score);
//   threads 128..     the query terms (4 threads per head) and folded weights;
//   thread 0          two MMAs (K = 2 x 32, M = 128 entries, N = U x HP);
//   warps 0..3        one entry per thread: read its U x HP columns of the
//                     accumulator, write the score (NaN when not a candidate).
// Grid mode (when every CTA of the launch fits on the GPU at once): the
// segment's CTAs select the top_k together, each keeping its 128 keys in
// registers, through three bounded segment barriers behind which the digit-1,
// -2 and -3 histograms of the segment are complete (gsel.cuh), then claim
// their outputs with one atomic per warp; the last CTA clears the histograms
// and counters.  Otherwise the CTA that finishes its segment last (an arrival
// counter after a memory fence) reads the segment's pool_k scores back and
// selects the top_k in one CTA (lsel.cuh), then clears the counter.
#include "common.cuh"
#include "gsel.cuh"
#include "kernels.h"
#include "lsel.cuh"
#include "tc.cuh"

namespace csa2 {

namespace {

constexpr int kThreads = 512;
constexpr int kTile = 128;                 // pool entries per CTA
constexpr int kMaxTerms = 3;
constexpr int kE = 32;                     // select: 512 x 32 = 16,384 elements per segment

struct Params {
    DevCache c;
    const __nv_bfloat16* q;   // [B*T][H_I][64]
    const float* hw;          // [B*T][H_I]
    int T, H_I, HP, U;        // HP: H_I rounded up to 16; U query terms
    const int32_t* pool;      // [B*T][pool_k]
    int pool_k, top_k;
    int32_t* topk;            // [B*T][top_k]
    float* scores;            // [B*T][pool_k] scratch
    uint32_t* counters;       // [B*T] arrival counters, zero between calls
    uint32_t* grid_hist;      // grid mode: [B*T][3][2048] digit histograms, zero between calls (nullptr: last-CTA mode)
    uint32_t* grid_cnt;       // grid mode: [B*T][kSelCounters] counters, zero between calls
    int scores_only;          // write the scores and stop (no selection)
    uint32_t* status;
    uint32_t wait_limit;      // tries of the wait that guards the epilogue (not of the drain)
    uint32_t tmem_cols;
};

struct __align__(1024) Smem {
    uint8_t a[kTile * 64];                          // keys: K-major, 64-byte swizzle
    uint8_t b[kMaxTerms * 64 * 64];                 // query terms: U x HP rows of 64 E4M3 values
    float wq[64];                                   // head weights times 2^-e (the query term scale)
    lsel::Smem<kThreads> sel;
    uint64_t mma_bar;
    uint32_t tmem_base;
    uint32_t last;
    uint32_t flag;
    uint32_t base[4];
    gsel::Cut cut;
};

__device__ __forceinline__ float e4m3_round(float x, uint8_t* code) {
    const uint16_t c = cvt_e4m3x2(0.0f, x);
    *code = (uint8_t)(c & 0xFF);
    return e4m3_to_float(*code);
}

// The top_k of the segment's keys, selected by all its CTAs together; the
// entry threads (tid < 128) hold one key each (0: not a candidate) and its
// position `id`.
__device__ void grid_topk(const Params& p, int seg, uint32_t key, int32_t id, Smem& sm) {
    const int tid = threadIdx.x, lane = tid & 31;
    const uint32_t C = gridDim.x;
    uint32_t* h1 = p.grid_hist + (int64_t)seg * 3 * 2048;
    uint32_t* h2 = h1 + 2048;
    uint32_t* h3 = h2 + 2048;
    uint32_t* cnt = p.grid_cnt + (int64_t)seg * kSelCounters;
    uint32_t* bar = cnt + 8;
    uint32_t* hc = sm.sel.hist;                     // a copy of one of the segment's histograms
    const uint32_t limit = p.wait_limit * 64u;
    uint32_t nbar = 0;
    bool ok = true;
    // level 1
    if (key) atomicAdd(h1 + (key >> 21), 1u);
    ok = gsel::seg_barrier(bar, ++nbar * C, limit, &sm.flag) && ok;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // every CTA is resident
    gsel::load_hist<kThreads>(hc, h1, 2048);
    const gsel::Cut c1 = gsel::threshold<kThreads>(hc, 0u, (uint32_t)p.top_k, sm.sel.wa, &sm.cut);
    const bool take1 = c1.need == 0 || c1.eq == c1.need - c1.above;
    if (blockIdx.x == 0)
        for (int k = (int)c1.need + tid; k < p.top_k; k += kThreads) p.topk[(int64_t)seg * p.top_k + k] = -1;
    // level 2: the elements of digit c1
    if (key && !take1 && (key >> 21) == c1.c) atomicAdd(h2 + ((key >> 10) & 0x7FFu), 1u);
    ok = gsel::seg_barrier(bar, ++nbar * C, limit, &sm.flag) && ok;
    gsel::load_hist<kThreads>(hc, h2, 2048);
    const uint32_t need2 = take1 ? 0u : c1.need - c1.above;
    const gsel::Cut c2 = gsel::threshold<kThreads>(hc, need2, 0u, sm.sel.wa, &sm.cut);
    const bool take2 = take1 || c2.eq == need2 - c2.above;
    // level 3: the elements of digits (c1, c2)
    const uint32_t pre = (c1.c << 11) | c2.c;
    if (key && !take2 && (key >> 10) == pre) atomicAdd(h3 + (key & 0x3FFu), 1u);
    ok = gsel::seg_barrier(bar, ++nbar * C, limit, &sm.flag) && ok;
    gsel::load_hist<kThreads>(hc, h3, 2048);
    const uint32_t need3 = take2 ? 0u : need2 - c2.above;
    const gsel::Cut c3 = gsel::threshold<kThreads>(hc, need3, 0u, sm.sel.wa, &sm.cut);
    // the cut as keys: every key >= lo is taken, and the first `ties` claimants of tie_key
    uint32_t lo, tie_key = 0u, ties = 0u;
    if (c1.need == 0) {
        lo = 0xFFFFFFFFu;
    } else if (take1) {
        lo = c1.c << 21;
    } else if (take2) {
        lo = (c1.c << 21) | (c2.c << 10);
    } else {
        tie_key = (pre << 10) | c3.c;
        lo = tie_key + 1u;
        ties = need3 - c3.above;
    }
    if (threadIdx.x < kTile) {                       // warps 0..3: the entry threads
        bool sel = key && key >= lo;
        const bool tie = key && key == tie_key;
        const uint32_t m = __ballot_sync(0xffffffffu, tie);
        if (m) {
            uint32_t base = 0;
            const int leader = __ffs(m) - 1;
            if (lane == leader) base = atomicAdd(cnt + 4, (uint32_t)__popc(m));
            base = __shfl_sync(0xffffffffu, base, leader);
            sel = sel || (tie && base + __popc(m & ((1u << lane) - 1u)) < ties);
        }
        const uint32_t ms = __ballot_sync(0xffffffffu, sel);
        uint32_t obase = 0;
        if (ms && lane == 0) obase = atomicAdd(cnt + 0, (uint32_t)__popc(ms));
        obase = __shfl_sync(0xffffffffu, obase, 0);
        const uint32_t pos = obase + __popc(ms & ((1u << lane) - 1u));
        if (sel && pos < (uint32_t)p.top_k) p.topk[(int64_t)seg * p.top_k + pos] = id;
    }
    if (!ok && tid == 0) flag(p.status, kStatusTimeout);
    // the last CTA leaves the segment's histograms and counters zero
    __threadfence();
    __syncthreads();
    if (tid == 0) sm.last = atomicAdd(bar, 1u) == (nbar + 1) * C - 1 ? 1u : 0u;
    __syncthreads();
    if (!sm.last) return;
    __threadfence();
    for (int k = tid; k < 3 * 2048; k += kThreads) h1[k] = 0u;
    if (tid < kSelCounters) cnt[tid] = 0u;
}

__global__ void __launch_bounds__(kThreads, 1) k_reindex_tc(const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int seg = blockIdx.y, b = seg / p.T, j = seg % p.T;
    const int NA = p.U * p.HP;                      // accumulator columns
    if (tid == 0) {
        tc::mbar_init(&sm.mma_bar, 1);
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, p.tmem_cols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem_base;
    // in grid mode the next kernel may launch only once every CTA of this one
    // is resident (after the first segment barrier)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (!p.grid_hist) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // ---- operands
    const int i = blockIdx.x * kTile + tid;         // this thread's pool entry (tid < 128)
    bool live = false;
    int32_t t = -1;
    if (tid < kTile) {
        const int64_t L = seq_len(p.c, b, p.status);
        const int64_t pq = L - p.T + j;
        t = i < p.pool_k ? __ldg(p.pool + (int64_t)seg * p.pool_k + i) : -1;
        int64_t slot = -1;
        if (t >= 0) {
            if (t > pq) {
                flag(p.status, kStatusBounds);      // a pool entry the query cannot see
            } else {
                slot = slot_of(p.c, b, t);
                if (slot < 0) flag(p.status, kStatusBounds);
            }
        }
        live = slot >= 0;
        uint4 k4[4] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u),
                       make_uint4(0u, 0u, 0u, 0u)};
        if (live) {
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.c.keys) + slot * 64);
#pragma unroll
            for (int k = 0; k < 4; ++k) k4[k] = __ldg(src + k);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) *reinterpret_cast<uint4*>(sm.a + tc::sw64_offset(tid, k)) = k4[k];
    } else if (tid < kTile + 4 * p.HP) {
        // query row h: 4 threads, 16 values each; per-row power-of-two scale
        // putting the row maximum in [128, 256), then U exact E4M3 terms
        const int qt = tid - kTile, h = qt >> 2, quarter = qt & 3;
        const bool real = h < p.H_I;
        float v[16];
        if (real) {
            const uint4* src = reinterpret_cast<const uint4*>(p.q + (((int64_t)seg * p.H_I + h) * 64 + quarter * 16));
            const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
            const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                v[2 * k] = __uint_as_float(w[k] << 16);
                v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
            }
        } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] = 0.0f;
        }
        float m = 0.0f;
#pragma unroll
        for (int k = 0; k < 16; ++k) m = fmaxf(m, fabsf(v[k]));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        int e = 0;
        if (m > 0.0f) {
            e = 7 - ((int)((__float_as_uint(m) >> 23) & 0xFF) - 127);
            e = e < -100 ? -100 : (e > 100 ? 100 : e);
        }
        const float up = __uint_as_float((uint32_t)(127 + e) << 23);
        const float down = __uint_as_float((uint32_t)(127 - e) << 23);
        uint8_t tq[kMaxTerms][16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            float r = v[k] * up;                    // exact: a power-of-two scale
#pragma unroll
            for (int u = 0; u < kMaxTerms; ++u) {
                // term u carries the remainder scaled by 16^u (exact)
                const float scale = (float)(1 << (4 * u));
                const float tv = e4m3_round(r * scale, &tq[u][k]);
                r -= tv / scale;
            }
        }
#pragma unroll
        for (int u = 0; u < kMaxTerms; ++u) {
            if (u >= p.U) break;
            uint32_t wds[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                wds[k] = (uint32_t)tq[u][4 * k] | ((uint32_t)tq[u][4 * k + 1] << 8) |
                         ((uint32_t)tq[u][4 * k + 2] << 16) | ((uint32_t)tq[u][4 * k + 3] << 24);
            *reinterpret_cast<uint4*>(sm.b + tc::sw64_offset(u * p.HP + h, quarter)) =
                make_uint4(wds[0], wds[1], wds[2], wds[3]);
        }
        if (quarter == 0) sm.wq[h] = real ? __ldg(p.hw + (int64_t)seg * p.H_I + h) * down : 0.0f;
    }
    tc::fence_proxy_async_smem();                   // keys and query terms are MMA operands
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();

    // ---- scores of the tile
    if (tid == 0) {
        const uint32_t idesc = tc::idesc_f8_f32(kTile, NA, 0u, 0u);
        const uint32_t aa = tc::smem_u32(sm.a), bb = tc::smem_u32(sm.b);
        tc::mma_f8(tmem, tc::desc_sw64(aa), tc::desc_sw64(bb), idesc, 0u);
        tc::mma_f8(tmem, tc::desc_sw64(aa + 32), tc::desc_sw64(bb + 32), idesc, 1u);
        tc::mma_commit(&sm.mma_bar);
    }
    bool ok = true;
    uint32_t my_key = 0;                            // grid mode: this entry's key (0: not a candidate)
    if (warp < 4) {
        ok = __all_sync(0xffffffffu, tc::mbar_wait(&sm.mma_bar, 0, p.wait_limit));
        tc::fence_after_sync();
        float s0 = 0.0f, s1 = 0.0f;
        if (ok) {
            const uint32_t abase = tmem + ((uint32_t)(warp * 32) << 16);
            for (int c0 = 0; c0 < p.HP; c0 += 16) {
                uint32_t r[kMaxTerms][16];
                tc::tmem_ld16_nowait(abase + (uint32_t)c0, r[0]);
                tc::tmem_ld16_nowait(abase + (uint32_t)(p.HP + c0), r[1]);
                if (p.U > 2) tc::tmem_ld16_nowait(abase + (uint32_t)(2 * p.HP + c0), r[2]);
                tc::tmem_ld_wait();
                const float4* w4 = reinterpret_cast<const float4*>(sm.wq + c0);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 ww = w4[q4];
                    float dot[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        float x = fmaf(__uint_as_float(r[1][4 * q4 + k]), 0.0625f, __uint_as_float(r[0][4 * q4 + k]));
                        if (p.U > 2) x = fmaf(__uint_as_float(r[2][4 * q4 + k]), 0.00390625f, x);
                        dot[k] = fmaxf(x, 0.0f);
                    }
                    s0 = fmaf(ww.x, dot[0], s0);
                    s1 = fmaf(ww.y, dot[1], s1);
                    s0 = fmaf(ww.z, dot[2], s0);
                    s1 = fmaf(ww.w, dot[3], s1);
                }
            }
        }
        // every entry of the tile gets a value: NaN marks one that is not a candidate
        const float sc = (ok && live) ? s0 + s1 : __int_as_float(0x7fc00000);
        if (p.grid_hist) my_key = select_key(sc, i < p.pool_k && ok && live);
        else if (i < p.pool_k) p.scores[(int64_t)seg * p.pool_k + i] = sc;
    }
    if (!ok && lane == 0) flag(p.status, kStatusTimeout);
    __threadfence();
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        // after a wait that gave up, the MMA may still be running: wait for it
        // (again bounded) before the tensor memory is freed
        if (!ok) tc::mbar_wait(&sm.mma_bar, 0, tc::kWaitLimit);
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, p.tmem_cols);
    }
    if (p.grid_hist) {
        grid_topk(p, seg, my_key, t, sm);
        return;
    }
    if (p.scores_only) return;
    if (tid == 0) sm.last = atomicAdd(p.counters + seg, 1u) == gridDim.x - 1 ? 1u : 0u;
    __syncthreads();
    if (!sm.last) return;

    // ---- the segment's last CTA: top_k of its pool_k scores
    __threadfence();
    uint32_t key[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) {
        const int k = e * kThreads + tid;
        key[e] = k < p.pool_k ? __float_as_uint(__ldcg(p.scores + (int64_t)seg * p.pool_k + k)) : 0u;
    }
#pragma unroll
    for (int e = 0; e < kE; ++e) {
        const int k = e * kThreads + tid;
        key[e] = select_key(__uint_as_float(key[e]), k < p.pool_k);   // NaN: padding or rejected
    }
    auto id_of = [&](int e) -> int32_t { return __ldg(p.pool + (int64_t)seg * p.pool_k + e * kThreads + tid); };
    const uint32_t take = lsel::select_mask<kThreads, kE>(key, (uint32_t)p.top_k, sm.sel);
    lsel::write_selected<kThreads, kE>(take, key, id_of, p.topk + (int64_t)seg * p.top_k, nullptr, p.top_k, sm.sel);
    if (tid == 0) p.counters[seg] = 0u;             // ready for the next call
}

}  // namespace

bool reindex_tc_supported(const DevCache& c, int H_I) {
    return c.key_dtype == 2 && c.idx_dim == 64 && H_I <= 64;
}

cudaError_t launch_reindex_tc(const DevCache& c, const void* q, const float* hw, int T, int H_I,
                              const int32_t* pool, int pool_k, int top_k, int32_t* topk, float* scores,
                              uint32_t* counters, uint32_t* grid_hist, uint32_t* grid_cnt, uint32_t* status,
                              cudaStream_t st) {
    Params p;
    p.c = c;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.hw = hw;
    p.T = T;
    p.H_I = H_I;
    p.HP = (H_I + 15) / 16 * 16;
    p.U = 3 * p.HP <= 256 ? 3 : 2;
    p.pool = pool;
    p.pool_k = pool_k;
    p.top_k = top_k;
    p.topk = topk;
    p.scores = scores;
    p.counters = counters;
    p.grid_hist = nullptr;
    p.grid_cnt = nullptr;
    p.scores_only = 0;
    p.status = status;
    p.wait_limit = wait_limit();
    uint32_t cols = 32;
    while (cols < (uint32_t)(p.U * p.HP)) cols <<= 1;
    p.tmem_cols = cols;
    const size_t smem = sizeof(Smem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_reindex_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned tiles = (unsigned)((pool_k + kTile - 1) / kTile);
    if (grid_hist && grid_cnt) {
        // grid mode when every CTA of the launch fits on the GPU at once
        static int64_t cap = -1;
        if (cap < 0) {
            int dev = 0, sms = 0, per = 0;
            cap = 0;
            if (cudaGetDevice(&dev) == cudaSuccess &&
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
                cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, k_reindex_tc, kThreads, smem) == cudaSuccess)
                cap = (int64_t)sms * per;
        }
        if ((int64_t)tiles * c.batch * T <= cap) {
            p.grid_hist = grid_hist;
            p.grid_cnt = grid_cnt;
        }
    }
    return launch_pdl(k_reindex_tc, dim3(tiles, (unsigned)(c.batch * T)), dim3(kThreads), smem, st, p);
}

cudaError_t launch_reindex_tc_scores(const DevCache& c, const void* q, const float* hw, int T, int H_I,
                                     const int32_t* pool, int pool_k, float* scores, uint32_t* status, cudaStream_t st) {
    Params p;
    p.c = c;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.hw = hw;
    p.T = T;
    p.H_I = H_I;
    p.HP = (H_I + 15) / 16 * 16;
    p.U = 3 * p.HP <= 256 ? 3 : 2;
    p.pool = pool;
    p.pool_k = pool_k;
    p.top_k = 0;
    p.topk = nullptr;
    p.scores = scores;
    p.counters = nullptr;
    p.grid_hist = nullptr;
    p.grid_cnt = nullptr;
    p.scores_only = 1;
    p.status = status;
    p.wait_limit = wait_limit();
    uint32_t cols = 32;
    while (cols < (uint32_t)(p.U * p.HP)) cols <<= 1;
    p.tmem_cols = cols;
    const size_t smem = sizeof(Smem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_reindex_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned tiles = (unsigned)((pool_k + kTile - 1) / kTile);
    return launch_pdl(k_reindex_tc, dim3(tiles, (unsigned)(c.batch * T)), dim3(kThreads), smem, st, p);
}

}  // namespace csa2

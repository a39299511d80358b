// Indexer scoring on the 5th-generation tensor cores (tcgen05, kind::f8f6f4)
// for E4M3 index keys:  s_t = sum_h w_h * max(0, q_h . k_t)  for every
// visible position.
//
// Role of the indexer: tldrocket.com, "DeepSeek AI Released DeepSeek-V4.1-Flash
// with 1M Context, FP4 KV Cache, and Cross-Layer Attention Reuse", paragraph 3
// (a Full layer scores the whole context into a candidate pool of <= 16,384
// positions); hackernews.kjhq.dev post 49735410, key point 3.
//
// The key stream is the HBM-bound hot loop (64 B per position).  The E4M3 keys
// are the MMA's A operand exactly as stored: TMA tensor loads (64-byte
// swizzle, no multicast; one 256-row box per stage of a contiguous cache, one
// 64-row box per page run of a paged one) fill a ring of 256-position stages
// that tcgen05.mma reads directly, two 128-position tiles per stage.  The bf16 queries become
// U E4M3 operands stacked along N: per (token, head) row the values are scaled
// by a power of two so the row maximum lies in [128, 256), then
//     t0 = E4M3(q),  t1 = E4M3(16 (q - t0)),  t2 = E4M3(256 (q - t0 - t1/16))
// (round to nearest), so q = t0 + t1/16 + t2/256.  A bf16 value has 8
// significant bits and each term takes 4, so the sum is exact for every value
// at or above 2^-14 of the row maximum, and off by at most 2^-25 of it below
// (U = 3; U = 2 when 3 N would not fit: exact above 2^-14, off by at most
// 2^-21 below).  Two MMAs per tile (K = 2 x 32, N = U x T x H_I) accumulate the
// term products in fp32; the epilogue adds the term columns with their exact
// power-of-two weights.
//
//   producer warp  : TMA loads into the ring (bounded mbarrier waits)
//   MMA warp       : four tcgen05.mma (two per tile) and one commit per stage
//                    into a double-buffered TMEM accumulator (one buffer
//                    when two would not fit the 512 columns)
//   epilogue warps : four warpgroups, one per (buffer, tile); the first
//                    thread to see a stage's accumulators releases its ring
//                    stage; they stage
//                    the query terms when the sequence changes; per tile
//                    tcgen05.ld of each position's row, ReLU + head-weighted
//                    sum, fp32 score store, level-1 radix histogram in smem.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa2 {

namespace {

constexpr int kTile = 128;                // positions per MMA (M)
constexpr int kStagePos = 256;            // positions per ring stage: two tiles, one TMA box when contiguous
constexpr int kStages = 8;
constexpr int kStageBytes = kStagePos * 64;
constexpr int kMaxTerms = 3;
constexpr int kThreads = 576;
constexpr int kWarpProducer = 0, kWarpMma = 1, kWarpEpi0 = 2;   // epilogue: warps 2-17, four warpgroups
constexpr int kEpiThreads = 512;
constexpr uint32_t kDrainLimit = 65536;

struct Params {
    DevCache c;
    const __nv_bfloat16* q;  // [B][T][H_I][64]
    const float* hw;         // [B][T][H_I]
    int T, H_I, HP, NP;      // HP: H_I rounded up to 16; NP = T * HP columns per term
    int U;                   // query terms stacked along N (MMA N = U * NP)
    float* scores;           // [(b*T + j) * cap + t]
    uint32_t* hist;          // [(b*T + j)][3][kRadixBins]; level 1 accumulated here; nullable
    uint32_t* status;
    uint32_t wait_limit;     // tries of the waits that guard work (not of the drains)
    int64_t items_per_seq, total_items;   // an item is one ring stage of one sequence
    int nbuf;                // TMEM accumulator buffers of 2 * U * NP columns
    uint32_t tmem_cols;
    uint32_t off_b, off_hist, off_wq, off_bar;
};

struct Item {
    int b;
    int64_t t0, L;
};

// The CTA's items blockIdx.x, blockIdx.x + gridDim.x, .. as (sequence, stage)
// pairs, advanced without a division per item.
struct ItemCursor {
    int64_t item, k;
    int b;
    __device__ explicit ItemCursor(const Params& p) : item(blockIdx.x) {
        b = (int)(item / p.items_per_seq);
        k = item - (int64_t)b * p.items_per_seq;
    }
    __device__ void next(const Params& p) {
        item += gridDim.x;
        k += gridDim.x;
        while (k >= p.items_per_seq) {
            k -= p.items_per_seq;
            ++b;
        }
    }
};

__device__ __forceinline__ bool get_item(const Params& p, const ItemCursor& cu, Item& it) {
    const int b = cu.b;
    const int64_t k = cu.k;
    int64_t L = __ldg(p.c.seq_lens + b);
    L = L < 0 ? 0 : (L > p.c.cap ? p.c.cap : L);
    const int64_t t0 = k * kStagePos;
    if (t0 >= L) return false;
    it.b = b;
    it.t0 = t0;
    it.L = L;
    return true;
}

struct Bars {
    uint64_t full[kStages], empty[kStages];   // empty: released by the epilogue
    uint64_t acc_full[2], acc_empty[2];
    uint64_t b_ready[2], b_free[2];
    uint64_t hist_done, hist_clear;
    uint64_t drain;
    uint32_t tmem_base;
};

__device__ __forceinline__ float e4m3_round(float x, uint8_t* code) {
    const uint16_t c = cvt_e4m3x2(0.0f, x);
    *code = (uint8_t)(c & 0xFF);
    return e4m3_to_float(*code);
}

// The U 8-bit query operands of one sequence, stacked: row u * NP + c holds
// term u of row c (c = token j * HP + head h; padding rows are zero); plus the
// folded weights w * 2^-e.  4 threads per row, 16 values each.
__device__ void prepare_queries(const Params& p, int b, uint8_t* bq, float* wq, int tid) {
    const int row_in_pass = tid >> 2, quarter = tid & 3;
    for (int r0 = 0; r0 < p.NP; r0 += 32) {
        const int c = r0 + row_in_pass;
        const int j = c / p.HP, h = c - j * p.HP;
        const bool real = c < p.NP && h < p.H_I;
        float v[16];
        if (real) {
            const uint4* src = reinterpret_cast<const uint4*>(
                p.q + ((((int64_t)b * p.T + j) * p.H_I + h) * 64 + quarter * 16));
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
            const int E = (int)((__float_as_uint(m) >> 23) & 0xFF) - 127;
            e = 7 - E;
            e = e < -100 ? -100 : (e > 100 ? 100 : e);
        }
        const float up = __uint_as_float((uint32_t)(127 + e) << 23);
        const float down = __uint_as_float((uint32_t)(127 - e) << 23);
        if (c < p.NP) {
            uint8_t t[kMaxTerms][16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                float r = v[k] * up;                        // exact: a power-of-two scale
#pragma unroll
                for (int u = 0; u < kMaxTerms; ++u) {
                    // term u carries the remainder scaled by 16^u (exact); the
                    // remainder update subtracts its exact value
                    const float scale = (float)(1 << (4 * u));
                    const float tv = e4m3_round(r * scale, &t[u][k]);
                    r -= tv / scale;
                }
            }
#pragma unroll
            for (int u = 0; u < kMaxTerms; ++u) {
                if (u >= p.U) break;
                uint32_t wds[4];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    wds[k] = (uint32_t)t[u][4 * k] | ((uint32_t)t[u][4 * k + 1] << 8) |
                             ((uint32_t)t[u][4 * k + 2] << 16) | ((uint32_t)t[u][4 * k + 3] << 24);
                *reinterpret_cast<uint4*>(bq + tc::sw64_offset(u * p.NP + c, quarter)) =
                    make_uint4(wds[0], wds[1], wds[2], wds[3]);
            }
            if (quarter == 0) wq[c] = real ? __ldg(p.hw + ((int64_t)b * p.T + j) * p.H_I + h) * down : 0.0f;
        }
    }
}

// Score of one position from its accumulator row (one query token, 32 head
// columns per term, three terms): x_h = t0 + t1 / 16 + t2 / 256 (the exact
// term weights), then sum_h w_h max(0, x_h), heads in pairs with f32x2 FMAs.
__device__ __forceinline__ float score_32x3(uint32_t abase, const float* wq) {
    const float4* w4 = reinterpret_cast<const float4*>(wq);
    const float2 k16 = make_float2(0.0625f, 0.0625f), k256 = make_float2(0.00390625f, 0.00390625f);
    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int half = 0; half < 2; ++half) {            // heads 16 half .. 16 half + 15
        uint32_t r[3][16];
#pragma unroll
        for (int u = 0; u < 3; ++u) tc::tmem_ld16_nowait(abase + (uint32_t)(32 * u + 16 * half), r[u]);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 4; ++i) {                 // heads 16 half + 4 i .. + 3
            const float4 w = w4[4 * half + i];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int c = 4 * i + 2 * h;
                float2 x = make_float2(__uint_as_float(r[0][c]), __uint_as_float(r[0][c + 1]));
                x = __ffma2_rn(make_float2(__uint_as_float(r[1][c]), __uint_as_float(r[1][c + 1])), k16, x);
                x = __ffma2_rn(make_float2(__uint_as_float(r[2][c]), __uint_as_float(r[2][c + 1])), k256, x);
                x.x = fmaxf(x.x, 0.0f);
                x.y = fmaxf(x.y, 0.0f);
                acc[(2 * i + h) & 3] = __ffma2_rn(h ? make_float2(w.z, w.w) : make_float2(w.x, w.y), x,
                                                  acc[(2 * i + h) & 3]);
            }
        }
    }
    return ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) + ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
}

template <int NBUF>
__global__ void __launch_bounds__(kThreads, 1)
k_score_full_tc(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap tmap_stage,
                const Params p) {
    pdl_begin();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sRing = smem;
    uint8_t* sB = smem + p.off_b;
    uint32_t* sHist = reinterpret_cast<uint32_t*>(smem + p.off_hist);
    float* sWq = reinterpret_cast<float*>(smem + p.off_wq);
    Bars* bars = reinterpret_cast<Bars*>(smem + p.off_bar);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bq_bytes = p.U * p.NP * 64;
    const int NA = p.U * p.NP;                  // accumulator columns per 128-position tile
    constexpr int nbuf = NBUF;                  // accumulator buffers (a buffer holds a stage's two tiles)

    for (int i = threadIdx.x; i < p.T * kRadixBins; i += kThreads) sHist[i] = 0;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) { tc::mbar_init(&bars->full[i], 1); tc::mbar_init(&bars->empty[i], 1); }
        // empty[s] is arrived by the one epilogue thread that first sees the stage's accumulators
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&bars->acc_full[i], 1);
            tc::mbar_init(&bars->acc_empty[i], 2 * 128);
            tc::mbar_init(&bars->b_ready[i], kEpiThreads);
            tc::mbar_init(&bars->b_free[i], 1);
        }
        tc::mbar_init(&bars->hist_done, kEpiThreads);
        tc::mbar_init(&bars->hist_clear, kEpiThreads);
        tc::mbar_init(&bars->drain, 1);
        tc::fence_mbar_init();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_stage)) : "memory");
    }
    if (warp == kWarpMma) tc::tmem_alloc(&bars->tmem_base, p.tmem_cols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = bars->tmem_base;

    if (warp == kWarpProducer) {
        if (lane == 0) {
            uint32_t g = 0;
            bool ok = true;
            for (ItemCursor cu(p); cu.item < p.total_items && ok; cu.next(p)) {
                Item it;
                if (!get_item(p, cu, it)) continue;
                const int s = g % kStages;
                if (!tc::mbar_wait(&bars->empty[s], ((g / kStages) & 1) ^ 1, p.wait_limit)) { ok = false; break; }
                uint8_t* dst = sRing + s * kStageBytes;
                const int64_t slot0 = p.c.page_table ? -1 : slot_of(p.c, it.b, it.t0);
                if (slot0 >= 0 && slot0 + kStagePos <= p.c.n_slots) {
                    // a contiguous cache: the stage is one 256-row box
                    tc::mbar_arrive_expect_tx(&bars->full[s], kStageBytes);
                    tc::tma_load_2d(dst, &tmap_stage, 0, (int32_t)slot0, &bars->full[s]);
                } else {
                    // a paged cache, or a stage that would reach past the cache:
                    // one 64-row box per run of 64 positions
                    int64_t slot[kStagePos / 64];
                    uint32_t bytes = 0;
#pragma unroll
                    for (int r = 0; r < kStagePos / 64; ++r) {
                        const int64_t p0 = it.t0 + 64 * r;
                        slot[r] = p0 < it.L ? slot_of(p.c, it.b, p0) : -1;
                        if (p0 < it.L && slot[r] < 0) flag(p.status, kStatusBounds);
                        if (slot[r] >= 0) bytes += 64u * 64u;
                    }
                    if (bytes == 0) {
                        tc::mbar_arrive(&bars->full[s]);
                    } else {
                        tc::mbar_arrive_expect_tx(&bars->full[s], bytes);
#pragma unroll
                        for (int r = 0; r < kStagePos / 64; ++r)
                            if (slot[r] >= 0) tc::tma_load_2d(dst + r * 4096, &tmap, 0, (int32_t)slot[r], &bars->full[s]);
                    }
                }
                ++g;
            }
            if (!ok) flag(p.status, kStatusTimeout);
            // loads still in flight must land before the CTA's shared memory goes away
            for (uint32_t k = g > (uint32_t)kStages ? g - kStages : 0; k < g; ++k)
                tc::mbar_wait(&bars->full[k % kStages], (k / kStages) & 1, kDrainLimit);
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_f8_f32(128, NA, 0u, 0u);
            const uint64_t dring = tc::desc_sw64(tc::smem_u32(sRing));
            uint32_t g = 0, n = 0;
            int cur_b = -1;
            bool ok = true;
            for (ItemCursor cu(p); cu.item < p.total_items && ok; cu.next(p)) {
                Item it;
                if (!get_item(p, cu, it)) continue;
                if (it.b != cur_b) {
                    if (cur_b >= 0) { tc::mma_commit(&bars->b_free[n & 1]); ++n; }
                    cur_b = it.b;
                    if (!tc::mbar_wait(&bars->b_ready[n & 1], (n >> 1) & 1, p.wait_limit)) { ok = false; break; }
                }
                const uint64_t db = tc::desc_sw64(tc::smem_u32(sB + (n & 1) * bq_bytes));
                const int s = g % kStages, buf = g % nbuf;
                const uint32_t use = g / nbuf;            // the buffer's use count
                if (!tc::mbar_wait(&bars->full[s], (g / kStages) & 1, p.wait_limit) ||
                    !tc::mbar_wait(&bars->acc_empty[buf], (use & 1) ^ 1, p.wait_limit)) { ok = false; break; }
                tc::fence_after_sync();
                const uint64_t da = tc::desc_at(dring, (uint32_t)s * kStageBytes);
                const uint32_t d = tmem + (uint32_t)(buf * 2 * NA);
#pragma unroll
                for (int x = 0; x < 2; ++x) {            // the stage's two 128-position tiles
                    const uint64_t dx = tc::desc_at(da, (uint32_t)x * (kTile * 64));
                    tc::mma_f8(d + (uint32_t)(x * NA), dx, db, idesc, 0u);
                    tc::mma_f8(d + (uint32_t)(x * NA), tc::desc_at(dx, 32), tc::desc_at(db, 32), idesc, 1u);
                }
                tc::mma_commit(&bars->acc_full[buf]);
                ++g;
            }
            if (!ok) flag(p.status, kStatusTimeout);
            tc::mma_commit(&bars->drain);
            tc::mbar_wait(&bars->drain, 0, kDrainLimit);
        }
    } else {
        // epilogue: four warpgroups; warpgroup w finishes tile w % 2 of the
        // stages held in accumulator buffer w / 2 (with one buffer, warpgroups
        // 2 and 3 only take part in the per-sequence steps); thread = TMEM lane
        // = position in the tile
        const int tid = threadIdx.x - kWarpEpi0 * 32;          // 0..511
        const int grp = tid >> 7;                               // warpgroup
        const int my_buf = grp >> 1, my_x = grp & 1;
        const bool works = my_buf < nbuf;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
        uint32_t g = 0, n = 0, nflush = 0;
        int cur_b = -1;
        bool ok = true;
        // Move the shared histogram of sequence b into the global one.  The
        // epilogue threads meet on two mbarriers (bounded waits).
        auto flush = [&](int b) -> bool {
            tc::mbar_arrive(&bars->hist_done);
            if (!tc::mbar_wait(&bars->hist_done, nflush & 1, p.wait_limit)) return false;
            if (p.hist) {
                for (int j = 0; j < p.T; ++j) {
                    uint32_t* gh = p.hist + ((int64_t)b * p.T + j) * 3 * kRadixBins;
                    for (int i = tid; i < kRadixBins; i += kEpiThreads) {
                        const uint32_t v = sHist[j * kRadixBins + i];
                        if (v) { atomicAdd(gh + i, v); sHist[j * kRadixBins + i] = 0; }
                    }
                }
            }
            tc::mbar_arrive(&bars->hist_clear);
            if (!tc::mbar_wait(&bars->hist_clear, nflush & 1, p.wait_limit)) return false;
            ++nflush;
            return true;
        };
        // all lanes of a warp take the same decision before tcgen05.ld (.aligned)
        auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
            const bool got = tc::mbar_wait(bar, parity, p.wait_limit);
            return __all_sync(0xffffffffu, got);
        };
        const float* wq = sWq;
        for (ItemCursor cu(p); cu.item < p.total_items && ok; cu.next(p)) {
            Item it;
            if (!get_item(p, cu, it)) continue;
            if (it.b != cur_b) {
                if (cur_b >= 0) {
                    if (!flush(cur_b)) { ok = false; break; }
                    ++n;
                }
                cur_b = it.b;
                // stage this sequence's query operands once the MMAs of the
                // sequence that used the buffer before are done
                const int qb = n & 1;
                if (!tc::mbar_wait(&bars->b_free[qb], ((n >> 1) & 1) ^ 1, p.wait_limit)) { ok = false; break; }
                if (grp == 0) prepare_queries(p, it.b, sB + qb * bq_bytes, sWq + qb * p.NP, tid);
                tc::fence_proxy_async_smem();
                tc::mbar_arrive(&bars->b_ready[qb]);
                // the same barrier publishes the weights to every epilogue thread
                if (!warp_wait(&bars->b_ready[qb], (n >> 1) & 1)) { ok = false; break; }
                wq = sWq + qb * p.NP;
            }
            const uint32_t gs = g++;
            if (!works || (int)(gs % nbuf) != my_buf) continue;   // another warpgroup's stage
            const uint32_t use = gs / nbuf;
            const int64_t t = it.t0 + (int64_t)my_x * kTile + row;
            // a position on a page outside the cache was not loaded (the
            // producer flagged it): its score is NaN, which is never selected
            const bool skipped = p.c.page_table != nullptr && t < it.L && slot_of(p.c, it.b, t) < 0;
            if (!warp_wait(&bars->acc_full[my_buf], use & 1)) { ok = false; break; }
            tc::fence_after_sync();
            // the MMAs of this stage are complete: its ring stage can be refilled
            if (my_x == 0 && (tid & 127) == 0) tc::mbar_arrive(&bars->empty[gs % kStages]);
            const uint32_t abase = lane_addr + (uint32_t)((my_buf * 2 + my_x) * NA);
            if (p.T == 1 && p.NP == 32 && p.U == 3) {
                // one query token, 32 head columns per term: every column of the
                // three terms in flight at once, the heads in pairs (f32x2)
                const float sc = skipped ? __int_as_float(0x7fc00000) : score_32x3(abase, wq);
                if (t <= it.L - 1) {
                    p.scores[(int64_t)it.b * p.c.cap + t] = sc;
                    if (p.hist && !skipped) atomicAdd(&sHist[ordered_key(sc) >> 21], 1u);
                }
            } else
            for (int j = 0; j < p.T; ++j) {
                float s0 = 0.0f, s1 = 0.0f;
                for (int c0 = j * p.HP; c0 < (j + 1) * p.HP; c0 += 16) {
                    // the 16 heads' columns of every term in flight, one wait
                    uint32_t r[kMaxTerms][16];
                    tc::tmem_ld16_nowait(abase + (uint32_t)c0, r[0]);
                    tc::tmem_ld16_nowait(abase + (uint32_t)(p.NP + c0), r[1]);
                    if (p.U > 2) tc::tmem_ld16_nowait(abase + (uint32_t)(2 * p.NP + c0), r[2]);
                    tc::tmem_ld_wait();
                    const float4* w4 = reinterpret_cast<const float4*>(wq + c0);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float4 ww = w4[i];
                        float dot[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            float x = fmaf(__uint_as_float(r[1][4 * i + k]), 0.0625f, __uint_as_float(r[0][4 * i + k]));
                            if (p.U > 2) x = fmaf(__uint_as_float(r[2][4 * i + k]), 0.00390625f, x);
                            dot[k] = fmaxf(x, 0.0f);
                        }
                        s0 = fmaf(ww.x, dot[0], s0);
                        s1 = fmaf(ww.y, dot[1], s1);
                        s0 = fmaf(ww.z, dot[2], s0);
                        s1 = fmaf(ww.w, dot[3], s1);
                    }
                }
                const float sc = skipped ? __int_as_float(0x7fc00000) : s0 + s1;
                const bool vis = t <= it.L - p.T + j;
                if (vis) p.scores[((int64_t)it.b * p.T + j) * p.c.cap + t] = sc;
                if (p.hist && vis && !skipped) atomicAdd(&sHist[j * kRadixBins + (ordered_key(sc) >> 21)], 1u);
            }
            tc::fence_before_sync();
            tc::mbar_arrive(&bars->acc_empty[my_buf]);
        }
        if (ok && cur_b >= 0 && !flush(cur_b)) ok = false;
        if (!ok) flag(p.status, kStatusTimeout);
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == kWarpMma) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, p.tmem_cols);
    }
}

struct SmemPlan {
    uint32_t off_b, off_hist, off_wq, off_bar, total;
};

int n_terms(int NP) { return 3 * NP <= 256 ? 3 : 2; }

SmemPlan smem_plan(int T, int NP) {
    SmemPlan s;
    uint32_t off = kStages * kStageBytes;
    s.off_b = off;
    off += 2 * n_terms(NP) * NP * 64;
    s.off_hist = off;
    off += T * kRadixBins * 4;
    s.off_wq = off;
    off += 2 * NP * 4;
    off = (off + 15) / 16 * 16;
    s.off_bar = off;
    off += sizeof(Bars);
    s.total = off + 1024;  // room to align the base to 1024 B
    return s;
}

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
    // the driver entry point, resolved through the runtime (no link-time driver dependency)
    static EncodeTiled fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeTiled) nullptr;
        return reinterpret_cast<EncodeTiled>(f);
    }();
    return fn;
}

}  // namespace

bool score_full_tc_supported(const DevCache& c, int T, int H_I) {
    const int HP = (H_I + 15) / 16 * 16;
    return c.key_dtype == 2 && c.idx_dim == 64 && 2 * T * HP <= 256 && smem_plan(T, T * HP).total <= 227 * 1024 &&
           c.n_slots < ((int64_t)1 << 31) && encode_fn() != nullptr;
}

cudaError_t launch_score_full_tc(const DevCache& c, const void* q, const float* hw, int T, int H_I, float* scores,
                                 uint32_t* hist, uint32_t* status, cudaStream_t st, int num_sms) {
    Params p;
    p.c = c;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.hw = hw;
    p.T = T;
    p.H_I = H_I;
    p.HP = (H_I + 15) / 16 * 16;
    p.NP = T * p.HP;
    p.U = n_terms(p.NP);
    p.scores = scores;
    p.hist = hist;
    p.status = status;
    p.wait_limit = wait_limit();
    p.items_per_seq = (c.cap + kStagePos - 1) / kStagePos;
    p.total_items = p.items_per_seq * c.batch;
    // two buffers of a stage's two tiles when they fit in the 512 TMEM columns
    p.nbuf = 4 * p.U * p.NP <= 512 ? 2 : 1;
    uint32_t cols = 32;
    while (cols < (uint32_t)(2 * p.nbuf * p.U * p.NP)) cols <<= 1;
    p.tmem_cols = cols;
    const SmemPlan sp = smem_plan(T, p.NP);
    p.off_b = sp.off_b;
    p.off_hist = sp.off_hist;
    p.off_wq = sp.off_wq;
    p.off_bar = sp.off_bar;

    // keys as a 2-D byte tensor [n_slots][64], 64-byte swizzle: 64-row boxes
    // (page runs) and 256-row boxes (a whole stage of a contiguous cache)
    CUtensorMap tmap, tmap_stage;
    const cuuint64_t gdim[2] = {64, (cuuint64_t)c.n_slots};
    const cuuint64_t gstride[1] = {64};
    const cuuint32_t box[2] = {64, 64}, box_stage[2] = {64, (cuuint32_t)kStagePos};
    const cuuint32_t estride[2] = {1, 1};
    EncodeTiled enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    if (enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, c.keys, gdim, gstride, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        enc(&tmap_stage, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, c.keys, gdim, gstride, box_stage, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;

    auto kern = p.nbuf == 2 ? k_score_full_tc<2> : k_score_full_tc<1>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp.total);
    if (e != cudaSuccess) return e;
    // one CTA per SM (its four epilogue warpgroups and up to 512 TMEM columns)
    int64_t grid = (int64_t)num_sms;
    if (grid > p.total_items) grid = p.total_items;
    if (grid < 1) grid = 1;
    return launch_pdl(kern, dim3((unsigned)grid), dim3(kThreads), sp.total, st, tmap, tmap_stage, p);
}

}  // namespace csa2

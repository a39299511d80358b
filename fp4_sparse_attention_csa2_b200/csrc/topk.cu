// Top-n selection by radix select on order-preserving 32-bit keys of fp32
// scores: the candidate pool (<= 16,384 of up to 1M scores) of a Full layer
// and the top-k of Full / Reindex layers (tldrocket.com, "DeepSeek AI Released
// DeepSeek-V4.1-Flash with 1M Context, FP4 KV Cache, and Cross-Layer Attention
// Reuse", paragraph 3; hackernews.kjhq.dev post 49735410, key point 2, "Top-K
// indices").
//
// The key is split into three digits: bits 31..21, 20..10 and 9..0.  For a
// digit histogram h and a number `need` still to select, the threshold digit c
// satisfies above(c) < need <= above(c) + h[c]; elements with a larger digit
// are selected, elements with digit c go on to the next digit, and at the last
// digit the remaining equal keys are exact ties of which the first claimants
// win.  Output order is unspecified; -1 pads the tail.
//
//   large segments (Full layer, up to 1M scores), when every CTA of the grid
//     fits on the GPU at once: one launch, each CTA holding its keys in
//     registers, two bounded segment barriers between the digit levels
//     (k_sel_grid; also for a list of positions, as a pool update's).
//   large segments otherwise: the level-1 histogram comes
//     from the scoring kernel; a streaming pass (many CTAs per segment) works
//     out each target's level-1 threshold, selects above it and compacts the
//     elements equal to it into candidate lists (histogramming their digit 2);
//     the pass's last CTA publishes the digit-2 plan.  A second pass over the
//     lists (many CTAs) selects above the digit-2 thresholds and keeps the
//     survivors, and its last CTA resolves digit 3 and exact ties.  The pool
//     and the layer's top-k are two targets of the same passes.
//   small segments (<= 16,384: the top-k of a pool, and the pool of a Full
//     layer over a short context): one CTA of 1,024 threads per segment
//     brackets the cutoff from a sample, compacts the elements inside the
//     bracket and resolves them by radix select in shared memory (lsel.cuh).
#include "common.cuh"
#include "gsel.cuh"
#include "kernels.h"
#include "lsel.cuh"

namespace csa2 {

namespace {

constexpr int kPassThreads = 256;
constexpr int kPassChunk = kPassThreads * 16;
constexpr int kSmallMax = 16384;

struct Elem {
    bool valid;
    int32_t id;
    uint32_t key;
};

__device__ __forceinline__ int64_t n_valid_positions(const SelSrc& s, int seg) {
    const int b = seg / s.T, j = seg % s.T;
    int64_t L = __ldg(s.seq_lens + b);
    if (L > s.cap) L = s.cap;
    const int64_t n = L - s.T + j + 1;
    return n < 0 ? 0 : n;
}

__device__ __forceinline__ Elem load_elem(const SelSrc& s, int seg, int64_t i, int64_t nvalid) {
    Elem e;
    if (s.ids == nullptr) {
        e.id = (int32_t)i;
        e.key = select_key(i < nvalid ? s.vals[seg * s.vals_stride + i] : 0.0f, i < nvalid);
        e.valid = e.key != 0u;
    } else {
        // entries outside [0, p] are padding or were flagged when scored
        e.id = s.ids[seg * s.ids_stride + i];
        const bool cand = e.id >= 0 && e.id < nvalid;
        e.key = select_key(cand ? s.vals[seg * s.vals_stride + (s.gather ? (int64_t)e.id : i)] : 0.0f, cand);
        e.valid = e.key != 0u;
    }
    return e;
}

// The score an ordered key came from (-0 comes back as +0).
__device__ __forceinline__ float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

__device__ __forceinline__ uint32_t digit(uint32_t key, int level) {
    return level == 1 ? (key >> 21) : level == 2 ? ((key >> 10) & 0x7FFu) : (key & 0x3FFu);
}

// Threshold digit of a 2048-bin histogram (global or shared memory) found by
// the whole block of NT threads.  Thread t owns the kRadixBins / NT bins just
// below 2048 - t * (kRadixBins / NT), so descending bins follow ascending
// threads, and one exclusive scan of the per-thread sums locates the bin c
// with above(c) < need <= above(c) + h[c].  need_in == 0 asks for
// need = min(total, n_out).  Every thread gets {c, above(c), h[c], need};
// with need == 0 there is nothing to select and c is meaningless.
struct Thr {
    uint32_t c, above, eq, need;
};

template <int NT>
__device__ __forceinline__ Thr block_threshold(const uint32_t* h, uint32_t need_in, uint32_t n_out, uint32_t* s_wsum,
                                               Thr* s_thr) {
    constexpr int per = kRadixBins / NT;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int lo = kRadixBins - per * (tid + 1);
    uint32_t bins[per];
    uint32_t sum = 0;
#pragma unroll
    for (int k = 0; k < per; ++k) {
        bins[k] = h[lo + k];
        sum += bins[k];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    uint32_t before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        const uint32_t v = s_wsum[w];
        before += w < warp ? v : 0u;
        total += v;
    }
    const uint32_t need = need_in ? need_in : (total < n_out ? total : n_out);
    const uint32_t excl = before + incl - sum;
    if (need > 0 && excl < need && need <= excl + sum) {
        uint32_t above = excl;
#pragma unroll
        for (int k = per - 1; k >= 0; --k) {
            if (need <= above + bins[k]) {
                s_thr->c = (uint32_t)(lo + k);
                s_thr->above = above;
                s_thr->eq = bins[k];
                break;
            }
            above += bins[k];
        }
    }
    __syncthreads();
    Thr r = *s_thr;
    r.need = need;
    __syncthreads();   // s_wsum and s_thr are rewritten by the next call
    return r;
}

// Exclusive prefix sum over the block of one value per thread; *total gets the sum.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* s_wsum, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    uint32_t before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        const uint32_t u = s_wsum[w];
        before += w < warp ? u : 0u;
        tot += u;
    }
    __syncthreads();   // s_wsum is rewritten by the next call
    *total = tot;
    return before + incl - v;
}

// Exclusive prefix over the block of four 16-bit counts packed in one 64-bit
// value (per-block sums must stay below 65,536); *total gets the sums.
template <int NT>
__device__ __forceinline__ uint64_t block_excl_scan4(uint64_t v, uint64_t* s_wsum, uint64_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    uint64_t before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        const uint64_t u = s_wsum[w];
        before += w < warp ? u : 0ull;
        tot += u;
    }
    __syncthreads();   // s_wsum is rewritten by the next call
    *total = tot;
    return before + incl - v;
}

__device__ __forceinline__ uint32_t field16(uint64_t v, int f) { return (uint32_t)(v >> (16 * f)) & 0xFFFFu; }

// Warp-aggregated claim: the lanes with `pred` get consecutive values of *counter.
__device__ __forceinline__ uint32_t warp_claim(bool pred, uint32_t* counter) {
    const int lane = threadIdx.x & 31;
    const uint32_t m = __ballot_sync(0xffffffffu, pred);
    uint32_t base = 0;
    if (m) {
        const int leader = __ffs(m) - 1;
        if (lane == leader) base = atomicAdd(counter, (uint32_t)__popc(m));
        base = __shfl_sync(0xffffffffu, base, leader);
    }
    return base + __popc(m & ((1u << lane) - 1u));
}

// ---------------------------------------------------------------- large segments
// Level-1 histogram, for sources that did not get one from the scoring kernel.
__global__ void __launch_bounds__(kPassThreads) k_sel_hist(SelSrc src, SelWork wk) {
    pdl_begin();
    __shared__ uint32_t h[kRadixBins];
    const int seg = blockIdx.y;
    for (int i = threadIdx.x; i < kRadixBins; i += kPassThreads) h[i] = 0;
    __syncthreads();
    const int64_t nvalid = n_valid_positions(src, seg);
    const int64_t base = (int64_t)blockIdx.x * kPassChunk;
    const int64_t end = min(base + kPassChunk, src.ids ? src.n : nvalid);
    for (int64_t i = base + threadIdx.x; i < end; i += kPassThreads) {
        Elem e = load_elem(src, seg, i, nvalid);
        if (e.valid) atomicAdd(&h[digit(e.key, 1)], 1u);
    }
    __syncthreads();
    uint32_t* gh = wk.hist + (int64_t)seg * 3 * kRadixBins;
    for (int i = threadIdx.x; i < kRadixBins; i += kPassThreads)
        if (h[i]) atomicAdd(gh + i, h[i]);
}

// Two selections of the same scores at once: target a (the pool, n_a) and
// target b (the top-k, n_b <= n_a; n_b == 0: none), with b a subset of a.
// Level-1 plan of one target from the level-1 histogram.
// Threshold digits of two targets in one 2048-bin histogram (global or shared
// memory) with one block-wide scan; need_in[t] == 0 asks for
// min(total, n_out[t]), and a target with need 0 gets no threshold.
template <int NT>
__device__ __forceinline__ void block_thresholds2(const uint32_t* h, const uint32_t need_in[2],
                                                  const uint32_t n_out[2], uint32_t* s_wsum, Thr* s_thr,
                                                  Thr out[2]) {
    constexpr int per = kRadixBins / NT;        // 2 or 8: one or two vector loads (many CTAs read one histogram)
    static_assert(per == 2 || per == 8, "bins per thread");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int lo = kRadixBins - per * (tid + 1);
    uint32_t bins[per];
    if (per == 8) {
        const uint4 v0 = reinterpret_cast<const uint4*>(h + lo)[0], v1 = reinterpret_cast<const uint4*>(h + lo)[1];
        const uint32_t b8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int k = 0; k < per; ++k) bins[k] = b8[k % 8];
    } else {
        const uint2 v = *reinterpret_cast<const uint2*>(h + lo);
        bins[0] = v.x;
        bins[per - 1] = v.y;
    }
    uint32_t sum = 0;
#pragma unroll
    for (int k = 0; k < per; ++k) sum += bins[k];
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    // warp totals: an inclusive scan by every warp over the NT / 32 totals
    uint32_t wt = lane < NT / 32 ? s_wsum[lane] : 0u;
#pragma unroll
    for (int o = 1; o < NT / 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, wt, o);
        if (lane >= o) wt += v;
    }
    const uint32_t total = __shfl_sync(0xffffffffu, wt, NT / 32 - 1);
    const uint32_t before = warp ? __shfl_sync(0xffffffffu, wt, (warp - 1) & 31) : 0u;
    const uint32_t excl = before + incl - sum;
    uint32_t need[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        need[t] = need_in[t] ? need_in[t] : (total < n_out[t] ? total : n_out[t]);
        if (need[t] > 0 && excl < need[t] && need[t] <= excl + sum) {
            uint32_t above = excl;
#pragma unroll
            for (int k = per - 1; k >= 0; --k) {
                if (need[t] <= above + bins[k]) {
                    s_thr[t].c = (uint32_t)(lo + k);
                    s_thr[t].above = above;
                    s_thr[t].eq = bins[k];
                    break;
                }
                above += bins[k];
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        out[t] = s_thr[t];
        out[t].need = need[t];
    }
    __syncthreads();   // s_wsum and s_thr are rewritten by the next call
}

// Two selections of the same scores at once: target a (the pool, n_a) and
// target b (the top-k, n_b <= n_a; n_b == 0: none), with b a subset of a.
// Level-1 plan of each target from the level-1 histogram.
struct Plan1 {
    uint32_t need, c, above, eq;   // eq: elements with digit c
    bool take_eq;                  // every digit-c element is needed (or nothing is)
};

template <int NT>
__device__ __forceinline__ void plans_level1(const uint32_t* h1, uint32_t n_a, uint32_t n_b, uint32_t* s_wsum,
                                             Thr* s_thr, Plan1& pa, Plan1& pb) {
    const uint32_t need_in[2] = {0u, 0u}, n_out[2] = {n_a, n_b};
    Thr t[2];
    block_thresholds2<NT>(h1, need_in, n_out, s_wsum, s_thr, t);
    Plan1* pp[2] = {&pa, &pb};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        Plan1 p = {0u, 0xFFFFFFFFu, 0u, 0u, true};
        if (t[i].need > 0) {
            p.need = t[i].need;
            p.c = t[i].c;
            p.above = t[i].above;
            p.eq = t[i].eq;
            p.take_eq = t[i].eq == t[i].need - t[i].above;
        }
        *pp[i] = p;
    }
}

// Level-2 plan of both targets (digit-2 thresholds on the candidate lists).
struct Plan2 {
    Plan1 p[2];
    bool shared;
    uint32_t len[2];        // candidate list lengths (0: the target is complete after level 1)
    uint32_t need2[2];      // still needed from the list
    Thr q[2];               // digit-2 thresholds
    bool eq2[2];            // every digit-2 == c2 candidate is needed
};

// The plan travels from pass 1's last CTA to pass 2 and the finisher as
// kPlanWords words after the segment's counters.
constexpr int kPlanWord0 = 9;
constexpr int kPlanWords = 19;
static_assert(kPlanWord0 + kPlanWords <= kSelCounters, "plan words");

// Level-1 words: both targets' level-1 plans and whether their candidate lists
// are one (written by pass 1's last CTA with the level-2 words).
__device__ __forceinline__ void plan_write1(uint32_t* w, const Plan1& pa, const Plan1& pb) {
    const Plan1* pp[2] = {&pa, &pb};
    for (int t = 0; t < 2; ++t) {
        w[5 * t + 0] = pp[t]->need;
        w[5 * t + 1] = pp[t]->c;
        w[5 * t + 2] = pp[t]->above;
        w[5 * t + 3] = pp[t]->eq;
        w[5 * t + 4] = pp[t]->take_eq;
    }
    w[18] = pb.c == pa.c && !pa.take_eq;
}

// Level-2 words (written by pass 1's last CTA): the digit-2 thresholds.
__device__ __forceinline__ void plan_write2(uint32_t* w, const Plan2& P) {
    for (int t = 0; t < 2; ++t) {
        w[10 + 4 * t + 0] = P.q[t].c;
        w[10 + 4 * t + 1] = P.q[t].above;
        w[10 + 4 * t + 2] = P.q[t].eq;
        w[10 + 4 * t + 3] = P.q[t].need;
    }
}

// Every thread gets the plan from the words (staged through shared memory).
__device__ __forceinline__ Plan2 plan_read(const uint32_t* w, uint32_t* s_words) {
    if (threadIdx.x < kPlanWords) s_words[threadIdx.x] = __ldcg(w + threadIdx.x);
    __syncthreads();
    Plan2 P;
    for (int t = 0; t < 2; ++t) {
        P.p[t].need = s_words[5 * t + 0];
        P.p[t].c = s_words[5 * t + 1];
        P.p[t].above = s_words[5 * t + 2];
        P.p[t].eq = s_words[5 * t + 3];
        P.p[t].take_eq = s_words[5 * t + 4] != 0u;
        P.q[t].c = s_words[10 + 4 * t + 0];
        P.q[t].above = s_words[10 + 4 * t + 1];
        P.q[t].eq = s_words[10 + 4 * t + 2];
        P.q[t].need = s_words[10 + 4 * t + 3];
    }
    P.shared = s_words[18] != 0u;
    for (int t = 0; t < 2; ++t) {
        P.len[t] = P.p[t].take_eq ? 0u : P.p[t].eq;
        P.need2[t] = P.len[t] ? P.p[t].need - P.p[t].above : 0u;
        P.eq2[t] = P.q[t].eq == P.need2[t] - P.q[t].above;
    }
    return P;
}

// Level 1 over every element, both targets: digits above a target's c1 are
// selected, digit-c1 elements are compacted into that target's candidate list
// (one list when both thresholds fall on the same digit that a does not take
// whole) and their digit 2 is histogrammed in shared memory, then added to the
// segment's level-2 histogram of that list.  The chunk's scores are loaded
// before the plan is known.  Each CTA claims its output and candidate slots
// with one atomic per counter (block-wide scans of per-thread counts; the four
// atomics issued by four threads).
constexpr int kPassPer = kPassChunk / kPassThreads;   // elements per thread and chunk

__global__ void __launch_bounds__(kPassThreads)
k_sel_pass1(SelSrc src, SelWork wk, int n_a, int32_t* __restrict__ out_a, float* __restrict__ vals_a,
            int64_t stride_a, int n_b, int32_t* __restrict__ out_b, int64_t stride_b) {
    pdl_begin();
    __shared__ uint32_t s_wsum[kPassThreads / 32];
    __shared__ uint64_t s_wsum64[kPassThreads / 32];
    __shared__ Thr s_thr[2];
    __shared__ uint32_t s_base[4];
    __shared__ __align__(16) uint32_t h2[2][kRadixBins];   // digit 2 of the candidates of list a, of list b
    extern __shared__ uint2 stage_dyn[];                      // 2 x kPassChunk: the stages of a and of b
    uint2* stage_a = stage_dyn;
    uint2* stage_b = stage_dyn + kPassChunk;
    const int seg = blockIdx.y, tid = threadIdx.x;
    for (int i = tid; i < 2 * kRadixBins; i += kPassThreads) (&h2[0][0])[i] = 0;   // ordered by the barriers below
    uint32_t* cnt = wk.cnt + (int64_t)seg * kSelCounters;
    const int64_t nvalid = n_valid_positions(src, seg);
    const int64_t n_items = src.ids ? src.n : nvalid;
    int64_t base = (int64_t)blockIdx.x * kPassChunk;
    // a chunk is fetched in two steps: every load is issued first (the ids, then
    // the values they select), the keys are formed only when they are needed,
    // so the first chunk's loads are in flight while the plan is read
    uint32_t keys[kPassPer];
    int32_t ids[kPassPer];
    float raw[kPassPer];
    auto issue_chunk = [&](int64_t b0) {
#pragma unroll
        for (int k = 0; k < kPassPer; ++k) {
            const int64_t i = b0 + k * kPassThreads + tid;
            ids[k] = i < n_items ? (src.ids ? src.ids[seg * src.ids_stride + i] : (int32_t)i) : -1;
        }
#pragma unroll
        for (int k = 0; k < kPassPer; ++k) {
            const int64_t i = b0 + k * kPassThreads + tid;
            const bool v = ids[k] >= 0 && ids[k] < nvalid;
            raw[k] = v ? src.vals[seg * src.vals_stride + (src.gather && src.ids ? (int64_t)ids[k] : i)] : 0.0f;
        }
    };
    auto form_keys = [&]() {
#pragma unroll
        for (int k = 0; k < kPassPer; ++k)   // a valid key is never 0
            keys[k] = select_key(raw[k], ids[k] >= 0 && ids[k] < nvalid);
    };
    if (base < n_items) issue_chunk(base);
    // level-1 plans of both targets from the scorer's histogram (two 16-byte
    // loads per thread, one block-wide scan), while the chunk's loads are in flight
    Plan1 pa, pb;
    plans_level1<kPassThreads>(wk.hist + (int64_t)seg * 3 * kRadixBins, (uint32_t)n_a, (uint32_t)n_b, s_wsum, s_thr,
                               pa, pb);
    int32_t* oa = out_a + (int64_t)seg * stride_a;
    int32_t* ob = out_b ? out_b + (int64_t)seg * stride_b : nullptr;
    float* va = vals_a ? vals_a + (int64_t)seg * stride_a : nullptr;
    if (blockIdx.x == 0) {
        for (int i = (int)pa.need + tid; i < n_a; i += kPassThreads) oa[i] = -1;
        for (int i = (int)pb.need + tid; i < n_b; i += kPassThreads) ob[i] = -1;
    }
    if (pa.need == 0) base = n_items;                 // nothing to select (every CTA still reports below)
    const bool shared = pb.c == pa.c && !pa.take_eq;   // b's candidates are a's
    uint2* cand_a = reinterpret_cast<uint2*>(wk.cand1) + seg * wk.cand_stride;
    uint2* cand_b = reinterpret_cast<uint2*>(wk.cand2) + seg * wk.cand_stride;
    for (; base < n_items; base += (int64_t)gridDim.x * kPassChunk) {
        if (base != (int64_t)blockIdx.x * kPassChunk) issue_chunk(base);
        form_keys();
        uint32_t na = 0, nca = 0, nb = 0, ncb = 0;
#pragma unroll
        for (int k = 0; k < kPassPer; ++k) {
            const bool valid = keys[k] != 0u;
            const uint32_t d = digit(keys[k], 1);
            na += valid && (d > pa.c || (d == pa.c && pa.take_eq));
            nca += valid && d == pa.c && !pa.take_eq;
            nb += valid && (d > pb.c || (d == pb.c && pb.take_eq));
            ncb += valid && !shared && d == pb.c && !pb.take_eq;
        }
        // per-thread counts <= 16 and per-block sums <= 4096: four fit one 64-bit word
        uint64_t tot;
        const uint64_t pre = block_excl_scan4<kPassThreads>(
            (uint64_t)na | ((uint64_t)nca << 16) | ((uint64_t)nb << 32) | ((uint64_t)ncb << 48), s_wsum64, &tot);
        if (tid < 4) {   // a outputs, a candidates, b outputs, b candidates
            const uint32_t v = field16(tot, tid);
            s_base[tid] = v ? atomicAdd(cnt + tid, v) : 0u;
        }
        // the CTA's outputs are gathered in shared memory first (a's and b's
        // outputs from the front of their stage, candidates from the back),
        // then written out as contiguous runs
        uint32_t os_a = field16(pre, 0), cs_a = field16(pre, 1), os_b = field16(pre, 2), cs_b = field16(pre, 3);
#pragma unroll
        for (int k = 0; k < kPassPer; ++k) {
            const uint32_t key = keys[k];
            if (!key) continue;
            const uint32_t d = digit(key, 1);
            if (d > pa.c || (d == pa.c && pa.take_eq)) {
                stage_a[os_a++] = make_uint2((uint32_t)ids[k], key);
            } else if (d == pa.c) {
                stage_a[kPassChunk - 1 - cs_a++] = make_uint2(key, (uint32_t)ids[k]);
            }
            if (d > pb.c || (d == pb.c && pb.take_eq)) {
                stage_b[os_b++] = make_uint2((uint32_t)ids[k], key);
            } else if (!shared && d == pb.c) {
                stage_b[kPassChunk - 1 - cs_b++] = make_uint2(key, (uint32_t)ids[k]);
            }
        }
        __syncthreads();   // the stages are complete; the bases have been claimed
        {
            const uint32_t n0 = field16(tot, 0), n1 = field16(tot, 1), n2 = field16(tot, 2), n3 = field16(tot, 3);
            // outputs stay inside their rows even when the level-1 histogram
            // undercounts (a scoring kernel whose wait gave up; the status says so)
            for (uint32_t i = tid; i < n0; i += kPassThreads) {
                const uint2 v = stage_a[i];
                const uint32_t o = s_base[0] + i;
                if (o >= (uint32_t)n_a) break;
                oa[o] = (int32_t)v.x;
                if (va) va[o] = key_value(v.y);
            }
            for (uint32_t i = tid; i < n1; i += kPassThreads) cand_a[s_base[1] + i] = stage_a[kPassChunk - 1 - i];
            for (uint32_t i = tid; i < n2 && s_base[2] + i < (uint32_t)n_b; i += kPassThreads)
                ob[s_base[2] + i] = (int32_t)stage_b[i].x;
            for (uint32_t i = tid; i < n3; i += kPassThreads) cand_b[s_base[3] + i] = stage_b[kPassChunk - 1 - i];
        }
        __syncthreads();   // s_base and the stages are rewritten by the next chunk
        // digit-2 histograms of the candidates just compacted
#pragma unroll
        for (int k = 0; k < kPassPer; ++k) {
            const uint32_t key = keys[k];
            const uint32_t d = digit(key, 1);
            if (key && d == pa.c && !pa.take_eq) atomicAdd(&h2[0][digit(key, 2)], 1u);
            if (key && !shared && d == pb.c && !pb.take_eq) atomicAdd(&h2[1][digit(key, 2)], 1u);
        }
    }
    __syncthreads();
    uint32_t* gh = wk.hist + (int64_t)seg * 3 * kRadixBins;
    for (int i = tid; i < 2 * kRadixBins; i += kPassThreads) {
        const uint32_t v = (&h2[0][0])[i];
        if (v) atomicAdd(gh + kRadixBins + i, v);   // level-2 histograms of list a, list b
    }
    // the CTA that reports last sees the complete level-2 histograms and
    // publishes the plan of both targets for pass 2 and the finisher
    __threadfence();
    __syncthreads();
    if (tid == 0) s_base[0] = atomicAdd(cnt + 8, 1u) == gridDim.x - 1 ? 1u : 0u;
    __syncthreads();
    if (!s_base[0]) return;
    __threadfence();
    {
        // all loads in flight at once (4 x 16 bytes per thread)
        constexpr int kVec = 2 * kRadixBins / 4 / kPassThreads;
        uint4 hv[kVec];
        const uint4* g4 = reinterpret_cast<const uint4*>(gh + kRadixBins);
#pragma unroll
        for (int k = 0; k < kVec; ++k) hv[k] = __ldcg(g4 + k * kPassThreads + tid);
#pragma unroll
        for (int k = 0; k < kVec; ++k) reinterpret_cast<uint4*>(&h2[0][0])[k * kPassThreads + tid] = hv[k];
    }
    __syncthreads();
    Plan2 P;
    P.p[0] = pa;
    P.p[1] = pb;
    P.shared = shared;
    const uint32_t none[2] = {0u, 0u};
    for (int t = 0; t < 2; ++t) {
        P.len[t] = P.p[t].take_eq ? 0u : P.p[t].eq;
        P.need2[t] = P.len[t] ? P.p[t].need - P.p[t].above : 0u;
    }
    if (shared) {
        block_thresholds2<kPassThreads>(h2[0], P.need2, none, s_wsum, s_thr, P.q);
    } else {
        Thr qa[2], qb[2];
        const uint32_t na_only[2] = {P.need2[0], 0u}, nb_only[2] = {P.need2[1], 0u};
        block_thresholds2<kPassThreads>(h2[0], na_only, none, s_wsum, s_thr, qa);
        block_thresholds2<kPassThreads>(h2[1], nb_only, none, s_wsum, s_thr, qb);
        P.q[0] = qa[0];
        P.q[1] = qb[0];
    }
    if (tid == 0) {
        plan_write1(cnt + kPlanWord0, pa, pb);
        plan_write2(cnt + kPlanWord0, P);
    }
}

// Digit 3 and exact ties of both targets among the digit-2 survivors, run by
// the CTA of pass 2 that finishes last (the survivors of smooth score
// distributions number a few dozen).  Exact ties at the last digit are ranked
// by claim order; when both targets cut inside the same group of equal keys,
// b takes the ranks below its need, which a takes too, so b stays a subset of
// a.  Finally the histograms and counters of the segment are cleared for the
// next selection.  h3: 2 x kRadixBins words of shared memory.
template <int NT>
__device__ void finish_level3(const SelWork& wk, int seg, const Plan2& P, int32_t* __restrict__ out_a,
                              float* __restrict__ vals_a, int64_t stride_a, int32_t* __restrict__ out_b,
                              int64_t stride_b, uint32_t* h3, uint32_t* s_wsum, Thr* s_thr, uint32_t* s_ctr) {
    const int tid = threadIdx.x;
    uint32_t* cnt = wk.cnt + (int64_t)seg * kSelCounters;
    uint32_t* h1 = wk.hist + (int64_t)seg * 3 * kRadixBins;
    for (int i = tid; i < 2 * kRadixBins; i += NT) h3[i] = 0;
    if (tid < 2) s_ctr[tid] = 0;
    bool lvl3[2];
    uint32_t need3[2], ns[2];
    for (int t = 0; t < 2; ++t) {
        lvl3[t] = P.len[t] && !P.eq2[t];
        need3[t] = lvl3[t] ? P.need2[t] - P.q[t].above : 0u;
        ns[t] = __ldcg(cnt + (t == 0 ? 4 : 5));           // survivors
    }
    __syncthreads();
    // with a shared list and one digit-2 threshold both targets have the same survivors
    const bool one_list = P.shared && lvl3[0] && lvl3[1] && P.q[0].c == P.q[1].c;
    const uint2* surv[2] = {reinterpret_cast<const uint2*>(wk.surv1) + seg * wk.cand_stride,
                            reinterpret_cast<const uint2*>(wk.surv2) + seg * wk.cand_stride};
    for (int t = 0; t < 2; ++t)
        if (lvl3[t])
            for (uint32_t i = tid; i < ns[t]; i += NT) atomicAdd(&h3[t * kRadixBins + digit(__ldcg(surv[t] + i).x, 3)], 1u);
    __syncthreads();
    Thr r3[2];
    {
        Thr ra[2], rb[2];
        const uint32_t none[2] = {0u, 0u};
        const uint32_t na_only[2] = {need3[0], 0u}, nb_only[2] = {need3[1], 0u};
        block_thresholds2<NT>(h3, na_only, none, s_wsum, s_thr, ra);
        block_thresholds2<NT>(h3 + kRadixBins, nb_only, none, s_wsum, s_thr, rb);
        r3[0] = ra[0];
        r3[1] = rb[0];
    }
    uint32_t ties[2];
    for (int t = 0; t < 2; ++t) ties[t] = lvl3[t] ? need3[t] - r3[t].above : 0u;
    const bool coupled = one_list && r3[0].c == r3[1].c;
    int32_t* out[2] = {out_a + (int64_t)seg * stride_a, out_b ? out_b + (int64_t)seg * stride_b : nullptr};
    float* va = vals_a ? vals_a + (int64_t)seg * stride_a : nullptr;
    for (int t = 0; t < 2; ++t) {
        if (!lvl3[t] || (one_list && t == 1)) continue;
        const uint32_t tmask = one_list ? 3u : (1u << t);
        for (uint32_t i0 = 0; i0 < ns[t]; i0 += NT) {
            const uint32_t i = i0 + tid;
            const bool in = i < ns[t];
            const uint2 kv = in ? __ldcg(surv[t] + i) : make_uint2(0u, 0u);
            const uint32_t d3 = digit(kv.x, 3);
            bool on[2], eqv[2];
            for (int u = 0; u < 2; ++u) {
                on[u] = in && ((tmask >> u) & 1u);
                eqv[u] = on[u] && d3 == r3[u].c;
            }
            const uint32_t rk_a = warp_claim(eqv[0], &s_ctr[0]);
            const uint32_t rk_b = coupled ? rk_a : warp_claim(eqv[1], &s_ctr[1]);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const uint32_t rk = u == 0 ? rk_a : rk_b;
                const bool tk = on[u] && (d3 > r3[u].c || (eqv[u] && rk < ties[u]));
                const uint32_t os = warp_claim(tk, cnt + (u == 0 ? 0 : 2));
                if (tk && (int64_t)os < (u == 0 ? stride_a : stride_b)) {
                    out[u][os] = (int32_t)kv.y;
                    if (u == 0 && va) va[os] = key_value(kv.x);
                }
            }
        }
    }
    // leave the workspace as csa2_workspace_init does: histograms and counters zero
    __syncthreads();
    for (int i = tid; i < 3 * kRadixBins; i += NT) h1[i] = 0;
    if (tid < kSelCounters) cnt[tid] = 0;
}

// Digit 2 of both targets over their candidate lists, many CTAs per segment:
// the lists' chunks of kPassChunk candidates (list a's, then list b's) are
// spread over the CTAs.  Digit 2 above a target's threshold is selected, the
// candidates equal to it survive into that target's survivor list.  Slots are
// claimed once per CTA and chunk, as in pass 1.  The last CTA to finish
// resolves digit 3 (finish_level3).
__global__ void __launch_bounds__(kPassThreads)
k_sel_pass2(SelWork wk, int n_a, int32_t* __restrict__ out_a, float* __restrict__ vals_a, int64_t stride_a,
            int n_b, int32_t* __restrict__ out_b, int64_t stride_b) {
    pdl_begin();
    __shared__ uint64_t s_wsum64[kPassThreads / 32];
    __shared__ uint32_t s_base[4];
    extern __shared__ uint2 stage_dyn[];                      // 2 x kPassChunk: the stages of a and of b
    uint2* stage_a = stage_dyn;
    uint2* stage_b = stage_dyn + kPassChunk;
    const int seg = blockIdx.y, tid = threadIdx.x;
    uint32_t* cnt = wk.cnt + (int64_t)seg * kSelCounters;
    __shared__ uint32_t s_words[kPlanWords];
    const Plan2 P = plan_read(cnt + kPlanWord0, s_words);
    const uint2* list[2] = {reinterpret_cast<const uint2*>(wk.cand1) + seg * wk.cand_stride,
                            reinterpret_cast<const uint2*>(wk.cand2) + seg * wk.cand_stride};
    uint2* surv[2] = {reinterpret_cast<uint2*>(wk.surv1) + seg * wk.cand_stride,
                      reinterpret_cast<uint2*>(wk.surv2) + seg * wk.cand_stride};
    int32_t* out[2] = {out_a + (int64_t)seg * stride_a, out_b ? out_b + (int64_t)seg * stride_b : nullptr};
    float* va = vals_a ? vals_a + (int64_t)seg * stride_a : nullptr;
    // chunks of list a serve b too when shared; list b has chunks of its own otherwise
    const uint32_t nch_a = (P.len[0] + kPassChunk - 1) / kPassChunk;
    const uint32_t nch_b = P.shared ? 0u : (P.len[1] + kPassChunk - 1) / kPassChunk;
    for (uint32_t vc = blockIdx.x; vc < nch_a + nch_b; vc += gridDim.x) {
        const int li = vc < nch_a ? 0 : 1;
        const uint32_t c0 = (li == 0 ? vc : vc - nch_a) * kPassChunk;
        const uint32_t n = li == 0 ? P.len[0] : P.len[1];
        const uint32_t tmask = li == 1 ? 2u : (P.shared ? 3u : 1u);
        const uint2* lst = li == 0 ? list[0] : list[1];
        uint2 kv[kPassPer];
        uint32_t cn[4] = {0u, 0u, 0u, 0u};   // a taken, a survivors, b taken, b survivors
#pragma unroll
        for (int k = 0; k < kPassPer; ++k) {   // every load issued before any is used
            const uint32_t i = c0 + k * kPassThreads + tid;
            kv[k] = i < n ? lst[i] : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int k = 0; k < kPassPer; ++k) {
            const uint32_t d2 = digit(kv[k].x, 2);
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const bool on = kv[k].x != 0u && P.len[t] && ((tmask >> t) & 1u);
                cn[2 * t] += on && (d2 > P.q[t].c || (d2 == P.q[t].c && P.eq2[t]));
                cn[2 * t + 1] += on && d2 == P.q[t].c && !P.eq2[t];
            }
        }
        uint64_t tot;
        const uint64_t pre = block_excl_scan4<kPassThreads>(
            (uint64_t)cn[0] | ((uint64_t)cn[1] << 16) | ((uint64_t)cn[2] << 32) | ((uint64_t)cn[3] << 48), s_wsum64,
            &tot);
        if (tid < 4) {   // a outputs, a survivors, b outputs, b survivors
            const int ctr = tid == 0 ? 0 : tid == 1 ? 4 : tid == 2 ? 2 : 5;
            const uint32_t v = field16(tot, tid);
            s_base[tid] = v ? atomicAdd(cnt + ctr, v) : 0u;
        }
        // outputs gathered in shared memory (front: taken, back: survivors),
        // then written out as contiguous runs
        uint32_t pos[4];
#pragma unroll
        for (int f = 0; f < 4; ++f) pos[f] = field16(pre, f);
#pragma unroll
        for (int k = 0; k < kPassPer; ++k) {
            const uint32_t d2 = digit(kv[k].x, 2);
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                uint2* stg = t == 0 ? stage_a : stage_b;
                const bool on = kv[k].x != 0u && P.len[t] && ((tmask >> t) & 1u);
                if (on && (d2 > P.q[t].c || (d2 == P.q[t].c && P.eq2[t]))) {
                    stg[pos[2 * t]++] = kv[k];
                } else if (on && d2 == P.q[t].c) {
                    stg[kPassChunk - 1 - pos[2 * t + 1]++] = kv[k];
                }
            }
        }
        __syncthreads();   // the stages are complete; the bases have been claimed
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const uint2* stg = t == 0 ? stage_a : stage_b;
            const uint32_t nt = field16(tot, 2 * t), ns = field16(tot, 2 * t + 1);
            const uint32_t cap = (uint32_t)(t == 0 ? n_a : n_b);
            for (uint32_t i = tid; i < nt && s_base[2 * t] + i < cap; i += kPassThreads) {
                const uint2 v = stg[i];
                out[t][s_base[2 * t] + i] = (int32_t)v.y;
                if (t == 0 && va) va[s_base[0] + i] = key_value(v.x);
            }
            for (uint32_t i = tid; i < ns; i += kPassThreads) surv[t][s_base[2 * t + 1] + i] = stg[kPassChunk - 1 - i];
        }
        __syncthreads();   // s_base and the stages are rewritten by the next chunk
    }
    // the CTA that reports last sees every survivor and finishes the selection
    __threadfence();
    __syncthreads();
    if (tid == 0) s_base[0] = atomicAdd(cnt + 7, 1u) == gridDim.x - 1 ? 1u : 0u;
    __syncthreads();
    if (!s_base[0]) return;
    __threadfence();
    __shared__ uint32_t s_wsum[kPassThreads / 32];
    __shared__ Thr s_thr[2];
    __shared__ uint32_t s_ctr[2];
    finish_level3<kPassThreads>(wk, seg, P, out_a, vals_a, stride_a, out_b, stride_b,
                                reinterpret_cast<uint32_t*>(stage_dyn), s_wsum, s_thr, s_ctr);
}

// ---------------------------------------------------------------- one CTA per segment
// Whole selection of one segment of at most 1024 * E elements by one CTA
// (lsel.cuh): the n_a best into out_a (scores into vals_a, nullable) and,
// with n_b > 0, the n_b best of those into out_b (a subset of out_a).
// Element i has value vals[seg * vals_stride + i] and id ids[seg *
// ids_stride + i] (ids == nullptr: id i, valid for i <= p); VEC: the value
// and id rows are 16-byte aligned, so four consecutive elements are one load.
constexpr int kLocalThreads = 1024;

template <int E, bool VEC>
__global__ void __launch_bounds__(kLocalThreads)
k_sel_local(SelSrc src, int n_a, int32_t* __restrict__ out_a, float* __restrict__ vals_a, int64_t stride_a, int n_b,
            int32_t* __restrict__ out_b, int64_t stride_b) {
    __shared__ lsel::Smem<kLocalThreads> sh;
    extern __shared__ int32_t s_ids[];               // [1024 * E] when the ids come from memory
    pdl_begin();
    const int seg = blockIdx.x;
    const int64_t nvalid = n_valid_positions(src, seg);
    const int64_t n = src.ids ? src.n : (src.n < nvalid ? src.n : nvalid);
    const float* vrow = src.vals + seg * src.vals_stride;
    const int32_t* irow = src.ids ? src.ids + seg * src.ids_stride : nullptr;
    uint32_t key[E];
    int32_t idv[E];
    // every load issued before any is used (indices clamped to the rows'
    // allocated length so that no load is conditional; elements at or beyond
    // n are masked afterwards)
    const int64_t row_len = irow && src.ids_stride < src.vals_stride ? src.ids_stride : src.vals_stride;
#pragma unroll
    for (int g = 0; g < (E + 3) / 4; ++g) {
        const int i0 = lsel::elem_index<kLocalThreads, E>(4 * g);
        if (VEC && E % 4 == 0) {
            const int ic = i0 + 3 < row_len ? i0 : 0;
            const uint4 v = *reinterpret_cast<const uint4*>(vrow + ic);
            key[4 * g] = v.x; key[4 * g + 1] = v.y; key[4 * g + 2] = v.z; key[4 * g + 3] = v.w;
            if (irow) {
                const int4 d = *reinterpret_cast<const int4*>(irow + ic);
                idv[4 * g] = d.x; idv[4 * g + 1] = d.y; idv[4 * g + 2] = d.z; idv[4 * g + 3] = d.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (4 * g + k >= E) break;
                const int i = lsel::elem_index<kLocalThreads, E>(4 * g + k);
                const int ic = i < row_len ? i : 0;
                key[4 * g + k] = __float_as_uint(vrow[ic]);
                if (irow) idv[4 * g + k] = irow[ic];
            }
        }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int i = lsel::elem_index<kLocalThreads, E>(e);
        int32_t id = irow ? idv[e] : i;
        if (i >= n) id = -1;
        key[e] = select_key(__uint_as_float(key[e]), id >= 0 && id < nvalid);
        if (irow) s_ids[e * kLocalThreads + threadIdx.x] = id;   // parked in shared memory until the output
    }
    auto id_of = [&](int e) -> int32_t {
        return irow ? s_ids[e * kLocalThreads + threadIdx.x] : lsel::elem_index<kLocalThreads, E>(e);
    };
    const uint32_t ta = lsel::select_mask<kLocalThreads, E>(key, (uint32_t)n_a, sh);
    lsel::write_selected<kLocalThreads, E>(ta, key, id_of, out_a + (int64_t)seg * stride_a,
                                           vals_a ? vals_a + (int64_t)seg * stride_a : nullptr, n_a, sh);
    if (n_b > 0) {
        // the second target chooses among the first one's picks only
#pragma unroll
        for (int e = 0; e < E; ++e) key[e] = ((ta >> e) & 1u) ? key[e] : 0u;
        const uint32_t tb = lsel::select_mask<kLocalThreads, E>(key, (uint32_t)n_b, sh);
        lsel::write_selected<kLocalThreads, E>(tb, key, id_of, out_b + (int64_t)seg * stride_b, nullptr, n_b, sh);
    }
}

template <int E>
cudaError_t launch_local_e(const SelSrc& src, int nseg, int n_a, int32_t* out_a, float* vals_a, int64_t stride_a,
                           int n_b, int32_t* out_b, int64_t stride_b, cudaStream_t st) {
    const bool vec = (reinterpret_cast<uintptr_t>(src.vals) & 15u) == 0 && src.vals_stride % 4 == 0 &&
                     (!src.ids || ((reinterpret_cast<uintptr_t>(src.ids) & 15u) == 0 && src.ids_stride % 4 == 0));
    const size_t smem = src.ids ? sizeof(int32_t) * kLocalThreads * E : 0;
    auto kern = vec ? k_sel_local<E, true> : k_sel_local<E, false>;
    if (smem > 48 * 1024 - sizeof(lsel::Smem<kLocalThreads>)) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(kern, dim3((unsigned)nseg), dim3(kLocalThreads), smem, st, src, n_a, out_a, vals_a, stride_a,
                      n_b, out_b, stride_b);
}

// ---------------------------------------------------------------- one grid per selection
// Both targets of a large segment in one launch, every key held in a register
// from its load to its decision: C CTAs per segment, each owning
// kGridThreads x E consecutive elements, meet at barriers (arrival counts in
// the segment's counters, bounded spins) behind which the segment's digit
// histograms are complete in global memory:
//   level 0  (only without the scorer's histogram) digit 1 of every element -> barrier
//   level 1  the digit-1 histogram -> both targets' (c1, above, eq); the
//            elements of digit c1 are histogrammed by digit 2          -> barrier A
//   level 2  the digit-2 histograms -> (c2, above); the elements of digit c2
//            are histogrammed by digit 3                               -> barrier B
//   level 3  the digit-3 histograms -> (c3, ties); exact ties at the last
//            digit are ranked by claim order, one rank shared by both targets
//            when they cut inside the same group of equal keys (so the top-k
//            stays inside the pool)
// then every CTA claims its outputs with one atomic per target, and the last
// CTA to finish clears the segment's histograms and counters.  All CTAs of a
// launch must be resident at once: the host launches it only when the whole
// grid fits on the GPU beside nothing else, and a CTA lets the next kernel
// launch only after barrier A, when every CTA of the grid has arrived.
constexpr int kGridThreads = 1024;

using gsel::seg_barrier;

__device__ __forceinline__ void load_hist(uint32_t* dst, const uint32_t* src, int n) {
    gsel::load_hist<kGridThreads>(dst, src, n);
}

// IDS: the elements are a list of positions (src.ids) with their values at
// the same index (src.gather == 0), as a pool update's candidates are.
template <int E, bool IDS>
__global__ void __launch_bounds__(kGridThreads, 1)
k_sel_grid(SelSrc src, SelWork wk, int n_a, int32_t* __restrict__ out_a, float* __restrict__ vals_a, int64_t stride_a,
           int n_b, int32_t* __restrict__ out_b, int64_t stride_b, int hist_ready, uint32_t wait_limit) {
    static_assert(E <= 16, "two decision bits per key in one 32-bit word");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ uint32_t s_wsum[kGridThreads / 32];
    __shared__ uint64_t s_wsum64[kGridThreads / 32];
    __shared__ Thr s_thr[2];
    __shared__ uint32_t s_misc[4];
    __shared__ __align__(16) uint32_t h[2][kRadixBins];    // this CTA's histograms
    __shared__ __align__(16) uint32_t hc[2][kRadixBins];   // a copy of the segment's
    const int seg = blockIdx.y, tid = threadIdx.x;
    const uint32_t C = gridDim.x;
    uint32_t* cnt = wk.cnt + (int64_t)seg * kSelCounters;
    uint32_t* h1g = wk.hist + (int64_t)seg * 3 * kRadixBins;
    uint32_t* h2g = h1g + kRadixBins;                      // [2][kRadixBins]: digit 2 of a's and b's candidates
    uint32_t* h3g = wk.hist3 + (int64_t)seg * 2 * kRadixBins;
    uint32_t* bar = cnt + 8;
    const uint32_t limit = wait_limit * 64u;              // a try sleeps 0.1-0.3 us: a fraction of a second by default
    const int64_t nvalid = n_valid_positions(src, seg);
    const int64_t base = (int64_t)blockIdx.x * kGridThreads * E;
    // every score load in flight before anything else (clamped, so that no load
    // is conditional); with the scorer's histogram the level-1 plan is worked
    // out while they land
    float raw[E];
    int32_t idv[IDS ? E : 1];
    const int64_t n_items = IDS ? src.n : nvalid;
#pragma unroll
    for (int k = 0; k < E; ++k) {
        const int64_t i = base + (int64_t)k * kGridThreads + tid;
        const int64_t ic = i < n_items ? i : 0;
        if (IDS) idv[k] = __ldcg(src.ids + seg * src.ids_stride + ic);
        raw[k] = __ldcg(src.vals + seg * src.vals_stride + ic);
    }
    for (int i = tid; i < 2 * kRadixBins; i += kGridThreads) (&h[0][0])[i] = 0u;
    Plan1 pa, pb;
    if (hist_ready) {
        load_hist(&hc[0][0], h1g, kRadixBins);
        plans_level1<kGridThreads>(&hc[0][0], (uint32_t)n_a, (uint32_t)n_b, s_wsum, s_thr, pa, pb);
    }
    uint32_t key[E];
#pragma unroll
    for (int k = 0; k < E; ++k) {   // a valid key is never 0
        const int64_t i = base + (int64_t)k * kGridThreads + tid;
        const bool v = IDS ? i < n_items && idv[k] >= 0 && idv[k] < nvalid : i < nvalid;
        key[k] = select_key(raw[k], v);
    }
    uint32_t nbar = 0;
    bool ok = true;
    // flush this CTA's histograms (the nonzero bins) into the segment's and clear them
    auto flush = [&](uint32_t* dst, int n) {
        __syncthreads();
        for (int i = tid; i < n; i += kGridThreads) {
            const uint32_t v = (&h[0][0])[i];
            if (v) {
                atomicAdd(dst + i, v);
                (&h[0][0])[i] = 0u;
            }
        }
    };
    if (!hist_ready) {
        __syncthreads();
#pragma unroll
        for (int k = 0; k < E; ++k)
            if (key[k]) atomicAdd(&h[0][digit(key[k], 1)], 1u);
        flush(h1g, kRadixBins);
        ok = seg_barrier(bar, ++nbar * C, limit, &s_misc[3]) && ok;
        load_hist(&hc[0][0], h1g, kRadixBins);
        plans_level1<kGridThreads>(&hc[0][0], (uint32_t)n_a, (uint32_t)n_b, s_wsum, s_thr, pa, pb);
    }

    // ---- level 1
    int32_t* oa = out_a + (int64_t)seg * stride_a;
    int32_t* ob = out_b ? out_b + (int64_t)seg * stride_b : nullptr;
    float* va = vals_a ? vals_a + (int64_t)seg * stride_a : nullptr;
    if (blockIdx.x == 0) {
        for (int i = (int)pa.need + tid; i < n_a; i += kGridThreads) oa[i] = -1;
        for (int i = (int)pb.need + tid; i < n_b; i += kGridThreads) ob[i] = -1;
    }
    const bool shared = pb.c == pa.c && !pa.take_eq;       // b's candidates are a's
    const uint32_t c1a = pa.take_eq ? 0xFFFFFFFFu : pa.c, c1b = shared || pb.take_eq ? 0xFFFFFFFFu : pb.c;
#pragma unroll
    for (int k = 0; k < E; ++k) {
        const uint32_t d1 = digit(key[k], 1), d2 = digit(key[k], 2);
        if (key[k] && d1 == c1a) atomicAdd(&h[0][d2], 1u);
        if (key[k] && d1 == c1b) atomicAdd(&h[1][d2], 1u);
    }
    flush(h2g, 2 * kRadixBins);
    ok = seg_barrier(bar, ++nbar * C, limit, &s_misc[3]) && ok;
    // every CTA of the grid is resident: the next kernel may launch
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // ---- level 2
    const Plan1 p1[2] = {pa, pb};
    uint32_t len[2], need2[2];
    for (int t = 0; t < 2; ++t) {
        len[t] = p1[t].take_eq ? 0u : p1[t].eq;
        need2[t] = len[t] ? p1[t].need - p1[t].above : 0u;
    }
    load_hist(&hc[0][0], h2g, 2 * kRadixBins);
    const uint32_t none[2] = {0u, 0u};
    Thr q[2];
    if (shared) {
        block_thresholds2<kGridThreads>(hc[0], need2, none, s_wsum, s_thr, q);
    } else {
        Thr qa[2], qb[2];
        const uint32_t na_only[2] = {need2[0], 0u}, nb_only[2] = {need2[1], 0u};
        block_thresholds2<kGridThreads>(hc[0], na_only, none, s_wsum, s_thr, qa);
        block_thresholds2<kGridThreads>(hc[1], nb_only, none, s_wsum, s_thr, qb);
        q[0] = qa[0];
        q[1] = qb[0];
    }
    bool eq2[2], lvl3[2];
    for (int t = 0; t < 2; ++t) {
        eq2[t] = q[t].eq == need2[t] - q[t].above;
        lvl3[t] = len[t] && !eq2[t];
    }
    // with one list and one digit-2 threshold both targets have the same survivors
    const bool one_list = shared && lvl3[0] && lvl3[1] && q[0].c == q[1].c;
    // the survivors of a target share their top 21 bits: (c1, c2)
    const uint32_t pre_a = lvl3[0] ? (pa.c << 11) | q[0].c : 0xFFFFFFFFu;
    const uint32_t pre_b = lvl3[1] && !one_list ? (pb.c << 11) | q[1].c : 0xFFFFFFFFu;
#pragma unroll
    for (int k = 0; k < E; ++k) {
        const uint32_t top = key[k] >> 10, d3 = digit(key[k], 3);
        if (key[k] && top == pre_a) atomicAdd(&h[0][d3], 1u);
        if (key[k] && top == pre_b) atomicAdd(&h[1][d3], 1u);
    }
    flush(h3g, 2 * kRadixBins);
    ok = seg_barrier(bar, ++nbar * C, limit, &s_misc[3]) && ok;

    // ---- level 3
    load_hist(&hc[0][0], h3g, 2 * kRadixBins);
    uint32_t need3[2];
    for (int t = 0; t < 2; ++t) need3[t] = lvl3[t] ? need2[t] - q[t].above : 0u;
    Thr r3[2];
    if (one_list) {
        block_thresholds2<kGridThreads>(hc[0], need3, none, s_wsum, s_thr, r3);
    } else {
        Thr ra[2], rb[2];
        const uint32_t na_only[2] = {need3[0], 0u}, nb_only[2] = {need3[1], 0u};
        block_thresholds2<kGridThreads>(hc[0], na_only, none, s_wsum, s_thr, ra);
        block_thresholds2<kGridThreads>(hc[1], nb_only, none, s_wsum, s_thr, rb);
        r3[0] = ra[0];
        r3[1] = rb[0];
    }
    uint32_t ties[2];
    for (int t = 0; t < 2; ++t) ties[t] = lvl3[t] ? need3[t] - r3[t].above : 0u;
    const bool coupled = one_list && r3[0].c == r3[1].c;   // both cut inside one group of equal keys

    // ---- decisions, claims and writes.  Each target's cut as two keys: every
    // key >= lo is taken; a key equal to tie_key (a cut at the last digit) is
    // taken by the first `ties` claimants
    uint32_t lo[2], tie_key[2];
    for (int t = 0; t < 2; ++t) {
        const Plan1& p = p1[t];
        tie_key[t] = 0u;                                   // never a valid key
        if (p.need == 0) {
            lo[t] = 0xFFFFFFFFu;                           // above every valid key
        } else if (p.take_eq) {
            lo[t] = p.c << 21;
        } else if (eq2[t]) {
            lo[t] = (p.c << 21) | (q[t].c << 10);
        } else {
            tie_key[t] = (p.c << 21) | (q[t].c << 10) | r3[t].c;
            lo[t] = tie_key[t] + 1u;
        }
    }
    uint32_t take = 0;                                     // bit 2k: target a takes key k, bit 2k + 1: b
    uint32_t na = 0, nb = 0;
#pragma unroll
    for (int k = 0; k < E; ++k) {
        const bool v = key[k] != 0u;
        bool sel[2], tie[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            sel[t] = v && key[k] >= lo[t];
            tie[t] = v && key[k] == tie_key[t];
        }
        const uint32_t rk_a = warp_claim(tie[0], cnt + 4);
        const uint32_t rk_b = coupled ? rk_a : warp_claim(tie[1], cnt + 5);
        sel[0] = sel[0] || (tie[0] && rk_a < ties[0]);
        sel[1] = sel[1] || (tie[1] && rk_b < ties[1]);
        take |= (sel[0] ? 1u : 0u) << (2 * k);
        take |= (sel[1] ? 2u : 0u) << (2 * k);
        na += sel[0];
        nb += sel[1];
    }
    uint64_t tot;
    const uint64_t pre = block_excl_scan4<kGridThreads>((uint64_t)na | ((uint64_t)nb << 16), s_wsum64, &tot);
    if (tid < 2) {
        const uint32_t v = field16(tot, tid);
        s_misc[tid] = v ? atomicAdd(cnt + 2 * tid, v) : 0u;   // a outputs, b outputs
    }
    __syncthreads();
    uint32_t oa_pos = s_misc[0] + field16(pre, 0), ob_pos = s_misc[1] + field16(pre, 1);
#pragma unroll
    for (int k = 0; k < E; ++k) {
        const int32_t id = IDS ? idv[k] : (int32_t)(base + (int64_t)k * kGridThreads + tid);
        if ((take >> (2 * k)) & 1u) {
            if (oa_pos < (uint32_t)n_a) {
                oa[oa_pos] = id;
                if (va) va[oa_pos] = key_value(key[k]);
            }
            ++oa_pos;
        }
        if ((take >> (2 * k + 1)) & 1u) {
            if (ob && ob_pos < (uint32_t)n_b) ob[ob_pos] = id;
            ++ob_pos;
        }
    }
    if (!ok && tid == 0) flag(wk.status, kStatusTimeout);

    // ---- the last CTA leaves the segment's histograms and counters zero
    __threadfence();
    __syncthreads();
    if (tid == 0) s_misc[2] = atomicAdd(bar, 1u) == (nbar + 1) * C - 1 ? 1u : 0u;
    __syncthreads();
    if (!s_misc[2]) return;
    __threadfence();
    for (int i = tid; i < 3 * kRadixBins; i += kGridThreads) h1g[i] = 0u;
    for (int i = tid; i < 2 * kRadixBins; i += kGridThreads) h3g[i] = 0u;
    if (tid < kSelCounters) cnt[tid] = 0u;
}

}  // namespace

cudaError_t launch_select_local(const SelSrc& src, int nseg, int n_a, int32_t* out_a, float* vals_a, int64_t stride_a,
                                int n_b, int32_t* out_b, int64_t stride_b, cudaStream_t st) {
    if (src.n <= 1024) return launch_local_e<1>(src, nseg, n_a, out_a, vals_a, stride_a, n_b, out_b, stride_b, st);
    if (src.n <= 4096) return launch_local_e<4>(src, nseg, n_a, out_a, vals_a, stride_a, n_b, out_b, stride_b, st);
    return launch_local_e<16>(src, nseg, n_a, out_a, vals_a, stride_a, n_b, out_b, stride_b, st);
}

cudaError_t launch_select(const SelSrc& src, const SelWork& wk, int nseg, int n_out, int32_t* out,
                          int64_t out_stride, cudaStream_t st, bool hist_ready, float* out_vals) {
    if (src.n <= kSmallMax)
        return launch_select_local(src, nseg, n_out, out, out_vals, out_stride, 0, nullptr, 0, st);
    return launch_select_dual(src, wk, nseg, n_out, out, out_vals, out_stride, 0, nullptr, 0, st, hist_ready);
}

namespace {

// CTAs of k_sel_grid<E> that fit on the device at once (0: unknown).
template <int E, bool IDS>
int64_t grid_capacity() {
    static int64_t cap = -1;
    if (cap < 0) {
        int dev = 0, sms = 0, per = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, k_sel_grid<E, IDS>, kGridThreads, 0) != cudaSuccess)
            return 0;
        cap = (int64_t)sms * per;
    }
    return cap;
}

template <int E, bool IDS>
bool try_grid(const SelSrc& src, const SelWork& wk, int nseg, int n_a, int32_t* out_a, float* vals_a, int64_t stride_a,
              int n_b, int32_t* out_b, int64_t stride_b, cudaStream_t st, bool hist_ready, cudaError_t* e) {
    const int64_t per_cta = (int64_t)kGridThreads * E;
    const int64_t C = (src.n + per_cta - 1) / per_cta;
    if (C < 1 || C * nseg > grid_capacity<E, IDS>()) return false;
    *e = launch_pdl(k_sel_grid<E, IDS>, dim3((unsigned)C, (unsigned)nseg), dim3(kGridThreads), 0, st, src, wk, n_a,
                    out_a, vals_a, stride_a, n_b, out_b, stride_b, hist_ready ? 1 : 0, wait_limit());
    return true;
}

}  // namespace

cudaError_t launch_select_dual(const SelSrc& src, const SelWork& wk, int nseg, int n_a, int32_t* out_a, float* vals_a,
                               int64_t stride_a, int n_b, int32_t* out_b, int64_t stride_b, cudaStream_t st,
                               bool hist_ready) {
    // the histograms and counters are zero on entry (workspace initialisation,
    // then every selection's last CTA clears what it used)
    cudaError_t e = cudaSuccess;
    if (src.ids == nullptr && wk.hist3 != nullptr) {
        // one grid, the keys in registers, when every CTA fits on the GPU at once
        // the fewest keys per thread (the most CTAs) with which the grid fits
        if (try_grid<1, false>(src, wk, nseg, n_a, out_a, vals_a, stride_a, n_b, out_b, stride_b, st, hist_ready, &e) ||
            try_grid<2, false>(src, wk, nseg, n_a, out_a, vals_a, stride_a, n_b, out_b, stride_b, st, hist_ready, &e) ||
            try_grid<4, false>(src, wk, nseg, n_a, out_a, vals_a, stride_a, n_b, out_b, stride_b, st, hist_ready, &e) ||
            try_grid<7, false>(src, wk, nseg, n_a, out_a, vals_a, stride_a, n_b, out_b, stride_b, st, hist_ready, &e) ||
            try_grid<16, false>(src, wk, nseg, n_a, out_a, vals_a, stride_a, n_b, out_b, stride_b, st, hist_ready, &e))
            return e;
    }
    if (src.ids != nullptr && src.gather == 0 && wk.hist3 != nullptr) {
        // a list of positions with their values at the same index
        if (try_grid<1, true>(src, wk, nseg, n_a, out_a, vals_a, stride_a, n_b, out_b, stride_b, st, hist_ready, &e) ||
            try_grid<2, true>(src, wk, nseg, n_a, out_a, vals_a, stride_a, n_b, out_b, stride_b, st, hist_ready, &e) ||
            try_grid<4, true>(src, wk, nseg, n_a, out_a, vals_a, stride_a, n_b, out_b, stride_b, st, hist_ready, &e) ||
            try_grid<7, true>(src, wk, nseg, n_a, out_a, vals_a, stride_a, n_b, out_b, stride_b, st, hist_ready, &e))
            return e;
    }
    // otherwise two streaming passes; without a histogram from the scoring
    // kernel, level 1 is built here
    const unsigned chunks = (unsigned)((src.n + kPassChunk - 1) / kPassChunk);
    dim3 grid(chunks ? chunks : 1, (unsigned)nseg);
    if (!hist_ready) {
        e = launch_pdl(k_sel_hist, dim3(grid), dim3(kPassThreads), 0, st, src, wk);
        if (e != cudaSuccess) return e;
    }
    constexpr size_t kStageSmem = 2 * kPassChunk * sizeof(uint2);
    e = cudaFuncSetAttribute(k_sel_pass1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStageSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k_sel_pass2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStageSmem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(k_sel_pass1, dim3(grid), dim3(kPassThreads), kStageSmem, st, src, wk, n_a, out_a, vals_a, stride_a,
                   n_b, out_b, stride_b);
    if (e != cudaSuccess) return e;
    // candidates: at most the segment size; spread over up to 148 CTAs
    const unsigned g2 = chunks < 148 ? (chunks ? chunks : 1) : 148;
    return launch_pdl(k_sel_pass2, dim3(g2, (unsigned)nseg), dim3(kPassThreads), kStageSmem, st, wk, n_a, out_a,
                      vals_a, stride_a, n_b, out_b, stride_b);
}

}  // namespace csa2

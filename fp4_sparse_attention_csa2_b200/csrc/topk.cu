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
//   large segments (Full layer, up to 1M scores): the level-1 histogram comes
//     from the scoring kernel; a streaming pass (many CTAs per segment) selects
//     above each target's level-1 threshold and compacts the elements equal to
//     it into candidate lists; a cluster of CTAs per segment then resolves
//     digits 2 and 3 on those lists.  The pool and the layer's top-k are two
//     targets of the same pass.
//   small segments (<= 16,384: the top-k of a pool): a cluster of 8 CTAs per
//     segment keeps every key in registers and resolves all three digits,
//     summing the CTAs' histograms through distributed shared memory.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace csa2 {

namespace cg = cooperative_groups;

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
        e.valid = i < nvalid;
        e.id = (int32_t)i;
        e.key = e.valid ? ordered_key(s.vals[seg * s.vals_stride + i]) : 0u;
    } else {
        // entries outside [0, p] are padding or were flagged when scored
        e.id = s.ids[seg * s.ids_stride + i];
        e.valid = e.id >= 0 && e.id < nvalid;
        e.key = e.valid ? ordered_key(s.vals[seg * s.vals_stride + (s.gather ? (int64_t)e.id : i)]) : 0u;
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

// Cluster geometry shared by the pool-sized selection and the resolve kernel.
constexpr int kClCtas = 8;
constexpr int kClThreads = 512;
constexpr int kClPer = kSmallMax / (kClCtas * kClThreads);   // elements per thread
constexpr int kClBinsPer = kRadixBins / kClThreads;          // histogram bins per thread

struct ClPlan {
    uint32_t c, above, eq, total;
};

// Threshold of the cluster-wide histogram `h` (this CTA's copy; the others
// are read through distributed shared memory).  need == 0 asks only for the
// total (used at level 1, where `need` follows from it).
__device__ __forceinline__ ClPlan cluster_threshold(cg::cluster_group& cl, uint32_t* h, uint32_t need_in,
                                                    uint32_t n_out, uint32_t* s_wsum, ClPlan* s_plan) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // thread t owns bins hi - 3 .. hi, hi = 2047 - 4 t: descending bins follow ascending t
    const int lo = kRadixBins - kClBinsPer * (tid + 1);
    uint4 g = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int r = 0; r < kClCtas; ++r) {
        const uint4 v = *reinterpret_cast<const uint4*>(cl.map_shared_rank(h + lo, r));
        g.x += v.x; g.y += v.y; g.z += v.z; g.w += v.w;
    }
    const uint32_t sum = g.x + g.y + g.z + g.w;
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    uint32_t before = 0, total = 0;
    for (int w = 0; w < kClThreads / 32; ++w) {
        const uint32_t v = s_wsum[w];
        before += w < warp ? v : 0u;
        total += v;
    }
    const uint32_t need = need_in ? need_in : (total < n_out ? total : n_out);
    const uint32_t excl = before + incl - sum;
    if (need > 0 && excl < need && need <= excl + sum) {
        const uint32_t b[4] = {g.w, g.z, g.y, g.x};   // bins lo + 3 .. lo, descending
        uint32_t above = excl;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (need <= above + b[k]) {
                s_plan->c = (uint32_t)(lo + 3 - k);
                s_plan->above = above;
                s_plan->eq = b[k];
                break;
            }
            above += b[k];
        }
    }
    if (tid == 0) s_plan->total = total;
    __syncthreads();
    const ClPlan pl = *s_plan;
    __syncthreads();   // s_wsum and s_plan are rewritten by the next call
    return pl;
}

// Two selections of the same scores at once: target a (the pool, n_a) and
// target b (the top-k, n_b <= n_a; n_b == 0: none), with b a subset of a.
// Level-1 plan of one target from the level-1 histogram.
struct Plan1 {
    uint32_t need, c, above, eq;   // eq: elements with digit c
    bool take_eq;                  // every digit-c element is needed (or nothing is)
};

template <int NT>
__device__ __forceinline__ Plan1 plan_level1(const uint32_t* h1, uint32_t n_out, uint32_t* s_wsum, Thr* s_thr) {
    Plan1 p = {0u, 0xFFFFFFFFu, 0u, 0u, true};
    if (n_out == 0) return p;
    const Thr t = block_threshold<NT>(h1, 0u, n_out, s_wsum, s_thr);
    p.need = t.need;
    if (t.need == 0) return p;
    p.c = t.c;
    p.above = t.above;
    p.eq = t.eq;
    p.take_eq = t.eq == t.need - t.above;
    return p;
}

// Level 1 over every element, both targets: digits above a target's c1 are
// selected, digit-c1 elements are compacted into that target's candidate list
// (one list when both thresholds fall on the same digit).  Each CTA claims its
// output and candidate slots with one atomic per counter (block-wide scans of
// per-thread counts), so the shared counters see one atomic per CTA and chunk.
constexpr int kPassPer = kPassChunk / kPassThreads;   // elements per thread and chunk

__global__ void __launch_bounds__(kPassThreads)
k_sel_pass1(SelSrc src, SelWork wk, int n_a, int32_t* __restrict__ out_a, float* __restrict__ vals_a,
            int64_t stride_a, int n_b, int32_t* __restrict__ out_b, int64_t stride_b) {
    pdl_begin();
    __shared__ uint32_t s_wsum[kPassThreads / 32];
    __shared__ Thr s_thr;
    __shared__ uint32_t s_base[4];
    const int seg = blockIdx.y, tid = threadIdx.x;
    uint32_t* cnt = wk.cnt + (int64_t)seg * kSelCounters;
    const uint32_t* h1 = wk.hist + (int64_t)seg * 3 * kRadixBins;
    const Plan1 pa = plan_level1<kPassThreads>(h1, (uint32_t)n_a, s_wsum, &s_thr);
    const Plan1 pb = plan_level1<kPassThreads>(h1, (uint32_t)n_b, s_wsum, &s_thr);
    int32_t* oa = out_a + (int64_t)seg * stride_a;
    int32_t* ob = out_b ? out_b + (int64_t)seg * stride_b : nullptr;
    float* va = vals_a ? vals_a + (int64_t)seg * stride_a : nullptr;
    if (blockIdx.x == 0) {
        for (int i = (int)pa.need + tid; i < n_a; i += kPassThreads) oa[i] = -1;
        for (int i = (int)pb.need + tid; i < n_b; i += kPassThreads) ob[i] = -1;
    }
    if (pa.need == 0) return;
    // b's candidates are a's when both thresholds fall on one digit that a does
    // not take whole
    const bool shared = pb.c == pa.c && !pa.take_eq;
    const int64_t nvalid = n_valid_positions(src, seg);
    const int64_t n_items = src.ids ? src.n : nvalid;
    uint2* cand_a = reinterpret_cast<uint2*>(wk.cand1) + seg * wk.cand_stride;
    uint2* cand_b = reinterpret_cast<uint2*>(wk.cand2) + seg * wk.cand_stride;
    for (int64_t base = (int64_t)blockIdx.x * kPassChunk; base < n_items; base += (int64_t)gridDim.x * kPassChunk) {
        uint32_t keys[kPassPer];
        int32_t ids[kPassPer];
        uint32_t na = 0, nca = 0, nb = 0, ncb = 0;
#pragma unroll
        for (int k = 0; k < kPassPer; ++k) {
            const int64_t i = base + k * kPassThreads + tid;
            Elem e = {false, -1, 0u};
            if (i < n_items) e = load_elem(src, seg, i, nvalid);
            keys[k] = e.valid ? e.key : 0u;   // a valid key is never 0
            ids[k] = e.id;
            const uint32_t d = digit(keys[k], 1);
            na += e.valid && (d > pa.c || (d == pa.c && pa.take_eq));
            nca += e.valid && d == pa.c && !pa.take_eq;
            nb += e.valid && (d > pb.c || (d == pb.c && pb.take_eq));
            ncb += e.valid && !shared && d == pb.c && !pb.take_eq;
        }
        // per-thread counts <= 16 and per-block sums <= 4096: two fit one word
        uint32_t tot_a, tot_b;
        const uint32_t pre_a = block_excl_scan<kPassThreads>((na << 16) | nca, s_wsum, &tot_a);
        const uint32_t pre_b = block_excl_scan<kPassThreads>((nb << 16) | ncb, s_wsum, &tot_b);
        if (tid == 0) {
            s_base[0] = (tot_a >> 16) ? atomicAdd(cnt + 0, tot_a >> 16) : 0u;
            s_base[1] = (tot_a & 0xFFFFu) ? atomicAdd(cnt + 1, tot_a & 0xFFFFu) : 0u;
            s_base[2] = (tot_b >> 16) ? atomicAdd(cnt + 2, tot_b >> 16) : 0u;
            s_base[3] = (tot_b & 0xFFFFu) ? atomicAdd(cnt + 3, tot_b & 0xFFFFu) : 0u;
        }
        __syncthreads();
        uint32_t os_a = s_base[0] + (pre_a >> 16), cs_a = s_base[1] + (pre_a & 0xFFFFu);
        uint32_t os_b = s_base[2] + (pre_b >> 16), cs_b = s_base[3] + (pre_b & 0xFFFFu);
        __syncthreads();   // s_base is rewritten by the next chunk
#pragma unroll
        for (int k = 0; k < kPassPer; ++k) {
            const uint32_t key = keys[k];
            if (!key) continue;
            const uint32_t d = digit(key, 1);
            if (d > pa.c || (d == pa.c && pa.take_eq)) {
                oa[os_a] = ids[k];
                if (va) va[os_a] = key_value(key);
                ++os_a;
            } else if (d == pa.c) {
                cand_a[cs_a++] = make_uint2(key, (uint32_t)ids[k]);
            }
            if (d > pb.c || (d == pb.c && pb.take_eq)) {
                ob[os_b++] = ids[k];
            } else if (!shared && d == pb.c) {
                cand_b[cs_b++] = make_uint2(key, (uint32_t)ids[k]);
            }
        }
    }
}

// Digits 2 and 3 of both targets on their candidate lists, one cluster of
// kClCtas CTAs per segment.  The lists are walked in chunks of kClChunk
// candidates (chunk n belongs to CTA n % kClCtas); the CTAs' shared-memory
// histograms are summed through distributed shared memory.  Output slots and
// tie ranks are claimed once per CTA and chunk (block-wide scans of
// per-thread counts) on counters in CTA 0's shared memory, after the slots
// pass 1 filled.  Exact ties at the last digit are ranked by claim order;
// when both targets cut inside the same group of equal keys, b takes the
// ranks below its need, which a takes too, so b stays a subset of a.
// Finally the histograms and counters of the segment are cleared for the
// next selection.
constexpr int kClPerItem = 4;                          // candidates per thread and chunk
constexpr int kClChunk = kClThreads * kClPerItem;

struct Resolve {
    // per target: digit-2 threshold and whether every digit-c2 element is
    // taken; digit-3 threshold, and the tie ranks that are taken
    uint32_t c2[2], c3[2], ties[2];
    bool eq2[2], lvl3[2];
    bool coupled;                       // b's ties are ranked with a's
    uint32_t base[2];                   // slots already filled by pass 1
    int32_t* out[2];
    float* vals_a;
};

// One pass over `list` (len candidates) for the targets in mask (bit t:
// target t).  level 2: take digit 2 above c2 (or equal, with eq2) and
// histogram digit 3 of the rest equal to c2 into h3[t]; level 3: among
// digit-2 == c2, take digit 3 above c3, and ties by rank.
template <int LEVEL>
__device__ __forceinline__ void resolve_pass(const Resolve& R, uint32_t mask, const uint2* list, uint32_t len,
                                             uint32_t rank, uint32_t* ctr, uint32_t (*h3)[kRadixBins],
                                             uint32_t* s_wsum, uint32_t* s_base) {
    const int tid = threadIdx.x;
    const uint32_t nch = (len + kClChunk - 1) / kClChunk;
    for (uint32_t ch = rank; ch < nch; ch += kClCtas) {        // the same trip count in every thread of a CTA
        uint2 kv[kClPerItem];
        bool in2[2][kClPerItem], eqv[2][kClPerItem];
        uint32_t ne[2] = {0u, 0u};
#pragma unroll
        for (int k = 0; k < kClPerItem; ++k) {
            const uint32_t i = ch * kClChunk + k * kClThreads + tid;
            const bool in = i < len;
            kv[k] = in ? list[i] : make_uint2(0u, 0u);
            const uint32_t d2 = digit(kv[k].x, 2), d3 = digit(kv[k].x, 3);
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const bool on = in && ((mask >> t) & 1u);
                in2[t][k] = on && d2 == R.c2[t];
                eqv[t][k] = LEVEL == 3 && in2[t][k] && d3 == R.c3[t];
                if (LEVEL == 2 && in2[t][k] && !R.eq2[t]) atomicAdd(&h3[t][d3], 1u);
                ne[t] += eqv[t][k] && !(t == 1 && R.coupled);
            }
        }
        uint32_t rk_next[2] = {0u, 0u};
        if (LEVEL == 3) {
            uint32_t tot;
            const uint32_t pre = block_excl_scan<kClThreads>((ne[0] << 16) | ne[1], s_wsum, &tot);
            if (tid == 0) {
                s_base[2] = (tot >> 16) ? atomicAdd(ctr + 2, tot >> 16) : 0u;
                s_base[3] = (tot & 0xFFFFu) ? atomicAdd(ctr + 3, tot & 0xFFFFu) : 0u;
            }
            __syncthreads();
            rk_next[0] = s_base[2] + (pre >> 16);
            rk_next[1] = s_base[3] + (pre & 0xFFFFu);
            __syncthreads();
        }
        uint32_t take[2] = {0u, 0u}, nt[2] = {0u, 0u};
#pragma unroll
        for (int k = 0; k < kClPerItem; ++k) {
            const uint32_t d2 = digit(kv[k].x, 2), d3 = digit(kv[k].x, 3);
            const uint32_t rk_a = eqv[0][k] ? rk_next[0]++ : 0xFFFFFFFFu;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const bool on = ((mask >> t) & 1u) && kv[k].x != 0u;
                bool tk;
                if (LEVEL == 2) {
                    tk = on && (d2 > R.c2[t] || (d2 == R.c2[t] && R.eq2[t]));
                } else {
                    const uint32_t rk = t == 0 ? rk_a : (R.coupled ? rk_a : (eqv[1][k] ? rk_next[1]++ : 0xFFFFFFFFu));
                    tk = in2[t][k] && (d3 > R.c3[t] || (eqv[t][k] && rk < R.ties[t]));
                }
                take[t] |= (uint32_t)tk << k;
                nt[t] += tk;
            }
        }
        uint32_t tot;
        const uint32_t pre = block_excl_scan<kClThreads>((nt[0] << 16) | nt[1], s_wsum, &tot);
        if (tid == 0) {
            s_base[0] = (tot >> 16) ? atomicAdd(ctr + 0, tot >> 16) : 0u;
            s_base[1] = (tot & 0xFFFFu) ? atomicAdd(ctr + 1, tot & 0xFFFFu) : 0u;
        }
        __syncthreads();
        uint32_t os[2] = {R.base[0] + s_base[0] + (pre >> 16), R.base[1] + s_base[1] + (pre & 0xFFFFu)};
        __syncthreads();   // s_base is rewritten by the next chunk
#pragma unroll
        for (int k = 0; k < kClPerItem; ++k) {
            if ((take[0] >> k) & 1u) {
                R.out[0][os[0]] = (int32_t)kv[k].y;
                if (R.vals_a) R.vals_a[os[0]] = key_value(kv[k].x);
                ++os[0];
            }
            if ((take[1] >> k) & 1u) R.out[1][os[1]++] = (int32_t)kv[k].y;
        }
    }
}

__global__ void __launch_bounds__(kClThreads)
k_sel_resolve(SelWork wk, int n_a, int32_t* __restrict__ out_a, float* __restrict__ vals_a, int64_t stride_a,
              int n_b, int32_t* __restrict__ out_b, int64_t stride_b) {
    cg::cluster_group cl = cg::this_cluster();
    __shared__ __align__(16) uint32_t hist[4][kRadixBins];   // digit 2 of a, of b; digit 3 of a, of b
    __shared__ uint32_t s_wsum[kClThreads / 32];
    __shared__ Thr s_thr;
    __shared__ ClPlan s_cl;
    __shared__ uint32_t s_ctr[4];     // CTA 0's: a slots, b slots, a tie ranks, b tie ranks
    __shared__ uint32_t s_base[4];
    const uint32_t rank = cl.block_rank();
    const int seg = blockIdx.y, tid = threadIdx.x;
    for (int i = tid; i < 4 * kRadixBins; i += kClThreads) (&hist[0][0])[i] = 0;
    if (tid < 4) s_ctr[tid] = 0;
    pdl_begin();
    uint32_t* cnt = wk.cnt + (int64_t)seg * kSelCounters;
    uint32_t* h1 = wk.hist + (int64_t)seg * 3 * kRadixBins;
    const Plan1 pa = plan_level1<kClThreads>(h1, (uint32_t)n_a, s_wsum, &s_thr);
    const Plan1 pb = plan_level1<kClThreads>(h1, (uint32_t)n_b, s_wsum, &s_thr);
    const bool shared = pb.c == pa.c && !pa.take_eq;   // as in k_sel_pass1
    const uint2* list_a = reinterpret_cast<const uint2*>(wk.cand1) + seg * wk.cand_stride;
    const uint2* list_b = shared ? list_a : reinterpret_cast<const uint2*>(wk.cand2) + seg * wk.cand_stride;
    const uint32_t len_a = pa.take_eq ? 0u : pa.eq, len_b = pb.take_eq ? 0u : pb.eq;
    uint32_t* ctr = cl.map_shared_rank(s_ctr, 0);
    Resolve R;
    R.base[0] = cnt[0];
    R.base[1] = cnt[2];
    R.out[0] = out_a + (int64_t)seg * stride_a;
    R.out[1] = out_b ? out_b + (int64_t)seg * stride_b : nullptr;
    R.vals_a = vals_a ? vals_a + (int64_t)seg * stride_a : nullptr;

    // digit 2 histograms (one for both targets when the list is shared)
    for (uint32_t i = rank * kClThreads + tid; i < len_a; i += kClCtas * kClThreads)
        atomicAdd(&hist[0][digit(list_a[i].x, 2)], 1u);
    if (!shared)
        for (uint32_t i = rank * kClThreads + tid; i < len_b; i += kClCtas * kClThreads)
            atomicAdd(&hist[1][digit(list_b[i].x, 2)], 1u);
    cl.sync();   // histograms complete everywhere; CTA 0's counters are zero
    const uint32_t need2[2] = {len_a ? pa.need - pa.above : 0u, len_b ? pb.need - pb.above : 0u};
    ClPlan q[2] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
    if (len_a) q[0] = cluster_threshold(cl, hist[0], need2[0], 0u, s_wsum, &s_cl);
    if (len_b) q[1] = cluster_threshold(cl, hist[shared ? 0 : 1], need2[1], 0u, s_wsum, &s_cl);
    for (int t = 0; t < 2; ++t) {
        R.c2[t] = q[t].c;
        R.eq2[t] = q[t].eq == need2[t] - q[t].above;
    }
    const uint32_t act_a = len_a ? 1u : 0u, act_b = len_b ? 2u : 0u;
    if (shared) {
        resolve_pass<2>(R, act_a | act_b, list_a, len_a, rank, ctr, &hist[2], s_wsum, s_base);
    } else {
        resolve_pass<2>(R, act_a, list_a, len_a, rank, ctr, &hist[2], s_wsum, s_base);
        resolve_pass<2>(R, act_b, list_b, len_b, rank, ctr, &hist[2], s_wsum, s_base);
    }
    cl.sync();   // digit-3 histograms complete everywhere
    for (int t = 0; t < 2; ++t) R.lvl3[t] = (t == 0 ? len_a : len_b) && !R.eq2[t];
    const uint32_t need3[2] = {R.lvl3[0] ? need2[0] - q[0].above : 0u, R.lvl3[1] ? need2[1] - q[1].above : 0u};
    ClPlan r3[2] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
    if (R.lvl3[0]) r3[0] = cluster_threshold(cl, hist[2], need3[0], 0u, s_wsum, &s_cl);
    if (R.lvl3[1]) r3[1] = cluster_threshold(cl, hist[3], need3[1], 0u, s_wsum, &s_cl);
    for (int t = 0; t < 2; ++t) {
        R.c3[t] = r3[t].c;
        R.ties[t] = R.lvl3[t] ? need3[t] - r3[t].above : 0u;
    }
    R.coupled = shared && R.lvl3[0] && R.lvl3[1] && R.c2[0] == R.c2[1] && R.c3[0] == R.c3[1];
    const uint32_t l3_a = R.lvl3[0] ? 1u : 0u, l3_b = R.lvl3[1] ? 2u : 0u;
    if (shared) {
        resolve_pass<3>(R, l3_a | l3_b, list_a, len_a, rank, ctr, &hist[2], s_wsum, s_base);
    } else {
        resolve_pass<3>(R, l3_a, list_a, len_a, rank, ctr, &hist[2], s_wsum, s_base);
        resolve_pass<3>(R, l3_b, list_b, len_b, rank, ctr, &hist[2], s_wsum, s_base);
    }
    // leave the workspace as csa2_workspace_init does: histograms and counters zero
    cl.sync();
    if (rank == 0) {
        for (int i = tid; i < 3 * kRadixBins; i += kClThreads) h1[i] = 0;
        if (tid < kSelCounters) cnt[tid] = 0;
    }
}

// ---------------------------------------------------------------- small segments
// Whole selection of one segment of at most kSmallMax elements by a cluster of
// kClCtas CTAs.  Element i belongs to CTA (i / kClThreads) % kClCtas, which
// keeps its key and id in registers.  Each level: every CTA histograms its own
// elements of the current prefix in shared memory, one cluster barrier, then
// every CTA sums the kClCtas histograms through distributed shared memory and
// finds the same threshold digit; the following pass selects digits above it
// and histograms the next digit of the elements equal to it.  Output slots and
// exact-tie ranks are claimed on counters in CTA 0.
__global__ void __launch_bounds__(kClThreads)
k_sel_small(SelSrc src, int n_out, int32_t* __restrict__ out, float* __restrict__ out_vals, int64_t out_stride) {
    cg::cluster_group cl = cg::this_cluster();
    __shared__ __align__(16) uint32_t hist[3][kRadixBins];
    __shared__ uint32_t s_wsum[kClThreads / 32];
    __shared__ ClPlan s_plan;
    __shared__ uint32_t s_cnt[2];               // CTA 0's: output slots, exact-tie ranks
    const uint32_t rank = cl.block_rank();
    const int seg = blockIdx.y, tid = threadIdx.x;
    for (int i = tid; i < 3 * kRadixBins; i += kClThreads) (&hist[0][0])[i] = 0;
    if (tid < 2) s_cnt[tid] = 0;
    pdl_begin();
    const int n = (int)src.n;
    const int64_t nvalid = n_valid_positions(src, seg);
    int32_t* o = out + (int64_t)seg * out_stride;
    float* ov = out_vals ? out_vals + (int64_t)seg * out_stride : nullptr;
    uint32_t* cnt_out = cl.map_shared_rank(&s_cnt[0], 0);
    uint32_t* cnt_tie = cl.map_shared_rank(&s_cnt[1], 0);

    int32_t ids[kClPer];
    uint32_t keys[kClPer];
#pragma unroll
    for (int k = 0; k < kClPer; ++k) {
        const int i = (k * kClCtas + (int)rank) * kClThreads + tid;
        ids[k] = i < n ? (src.ids ? __ldg(src.ids + seg * src.ids_stride + i) : i) : -1;
    }
#pragma unroll
    for (int k = 0; k < kClPer; ++k) {
        const int i = (k * kClCtas + (int)rank) * kClThreads + tid;
        const bool valid = i < n && ids[k] >= 0 && ids[k] < nvalid;
        keys[k] = valid ? ordered_key(src.vals[seg * src.vals_stride + (src.gather || !src.ids ? (int64_t)ids[k] : i)])
                        : 0u;                     // the ordered key of a finite float is never 0
        if (valid) atomicAdd(&hist[0][digit(keys[k], 1)], 1u);
    }
    cl.sync();   // every CTA's level-1 histogram (and CTA 0's zeroed counters) complete
    ClPlan pl = cluster_threshold(cl, hist[0], 0u, (uint32_t)n_out, s_wsum, &s_plan);
    const uint32_t need0 = pl.total < (uint32_t)n_out ? pl.total : (uint32_t)n_out;
    for (int i = (int)need0 + (int)rank * kClThreads + tid; i < n_out; i += kClCtas * kClThreads) o[i] = -1;
    uint32_t need = need0, prefix = 0, mask = 0;
    bool done = need0 == 0;
    for (int level = 1; level <= 3 && !done; ++level) {
        if (level > 1) {
            cl.sync();   // the level's histograms complete in every CTA
            pl = cluster_threshold(cl, hist[level - 1], need, (uint32_t)n_out, s_wsum, &s_plan);
        }
        const uint32_t shift = level == 1 ? 21 : level == 2 ? 10 : 0;
        const uint32_t dmask = level == 3 ? 0x3FFu : 0x7FFu;
        const bool all_eq = pl.eq == need - pl.above;
        // select the elements of the current prefix whose digit is above c (and
        // those equal to c when exactly the missing number of them exist); the
        // others equal to c go on to the next digit
#pragma unroll
        for (int k = 0; k < kClPer; ++k) {
            const uint32_t key = keys[k];
            const bool in = key && (key & mask) == prefix;
            const uint32_t d = (key >> shift) & dmask;
            const bool take = in && (d > pl.c || (d == pl.c && all_eq));
            if (level < 3 && in && d == pl.c && !all_eq) atomicAdd(&hist[level][digit(key, level + 1)], 1u);
            const uint32_t os = warp_claim(take, cnt_out);
            if (take) {
                o[os] = ids[k];
                if (ov) ov[os] = key_value(key);
            }
        }
        if (all_eq) {
            done = true;
        } else {
            need -= pl.above;
            prefix |= pl.c << shift;
            mask |= dmask << shift;
            if (level == 3) {
                // exact ties of the full key: the first `need` claimants win
#pragma unroll
                for (int k = 0; k < kClPer; ++k) {
                    const uint32_t key = keys[k];
                    const bool eq = key && key == prefix;
                    const uint32_t ts = warp_claim(eq, cnt_tie);
                    const bool take = eq && ts < need;
                    const uint32_t os = warp_claim(take, cnt_out);
                    if (take) {
                        o[os] = ids[k];
                        if (ov) ov[os] = key_value(key);
                    }
                }
            }
        }
    }
    cl.sync();   // no CTA leaves while another may still read its shared memory
}

}  // namespace

cudaError_t launch_select(const SelSrc& src, const SelWork& wk, int nseg, int n_out, int32_t* out,
                          int64_t out_stride, cudaStream_t st, bool hist_ready, float* out_vals) {
    if (src.n <= kSmallMax)
        return launch_pdl_cluster(k_sel_small, dim3(kClCtas, (unsigned)nseg), dim3(kClThreads), 0, st, kClCtas, src,
                                  n_out, out, out_vals, out_stride);
    return launch_select_dual(src, wk, nseg, n_out, out, out_vals, out_stride, 0, nullptr, 0, st, hist_ready);
}

cudaError_t launch_select_dual(const SelSrc& src, const SelWork& wk, int nseg, int n_a, int32_t* out_a, float* vals_a,
                               int64_t stride_a, int n_b, int32_t* out_b, int64_t stride_b, cudaStream_t st,
                               bool hist_ready) {
    // the histograms and counters are zero on entry (workspace initialisation,
    // then every k_sel_resolve clears what its selection used); without a
    // histogram from the scoring kernel, build level 1 here
    cudaError_t e;
    const unsigned chunks = (unsigned)((src.n + kPassChunk - 1) / kPassChunk);
    dim3 grid(chunks ? chunks : 1, (unsigned)nseg);
    if (!hist_ready) {
        e = launch_pdl(k_sel_hist, dim3(grid), dim3(kPassThreads), 0, st, src, wk);
        if (e != cudaSuccess) return e;
    }
    e = launch_pdl(k_sel_pass1, dim3(grid), dim3(kPassThreads), 0, st, src, wk, n_a, out_a, vals_a, stride_a, n_b,
                   out_b, stride_b);
    if (e != cudaSuccess) return e;
    return launch_pdl_cluster(k_sel_resolve, dim3(kClCtas, (unsigned)nseg), dim3(kClThreads), 0, st, kClCtas, wk, n_a,
                              out_a, vals_a, stride_a, n_b, out_b, stride_b);
}

}  // namespace csa2

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
//     from the scoring kernel; a streaming pass (many CTAs per segment)
//     selects above c1 and compacts the digit-c1 elements into a candidate
//     list; one CTA per segment then resolves digits 2 and 3 on that list.
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
constexpr int kFinThreads = 1024;
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

// Level 1 over every element: select digit > c1, compact digit == c1 into the
// candidate list and histogram their digit 2.  Each CTA claims its output and
// candidate slots with one atomic per counter (a block-wide scan of per-thread
// counts), so the shared counters see one atomic per CTA and chunk.
constexpr int kPassPer = kPassChunk / kPassThreads;   // elements per thread and chunk

__global__ void __launch_bounds__(kPassThreads)
k_sel_pass1(SelSrc src, SelWork wk, int n_out, int32_t* __restrict__ out, float* __restrict__ out_vals,
            int64_t out_stride) {
    pdl_begin();
    __shared__ uint32_t h2[kRadixBins];
    __shared__ uint32_t s_wsum[kPassThreads / 32];
    __shared__ Thr s_thr;
    __shared__ uint32_t s_base[2];
    const int seg = blockIdx.y, tid = threadIdx.x;
    uint32_t* cnt = wk.cnt + (int64_t)seg * 4;
    for (int i = tid; i < kRadixBins; i += kPassThreads) h2[i] = 0;   // ordered by the barriers below
    const Thr t1 = block_threshold<kPassThreads>(wk.hist + (int64_t)seg * 3 * kRadixBins, 0u, (uint32_t)n_out, s_wsum,
                                                 &s_thr);
    const uint32_t need0 = t1.need;
    int32_t* o = out + (int64_t)seg * out_stride;
    float* ov = out_vals ? out_vals + (int64_t)seg * out_stride : nullptr;
    if (blockIdx.x == 0)
        for (int i = (int)need0 + tid; i < n_out; i += kPassThreads) o[i] = -1;
    if (need0 == 0) return;
    const uint32_t c1 = t1.c;
    const bool take_eq = t1.eq == need0 - t1.above;   // every digit-c1 element is needed
    const int64_t nvalid = n_valid_positions(src, seg);
    const int64_t n_items = src.ids ? src.n : nvalid;
    uint2* cand = reinterpret_cast<uint2*>(wk.cand1) + seg * wk.cand_stride;
    bool any_cand = false;
    for (int64_t base = (int64_t)blockIdx.x * kPassChunk; base < n_items; base += (int64_t)gridDim.x * kPassChunk) {
        uint32_t keys[kPassPer];
        int32_t ids[kPassPer];
        uint32_t nt = 0, nc = 0;
#pragma unroll
        for (int k = 0; k < kPassPer; ++k) {
            const int64_t i = base + k * kPassThreads + tid;
            Elem e = {false, -1, 0u};
            if (i < n_items) e = load_elem(src, seg, i, nvalid);
            keys[k] = e.valid ? e.key : 0u;   // a valid key is never 0
            ids[k] = e.id;
            const uint32_t d = digit(keys[k], 1);
            const bool take = e.valid && (d > c1 || (d == c1 && take_eq));
            const bool to_cand = e.valid && d == c1 && !take_eq;
            nt += take;
            nc += to_cand;
            if (to_cand) atomicAdd(&h2[digit(keys[k], 2)], 1u);
        }
        // per-thread counts <= 16 and per-block sums <= 4096: both fit 16 bits
        uint32_t tot;
        const uint32_t pre = block_excl_scan<kPassThreads>((nt << 16) | nc, s_wsum, &tot);
        if (tid == 0) {
            s_base[0] = (tot >> 16) ? atomicAdd(cnt, tot >> 16) : 0u;
            s_base[1] = (tot & 0xFFFFu) ? atomicAdd(cnt + 1, tot & 0xFFFFu) : 0u;
        }
        __syncthreads();
        uint32_t os = s_base[0] + (pre >> 16), cs = s_base[1] + (pre & 0xFFFFu);
        __syncthreads();   // s_base is rewritten by the next chunk
#pragma unroll
        for (int k = 0; k < kPassPer; ++k) {
            const uint32_t d = digit(keys[k], 1);
            if (keys[k] && (d > c1 || (d == c1 && take_eq))) {
                o[os] = ids[k];
                if (ov) ov[os] = key_value(keys[k]);
                ++os;
            } else if (keys[k] && d == c1) {
                cand[cs++] = make_uint2(keys[k], (uint32_t)ids[k]);
            }
        }
        any_cand |= (tot & 0xFFFFu) != 0;
    }
    if (take_eq || !any_cand) return;   // the same in every thread of the block
    __syncthreads();
    uint32_t* gh2 = wk.hist + ((int64_t)seg * 3 + 1) * kRadixBins;
    for (int i = tid; i < kRadixBins; i += kPassThreads)
        if (h2[i]) atomicAdd(gh2 + i, h2[i]);
}

// Threshold plan of levels 1 and 2 from the global histograms.
// run == 0: level 1 already selected everything.
struct Plan2 {
    uint32_t run, c2, need2, n_cand, eq2, take_eq2;
};

template <int NT>
__device__ __forceinline__ Plan2 block_plan2(const uint32_t* h1, const uint32_t* h2, int n_out, uint32_t* s_wsum,
                                             Thr* s_thr) {
    Plan2 pl = {0u, 0u, 0u, 0u, 0u, 0u};
    const Thr t1 = block_threshold<NT>(h1, 0u, (uint32_t)n_out, s_wsum, s_thr);
    if (t1.need == 0 || t1.eq == t1.need - t1.above) return pl;
    const uint32_t need1 = t1.need - t1.above;
    const Thr t2 = block_threshold<NT>(h2, need1, (uint32_t)n_out, s_wsum, s_thr);
    pl.run = 1;
    pl.n_cand = t1.eq;
    pl.c2 = t2.c;
    pl.need2 = need1 - t2.above;
    pl.eq2 = t2.eq;
    pl.take_eq2 = t2.eq == pl.need2;
    return pl;
}

// Digit 2 over the (key, id) candidates of level 1, many CTAs per segment,
// slots claimed per CTA as in pass 1.
__global__ void __launch_bounds__(kPassThreads)
k_sel_pass2(SelWork wk, int n_out, int32_t* __restrict__ out, float* __restrict__ out_vals, int64_t out_stride) {
    pdl_begin();
    __shared__ uint32_t h3[kRadixBins];
    __shared__ uint32_t s_wsum[kPassThreads / 32];
    __shared__ Thr s_thr;
    __shared__ uint32_t s_base[2];
    const int seg = blockIdx.y, tid = threadIdx.x;
    uint32_t* cnt = wk.cnt + (int64_t)seg * 4;
    for (int i = tid; i < kRadixBins; i += kPassThreads) h3[i] = 0;
    const uint32_t* gh = wk.hist + (int64_t)seg * 3 * kRadixBins;
    const Plan2 pl = block_plan2<kPassThreads>(gh, gh + kRadixBins, n_out, s_wsum, &s_thr);
    if (!pl.run) return;
    const bool take_eq = pl.take_eq2 != 0;
    const uint2* cand = reinterpret_cast<const uint2*>(wk.cand1) + seg * wk.cand_stride;
    uint2* cand2 = reinterpret_cast<uint2*>(wk.cand2) + seg * wk.cand_stride;
    int32_t* o = out + (int64_t)seg * out_stride;
    float* ov = out_vals ? out_vals + (int64_t)seg * out_stride : nullptr;
    bool any = false;
    for (uint32_t base = blockIdx.x * kPassChunk; base < pl.n_cand; base += gridDim.x * kPassChunk) {
        uint2 kv[kPassPer];
        uint32_t nt = 0, nk = 0;
#pragma unroll
        for (int k = 0; k < kPassPer; ++k) {
            const uint32_t it = base + k * kPassThreads + tid;
            kv[k] = it < pl.n_cand ? cand[it] : make_uint2(0u, 0u);
            const uint32_t d = digit(kv[k].x, 2);
            const bool in = kv[k].x != 0u;
            const bool take = in && (d > pl.c2 || (d == pl.c2 && take_eq));
            const bool keep = in && d == pl.c2 && !take_eq;
            nt += take;
            nk += keep;
            if (keep) atomicAdd(&h3[digit(kv[k].x, 3)], 1u);
        }
        uint32_t tot;
        const uint32_t pre = block_excl_scan<kPassThreads>((nt << 16) | nk, s_wsum, &tot);
        if (tid == 0) {
            s_base[0] = (tot >> 16) ? atomicAdd(cnt, tot >> 16) : 0u;
            s_base[1] = (tot & 0xFFFFu) ? atomicAdd(cnt + 2, tot & 0xFFFFu) : 0u;
        }
        __syncthreads();
        uint32_t os = s_base[0] + (pre >> 16), ks = s_base[1] + (pre & 0xFFFFu);
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kPassPer; ++k) {
            const uint32_t d = digit(kv[k].x, 2);
            if (kv[k].x && (d > pl.c2 || (d == pl.c2 && take_eq))) {
                o[os] = (int32_t)kv[k].y;
                if (ov) ov[os] = key_value(kv[k].x);
                ++os;
            } else if (kv[k].x && d == pl.c2) {
                cand2[ks++] = kv[k];
            }
        }
        any |= (tot & 0xFFFFu) != 0;
    }
    if (take_eq || !any) return;
    __syncthreads();
    uint32_t* gh3 = wk.hist + ((int64_t)seg * 3 + 2) * kRadixBins;
    for (int i = tid; i < kRadixBins; i += kPassThreads)
        if (h3[i]) atomicAdd(gh3 + i, h3[i]);
}

// Digit 3 (exact ties last) of one segment, one CTA; then the histograms and
// counters of the segment are cleared for the next selection.
__global__ void __launch_bounds__(kFinThreads)
k_sel_finish(SelWork wk, int n_out, int32_t* __restrict__ out, float* __restrict__ out_vals, int64_t out_stride) {
    pdl_begin();
    __shared__ uint32_t s_wsum[kFinThreads / 32];
    __shared__ Thr s_thr;
    const int seg = blockIdx.x, tid = threadIdx.x;
    uint32_t* h1 = wk.hist + (int64_t)seg * 3 * kRadixBins;
    uint32_t* cnt = wk.cnt + (int64_t)seg * 4;
    const Plan2 pl = block_plan2<kFinThreads>(h1, h1 + kRadixBins, n_out, s_wsum, &s_thr);
    if (pl.run && !pl.take_eq2) {
        const Thr t3 = block_threshold<kFinThreads>(h1 + 2 * kRadixBins, pl.need2, (uint32_t)n_out, s_wsum, &s_thr);
        const uint32_t c3 = t3.c, need3 = pl.need2 - t3.above, n2 = pl.eq2;
        const uint2* cand2 = reinterpret_cast<const uint2*>(wk.cand2) + seg * wk.cand_stride;
        int32_t* o = out + (int64_t)seg * out_stride;
        for (uint32_t it0 = 0; it0 < n2; it0 += kFinThreads) {
            const uint32_t it = it0 + tid;
            const bool in = it < n2;
            const uint2 kv = in ? cand2[it] : make_uint2(0u, 0u);
            const uint32_t d = digit(kv.x, 3);
            const bool eq = in && d == c3;
            const uint32_t tie = warp_claim(eq, cnt + 3);
            const bool take = in && (d > c3 || (eq && tie < need3));
            const uint32_t os = warp_claim(take, cnt);
            if (take) {
                o[os] = (int32_t)kv.y;
                if (out_vals) out_vals[(int64_t)seg * out_stride + os] = key_value(kv.x);
            }
        }
    }
    // leave the workspace as csa2_workspace_init does: histograms and counters zero
    __syncthreads();
    for (int i = tid; i < 3 * kRadixBins; i += kFinThreads) h1[i] = 0;
    if (tid < 4) cnt[tid] = 0;
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
    cudaError_t e;
    if (src.n <= kSmallMax)
        return launch_pdl_cluster(k_sel_small, dim3(kClCtas, (unsigned)nseg), dim3(kClThreads), 0, st, kClCtas, src,
                                  n_out, out, out_vals, out_stride);
    // the histograms and counters are zero on entry (workspace initialisation,
    // then every k_sel_finish clears what its selection used); without a
    // histogram from the scoring kernel, build level 1 here
    const unsigned chunks = (unsigned)((src.n + kPassChunk - 1) / kPassChunk);
    dim3 grid(chunks ? chunks : 1, (unsigned)nseg);
    if (!hist_ready) {
        e = launch_pdl(k_sel_hist, dim3(grid), dim3(kPassThreads), 0, st, src, wk);
        if (e != cudaSuccess) return e;
    }
    e = launch_pdl(k_sel_pass1, dim3(grid), dim3(kPassThreads), 0, st, src, wk, n_out, out, out_vals, out_stride);
    if (e != cudaSuccess) return e;
    // level-1 candidates: at most the segment size; spread over up to 148 CTAs
    const unsigned g2 = chunks < 148 ? (chunks ? chunks : 1) : 148;
    e = launch_pdl(k_sel_pass2, dim3(g2, (unsigned)nseg), dim3(kPassThreads), 0, st, wk, n_out, out, out_vals,
                   out_stride);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_sel_finish, dim3(nseg), dim3(kFinThreads), 0, st, wk, n_out, out, out_vals, out_stride);
}

}  // namespace csa2

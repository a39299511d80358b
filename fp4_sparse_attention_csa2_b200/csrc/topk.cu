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
//   small segments (<= 16,384: the top-k of a pool): one CTA per segment keeps
//     every key in shared memory and resolves all three digits there.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

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

__device__ __forceinline__ uint32_t digit(uint32_t key, int level) {
    return level == 1 ? (key >> 21) : level == 2 ? ((key >> 10) & 0x7FFu) : (key & 0x3FFu);
}

// One warp: threshold digit of a 2048-bin histogram (global or shared).  Lane l
// owns the 64 bins [2047 - 64 l - 63, 2047 - 64 l].  Returns (c, above(c)) in
// every lane; requires 1 <= need <= sum(h).
__device__ __forceinline__ uint2 warp_threshold(const uint32_t* h, uint32_t need) {
    const int lane = threadIdx.x & 31;
    const int hi = kRadixBins - 1 - 64 * lane;
    uint32_t sum = 0;
#pragma unroll 16
    for (int k = 0; k < 64; ++k) sum += h[hi - k];
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - sum;
    const bool mine = excl < need && need <= incl;
    const int owner = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    uint2 r = make_uint2(0u, 0u);
    if (mine) {
        uint32_t above = excl;
        for (int k = 0; k < 64; ++k) {
            const uint32_t c = h[hi - k];
            if (need <= above + c) { r = make_uint2((uint32_t)(hi - k), above); break; }
            above += c;
        }
    }
    r.x = __shfl_sync(0xffffffffu, r.x, owner & 31);
    r.y = __shfl_sync(0xffffffffu, r.y, owner & 31);
    return r;
}

__device__ __forceinline__ uint32_t warp_sum_hist(const uint32_t* h) {
    uint32_t v = 0;
    for (int i = threadIdx.x & 31; i < kRadixBins; i += 32) v += h[i];
    return __reduce_add_sync(0xffffffffu, v);
}

// Copy `levels` consecutive 2048-bin histograms from global to shared memory
// (coalesced, the whole block), so the threshold scans run on shared memory.
__device__ __forceinline__ void stage_hist(uint32_t* dst, const uint32_t* src, int levels, int nthreads) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    for (int i = threadIdx.x; i < levels * kRadixBins / 4; i += nthreads) d4[i] = s4[i];
    __syncthreads();
}

// Histogram increment by a whole warp: lanes with the same bin add once.
__device__ __forceinline__ void warp_hist_add(uint32_t* hist, bool pred, uint32_t bin) {
    const uint32_t key = pred ? bin : 0xFFFFFFFFu;
    const uint32_t peers = __match_any_sync(0xffffffffu, key);
    if (pred && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(hist + bin, (uint32_t)__popc(peers));
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

// Level 1 over every element: select digit > c1, compact digit == c1.
__global__ void __launch_bounds__(kPassThreads)
k_sel_pass1(SelSrc src, SelWork wk, int n_out, int32_t* __restrict__ out, int64_t out_stride) {
    pdl_begin();
    __shared__ uint32_t s_plan[3];   // c1, elements to select, take every digit-c1 element
    __shared__ uint32_t h2[kRadixBins];
    __shared__ __align__(16) uint32_t h1[kRadixBins];
    const int seg = blockIdx.y;
    uint32_t* cnt = wk.cnt + (int64_t)seg * 4;
    stage_hist(h1, wk.hist + (int64_t)seg * 3 * kRadixBins, 1, kPassThreads);
    if (threadIdx.x < 32) {
        const uint32_t total = warp_sum_hist(h1);
        const uint32_t need = total < (uint32_t)n_out ? total : (uint32_t)n_out;
        uint2 t = make_uint2(0xFFFFFFFFu, 0u);
        if (need > 0) t = warp_threshold(h1, need);
        if (threadIdx.x == 0) {
            s_plan[0] = t.x;
            s_plan[1] = need;
            s_plan[2] = need > 0 ? (h1[t.x] == need - t.y) : 1u;
        }
    }
    for (int i = threadIdx.x; i < kRadixBins; i += kPassThreads) h2[i] = 0;
    __syncthreads();
    const uint32_t c1 = s_plan[0], need0 = s_plan[1];
    const bool take_eq = s_plan[2] != 0;
    int32_t* o = out + (int64_t)seg * out_stride;
    if (blockIdx.x == 0)
        for (int i = need0 + threadIdx.x; i < n_out; i += kPassThreads) o[i] = -1;
    if (need0 == 0) return;
    const int64_t nvalid = n_valid_positions(src, seg);
    const int64_t n_items = src.ids ? src.n : nvalid;
    uint2* cand = reinterpret_cast<uint2*>(wk.cand1) + seg * wk.cand_stride;
    for (int64_t base = (int64_t)blockIdx.x * kPassChunk; base < n_items; base += (int64_t)gridDim.x * kPassChunk) {
        const int64_t end = min(base + kPassChunk, n_items);
        for (int64_t it0 = base; it0 < end; it0 += kPassThreads) {
            const int64_t i = it0 + threadIdx.x;
            Elem e = {false, -1, 0u};
            if (i < end) e = load_elem(src, seg, i, nvalid);
            const uint32_t d = e.valid ? digit(e.key, 1) : 0u;
            const bool eq = e.valid && d == c1;
            const bool take = e.valid && (d > c1 || (eq && take_eq));
            const bool to_cand = eq && !take_eq;
            const uint32_t cs = warp_claim(to_cand, cnt + 1);
            if (to_cand) cand[cs] = make_uint2(e.key, (uint32_t)e.id);
            warp_hist_add(h2, to_cand, digit(e.key, 2));
            const uint32_t os = warp_claim(take, cnt);
            if (take) o[os] = e.id;
        }
    }
    if (take_eq) return;
    __syncthreads();
    uint32_t* gh2 = wk.hist + ((int64_t)seg * 3 + 1) * kRadixBins;
    for (int i = threadIdx.x; i < kRadixBins; i += kPassThreads)
        if (h2[i]) atomicAdd(gh2 + i, h2[i]);
}

// Threshold plan of levels 1 and 2 from the global histograms (one warp).
// run = 0: level 1 already selected everything.
struct Plan2 {
    uint32_t run, c2, need2, n_cand, eq2;
};

__device__ __forceinline__ Plan2 plan_level2(const uint32_t* h1, const uint32_t* h2, int n_out) {
    Plan2 pl = {0u, 0u, 0u, 0u, 0u};
    const uint32_t total = warp_sum_hist(h1);
    const uint32_t need = total < (uint32_t)n_out ? total : (uint32_t)n_out;
    if (need > 0) {
        const uint2 t1 = warp_threshold(h1, need);
        pl.n_cand = h1[t1.x];
        const uint32_t need1 = need - t1.y;
        if (pl.n_cand != need1) {
            const uint2 t2 = warp_threshold(h2, need1);
            pl.run = 1;
            pl.c2 = t2.x;
            pl.need2 = need1 - t2.y;
            pl.eq2 = h2[t2.x];
        }
    }
    return pl;
}

// Digit 2 over the (key, id) candidates of level 1, many CTAs per segment.
__global__ void __launch_bounds__(kPassThreads)
k_sel_pass2(SelWork wk, int n_out, int32_t* __restrict__ out, int64_t out_stride) {
    pdl_begin();
    __shared__ Plan2 s_pl;
    __shared__ uint32_t h3[kRadixBins];
    __shared__ __align__(16) uint32_t h12[2 * kRadixBins];
    const int seg = blockIdx.y;
    uint32_t* cnt = wk.cnt + (int64_t)seg * 4;
    stage_hist(h12, wk.hist + (int64_t)seg * 3 * kRadixBins, 2, kPassThreads);
    if (threadIdx.x < 32) {
        const Plan2 pl = plan_level2(h12, h12 + kRadixBins, n_out);
        if (threadIdx.x == 0) s_pl = pl;
    }
    for (int i = threadIdx.x; i < kRadixBins; i += kPassThreads) h3[i] = 0;
    __syncthreads();
    const Plan2 pl = s_pl;
    if (!pl.run) return;
    const bool take_eq = pl.eq2 == pl.need2;
    const uint2* cand = reinterpret_cast<const uint2*>(wk.cand1) + seg * wk.cand_stride;
    uint2* cand2 = reinterpret_cast<uint2*>(wk.cand2) + seg * wk.cand_stride;
    int32_t* o = out + (int64_t)seg * out_stride;
    bool any = false;
    for (uint32_t base = blockIdx.x * kPassChunk; base < pl.n_cand; base += gridDim.x * kPassChunk) {
        const uint32_t end = min(base + (uint32_t)kPassChunk, pl.n_cand);
        for (uint32_t it0 = base; it0 < end; it0 += kPassThreads) {
            const uint32_t it = it0 + threadIdx.x;
            const bool in = it < end;
            const uint2 kv = in ? cand[it] : make_uint2(0u, 0u);
            const uint32_t d = digit(kv.x, 2);
            const bool eq = in && d == pl.c2;
            const bool take = in && (d > pl.c2 || (eq && take_eq));
            const bool keep = eq && !take_eq;
            const uint32_t ks = warp_claim(keep, cnt + 2);
            if (keep) {
                cand2[ks] = kv;
                any = true;
            }
            warp_hist_add(h3, keep, digit(kv.x, 3));
            const uint32_t os = warp_claim(take, cnt);
            if (take) o[os] = (int32_t)kv.y;
        }
    }
    if (take_eq || !__syncthreads_or(any)) return;
    uint32_t* gh3 = wk.hist + ((int64_t)seg * 3 + 2) * kRadixBins;
    for (int i = threadIdx.x; i < kRadixBins; i += kPassThreads)
        if (h3[i]) atomicAdd(gh3 + i, h3[i]);
}

// Digit 3 (exact ties last) of one segment, one CTA; then the histograms and
// counters of the segment are cleared for the next selection.
__global__ void __launch_bounds__(kFinThreads)
k_sel_finish(SelWork wk, int n_out, int32_t* __restrict__ out, int64_t out_stride) {
    pdl_begin();
    __shared__ Plan2 s_pl;
    __shared__ uint32_t s_plan[2];
    __shared__ __align__(16) uint32_t hs[3 * kRadixBins];
    const int seg = blockIdx.x;
    uint32_t* h1 = wk.hist + (int64_t)seg * 3 * kRadixBins;
    uint32_t* cnt = wk.cnt + (int64_t)seg * 4;
    stage_hist(hs, h1, 3, kFinThreads);
    if (threadIdx.x < 32) {
        const Plan2 pl = plan_level2(hs, hs + kRadixBins, n_out);
        if (threadIdx.x == 0) s_pl = pl;
    }
    __syncthreads();
    const Plan2 pl = s_pl;
    if (pl.run && pl.eq2 != pl.need2) {
        const uint32_t* h3 = hs + 2 * kRadixBins;
        if (threadIdx.x < 32) {
            const uint2 t3 = warp_threshold(h3, pl.need2);
            if (threadIdx.x == 0) {
                s_plan[0] = t3.x;
                s_plan[1] = pl.need2 - t3.y;
            }
        }
        __syncthreads();
        const uint32_t c3 = s_plan[0], need3 = s_plan[1], n2 = pl.eq2;
        const uint2* cand2 = reinterpret_cast<const uint2*>(wk.cand2) + seg * wk.cand_stride;
        int32_t* o = out + (int64_t)seg * out_stride;
        for (uint32_t it0 = 0; it0 < n2; it0 += kFinThreads) {
            const uint32_t it = it0 + threadIdx.x;
            const bool in = it < n2;
            const uint2 kv = in ? cand2[it] : make_uint2(0u, 0u);
            const uint32_t d = digit(kv.x, 3);
            const bool eq = in && d == c3;
            const uint32_t tie = warp_claim(eq, cnt + 3);
            const bool take = in && (d > c3 || (eq && tie < need3));
            const uint32_t os = warp_claim(take, cnt);
            if (take) o[os] = (int32_t)kv.y;
        }
    }
    // leave the workspace as csa2_workspace_init does: histograms and counters zero
    __syncthreads();
    for (int i = threadIdx.x; i < 3 * kRadixBins; i += kFinThreads) h1[i] = 0;
    if (threadIdx.x < 4) cnt[threadIdx.x] = 0;
}

// ---------------------------------------------------------------- small segments
// Whole selection of one segment of at most kSmallMax elements in one CTA.
__global__ void __launch_bounds__(kFinThreads)
k_sel_small(SelSrc src, int n_out, int32_t* __restrict__ out, int64_t out_stride) {
    pdl_begin();
    extern __shared__ uint32_t sm[];
    uint32_t* keys = sm;                        // [n]; 0 marks an invalid element
    uint32_t* hist = sm + src.n;                // [kRadixBins]
    __shared__ uint32_t s_plan[3];
    __shared__ uint32_t s_cnt[2];
    const int seg = blockIdx.x;
    const int n = (int)src.n;
    const int64_t nvalid = n_valid_positions(src, seg);
    int32_t* o = out + (int64_t)seg * out_stride;
    for (int i = threadIdx.x; i < kRadixBins; i += kFinThreads) hist[i] = 0;
    if (threadIdx.x < 2) s_cnt[threadIdx.x] = 0;
    __syncthreads();
    uint32_t mine = 0;
    // 16 elements per thread (n <= 16384): ids first, then the values they select
    constexpr int kPer = kSmallMax / kFinThreads;
    int32_t ids[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int i = k * kFinThreads + threadIdx.x;
        ids[k] = i < n ? (src.ids ? __ldg(src.ids + seg * src.ids_stride + i) : i) : -1;   // the output id
    }
    float vals[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int i = k * kFinThreads + threadIdx.x;
        const bool valid = i < n && ids[k] >= 0 && ids[k] < nvalid;
        vals[k] = valid ? src.vals[seg * src.vals_stride + (src.gather || !src.ids ? (int64_t)ids[k] : i)] : 0.0f;
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int i = k * kFinThreads + threadIdx.x;
        const bool valid = i < n && ids[k] >= 0 && ids[k] < nvalid;
        const uint32_t key = valid ? ordered_key(vals[k]) : 0u;
        if (i < n) keys[i] = key;            // the ordered key of a finite float is never 0
        warp_hist_add(hist, valid, digit(key, 1));
        mine += valid;
    }
    mine = __reduce_add_sync(0xffffffffu, mine);
    if ((threadIdx.x & 31) == 0 && mine) atomicAdd(&s_cnt[1], mine);
    __syncthreads();
    const uint32_t total = s_cnt[1];
    const uint32_t need0 = total < (uint32_t)n_out ? total : (uint32_t)n_out;
    for (int i = need0 + threadIdx.x; i < n_out; i += kFinThreads) o[i] = -1;
    if (need0 == 0) return;
    // digits fixed so far, as (prefix, mask) over the key
    uint32_t prefix = 0, mask = 0, need = need0;
    for (int level = 1; level <= 3; ++level) {
        if (level > 1) {
            __syncthreads();
            for (int i = threadIdx.x; i < kRadixBins; i += kFinThreads) hist[i] = 0;
            __syncthreads();
            for (int i0 = 0; i0 < n; i0 += kFinThreads) {
                const int i = i0 + threadIdx.x;
                const uint32_t k = i < n ? keys[i] : 0u;
                warp_hist_add(hist, k && (k & mask) == prefix, digit(k, level));
            }
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            const uint2 t = warp_threshold(hist, need);
            if (threadIdx.x == 0) {
                s_plan[0] = t.x;
                s_plan[1] = t.y;
                s_plan[2] = hist[t.x];
            }
        }
        __syncthreads();
        const uint32_t c = s_plan[0], above = s_plan[1], eqn = s_plan[2];
        const uint32_t shift = level == 1 ? 21 : level == 2 ? 10 : 0;
        const uint32_t dmask = level == 3 ? 0x3FFu : 0x7FFu;
        const bool all_eq = eqn == need - above;
        // select the elements of the current prefix whose digit is above c
        // (and those equal to c when exactly the missing number of them exist)
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int i = k * kFinThreads + threadIdx.x;
            const uint32_t key = i < n ? keys[i] : 0u;
            const bool in = key && (key & mask) == prefix;
            const uint32_t d = (key >> shift) & dmask;
            const bool take = in && (d > c || (d == c && all_eq));
            const uint32_t os = warp_claim(take, &s_cnt[0]);
            if (take) o[os] = ids[k];
        }
        if (all_eq) break;
        need -= above;
        prefix |= c << shift;
        mask |= dmask << shift;
        if (level == 3) {
            // exact ties of the full key: the first `need` claimants win
            __syncthreads();
            if (threadIdx.x == 0) s_cnt[1] = 0;
            __syncthreads();
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int i = k * kFinThreads + threadIdx.x;
                const uint32_t key = i < n ? keys[i] : 0u;
                const bool eq = key && key == prefix;
                const uint32_t ts = warp_claim(eq, &s_cnt[1]);
                const bool take = eq && ts < need;
                const uint32_t os = warp_claim(take, &s_cnt[0]);
                if (take) o[os] = ids[k];
            }
        }
    }
}

}  // namespace

cudaError_t launch_select(const SelSrc& src, const SelWork& wk, int nseg, int n_out, int32_t* out,
                          int64_t out_stride, cudaStream_t st, bool hist_ready) {
    cudaError_t e;
    if (src.n <= kSmallMax) {
        const size_t smem = sizeof(uint32_t) * ((size_t)src.n + kRadixBins);
        if (smem > 48 * 1024) {
            e = cudaFuncSetAttribute(k_sel_small, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
        }
        return launch_pdl(k_sel_small, dim3(nseg), dim3(kFinThreads), smem, st, src, n_out, out, out_stride);
    }
    // the histograms and counters are zero on entry (workspace initialisation,
    // then every k_sel_finish clears what its selection used); without a
    // histogram from the scoring kernel, build level 1 here
    const unsigned chunks = (unsigned)((src.n + kPassChunk - 1) / kPassChunk);
    dim3 grid(chunks ? chunks : 1, (unsigned)nseg);
    if (!hist_ready) {
        e = launch_pdl(k_sel_hist, dim3(grid), dim3(kPassThreads), 0, st, src, wk);
        if (e != cudaSuccess) return e;
    }
    e = launch_pdl(k_sel_pass1, dim3(grid), dim3(kPassThreads), 0, st, src, wk, n_out, out, out_stride);
    if (e != cudaSuccess) return e;
    // level-1 candidates: at most the segment size; spread over up to 148 CTAs
    const unsigned g2 = chunks < 148 ? (chunks ? chunks : 1) : 148;
    e = launch_pdl(k_sel_pass2, dim3(g2, (unsigned)nseg), dim3(kPassThreads), 0, st, wk, n_out, out, out_stride);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_sel_finish, dim3(nseg), dim3(kFinThreads), 0, st, wk, n_out, out, out_stride);
}

}  // namespace csa2

// Top-n selection by radix select on order-preserving 32-bit keys of fp32
// scores: the candidate pool (<= 16,384 of up to 1M scores) of a Full layer
// and the top-k of Full / Reindex layers (tldrocket.com, "DeepSeek AI Released
// DeepSeek-V4.1-Flash with 1M Context, FP4 KV Cache, and Cross-Layer Attention
// Reuse", paragraph 3; hackernews.kjhq.dev post 49735410, key point 2, "Top-K
// indices").
//
// The 32-bit key is split into three digits: bits 31..21, 20..10 and 9..0.
//   hist pass : histogram of digit 1 over every valid element.
//   level 1   : every CTA finds, from the histogram, the digit value c1 that
//               holds the n-th largest key.  Elements above c1 are selected;
//               elements equal to c1 are either all selected (when exactly the
//               missing number of them exist) or appended to a candidate list
//               and histogrammed on digit 2.
//   level 2/3 : the same on the candidate list with the next digit; at level 3
//               the remaining equal keys are exact ties and the first ones to
//               claim a slot are selected.
// Output order is unspecified; -1 pads the tail.  Every CTA re-derives the
// thresholds from the (small) histograms, so no pass waits on another CTA.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

namespace {

constexpr int kThreads = 256;
constexpr int kPerThread = 16;
constexpr int kChunk = kThreads * kPerThread;  // elements per CTA and pass

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

// Block-wide: find c with above(c) < need <= above(c) + h[c], where above(c) is
// the number of elements in bins > c.  Writes c and above(c) to out[0..1].
// Requires 1 <= need <= sum(h).  256 threads, 2048 bins.
__device__ void find_threshold(const uint32_t* __restrict__ h, uint32_t need, uint32_t* s_scan, uint32_t* out) {
    const int tid = threadIdx.x;
    // thread tid owns bins [2040 - 8*tid, 2047 - 8*tid] (thread 0: the top bins)
    const int hi = kRadixBins - 1 - 8 * tid;
    uint32_t local[8];
    uint32_t sum = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) { local[k] = h[hi - k]; sum += local[k]; }
    s_scan[tid] = sum;
    __syncthreads();
    // inclusive scan over 256 thread sums (Hillis-Steele)
    for (int off = 1; off < kThreads; off <<= 1) {
        uint32_t v = tid >= off ? s_scan[tid - off] : 0u;
        __syncthreads();
        s_scan[tid] += v;
        __syncthreads();
    }
    uint32_t above = tid ? s_scan[tid - 1] : 0u;   // elements in bins above this thread's range
    if (above < need && need <= s_scan[tid]) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (above < need && need <= above + local[k]) {
                out[0] = (uint32_t)(hi - k);
                out[1] = above;
                break;
            }
            above += local[k];
        }
    }
    __syncthreads();
}

__device__ uint32_t block_sum_hist(const uint32_t* __restrict__ h, uint32_t* s_red) {
    uint32_t v = 0;
    for (int i = threadIdx.x; i < kRadixBins; i += kThreads) v += h[i];
    v = __reduce_add_sync(0xffffffffu, v);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = v;
    __syncthreads();
    uint32_t tot = 0;
    for (int w = 0; w < kThreads / 32; ++w) tot += s_red[w];
    __syncthreads();
    return tot;
}

// Thresholds of levels 1..level (shared with the block).
struct Plan {
    uint32_t need0;          // total to select: min(n_out, n_valid)
    uint32_t c[4];           // c[l]: threshold digit at level l
    uint32_t need[4];        // need[l]: still missing after taking digits > c[l]
    uint32_t cnt_eq[4];      // hist_l[c_l]
    bool direct[4];          // level l takes all of its equal-digit elements
};

__device__ void make_plan(const uint32_t* hist, int n_out, int level, Plan* p, uint32_t* s_scan, uint32_t* s_red,
                          uint32_t* s_out) {
    const uint32_t total = block_sum_hist(hist, s_red);
    uint32_t need = total < (uint32_t)n_out ? total : (uint32_t)n_out;
    if (threadIdx.x == 0) p->need0 = need;
    for (int l = 1; l <= level; ++l) {
        if (need == 0) {
            if (threadIdx.x == 0) { p->c[l] = 0xFFFFFFFFu; p->need[l] = 0; p->cnt_eq[l] = 0; p->direct[l] = true; }
            __syncthreads();
            continue;
        }
        const uint32_t* h = hist + (l - 1) * kRadixBins;
        find_threshold(h, need, s_scan, s_out);
        const uint32_t c = s_out[0], above = s_out[1];
        const uint32_t rem = need - above;
        const uint32_t eq = h[c];
        if (threadIdx.x == 0) {
            p->c[l] = c;
            p->cnt_eq[l] = eq;
            p->direct[l] = (eq == rem) || l == 3;
            p->need[l] = rem;
        }
        __syncthreads();
        // elements equal at this level: all selected when `direct`, otherwise the
        // next level needs `rem` of them; a direct level ends the search
        need = p->direct[l] ? 0 : rem;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kThreads)
k_sel_hist(SelSrc src, SelWork wk) {
    __shared__ uint32_t h[kRadixBins];
    const int seg = blockIdx.y;
    for (int i = threadIdx.x; i < kRadixBins; i += kThreads) h[i] = 0;
    __syncthreads();
    const int64_t nvalid = n_valid_positions(src, seg);
    const int64_t base = (int64_t)blockIdx.x * kChunk;
    const int64_t end = min(base + kChunk, src.ids ? src.n : nvalid);
    for (int64_t i = base + threadIdx.x; i < end; i += kThreads) {
        Elem e = load_elem(src, seg, i, nvalid);
        if (e.valid) atomicAdd(&h[digit(e.key, 1)], 1u);
    }
    __syncthreads();
    uint32_t* gh = wk.hist + (int64_t)seg * 3 * kRadixBins;
    for (int i = threadIdx.x; i < kRadixBins; i += kThreads)
        if (h[i]) atomicAdd(gh + i, h[i]);
}

template <int LEVEL>
__global__ void __launch_bounds__(kThreads)
k_sel_pass(SelSrc src, SelWork wk, int n_out, int32_t* __restrict__ out, int64_t out_stride) {
    __shared__ uint32_t s_scan[kThreads];
    __shared__ uint32_t s_red[kThreads / 32];
    __shared__ uint32_t s_out[2];
    __shared__ Plan plan;
    __shared__ uint32_t hnext[kRadixBins];
    const int seg = blockIdx.y;
    const uint32_t* hist = wk.hist + (int64_t)seg * 3 * kRadixBins;
    uint32_t* cnt = wk.cnt + (int64_t)seg * 4;
    make_plan(hist, n_out, LEVEL, &plan, s_scan, s_red, s_out);

    int32_t* o = out + (int64_t)seg * out_stride;
    if (LEVEL == 1 && blockIdx.x == 0)
        for (int i = plan.need0 + threadIdx.x; i < n_out; i += kThreads) o[i] = -1;

    // levels before this one must have left candidates for it
    for (int l = 1; l < LEVEL; ++l)
        if (plan.direct[l] || plan.need0 == 0) return;
    if (plan.need0 == 0) return;

    const bool more = !plan.direct[LEVEL];
    if (more)
        for (int i = threadIdx.x; i < kRadixBins; i += kThreads) hnext[i] = 0;
    __syncthreads();

    const uint32_t c = plan.c[LEVEL];
    const uint32_t need_here = plan.need[LEVEL];
    const int64_t nvalid = n_valid_positions(src, seg);
    const int64_t n_items = LEVEL == 1 ? (src.ids ? src.n : nvalid) : (int64_t)plan.cnt_eq[LEVEL - 1];
    const uint32_t* cand_in = LEVEL == 2 ? wk.cand1 + seg * wk.cand_stride : wk.cand2 + seg * wk.cand_stride;
    uint32_t* cand_out = LEVEL == 1 ? wk.cand1 + seg * wk.cand_stride : wk.cand2 + seg * wk.cand_stride;

    const int lane = threadIdx.x & 31;
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int64_t base = (int64_t)blockIdx.x * kChunk; base < n_items; base += (int64_t)gridDim.x * kChunk) {
        const int64_t end = min(base + kChunk, n_items);
        for (int64_t it0 = base; it0 < end; it0 += kThreads) {
            const int64_t it = it0 + threadIdx.x;
            Elem e;
            e.valid = false;
            int64_t i = 0;
            if (it < end) {
                i = LEVEL == 1 ? it : (int64_t)cand_in[it];
                e = load_elem(src, seg, i, nvalid);
            }
            const uint32_t d = e.valid ? digit(e.key, LEVEL) : 0u;
            const bool eq = e.valid && d == c;
            bool take = e.valid && d > c;
            bool to_cand = false;
            if (eq && LEVEL < 3) {
                if (more) to_cand = true;   // resolved by the next digit
                else take = true;           // exactly the missing number of them
            }
            // exact ties at the last level: the first `need_here` claimants win
            if (LEVEL == 3) {
                const uint32_t m = __ballot_sync(0xffffffffu, eq);
                if (m) {
                    const int leader = __ffs(m) - 1;
                    uint32_t b0 = 0;
                    if (lane == leader) b0 = atomicAdd(cnt + 3, (uint32_t)__popc(m));
                    b0 = __shfl_sync(0xffffffffu, b0, leader);
                    if (eq && b0 + __popc(m & lt_mask) < need_here) take = true;
                }
            }
            if (LEVEL < 3) {
                const uint32_t m = __ballot_sync(0xffffffffu, to_cand);
                if (m) {
                    const int leader = __ffs(m) - 1;
                    uint32_t b0 = 0;
                    if (lane == leader) b0 = atomicAdd(cnt + LEVEL, (uint32_t)__popc(m));
                    b0 = __shfl_sync(0xffffffffu, b0, leader);
                    if (to_cand) {
                        cand_out[b0 + __popc(m & lt_mask)] = (uint32_t)i;
                        atomicAdd(&hnext[digit(e.key, LEVEL + 1)], 1u);
                    }
                }
            }
            const uint32_t mt = __ballot_sync(0xffffffffu, take);
            if (mt) {
                const int leader = __ffs(mt) - 1;
                uint32_t b0 = 0;
                if (lane == leader) b0 = atomicAdd(cnt, (uint32_t)__popc(mt));
                b0 = __shfl_sync(0xffffffffu, b0, leader);
                if (take) o[b0 + __popc(mt & lt_mask)] = e.id;
            }
        }
    }
    if (LEVEL < 3 && more) {
        __syncthreads();
        uint32_t* gh = wk.hist + ((int64_t)seg * 3 + LEVEL) * kRadixBins;
        for (int i = threadIdx.x; i < kRadixBins; i += kThreads)
            if (hnext[i]) atomicAdd(gh + i, hnext[i]);
    }
}

}  // namespace

cudaError_t launch_select(const SelSrc& src, const SelWork& wk, int nseg, int n_out, int32_t* out,
                          int64_t out_stride, cudaStream_t st, bool hist_ready) {
    cudaError_t e;
    if (!hist_ready) {
        e = cudaMemsetAsync(wk.hist, 0, sizeof(uint32_t) * (size_t)nseg * 3 * kRadixBins, st);
        if (e != cudaSuccess) return e;
    }
    e = cudaMemsetAsync(wk.cnt, 0, sizeof(uint32_t) * (size_t)nseg * 4, st);
    if (e != cudaSuccess) return e;
    const unsigned chunks = (unsigned)((src.n + kChunk - 1) / kChunk);
    dim3 grid(chunks ? chunks : 1, (unsigned)nseg);
    if (!hist_ready) k_sel_hist<<<grid, kThreads, 0, st>>>(src, wk);
    k_sel_pass<1><<<grid, kThreads, 0, st>>>(src, wk, n_out, out, out_stride);
    k_sel_pass<2><<<grid, kThreads, 0, st>>>(src, wk, n_out, out, out_stride);
    k_sel_pass<3><<<grid, kThreads, 0, st>>>(src, wk, n_out, out, out_stride);
    return cudaGetLastError();
}

}  // namespace csa2

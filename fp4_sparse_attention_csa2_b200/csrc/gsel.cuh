// Pieces of a selection run by every CTA of a segment together (the keys stay
// where they were computed): the segment barrier, histogram reads from L2,
// and one target's threshold digit in a 2048-bin histogram.  Used by the
// one-grid Full-layer selection (topk.cu) and the Reindex kernel's grid mode
// (reindex_tc.cu).  The digit scheme is the one of topk.cu: bits 31..21,
// 20..10 and 9..0 of the order-preserving key.
#pragma once
#include <cstdint>

namespace csa2 {
namespace gsel {

// Arrive at the segment barrier (counter ctr) and wait, bounded, until it
// counts `target` arrivals; false when the wait gave up.  Every thread's
// global writes before the call are visible to the other CTAs after it.
// (Fencing in thread 0 alone, after the CTA barrier, measured slower.)
__device__ __forceinline__ bool seg_barrier(uint32_t* ctr, uint32_t target, uint32_t limit, uint32_t* s_flag) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        atomicAdd(ctr, 1u);
        uint32_t v = 0;
        for (uint32_t i = 0;; ++i) {
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
            if (v >= target || i >= limit) break;
            if (i >= 64) __nanosleep(128);                 // poll back to back at first
        }
        *s_flag = v >= target ? 1u : 0u;
    }
    __syncthreads();
    return *s_flag != 0u;
}

// n words (a multiple of 4) of a histogram written by other CTAs into shared memory (L2 reads).
template <int NT>
__device__ __forceinline__ void load_hist(uint32_t* dst, const uint32_t* src, int n) {
    for (int i = threadIdx.x; i < n / 4; i += NT)
        reinterpret_cast<uint4*>(dst)[i] = __ldcg(reinterpret_cast<const uint4*>(src) + i);
    __syncthreads();
}

struct Cut {
    uint32_t c, above, eq, need;   // threshold digit c: above(c) < need <= above(c) + h[c]
};

// One target's threshold digit in the 2048-bin histogram h (shared memory)
// with need = need_in, or min(total, n_out) when need_in is 0.  Thread t owns
// the 2048 / NT bins just below 2048 - t (2048 / NT): descending bins follow
// ascending threads, one block-wide scan.  s_wsum: NT / 32 words.
template <int NT>
__device__ __forceinline__ Cut threshold(const uint32_t* h, uint32_t need_in, uint32_t n_out, uint32_t* s_wsum,
                                         Cut* s_cut) {
    constexpr int per = 2048 / NT;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int lo = 2048 - per * (tid + 1);
    uint32_t bins[per], sum = 0;
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
    if (tid == 0) *s_cut = Cut{0u, 0u, 0u, 0u};
    __syncthreads();
    uint32_t wt = lane < NT / 32 ? s_wsum[lane] : 0u;
#pragma unroll
    for (int o = 1; o < NT / 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, wt, o);
        if (lane >= o) wt += v;
    }
    const uint32_t total = __shfl_sync(0xffffffffu, wt, NT / 32 - 1);
    const uint32_t before = warp ? __shfl_sync(0xffffffffu, wt, (warp - 1) & 31) : 0u;
    const uint32_t excl = before + incl - sum;
    const uint32_t need = need_in ? need_in : (total < n_out ? total : n_out);
    if (need > 0 && excl < need && need <= excl + sum) {
        uint32_t above = excl;
#pragma unroll
        for (int k = per - 1; k >= 0; --k) {
            if (need <= above + bins[k]) {
                *s_cut = Cut{(uint32_t)(lo + k), above, bins[k], need};
                break;
            }
            above += bins[k];
        }
    }
    __syncthreads();
    Cut r = *s_cut;
    r.need = need;
    __syncthreads();   // s_wsum and s_cut are rewritten by the next call
    return r;
}

}  // namespace gsel
}  // namespace csa2

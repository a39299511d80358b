// Selection of the n largest of at most NT * E keys by one CTA of NT
// threads, every key (and its id) held in registers, E per thread.  Used for
// the top-k of a pool (at most 16,384 elements: the Reindex layer) and the
// pool and top-k of a Full layer over a short context.
//
// Keys are order-preserving 32-bit images of the scores (select_key; 0 marks
// an element that is not a candidate).  Keys are binned by their distance
// from the largest key on a floating scale (64 bins per power of two, see
// dist_bin), so bins are narrow near the top, where the cutoff of the n
// largest lies, and wide far from it.  The work that touches every element
// is one branch-free pass without atomics:
//   1. a sample of NT keys (one per thread) is histogrammed; two bins that
//      bracket the sample's cutoff, with a margin of about three binomial
//      standard deviations, are read off it;
//   2. one pass classifies every element: nearer than the bracket (taken),
//      inside it (candidate), farther (dropped), and counts the first two;
//   3. if the bracket holds the cutoff (taken < n <= taken + candidates) and
//      the candidates fit the list, they are compacted into a shared-memory
//      list and the rest of the selection is a radix select over that list
//      on digits of the key relative to the list's smallest key (11 bits at a
//      time); exact ties left after the last digit are taken in list order.
// When the bracket misses (a sample unlike the whole, or too many keys tied
// inside it), a histogram of every element's bin replaces the sample's and
// the later levels walk the registers.
#pragma once
#include <cstdint>

#include "common.cuh"

namespace csa2 {
namespace lsel {

constexpr int kBins = 2048;
constexpr uint32_t kFull = 0xffffffffu;

constexpr int kList = 4096;

template <int NT>
struct Smem {
    uint32_t hist[kBins];
    uint32_t wa[NT / 32], wb[NT / 32], wc[NT / 32];
    uint32_t bc[4];
    uint32_t lkey[kList];      // the first level's leftover candidates: key,
    uint32_t lref[kList];      // and thread << 5 | element
    uint32_t take[NT];         // per thread: elements taken from the list
    uint32_t nlist;
};

// Exclusive prefix over the block of one value per thread; *total gets the
// sum.  Two barriers and one warp-wide scan: each warp's total goes to shared
// memory, warp 0 scans the NT / 32 totals, every thread reads its warp's
// prefix back (no thread walks all the totals).
template <int NT>
__device__ __forceinline__ uint32_t excl_scan(uint32_t v, Smem<NT>& sh, uint32_t* total) {
    static_assert(NT / 32 <= 32, "one warp scans the warp totals");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) sh.wa[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const uint32_t t = lane < NT / 32 ? sh.wa[lane] : 0u;
        uint32_t x = t;
#pragma unroll
        for (int o = 1; o < NT / 32; o <<= 1) {
            const uint32_t u = __shfl_up_sync(kFull, x, o);
            if (lane >= o) x += u;
        }
        if (lane < NT / 32) sh.wb[lane] = x - t;               // exclusive prefix of warp `lane`
        if (lane == NT / 32 - 1) sh.bc[3] = x;
    }
    __syncthreads();
    const uint32_t before = sh.wb[warp];
    *total = sh.bc[3];
    __syncthreads();   // wa, wb and bc[3] are rewritten by the next call
    return before + incl - v;
}

// The threshold bin c of the histogram for `need` (0 < need <= total):
// above(c) < need <= above(c) + h[c].  Thread t owns the kBins / NT bins just
// below kBins - t * (kBins / NT), so descending bins follow ascending threads.
template <int NT>
__device__ __forceinline__ void threshold(Smem<NT>& sh, uint32_t need, uint32_t& c, uint32_t& above,
                                          uint32_t& eq) {
    constexpr int per = kBins / NT;
    const int tid = threadIdx.x;
    const int lo = kBins - per * (tid + 1);
    uint32_t bins[per], sum = 0;
#pragma unroll
    for (int k = 0; k < per; ++k) {
        bins[k] = sh.hist[lo + k];
        sum += bins[k];
    }
    uint32_t total;
    const uint32_t excl = excl_scan<NT>(sum, sh, &total);
    if (excl < need && need <= excl + sum) {
        uint32_t a = excl;
#pragma unroll
        for (int k = per - 1; k >= 0; --k) {
            if (need <= a + bins[k]) {
                sh.bc[0] = (uint32_t)(lo + k);
                sh.bc[1] = a;
                sh.bc[2] = bins[k];
                break;
            }
            a += bins[k];
        }
    }
    __syncthreads();
    c = sh.bc[0];
    above = sh.bc[1];
    eq = sh.bc[2];
    __syncthreads();   // bc is rewritten by the next call
}

// Histogram of one digit over the list entries i < n (all threads).
template <int NT>
__device__ __forceinline__ void list_hist(Smem<NT>& sh, int n, uint32_t kmin, int s, uint32_t prefix_mask,
                                          uint32_t prefix) {
    for (int i = threadIdx.x; i < kBins; i += NT) sh.hist[i] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += NT) {
        const uint32_t rel = sh.lkey[i] - kmin;
        if ((rel & prefix_mask) == prefix) atomicAdd(&sh.hist[(rel >> s) & (kBins - 1)], 1u);
    }
    __syncthreads();
}

// First-level bin of a key: its distance from the largest key kmax on a
// floating scale, 64 bins per power of two (0 for the largest key itself).
// Monotone: a larger key never gets a larger bin.
__device__ __forceinline__ uint32_t dist_bin(uint32_t kmax, uint32_t key) {
    const uint32_t d = kmax - key;
    const uint32_t e = 31u - (uint32_t)__clz(d | 1u);      // bit length - 1
    const uint32_t sh = e > 6u ? e - 6u : 0u;
    const uint32_t far = ((e - 5u) << 6) | ((d >> sh) & 63u);
    return d < 64u ? d : far;                            // bins 0..63 hold the distance itself
}

// Smallest and largest distance of a dist_bin bin (the inverse of dist_bin).
__device__ __forceinline__ uint32_t bin_start(uint32_t b) {
    if (b < 64u) return b;
    const uint32_t e = (b >> 6) + 5u, m = b & 63u;               // distance in [2^e, 2^(e+1))
    return (64u | m) << (e - 6u);
}
__device__ __forceinline__ uint32_t bin_end(uint32_t b) {
    if (b < 64u) return b;
    const uint32_t e = (b >> 6) + 5u;
    return bin_start(b) + ((1u << (e - 6u)) - 1u);
}

// Sum of one value per thread over the block (every thread gets it).
template <int NT>
__device__ __forceinline__ uint32_t block_sum(uint32_t v, Smem<NT>& sh) {
    uint32_t total;
    excl_scan<NT>(v, sh, &total);
    return total;
}

template <int NT, int E>
__device__ uint32_t select_mask_hist(const uint32_t (&key)[E], uint32_t need, Smem<NT>& sh);

// Mark in sh.take the `rem` largest of the n list entries (0 < rem < n; ties
// in list order): radix levels on digits of (key - smallest list key).
template <int NT>
__device__ void resolve_list(Smem<NT>& sh, int n, uint32_t rem) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t lmin = 0xFFFFFFFFu, lmax = 0u;
    for (int i = tid; i < n; i += NT) {
        lmin = min(lmin, sh.lkey[i]);
        lmax = max(lmax, sh.lkey[i]);
    }
    lmin = __reduce_min_sync(kFull, lmin);
    lmax = __reduce_max_sync(kFull, lmax);
    if (lane == 0) {
        sh.wb[warp] = lmin;
        sh.wc[warp] = lmax;
    }
    __syncthreads();
    lmin = 0xFFFFFFFFu;
    lmax = 0u;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        lmin = min(lmin, sh.wb[w]);
        lmax = max(lmax, sh.wc[w]);
    }
    const uint32_t R = lmax - lmin;
    const int nb = R ? 32 - __clz(R) : 0;
    int s = nb;                                      // bits at and above s are equal in every entry in play
    uint32_t pmask = nb >= 32 ? 0u : ~0u << nb, prefix = 0u;
    bool done = false;
    while (!done) {
        const int s2 = s > 11 ? s - 11 : 0;
        list_hist<NT>(sh, n, lmin, s2, pmask, prefix);
        uint32_t c2, a2, e2;
        threshold<NT>(sh, rem, c2, a2, e2);
        const bool all2 = e2 == rem - a2;
        const bool last = s2 == 0;
        // take the entries above c2 (and at c2 when they are all needed); at
        // the last digit the entries at c2 are exact ties: the first rem - a2
        // of them in list order
        for (int i = tid; i < n; i += NT) {
            const uint32_t rel = sh.lkey[i] - lmin;
            if ((rel & pmask) != prefix) continue;
            const uint32_t d = (rel >> s2) & (kBins - 1);
            bool tk = d > c2 || (d == c2 && all2);
            if (!tk && d == c2 && last) {
                uint32_t rank = 0;
                for (int k = 0; k < i; ++k) {
                    const uint32_t rk = sh.lkey[k] - lmin;
                    rank += (rk & pmask) == prefix && ((rk >> s2) & (kBins - 1)) == c2;
                }
                tk = rank < rem - a2;
            }
            if (tk) atomicOr(&sh.take[sh.lref[i] >> 5], 1u << (sh.lref[i] & 31u));
        }
        rem -= a2;
        done = all2 || last;
        pmask = ~0u << s2;
        prefix = prefix | (c2 << s2);
        s = s2;
        __syncthreads();
    }
}

// Bit e of the result is set when this thread's element e is among the `need`
// largest keys of the block (fewer when fewer are valid).
template <int NT, int E>
__device__ uint32_t select_mask(const uint32_t (&key)[E], uint32_t need, Smem<NT>& sh) {
    static_assert(E <= 32, "at most 32 elements per thread");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t valid = 0u, kmax = 0u;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        valid |= (uint32_t)(key[e] != 0u) << e;
        kmax = max(kmax, key[e]);
    }
    uint32_t cnt = __reduce_add_sync(kFull, (uint32_t)__popc(valid));
    kmax = __reduce_max_sync(kFull, kmax);
    if (lane == 0) {
        sh.wa[warp] = cnt;
        sh.wc[warp] = kmax;
    }
    for (int i = tid; i < kBins; i += NT) sh.hist[i] = 0u;
    sh.take[tid] = 0u;
    __syncthreads();
    cnt = 0;
    kmax = 0u;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        cnt += sh.wa[w];
        kmax = max(kmax, sh.wc[w]);
    }
    if (need >= cnt || need == 0) {
        __syncthreads();
        return need ? valid : 0u;
    }
    // ---- 1. a sample: element tid % E of every thread (an unrolled select,
    // no dynamically indexed register array)
    uint32_t ks = 0u;
#pragma unroll
    for (int e = 0; e < E; ++e) ks = (e == tid % E) ? key[e] : ks;
    if (ks) atomicAdd(&sh.hist[kBins - 1 - dist_bin(kmax, ks)], 1u);
    __syncthreads();
    const uint32_t ns = block_sum<NT>((uint32_t)(ks != 0u), sh);
    const float f = (float)need / (float)cnt;
    const float rs = f * (float)ns;
    const float m = 4.0f + 3.0f * sqrtf(rs * (1.0f - f));
    const uint32_t r_hi = (uint32_t)fmaxf(1.0f, floorf(rs - m));
    const uint32_t r_lo = (uint32_t)fminf((float)ns, ceilf(rs + m));
    uint32_t c_hi = 0, c_lo = 0, a_tmp, e_tmp;
    bool sampled = ns > 0 && r_hi <= r_lo;
    if (sampled) {
        threshold<NT>(sh, r_hi, c_hi, a_tmp, e_tmp);
        threshold<NT>(sh, r_lo, c_lo, a_tmp, e_tmp);
    }
    const uint32_t bh = kBins - 1 - c_hi, bl = kBins - 1 - c_lo;   // distance bins, bh <= bl
    // bins are monotone in the key: bin < bh <=> key > k_take, bin <= bl <=> key >= k_lo
    const uint32_t k_take = kmax - bin_start(bh) + 1u;           // keys at or above are nearer than bh
    const uint32_t k_lo = bin_end(bl) >= kmax ? 1u : kmax - bin_end(bl);   // keys at or above: a bin <= bl
    // ---- 2. one pass over every element: taken (key >= k_take), candidate (k_lo <= key < k_take)
    uint32_t take = 0u, cand = 0u;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        take |= (uint32_t)(key[e] != 0u && key[e] >= k_take) << e;
        cand |= (uint32_t)(key[e] != 0u && key[e] >= k_lo && key[e] < k_take) << e;
    }
    uint32_t A = 0, B = 0;
    uint32_t slot = 0;
    if (sampled) {
        // counts fit 16 bits (at most 1024 * 32 elements): one scan of both
        uint32_t tot;
        const uint32_t pre = excl_scan<NT>((uint32_t)__popc(take) | ((uint32_t)__popc(cand) << 16), sh, &tot);
        A = tot & 0xFFFFu;
        B = tot >> 16;
        slot = pre >> 16;
    }
    if (sampled && A < need && need <= A + B && B <= (uint32_t)kList) {
        // ---- 3. compact the candidates, resolve need - A among them
        uint32_t cm = cand;
        while (cm) {
            const int e = __ffs(cm) - 1;
            cm &= cm - 1u;
            uint32_t ke = 0u;
#pragma unroll
            for (int k = 0; k < E; ++k) ke = (k == e) ? key[k] : ke;
            sh.lkey[slot] = ke;
            sh.lref[slot] = ((uint32_t)tid << 5) | (uint32_t)e;
            ++slot;
        }
        __syncthreads();
        const uint32_t rem = need - A;
        if (rem == B) {
            take |= cand;
        } else {
            resolve_list<NT>(sh, (int)B, rem);
            take |= sh.take[tid];
        }
        __syncthreads();
        return take;
    }
    __syncthreads();
    return select_mask_hist<NT, E>(key, need, sh);
}

// The selection with a histogram of every element's bin at the first level
// (the fallback of select_mask).  Same contract as select_mask.
template <int NT, int E>
__device__ uint32_t select_mask_hist(const uint32_t (&key)[E], uint32_t need, Smem<NT>& sh) {
    static_assert(E <= 32, "at most 32 elements per thread");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t cnt = 0, kmax = 0u, valid = 0u;
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (key[e]) {
            ++cnt;
            kmax = max(kmax, key[e]);
            valid |= 1u << e;
        }
    cnt = __reduce_add_sync(kFull, cnt);
    kmax = __reduce_max_sync(kFull, kmax);
    if (lane == 0) {
        sh.wa[warp] = cnt;
        sh.wc[warp] = kmax;
    }
    for (int i = tid; i < kBins; i += NT) sh.hist[i] = 0u;
    if (tid == 0) sh.nlist = 0u;
    sh.take[tid] = 0u;
    __syncthreads();
    cnt = 0;
    kmax = 0u;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        cnt += sh.wa[w];
        kmax = max(kmax, sh.wc[w]);
    }
    if (need >= cnt || need == 0) {
        __syncthreads();
        return need ? valid : 0u;
    }

    // ---- level 1 over every element: bins of the distance from the maximum
    // (bin 0 = nearest); the threshold is found on the reversed index so
    // that "above" counts the nearer bins
#pragma unroll
    for (int e = 0; e < E; ++e)
        if ((valid >> e) & 1u) atomicAdd(&sh.hist[kBins - 1 - dist_bin(kmax, key[e])], 1u);
    __syncthreads();
    uint32_t c, above, eq;
    threshold<NT>(sh, need, c, above, eq);
    const uint32_t cb = kBins - 1 - c;                   // the threshold bin as a distance bin
    uint32_t take = 0u, inplay = 0u;
    const bool all_eq = eq == need - above;
    const bool compact = !all_eq && eq <= (uint32_t)kList;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        if (!((valid >> e) & 1u)) continue;
        const uint32_t bn = dist_bin(kmax, key[e]);
        if (bn < cb || (bn == cb && all_eq)) {
            take |= 1u << e;
        } else if (bn == cb) {
            if (compact) {
                const uint32_t slot = atomicAdd(&sh.nlist, 1u);
                sh.lkey[slot] = key[e];
                sh.lref[slot] = ((uint32_t)tid << 5) | (uint32_t)e;
            } else {
                inplay |= 1u << e;
            }
        }
    }
    if (all_eq) {
        __syncthreads();
        return take;
    }
    uint32_t rem = need - above;

    // the keys still in play lie between the smallest and largest key of bin cb
    if (compact) {
        // ---- later levels over the list of the eq candidates of bin cb
        __syncthreads();
        resolve_list<NT>(sh, (int)eq, rem);
        take |= sh.take[tid];
        __syncthreads();
        return take;
    }

    // ---- later levels over the registers (more than kList keys in bin cb):
    // radix digits of (key - kmin_in_play), 11 bits at a time
    uint32_t pmin = 0xFFFFFFFFu, pmax = 0u;
#pragma unroll
    for (int e = 0; e < E; ++e)
        if ((inplay >> e) & 1u) {
            pmin = min(pmin, key[e]);
            pmax = max(pmax, key[e]);
        }
    pmin = __reduce_min_sync(kFull, pmin);
    pmax = __reduce_max_sync(kFull, pmax);
    if (lane == 0) {
        sh.wb[warp] = pmin;
        sh.wc[warp] = pmax;
    }
    __syncthreads();
    pmin = 0xFFFFFFFFu;
    pmax = 0u;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        pmin = min(pmin, sh.wb[w]);
        pmax = max(pmax, sh.wc[w]);
    }
    const uint32_t R = pmax - pmin;
    int s = R ? 32 - __clz(R) : 0;
    while (s > 0) {
        s = s > 11 ? s - 11 : 0;
        __syncthreads();                                 // hist is free again
        for (int i = tid; i < kBins; i += NT) sh.hist[i] = 0u;
        __syncthreads();
#pragma unroll
        for (int e = 0; e < E; ++e)
            if ((inplay >> e) & 1u) atomicAdd(&sh.hist[((key[e] - pmin) >> s) & (kBins - 1)], 1u);
        __syncthreads();
        uint32_t c2, a2, e2;
        threshold<NT>(sh, rem, c2, a2, e2);
        const bool all2 = e2 == rem - a2;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            if (!((inplay >> e) & 1u)) continue;
            const uint32_t d = ((key[e] - pmin) >> s) & (kBins - 1);
            if (d > c2 || (d == c2 && all2)) {
                take |= 1u << e;
                inplay &= ~(1u << e);
            } else if (d < c2) {
                inplay &= ~(1u << e);
            }
        }
        rem -= a2;
        if (all2) return take;
    }
    // exact ties at the cutoff: the first `rem` in claim order
    uint32_t total;
    uint32_t rank = excl_scan<NT>((uint32_t)__popc(inplay), sh, &total);
#pragma unroll
    for (int e = 0; e < E; ++e)
        if ((inplay >> e) & 1u) {
            if (rank < rem) take |= 1u << e;
            ++rank;
        }
    return take;
}

// Write the selected elements' ids (id_of(e) for this thread's element e;
// and, with vals, their scores) to out[0..) in claim order, then -1 up to
// n_out.  Returns the number written.
template <int NT, int E, typename IdOf>
__device__ uint32_t write_selected(uint32_t take, const uint32_t (&key)[E], IdOf id_of, int32_t* out, float* vals,
                                   int n_out, Smem<NT>& sh) {
    uint32_t total;
    uint32_t pos = excl_scan<NT>((uint32_t)__popc(take), sh, &total);
#pragma unroll
    for (int e = 0; e < E; ++e)
        if ((take >> e) & 1u) {
            out[pos] = id_of(e);
            if (vals) vals[pos] = key_score(key[e]);
            ++pos;
        }
    for (int i = (int)total + threadIdx.x; i < n_out; i += NT) out[i] = -1;
    return total;
}

// Index of element e of this thread in the layout the loaders use: with E a
// multiple of 4, groups of four consecutive elements per thread, so that they
// can be read with one 16-byte load -- element (e / 4) * 4 NT + 4 tid + e % 4;
// otherwise element e * NT + tid.  Either way the NT * E indices are covered once.
template <int NT, int E>
__device__ __forceinline__ int elem_index(int e) {
    if (E % 4 == 0) return (e >> 2) * (4 * NT) + 4 * (int)threadIdx.x + (e & 3);
    return e * NT + (int)threadIdx.x;
}

// The same with the ids in registers.
template <int NT, int E>
__device__ uint32_t write_selected(uint32_t take, const uint32_t (&key)[E], const int32_t (&id)[E], int32_t* out,
                                   float* vals, int n_out, Smem<NT>& sh) {
    uint32_t total;
    uint32_t pos = excl_scan<NT>((uint32_t)__popc(take), sh, &total);
#pragma unroll
    for (int e = 0; e < E; ++e)
        if ((take >> e) & 1u) {
            out[pos] = id[e];
            if (vals) vals[pos] = key_score(key[e]);
            ++pos;
        }
    for (int i = (int)total + threadIdx.x; i < n_out; i += NT) out[i] = -1;
    return total;
}

}  // namespace lsel
}  // namespace csa2

// Context-parallel decode: the per-rank steps around the exchanges when the
// positions of one sequence are spread over several devices (tldrocket.com,
// "DeepSeek AI Released DeepSeek-V4.1-Flash with 1M Context, FP4 KV Cache, and
// Cross-Layer Attention Reuse", paragraphs 1 and 3; zerohour.day: a context of
// one million tokens).  Scoring, selection and attention on a shard are the
// single-device kernels; what is here maps positions between a shard and the
// sequence, reorders the all-gathered candidates per sequence, builds the
// shard's part of the attended set and merges the attention parts.
//
// All of it is a few hundred KB per layer at most: plain coalesced
// element-per-thread kernels, launched with programmatic dependent launch.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

namespace {

constexpr int kThreads = 256;

unsigned blocks_for(int64_t n) { return (unsigned)((n + kThreads - 1) / kThreads); }

// cand[b][i] <- (ids[b][i] + pos0[b], vals[b][i]) for a selected entry, (-1, 0)
// for padding.
__global__ void __launch_bounds__(kThreads)
k_cp_pack(const int32_t* __restrict__ ids, const float* __restrict__ vals, int64_t in_stride,
          const int32_t* __restrict__ pos0, int batch, int n, CpCand* __restrict__ cand) {
    pdl_begin();
    const int64_t e = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (e >= (int64_t)batch * n) return;
    const int b = (int)(e / n), i = (int)(e % n);
    const int32_t id = ids[b * in_stride + i];
    CpCand c;
    c.pos = id >= 0 ? id + __ldg(pos0 + b) : -1;
    c.score = id >= 0 ? vals[b * in_stride + i] : 0.0f;
    cand[e] = c;
}

// local[b][i] <- the shard position of global pool entry pool[b][i] when the
// shard holds it, else -1.
__global__ void __launch_bounds__(kThreads)
k_cp_localize(const int32_t* __restrict__ pool, const int32_t* __restrict__ pos0,
              const int32_t* __restrict__ shard_lens, int batch, int n, int32_t* __restrict__ local) {
    pdl_begin();
    const int64_t e = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (e >= (int64_t)batch * n) return;
    const int b = (int)(e / n);
    const int64_t t = (int64_t)pool[e] - __ldg(pos0 + b);
    local[e] = (pool[e] >= 0 && t >= 0 && t < __ldg(shard_lens + b)) ? (int32_t)t : -1;
}

// A Reindex layer's share of the pool scores: out[b][i] <- the score of pool
// entry i when this shard holds it (NaN when the shard could not score it),
// 0 when another shard holds it or it is padding.  Summed over the ranks (an
// all-reduce), every entry then carries its owner's score exactly: the other
// terms are zeros.
__global__ void __launch_bounds__(kThreads)
k_cp_owned_scores(const int32_t* __restrict__ local, const float* __restrict__ sc, int64_t n,
                  float* __restrict__ out) {
    pdl_begin();
    const int64_t e = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (e >= n) return;
    out[e] = local[e] >= 0 ? sc[e] : 0.0f;
}

// All-gathered candidates [R][batch][n] -> per sequence [batch][R * n]: ids
// and scores in the layout the selection kernels read.
__global__ void __launch_bounds__(kThreads)
k_cp_unpack(const CpCand* __restrict__ cand, int R, int batch, int n, int32_t* __restrict__ ids,
            float* __restrict__ vals) {
    pdl_begin();
    const int64_t e = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t m = (int64_t)R * n;
    if (e >= (int64_t)batch * m) return;
    const int64_t b = e / m, k = e % m;
    const int64_t r = k / n, i = k % n;
    const CpCand c = cand[(r * batch + b) * n + i];
    ids[e] = c.pos;
    vals[e] = c.score;
}

// The shard's part of the attended set of the query at p = Lg[b] - 1, in
// shard positions: entries [0, window) are the window positions p - window +
// 1 + i that the shard holds, entries [window, window + top_k) the top-k
// entries before the window that it holds; -1 elsewhere.  The window and the
// top-k part are disjoint, so the attention over the list (no window of its
// own) counts every position of S ∩ shard once.
__global__ void __launch_bounds__(kThreads)
k_cp_attn_list(const int32_t* __restrict__ topk, int top_k, int window, const int32_t* __restrict__ pos0,
               const int32_t* __restrict__ shard_lens, const int32_t* __restrict__ lens_global, int batch,
               int32_t* __restrict__ list, uint32_t* __restrict__ status) {
    pdl_begin();
    const int n = window + top_k;
    const int64_t e = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (e >= (int64_t)batch * n) return;
    const int b = (int)(e / n), i = (int)(e % n);
    const int64_t Lg = __ldg(lens_global + b);
    const int64_t p = Lg - 1;
    const int64_t w0 = p - window + 1 > 0 ? p - window + 1 : 0;
    int64_t g = -1;
    if (i < window) {
        g = w0 + i;
        if (g > p) g = -1;
    } else {
        const int32_t t = topk[(int64_t)b * top_k + (i - window)];
        if (t < -1 || t >= Lg) flag(status, kStatusBounds);
        else if (t >= 0 && t < w0) g = t;
    }
    const int64_t s = g - __ldg(pos0 + b);
    list[e] = (g >= 0 && s >= 0 && s < __ldg(shard_lens + b)) ? (int32_t)s : -1;
}

// out[b][h][d] = sum_r exp(lse_r - lse) out_r[b][h][d], lse = log sum_r
// exp(lse_r), one thread per output element.  The parts are taken kMergeU at a
// time, every load of a group issued before any is used, and merged online
// (running maximum m, sum and accumulator rescaled by exp(m_old - m_new)).
constexpr int kMergeU = 8;

__global__ void __launch_bounds__(kThreads)
k_lse_merge(int R, int batch, int H, int D, const float* __restrict__ outs, int64_t out_stride,
            const float* __restrict__ lses, int64_t lse_stride, float* __restrict__ out, float* __restrict__ lse) {
    pdl_begin();
    const int64_t e = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (e >= (int64_t)batch * H * D) return;
    const int64_t bh = e / D;
    const int d = (int)(e % D);
    float m = -INFINITY, sum = 0.0f, acc = 0.0f;
    for (int r0 = 0; r0 < R; r0 += kMergeU) {
        float l[kMergeU], o[kMergeU];
#pragma unroll
        for (int k = 0; k < kMergeU; ++k) {
            const bool in = r0 + k < R;
            l[k] = in ? lses[(r0 + k) * lse_stride + bh] : -INFINITY;
            o[k] = in ? outs[(r0 + k) * out_stride + e] : 0.0f;
        }
        float mn = m;
#pragma unroll
        for (int k = 0; k < kMergeU; ++k) mn = fmaxf(mn, l[k]);
        if (mn == -INFINITY) continue;                 // nothing attended so far
        const float c = expf(m - mn);                  // 0 while m is -inf
        sum *= c;
        acc *= c;
#pragma unroll
        for (int k = 0; k < kMergeU; ++k) {
            const float wk = expf(l[k] - mn);          // 0 for an empty part
            sum += wk;
            acc += wk * o[k];
        }
        m = mn;
    }
    out[e] = m == -INFINITY ? 0.0f : acc / sum;
    if (lse && d == 0) lse[bh] = m == -INFINITY ? -INFINITY : m + logf(sum);
}

}  // namespace

cudaError_t launch_cp_pack(const int32_t* ids, const float* vals, int64_t in_stride, const int32_t* pos0, int batch,
                           int n, CpCand* cand, cudaStream_t st) {
    return launch_pdl(k_cp_pack, dim3(blocks_for((int64_t)batch * n)), dim3(kThreads), 0, st, ids, vals, in_stride,
                      pos0, batch, n, cand);
}

cudaError_t launch_cp_localize(const int32_t* pool, const int32_t* pos0, const int32_t* shard_lens, int batch, int n,
                               int32_t* local, cudaStream_t st) {
    return launch_pdl(k_cp_localize, dim3(blocks_for((int64_t)batch * n)), dim3(kThreads), 0, st, pool, pos0,
                      shard_lens, batch, n, local);
}

cudaError_t launch_cp_owned_scores(const int32_t* local, const float* sc, int64_t n, float* out, cudaStream_t st) {
    return launch_pdl(k_cp_owned_scores, dim3(blocks_for(n)), dim3(kThreads), 0, st, local, sc, n, out);
}

cudaError_t launch_cp_unpack(const CpCand* cand, int R, int batch, int n, int32_t* ids, float* vals,
                             cudaStream_t st) {
    return launch_pdl(k_cp_unpack, dim3(blocks_for((int64_t)batch * R * n)), dim3(kThreads), 0, st, cand, R, batch,
                      n, ids, vals);
}

cudaError_t launch_cp_attn_list(const int32_t* topk, int top_k, int window, const int32_t* pos0,
                                const int32_t* shard_lens, const int32_t* lens_global, int batch, int32_t* list,
                                uint32_t* status, cudaStream_t st) {
    return launch_pdl(k_cp_attn_list, dim3(blocks_for((int64_t)batch * (window + top_k))), dim3(kThreads), 0, st,
                      topk, top_k, window, pos0, shard_lens, lens_global, batch, list, status);
}

cudaError_t launch_lse_merge(int R, int batch, int H, int D, const float* outs, int64_t out_stride, const float* lses,
                             int64_t lse_stride, float* out, float* lse, cudaStream_t st) {
    return launch_pdl(k_lse_merge, dim3(blocks_for((int64_t)batch * H * D)), dim3(kThreads), 0, st, R, batch, H, D,
                      outs, out_stride, lses, lse_stride, out, lse);
}

}  // namespace csa2

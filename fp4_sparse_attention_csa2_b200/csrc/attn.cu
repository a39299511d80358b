// Sparse + sliding-window attention over the FP4 global cache.
//
// Method: hackernews.kjhq.dev post 49735410, key point 2 (local sliding windows
// plus global sparse retrieval, layers sharing one main KV and its Top-K
// indices); tldrocket.com, "DeepSeek AI Released DeepSeek-V4.1-Flash with 1M
// Context, FP4 KV Cache, and Cross-Layer Attention Reuse", paragraphs 2-4
// (128-token window in every layer; E2M1 values with one E4M3 scale per 16
// channels).
//
// Each (sequence, query token) owns a virtual list of W + k entries: the W
// window positions p, p-1, ..., p-W+1 followed by its k top-k positions; a
// top-k position that lies in the window, is -1 or is beyond p is masked, so
// the attended set is window ∪ top-k without double counting.  The list is cut
// into chunks of kRows entries; one CTA gathers the FP4 rows of its chunk,
// dequantises them in shared memory and writes a partial (max, sum, unnormalised
// output) per head.  A second kernel merges the partials (split softmax).
// With a layer-local bf16 ring ([FANOUT] item 2) the window entries' rows are
// read from the ring instead (fp32 arithmetic: no range limit beyond fp32's).
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

namespace {

constexpr int kRows = 32;      // entries per CTA
constexpr int kThreads = 256;

__device__ __forceinline__ int32_t entry_position(const int32_t* topk, int top_k, int window, int64_t p, int64_t L,
                                                  int v, uint32_t* status) {
    if (v < window) {
        const int64_t t = p - v;
        return t >= 0 ? (int32_t)t : -1;
    }
    const int32_t t = __ldg(topk + (v - window));
    if (t < -1 || t >= L) { flag(status, kStatusBounds); return -1; }
    if (t < 0 || t > p || t > p - window) return -1;   // padding, future, or already in the window
    return t;
}

// grid (nchunk, batch*T); dynamic smem: H*(D+4) + kRows*(D+4) + H*kRows floats + kRows ints
__global__ void __launch_bounds__(kThreads)
k_attn_partial(DevCache c, const __nv_bfloat16* __restrict__ q, int T, int H, const int32_t* __restrict__ topk,
               int top_k, int window, float scale, const __nv_bfloat16* __restrict__ ring, int64_t ring_len,
               float* __restrict__ part_o, float* __restrict__ part_ml, int nchunk, uint32_t* status) {
    pdl_begin();
    extern __shared__ float smem[];
    const int D = c.dim;
    const int DP = D + 4;
    float* qs = smem;                      // [H][DP]
    float* vs = qs + H * DP;               // [kRows][DP]
    float* ps = vs + kRows * DP;           // [H][kRows]
    int* pos = reinterpret_cast<int*>(ps + H * kRows);
    const int seg = blockIdx.y, chunk = blockIdx.x;
    const int b = seg / T, j = seg % T;
    const int64_t L = seq_len(c, b, status);
    const int64_t p = L - T + j;

    if (threadIdx.x < kRows) {
        const int v = chunk * kRows + threadIdx.x;
        int32_t t = -1;
        if (p >= 0 && v < window + top_k)
            t = entry_position(topk + (int64_t)seg * top_k, top_k, window, p, L, v, status);
        pos[threadIdx.x] = t;
    }
    const __nv_bfloat16* qg = q + (int64_t)seg * H * D;
    for (int i = threadIdx.x; i < H * D; i += kThreads) qs[(i / D) * DP + i % D] = __bfloat162float(qg[i]);
    __syncthreads();

    // gather + dequantise: one thread per 16-channel block of one row
    const int nblk = D >> 4;
    for (int w = threadIdx.x; w < kRows * nblk; w += kThreads) {
        const int r = w / nblk, blk = w % nblk;
        float* dst = vs + r * DP + blk * 16;
        const int32_t t = pos[r];
        if (ring && t >= 0 && chunk * kRows + r < window) {
            // a window entry: this layer's bf16 row, ring slot t mod ring_len
            const uint4* src = reinterpret_cast<const uint4*>(ring + ((int64_t)b * ring_len + t % ring_len) * D + blk * 16);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4 u = __ldg(src + h);
                const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    dst[h * 8 + 2 * k] = __uint_as_float(wv[k] << 16);
                    dst[h * 8 + 2 * k + 1] = __uint_as_float(wv[k] & 0xFFFF0000u);
                }
            }
            continue;
        }
        int64_t slot = t >= 0 ? slot_of(c, b, t) : -1;
        if (t >= 0 && slot < 0) flag(status, kStatusBounds);
        if (slot < 0) {
#pragma unroll
            for (int k = 0; k < 16; ++k) dst[k] = 0.0f;
            continue;
        }
        const uint8_t* row = c.rows + slot * c.row_stride;
        const uint2 codes = *reinterpret_cast<const uint2*>(row + blk * 8);
        const float s = e4m3_to_float(row[(D >> 1) + blk]);
        const uint32_t cw[2] = {codes.x, codes.y};
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float2 f = __half22float2(e2m1x2_to_half2((uint8_t)(cw[h] >> (8 * k))));
                dst[h * 8 + 2 * k] = f.x * s;
                dst[h * 8 + 2 * k + 1] = f.y * s;
            }
    }
    __syncthreads();

    // logits z[h][r] = scale * q_h . v_r ; thread (h, rg) handles rows rg, rg+4, ...
    for (int w = threadIdx.x; w < H * 4; w += kThreads) {
        const int h = w >> 2, rg = w & 3;
        float acc[kRows / 4];
#pragma unroll
        for (int i = 0; i < kRows / 4; ++i) acc[i] = 0.0f;
        const float* qh = qs + h * DP;
        for (int d = 0; d < D; d += 4) {
            const float4 qv = *reinterpret_cast<const float4*>(qh + d);
#pragma unroll
            for (int i = 0; i < kRows / 4; ++i) {
                const float4 vv = *reinterpret_cast<const float4*>(vs + (rg + 4 * i) * DP + d);
                acc[i] = fmaf(qv.x, vv.x, fmaf(qv.y, vv.y, fmaf(qv.z, vv.z, fmaf(qv.w, vv.w, acc[i]))));
            }
        }
#pragma unroll
        for (int i = 0; i < kRows / 4; ++i) {
            const int r = rg + 4 * i;
            ps[h * kRows + r] = pos[r] >= 0 ? acc[i] * scale * 1.4426950408889634f : -INFINITY;   // base 2
        }
    }
    __syncthreads();

    // per-head partial softmax statistics over this chunk
    float* ml = part_ml + ((int64_t)seg * nchunk + chunk) * H * 2;
    for (int h = threadIdx.x; h < H; h += kThreads) {
        float m = -INFINITY;
        for (int r = 0; r < kRows; ++r) m = fmaxf(m, ps[h * kRows + r]);
        float l = 0.0f;
        for (int r = 0; r < kRows; ++r) {
            const float e = m == -INFINITY ? 0.0f : exp2f(ps[h * kRows + r] - m);
            ps[h * kRows + r] = e;
            l += e;
        }
        ml[2 * h] = m;
        ml[2 * h + 1] = l;
    }
    __syncthreads();

    // unnormalised partial output O[h][d] = sum_r e[h][r] v_r[d]
    float* po = part_o + ((int64_t)seg * nchunk + chunk) * H * D;
    const int D4 = D >> 2;
    for (int w = threadIdx.x; w < H * D4; w += kThreads) {
        const int h = w / D4, d = (w % D4) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < kRows; ++r) {
            const float e = ps[h * kRows + r];
            const float4 vv = *reinterpret_cast<const float4*>(vs + r * DP + d);
            acc.x = fmaf(e, vv.x, acc.x);
            acc.y = fmaf(e, vv.y, acc.y);
            acc.z = fmaf(e, vv.z, acc.z);
            acc.w = fmaf(e, vv.w, acc.w);
        }
        *reinterpret_cast<float4*>(po + (int64_t)h * D + d) = acc;   // partials are [head][d]
    }
}

// Split-softmax merge.  Output (head h, channel d) of one (sequence, query
// token): with chunk c's partial output O_c[h][d] (not normalised) and its
// per-head (m_c, l_c) in base-2 units,
//     M = max_c m_c,  L = sum_c 2^(m_c - M) l_c,  out = sum_c 2^(m_c - M) O_c / L,
// lse = M ln 2 + ln L.  G consecutive threads share an output, thread `part`
// taking chunks part, part + G, ..; each thread issues all its loads at once
// (up to kBatch; indices clamped, so no load is conditional) and the G shares
// (M, L, acc) are combined by shuffles.  A warp's loads of one chunk are
// consecutive channels of one head.  grid (batch*T, ceil(H*D*G / 256)).
constexpr int kBatch = 18;

__device__ __forceinline__ void merge_part(const float* po, const float* ml, int nchunk, int part, int G, int64_t cs_o,
                                           int64_t cs_ml, float& M, float& Lsum, float& acc) {
    M = -INFINITY;
    Lsum = 0.0f;
    acc = 0.0f;
    for (int c0 = part; c0 < nchunk; c0 += kBatch * G) {
        float o[kBatch], m[kBatch], l[kBatch];
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const int ck = c0 + k * G;
            const int c = ck < nchunk ? ck : part;
            const float2 v = *reinterpret_cast<const float2*>(ml + (int64_t)c * cs_ml);
            o[k] = po[(int64_t)c * cs_o];
            m[k] = ck < nchunk ? v.x : -INFINITY;
            l[k] = v.y;
        }
        float mb = M;
#pragma unroll
        for (int k = 0; k < kBatch; ++k) mb = fmaxf(mb, m[k]);
        if (mb == -INFINITY) continue;                          // nothing attended so far
        const float rs = M == -INFINITY ? 0.0f : exp2f(M - mb);
        acc *= rs;
        Lsum *= rs;
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const float w = m[k] == -INFINITY ? 0.0f : exp2f(m[k] - mb);
            acc = fmaf(w, o[k], acc);
            Lsum = fmaf(w, l[k], Lsum);
        }
        M = mb;
    }
}

// Combine two shares (M, L, acc) of one output: both rescaled to the larger maximum.
__device__ __forceinline__ void merge_pair(float& M, float& Lsum, float& acc, float M2, float L2, float a2) {
    const float mb = fmaxf(M, M2);
    if (mb == -INFINITY) return;
    const float w1 = M == -INFINITY ? 0.0f : exp2f(M - mb), w2 = M2 == -INFINITY ? 0.0f : exp2f(M2 - mb);
    acc = acc * w1 + a2 * w2;
    Lsum = Lsum * w1 + L2 * w2;
    M = mb;
}

__global__ void __launch_bounds__(256)
k_attn_combine(int D, int H, const float* __restrict__ part_o, const float* __restrict__ part_ml, int nchunk, int G,
               float* __restrict__ out, float* __restrict__ lse) {
    pdl_begin();
    const int seg = blockIdx.x;
    const int t = blockIdx.y * 256 + threadIdx.x;
    const int part = t % G;
    const int nout = H * D;
    const int o = t / G;
    const int oc = o < nout ? o : nout - 1;                 // every lane takes part in the shuffles
    const int h = oc / D, d = oc - h * D;
    const int64_t cs_o = (int64_t)H * D, cs_ml = (int64_t)H * 2;
    float M, Lsum, acc;
    merge_part(part_o + (int64_t)seg * nchunk * cs_o + (int64_t)h * D + d,
               part_ml + (int64_t)seg * nchunk * cs_ml + (int64_t)h * 2, nchunk, part, G, cs_o, cs_ml, M, Lsum, acc);
    for (int x = 1; x < G; x <<= 1)
        merge_pair(M, Lsum, acc, __shfl_xor_sync(0xffffffffu, M, x), __shfl_xor_sync(0xffffffffu, Lsum, x),
                   __shfl_xor_sync(0xffffffffu, acc, x));
    if (o < nout && part == 0) {
        out[((int64_t)seg * H + h) * D + d] = Lsum > 0.0f ? acc / Lsum : 0.0f;
        if (lse && d == 0) lse[(int64_t)seg * H + h] = Lsum > 0.0f ? M * 0.6931471805599453f + logf(Lsum) : -INFINITY;
    }
}

}  // namespace

int attn_rows_per_chunk() { return kRows; }

cudaError_t launch_attn_combine(const DevCache& c, int T, int H, const AttnWork& aw, float* out, float* lse,
                                cudaStream_t st) {
    const int64_t nseg = (int64_t)c.batch * T;
    // threads per output: enough that each thread's chunks are one batch of loads
    int G = 1;
    while (G < 32 && aw.nchunk > kBatch * G) G <<= 1;
    const unsigned blocks = (unsigned)(((int64_t)H * c.dim * G + 255) / 256);
    return launch_pdl(k_attn_combine, dim3((unsigned)nseg, blocks), dim3(256), 0, st, c.dim, H, aw.part_o, aw.part_ml,
                      aw.nchunk, G, out, lse);
}

cudaError_t launch_attention(const DevCache& c, const void* q, int T, int H, const int32_t* topk, int top_k,
                             int window, float sm_scale, const Ring& ring, float* out, float* lse,
                             const AttnWork& aw_in, uint32_t* status, cudaStream_t st, int num_sms) {
    AttnWork aw = aw_in;
    cudaError_t e;
    if (attn_tc_supported(c, H)) {
        const int rows = attn_tc_rows_per_chunk();
        aw.nchunk = (window + top_k + rows - 1) / rows;
        if (aw.nchunk < 1) aw.nchunk = 1;
        e = launch_attention_tc(c, q, T, H, topk, top_k, window, sm_scale, ring, aw, status, st, num_sms);
    } else {
        const int D = c.dim;
        aw.nchunk = (window + top_k + kRows - 1) / kRows;
        if (aw.nchunk < 1) aw.nchunk = 1;
        const size_t smem = sizeof(float) * ((size_t)H * (D + 4) + (size_t)kRows * (D + 4) + (size_t)H * kRows) +
                            sizeof(int) * kRows;
        e = cudaFuncSetAttribute(k_attn_partial, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        dim3 grid((unsigned)aw.nchunk, (unsigned)(c.batch * T));
        e = launch_pdl(k_attn_partial, dim3(grid), dim3(kThreads), smem, st, c, static_cast<const __nv_bfloat16*>(q),
                       T, H, topk, top_k, window, sm_scale, ring.rows, ring.len, aw.part_o, aw.part_ml, aw.nchunk,
                       status);
    }
    if (e != cudaSuccess) return e;
    return launch_attn_combine(c, T, H, aw, out, lse, st);
}

}  // namespace csa2

namespace csa2 {

namespace {

// Rows of new tokens into a layer's ring: row i of sequence b (position
// start_pos[b] + i) to ring row (start_pos[b] + i) mod len.  One warp per row,
// 16-byte loads and stores.
__global__ void __launch_bounds__(256)
k_ring_append(__nv_bfloat16* __restrict__ ring, int64_t len, int batch, int dim, const __nv_bfloat16* __restrict__ x,
              const int32_t* __restrict__ start_pos, int n_new) {
    pdl_begin();
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= (int64_t)batch * n_new) return;
    const int b = (int)(row / n_new), i = (int)(row % n_new);
    const int64_t pos = (int64_t)__ldg(start_pos + b) + i;
    if (pos < 0) return;
    const uint4* src = reinterpret_cast<const uint4*>(x + row * dim);
    uint4* dst = reinterpret_cast<uint4*>(ring + ((int64_t)b * len + pos % len) * dim);
    for (int k = threadIdx.x & 31; k < dim / 8; k += 32) dst[k] = __ldg(src + k);
}

}  // namespace

cudaError_t launch_ring_append(const Ring& ring, int batch, int dim, const void* x, const int32_t* start_pos,
                               int n_new, cudaStream_t st) {
    const int64_t rows = (int64_t)batch * n_new;
    return launch_pdl(k_ring_append, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0, st,
                      ring.rows, ring.len, batch, dim,
                      static_cast<const __nv_bfloat16*>(x), start_pos, n_new);
}

}  // namespace csa2

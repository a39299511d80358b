// Indexer scoring on CUDA cores:  s_t = sum_h w_h * max(0, q_h . k_t).
//
// Role of the indexer: tldrocket.com, "DeepSeek AI Released DeepSeek-V4.1-Flash
// with 1M Context, FP4 KV Cache, and Cross-Layer Attention Reuse", paragraph 3
// (a Full layer scores the context into a pool of <= 16,384 positions, a
// Reindex layer rescores that pool); hackernews.kjhq.dev post 49735410, key
// point 3.  The scoring function itself is not given by the pages; this is the
// ReLU-gated, head-weighted dot product.
//
// Full scoring (fp32 keys): one thread scores one position for every query
// token of its sequence.  Pool scoring (Reindex): four threads share one pool
// entry, a quarter of the heads each (one thread per entry when many
// segments already fill the GPU).  The queries sit in shared memory as fp32
// and are read as broadcasts; the key (64 values) sits in registers.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

namespace {

constexpr int kDI = 64;

__device__ __forceinline__ void load_key(const DevCache& c, int64_t slot, float* k) {
    if (c.key_dtype == 2) {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(c.keys) + slot * kDI);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            uint4 u = __ldg(src + v);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float2 a = __half22float2(e4m3x2_to_half2((uint16_t)(w[q] & 0xFFFF)));
                float2 b = __half22float2(e4m3x2_to_half2((uint16_t)(w[q] >> 16)));
                k[v * 16 + q * 4 + 0] = a.x;
                k[v * 16 + q * 4 + 1] = a.y;
                k[v * 16 + q * 4 + 2] = b.x;
                k[v * 16 + q * 4 + 3] = b.y;
            }
        }
    } else {
        const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(c.keys) + slot * kDI);
#pragma unroll
        for (int v = 0; v < 16; ++v) {
            float4 f = __ldg(src + v);
            k[4 * v] = f.x; k[4 * v + 1] = f.y; k[4 * v + 2] = f.z; k[4 * v + 3] = f.w;
        }
    }
}

__device__ __forceinline__ float query_value(const void* q, int q_f32, int64_t i) {
    return q_f32 ? static_cast<const float*>(q)[i] : __bfloat162float(static_cast<const __nv_bfloat16*>(q)[i]);
}

__device__ __forceinline__ float score_one(const float* qs, const float* hw, int H_I, const float* k) {
    float s = 0.0f;
    for (int h = 0; h < H_I; ++h) {
        const float* qh = qs + h * kDI;
        float dot = 0.0f;
#pragma unroll
        for (int d = 0; d < kDI; ++d) dot = fmaf(qh[d], k[d], dot);
        s = fmaf(hw[h], fmaxf(dot, 0.0f), s);
    }
    return s;
}

// grid (ceil(cap / 256), batch); dynamic smem: T*H_I*64 + T*H_I floats
__global__ void __launch_bounds__(256)
k_score_full(DevCache c, const void* __restrict__ q, int q_f32, const float* __restrict__ hw, int T, int H_I,
             float* __restrict__ scores, uint32_t* status) {
    pdl_begin();
    extern __shared__ float smem[];
    float* qs = smem;
    float* ws = smem + T * H_I * kDI;
    const int b = blockIdx.y;
    const int64_t qoff = (int64_t)b * T * H_I * kDI;
    for (int i = threadIdx.x; i < T * H_I * kDI; i += blockDim.x) qs[i] = query_value(q, q_f32, qoff + i);
    for (int i = threadIdx.x; i < T * H_I; i += blockDim.x) ws[i] = hw[(int64_t)b * T * H_I + i];
    __syncthreads();
    const int64_t L = seq_len(c, b, status);
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= L) return;
    const int64_t slot = slot_of(c, b, t);
    if (slot < 0) {
        // a page outside the cache: the position is skipped (NaN is never selected)
        flag(status, kStatusBounds);
        for (int j = 0; j < T; ++j)
            if (t <= L - T + j) scores[((int64_t)b * T + j) * c.cap + t] = __int_as_float(0x7fc00000);
        return;
    }
    float k[kDI];
    load_key(c, slot, k);
    for (int j = 0; j < T; ++j) {
        if (t > L - T + j) continue;  // causal among the T query tokens
        scores[((int64_t)b * T + j) * c.cap + t] = score_one(qs + j * H_I * kDI, ws + j * H_I, H_I, k);
    }
}

// Pool scoring: SPLIT consecutive threads share one pool entry, each taking
// every SPLIT-th head, and add their parts with shuffles (SPLIT = 4 spreads a
// single 16,384-entry pool over every SM; SPLIT = 1 when many segments
// already fill the GPU, so no key is converted twice).  A CTA of 256 threads
// covers 256 / SPLIT entries.  The queries sit in shared memory with a row
// pitch of kQPitch floats, so the SPLIT heads read at once fall in different
// banks.  Dynamic smem: H_I * kQPitch + H_I floats.
constexpr int kQPitch = kDI + 4;

template <int SPLIT>
__global__ void __launch_bounds__(256)
k_score_pool(DevCache c, const void* __restrict__ q, int q_f32, const float* __restrict__ hw, int T, int H_I,
             const int32_t* __restrict__ pool, int pool_k, float* __restrict__ scores, uint32_t* status) {
    pdl_begin();
    extern __shared__ float smem[];
    float* qs = smem;
    float* ws = smem + H_I * kQPitch;
    const int seg = blockIdx.y;
    const int b = seg / T, j = seg % T;
    for (int i = threadIdx.x; i < H_I * kDI; i += blockDim.x)
        qs[(i / kDI) * kQPitch + i % kDI] = query_value(q, q_f32, (int64_t)seg * H_I * kDI + i);
    for (int i = threadIdx.x; i < H_I; i += blockDim.x) ws[i] = hw[(int64_t)seg * H_I + i];
    __syncthreads();
    const int64_t L = seq_len(c, b, status);
    const int part = threadIdx.x % SPLIT;
    // the SPLIT threads of an entry sit in one warp and stay together to the shuffles
    const int i = blockIdx.x * (256 / SPLIT) + threadIdx.x / SPLIT;
    bool live = i < pool_k;
    int64_t slot = -1;
    if (live) {
        const int32_t t = pool[(int64_t)seg * pool_k + i];
        if (t < 0) {
            live = false;
        } else if (t > L - T + j) {
            if (part == 0) flag(status, kStatusBounds);
            live = false;
        } else {
            slot = slot_of(c, b, t);
            if (slot < 0) {
                if (part == 0) flag(status, kStatusBounds);
                live = false;
            }
        }
    }
    float s = 0.0f;
    if (live) {
        float k[kDI];
        load_key(c, slot, k);
        for (int h = part; h < H_I; h += SPLIT) {
            const float* qh = qs + h * kQPitch;
            float dot = 0.0f;
#pragma unroll
            for (int d = 0; d < kDI; ++d) dot = fmaf(qh[d], k[d], dot);
            s = fmaf(ws[h], fmaxf(dot, 0.0f), s);
        }
    }
#pragma unroll
    for (int o = 1; o < SPLIT; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    // every entry gets a value: NaN marks one that is padding or was skipped,
    // and the selection never takes it (nothing stale from an earlier call is read)
    if (i < pool_k && part == 0) scores[(int64_t)seg * pool_k + i] = live ? s : __int_as_float(0x7fc00000);
}

// One thread per candidate slot; grid (ceil(m / 256), batch * T).
__global__ void __launch_bounds__(256)
k_pool_candidates(DevCache c, int T, const int32_t* __restrict__ pool_prev, int pool_k, int n_new,
                  int32_t* __restrict__ ids, uint32_t* status) {
    pdl_begin();
    const int seg = blockIdx.y, b = seg / T, j = seg % T;
    const int m = pool_k + n_new;
    const int i = blockIdx.x * 256 + threadIdx.x;
    if (i >= m) return;
    const int64_t L = seq_len(c, b, status);
    const int64_t p = L - T + j, t_new0 = L - n_new;
    int32_t t = -1;
    if (i < pool_k) {
        t = pool_prev[(int64_t)seg * pool_k + i];
        if (t < -1 || (t >= 0 && (t >= t_new0 || t > p))) {
            flag(status, kStatusBounds);
            t = -1;
        }
    } else {
        const int64_t tn = t_new0 + (i - pool_k);
        t = tn >= 0 && tn <= p ? (int32_t)tn : -1;
    }
    ids[(int64_t)seg * m + i] = t;
}

__global__ void k_chunk_len(const int32_t* __restrict__ seq_len, int drop, int32_t* __restrict__ len) {
    pdl_begin();
    const int32_t v = *seq_len - drop;
    *len = v > 0 ? v : 0;
}

}  // namespace

cudaError_t launch_chunk_len(const int32_t* seq_len, int drop, int32_t* len, cudaStream_t st) {
    return launch_pdl(k_chunk_len, dim3(1), dim3(1), 0, st, seq_len, drop, len);
}

cudaError_t launch_pool_candidates(const DevCache& c, int T, const int32_t* pool_prev, int pool_k, int n_new,
                                   int32_t* ids, uint32_t* status, cudaStream_t st) {
    const int m = pool_k + n_new;
    dim3 grid((unsigned)((m + 255) / 256), (unsigned)(c.batch * T));
    return launch_pdl(k_pool_candidates, dim3(grid), dim3(256), 0, st, c, T, pool_prev, pool_k, n_new, ids, status);
}

cudaError_t launch_score_full(const DevCache& c, const void* q, int q_f32, const float* hw, int T, int H_I,
                              float* scores, uint32_t* status, cudaStream_t st, int /*num_sms*/) {
    const size_t smem = sizeof(float) * (size_t)T * H_I * (kDI + 1);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_score_full, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((unsigned)((c.cap + 255) / 256), (unsigned)c.batch);
    return launch_pdl(k_score_full, dim3(grid), dim3(256), smem, st, c, q, q_f32, hw, T, H_I, scores, status);
}

cudaError_t launch_score_pool(const DevCache& c, const void* q, int q_f32, const float* hw, int T, int H_I,
                              const int32_t* pool, int pool_k, float* scores, uint32_t* status, cudaStream_t st) {
    const size_t smem = sizeof(float) * (size_t)H_I * (kQPitch + 1);
    const int64_t nseg = (int64_t)c.batch * T;
    // four threads per entry while one thread per entry would leave SMs idle
    // (fewer than about 4 x 148 CTAs of 256 entries)
    const bool split = nseg * ((pool_k + 255) / 256) < 4 * 148;
    const int per_cta = split ? 256 / 4 : 256;
    dim3 grid((unsigned)((pool_k + per_cta - 1) / per_cta), (unsigned)nseg);
    if (split)
        return launch_pdl(k_score_pool<4>, dim3(grid), dim3(256), smem, st, c, q, q_f32, hw, T, H_I, pool, pool_k,
                          scores, status);
    return launch_pdl(k_score_pool<1>, dim3(grid), dim3(256), smem, st, c, q, q_f32, hw, T, H_I, pool, pool_k, scores,
                      status);
}

}  // namespace csa2

// Sparse + sliding-window attention on the tcgen05 tensor cores.
//
// Method: hackernews.kjhq.dev post 49735410, key point 2 (local sliding windows
// plus global sparse retrieval over one shared main KV); tldrocket.com,
// "DeepSeek AI Released DeepSeek-V4.1-Flash with 1M Context, FP4 KV Cache, and
// Cross-Layer Attention Reuse", paragraphs 2-4 (128-token window in every
// layer; E2M1 values with one E4M3 scale per 16 channels, used as key and
// value of every head).
//
// One CTA owns 128 entries of the (window ++ top-k) list of one (sequence,
// query token) and one group of HG heads (HG = 16, 32 or H: fewer heads per
// CTA when the (chunk, segment) grid alone would leave SMs idle) -- a top-k
// entry that is -1, beyond p or inside the window is masked, so the attended
// set is window ∪ top-k without double counting:
//   1. gather the FP4 rows (16-byte loads), dequantise exactly to fp16 into a
//      128 x D tile laid out K-major with the 128-byte swizzle; meanwhile
//      convert the group's bf16 queries to fp16 scaled by a power of two per
//      head (exact) in the same layout;
//   2. S[pos, head] = V Q^T : tcgen05.mma M=128 (positions), N=HG, K=D;
//   3. logits to shared memory transposed; per-head max and exp over the 128
//      positions; P (fp16) written K-major;
//   4. O^T[d, head] = V^T P^T : the same V bytes read through an MN-major
//      descriptor, one M=128 slab of d per accumulator;
//   5. unnormalised partial output ([d][head]) and (max, sum) per head in
//      base-2 units to the workspace, merged by the split-softmax combine kernel.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa2 {

namespace {

constexpr int kRows = 128;
constexpr int kThreads = 256;
constexpr int kZStride = kRows + 4;   // padded row of the transposed logits (floats)

struct Params {
    DevCache c;
    const __nv_bfloat16* q;   // [B*T][H][D]
    const int32_t* topk;      // [B*T][top_k]
    int T, H, HG, top_k, window, nchunk;
    float scale;
    float* part_o;            // [seg][chunk][D][H]
    float* part_ml;           // [seg][chunk][H][2]
    uint32_t* status;
    uint32_t off_q, off_misc, tmem_cols;
};

struct Misc {
    float fac[64];               // per head of the group: softmax scale * log2(e) / query scale
    float red[16][64];           // per head partial max / sum of the threads that share it
    int32_t pos[kRows];
    uint64_t mma_bar;
    uint32_t tmem_base;
};

__device__ __forceinline__ uint32_t cvt_e2m1x2_f16x2(uint32_t byte) {
    uint32_t r;
    const uint16_t in = (uint16_t)(byte & 0xFF);
    asm("{\n\t.reg .b8 b, u;\n\tmov.b16 {b, u}, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(r) : "h"(in));
    return r;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    __half2 x, y;
    memcpy(&x, &a, 4);
    memcpy(&y, &b, 4);
    __half2 z = __hmul2(x, y);
    uint32_t r;
    memcpy(&r, &z, 4);
    return r;
}

__global__ void __launch_bounds__(kThreads, 1) k_attn_tc(const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int D = p.c.dim, H = p.H, HG = p.HG;
    const int nkb = D / 64;                     // 64-wide K blocks of the V tile
    uint8_t* sV = smem;                         // nkb x [128 rows x 128 B]
    uint8_t* sQ = smem + p.off_q;               // nkb x [HG rows x 128 B]; later logits + P
    float* sZ = reinterpret_cast<float*>(sQ);   // [HG][kZStride] (after S is computed)
    uint8_t* sP = sQ + ((HG * kZStride * 4 + 1023) & ~1023);   // 2 x [HG rows x 128 B]
    Misc* misc = reinterpret_cast<Misc*>(smem + p.off_misc);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int chunk = blockIdx.x, seg = blockIdx.y, h_base = blockIdx.z * HG;
    if (tid == 0) {
        tc::mbar_init(&misc->mma_bar, 1);
        tc::fence_mbar_init();
    }
    // everything below may read what the preceding kernel wrote (and the
    // tensor memory is allocated only once that kernel has released its own)
    pdl_begin();
    const int b = seg / p.T, j = seg % p.T;
    const int64_t L = seq_len(p.c, b, p.status);
    const int64_t pq = L - p.T + j;
    if (warp == 0) tc::tmem_alloc(&misc->tmem_base, p.tmem_cols);
    if (tid < kRows) {
        const int v = chunk * kRows + tid;
        int32_t t = -1;
        if (pq >= 0 && v < p.window + p.top_k) {
            if (v < p.window) {
                t = pq - v >= 0 ? (int32_t)(pq - v) : -1;
            } else {
                t = __ldg(p.topk + (int64_t)seg * p.top_k + (v - p.window));
                if (t < -1 || t >= L) { flag(p.status, kStatusBounds); t = -1; }
                else if (t > pq || t > pq - p.window) t = -1;   // future, or already in the window
            }
        }
        misc->pos[tid] = t;
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = misc->tmem_base;

    // ---- gather: every load of this thread is issued before any is used
    // item = (row, 16-byte code chunk = 32 channels); at most 8 items per thread
    const int nchunk16 = D / 32;
    const int n_items = kRows * nchunk16 / kThreads;
    uint4 gcode[8];
    uint16_t gscale[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if (k < n_items) {
            const int w = k * kThreads + tid;
            const int r = w / nchunk16, cc = w - r * nchunk16;
            const int32_t t = misc->pos[r];
            const int64_t slot = t >= 0 ? slot_of(p.c, b, t) : -1;
            if (t >= 0 && slot < 0) flag(p.status, kStatusBounds);
            if (slot >= 0) {
                const uint8_t* row = p.c.rows + slot * p.c.row_stride;
                gcode[k] = __ldg(reinterpret_cast<const uint4*>(row + cc * 16));
                gscale[k] = __ldg(reinterpret_cast<const uint16_t*>(row + (D >> 1) + 2 * cc));
            } else {
                gcode[k] = make_uint4(0u, 0u, 0u, 0u);
                gscale[k] = 0;                                  // E4M3 zero scale: the row dequantises to 0
            }
        }
    }

    // ---- queries of the group (their loads overlap the gathers in flight):
    // H rows of fp16 scaled by 2^e per head, the row maximum in [2^14, 2^15)
    // so that every bf16 value down to 2^-32 of it is exact; tph consecutive
    // threads share one head, D / tph consecutive values each
    {
        const int tph = kThreads / HG;               // 4, 8 or 16
        const int hl = tid / tph, part = tid % tph;
        const int span = D / tph;                    // a multiple of 8, at most 128
        const __nv_bfloat16* src = p.q + ((int64_t)seg * H + h_base + hl) * D + part * span;
        uint4 qv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (8 * i < span) qv[i] = __ldg(reinterpret_cast<const uint4*>(src + 8 * i));
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (8 * i < span) {
                const uint32_t wv[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    m = fmaxf(m, fmaxf(fabsf(__uint_as_float(wv[k] << 16)), fabsf(__uint_as_float(wv[k] & 0xFFFF0000u))));
            }
        }
        for (int o = 1; o < tph; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        int e = 0;
        if (m > 0.0f) {
            e = 14 - ((int)((__float_as_uint(m) >> 23) & 0xFF) - 127);
            e = e < -100 ? -100 : (e > 100 ? 100 : e);
        }
        const float up = __uint_as_float((uint32_t)(127 + e) << 23);
        // logits in base-2 units: softmax_scale * log2(e) / 2^e
        if (part == 0) misc->fac[hl] = p.scale * 1.4426950408889634f * __uint_as_float((uint32_t)(127 - e) << 23);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (8 * i < span) {
                const uint32_t wv[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
                uint32_t hv[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    __half2 hh = __floats2half2_rn(__uint_as_float(wv[k] << 16) * up,
                                                   __uint_as_float(wv[k] & 0xFFFF0000u) * up);
                    memcpy(&hv[k], &hh, 4);
                }
                const int d = part * span + 8 * i;        // 8 values: one 16-byte chunk
                *reinterpret_cast<uint4*>(sQ + (d >> 6) * (HG * 128) + tc::sw128_offset(hl, (d & 63) >> 3)) =
                    make_uint4(hv[0], hv[1], hv[2], hv[3]);
            }
        }
    }

    // ---- dequantise: value(code) * value(scale), exact in fp16, into the swizzled V tile
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if (k < n_items) {
            const int w = k * kThreads + tid;
            const int r = w / nchunk16, cc = w - r * nchunk16;
            uint32_t s2;
            asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(s2) : "h"(gscale[k]));
            const uint32_t s_lo = (s2 & 0xFFFFu) * 0x10001u;            // (s0, s0)
            const uint32_t s_hi = (s2 >> 16) * 0x10001u;                // (s1, s1)
            const uint32_t cw[4] = {gcode[k].x, gcode[k].y, gcode[k].z, gcode[k].w};
            uint32_t hv[16];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int bb = 0; bb < 4; ++bb)
                    hv[4 * q + bb] = hmul2_u32(cvt_e2m1x2_f16x2(cw[q] >> (8 * bb)), q < 2 ? s_lo : s_hi);
            uint8_t* blk = sV + (cc >> 1) * (kRows * 128);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<uint4*>(blk + tc::sw128_offset(r, 4 * (cc & 1) + q)) =
                    make_uint4(hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3]);
        }
    }
    tc::fence_proxy_async_smem();
    __syncthreads();

    // ---- S = V Q^T
    bool ok = true;
    if (warp == 4 && lane == 0) {
        tc::fence_after_sync();
        const uint32_t idesc = tc::idesc_f16_f32(kRows, HG);
        const uint32_t v0 = tc::smem_u32(sV), q0 = tc::smem_u32(sQ);
        for (int kb = 0; kb < nkb; ++kb)
#pragma unroll
            for (int k = 0; k < 4; ++k)
                tc::mma_f16(tmem, tc::desc_sw128(v0 + kb * (kRows * 128) + 32 * k),
                            tc::desc_sw128(q0 + kb * (HG * 128) + 32 * k), idesc, (kb | k) != 0);
        tc::mma_commit(&misc->mma_bar);
    }
    ok = tc::mbar_wait(&misc->mma_bar, 0);
    ok = __syncthreads_and(ok);
    tc::fence_after_sync();

    // ---- logits to shared memory, transposed: z[h][pos]; lane = position, the
    // two warpgroups take one half of the group's heads each (HG >= 32)
    const int ngrp = HG >= 32 ? 2 : 1;
    const int wgrp = warp >> 2, quad = warp & 3;
    if (ok && wgrp < ngrp) {
        const int r = quad * 32 + lane;
        const bool valid = misc->pos[r] >= 0;
        const int hc = HG / ngrp;
        for (int c0 = wgrp * hc; c0 < (wgrp + 1) * hc; c0 += 16) {
            float v[16];
            tc::tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + c0, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) sZ[(c0 + i) * kZStride + r] = valid ? v[i] * misc->fac[c0 + i] : -INFINITY;
        }
    }
    __syncthreads();

    // ---- softmax statistics: nq = 256 / HG threads per head, each over 128 / nq positions
    const int nq = kThreads / HG, per = kRows / nq;
    const int h = tid % HG, qt = tid / HG;
    const float* z = sZ + h * kZStride + qt * per;
    float m = -INFINITY, l = 0.0f;
    if (ok) {
        for (int i = 0; i < per; ++i) m = fmaxf(m, z[i]);
        misc->red[qt][h] = m;
    }
    __syncthreads();
    if (ok) {
        for (int k = 0; k < nq; ++k) m = fmaxf(m, misc->red[k][h]);
        uint8_t* blk = sP + ((qt * per) >> 6) * (HG * 128);
        const int c_first = ((qt * per) & 63) >> 3;
        for (int c = 0; c < per / 8; ++c) {
            uint32_t hv[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float e0 = m == -INFINITY ? 0.0f : exp2f(z[8 * c + 2 * k] - m);
                const float e1 = m == -INFINITY ? 0.0f : exp2f(z[8 * c + 2 * k + 1] - m);
                __half2 hh = __floats2half2_rn(e0, e1);
                const float2 back = __half22float2(hh);   // sum what the MMA will use
                l += back.x + back.y;
                memcpy(&hv[k], &hh, 4);
            }
            *reinterpret_cast<uint4*>(blk + tc::sw128_offset(h, c_first + c)) =
                make_uint4(hv[0], hv[1], hv[2], hv[3]);
        }
    }
    __syncthreads();   // all reads of red[] (the maxima) are done before it is reused for sums
    if (ok) misc->red[qt][h] = l;
    tc::fence_proxy_async_smem();
    __syncthreads();
    if (ok && tid < HG) {
        float* ml = p.part_ml + (((int64_t)seg * p.nchunk + chunk) * H + h_base + tid) * 2;
        float sum = 0.0f;
        for (int k = 0; k < nq; ++k) sum += misc->red[k][tid];
        ml[0] = m;                                   // thread tid < HG holds local head tid's maximum
        ml[1] = sum;
    }

    // ---- O^T = V^T P^T, one 128-wide slab of d per accumulator
    if (ok && warp == 4 && lane == 0) {
        tc::fence_after_sync();
        const uint32_t idesc = tc::idesc_f16_f32(kRows, HG, /*a_mn=*/true, /*b_mn=*/false);
        const uint32_t v0 = tc::smem_u32(sV), p0 = tc::smem_u32(sP);
        for (int s = 0; s < D / 128; ++s)
            for (int ks = 0; ks < kRows / 16; ++ks)
                tc::mma_f16(tmem + (uint32_t)(HG + s * HG),
                            tc::desc_mn_sw128(v0 + (2 * s) * (kRows * 128) + ks * 2048, kRows * 128, 1024),
                            tc::desc_sw128(p0 + (ks >> 2) * (HG * 128) + 32 * (ks & 3)), idesc, ks != 0);
        tc::mma_commit(&misc->mma_bar);
    }
    if (ok) ok = tc::mbar_wait(&misc->mma_bar, 1);
    ok = __syncthreads_and(ok);
    tc::fence_after_sync();

    // ---- unnormalised partial output, [d][head] (lane = d within the slab; the
    // two warpgroups take one half of the group's heads each; 16-byte stores)
    if (ok && wgrp < ngrp) {
        float* po = p.part_o + ((int64_t)seg * p.nchunk + chunk) * H * D + h_base;
        const int hc = HG / ngrp;
        for (int s2 = 0; s2 < D / 128; ++s2) {
            const int d = s2 * 128 + quad * 32 + lane;
            for (int c0 = wgrp * hc; c0 < (wgrp + 1) * hc; c0 += 16) {
                float v[16];
                tc::tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(HG + s2 * HG + c0), v);
                float4* dst = reinterpret_cast<float4*>(po + (int64_t)d * H + c0);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
        }
    }
    if (!ok && tid == 0) flag(p.status, kStatusTimeout);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, p.tmem_cols);
    }
}

size_t attn_tc_smem(int D, int HG, uint32_t* off_q, uint32_t* off_misc) {
    const uint32_t v = (uint32_t)(D / 64) * kRows * 128;
    const uint32_t qbytes = (uint32_t)(D / 64) * HG * 128;
    const uint32_t zbytes = (((uint32_t)HG * kZStride * 4 + 1023) & ~1023u) + 2u * HG * 128;
    const uint32_t qreg = ((qbytes > zbytes ? qbytes : zbytes) + 1023) & ~1023u;
    *off_q = v;
    *off_misc = v + qreg;
    return (size_t)v + qreg + sizeof(Misc) + 1024;
}

}  // namespace

bool attn_tc_supported(const DevCache& c, int H) {
    uint32_t a, b;
    return c.dim % 128 == 0 && c.dim <= 512 && (H == 16 || H == 32 || H == 64) &&
           attn_tc_smem(c.dim, H, &a, &b) <= 227 * 1024;
}

int attn_tc_rows_per_chunk() { return kRows; }

int attn_tc_heads_per_cta(int H, int nchunk, int nseg, int num_sms) {
    int hg = H;
    while (hg > 16 && (int64_t)nchunk * nseg * (H / hg) < num_sms) hg >>= 1;
    return hg;
}

cudaError_t launch_attention_tc(const DevCache& c, const void* q, int T, int H, const int32_t* topk, int top_k,
                                int window, float sm_scale, const AttnWork& aw, uint32_t* status, cudaStream_t st,
                                int num_sms) {
    Params p;
    p.c = c;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.topk = topk;
    p.T = T;
    p.H = H;
    p.HG = attn_tc_heads_per_cta(H, aw.nchunk, c.batch * T, num_sms);
    p.top_k = top_k;
    p.window = window;
    p.nchunk = aw.nchunk;
    p.scale = sm_scale;
    p.part_o = aw.part_o;
    p.part_ml = aw.part_ml;
    p.status = status;
    uint32_t cols = 32;
    while (cols < (uint32_t)(p.HG + (c.dim / 128) * p.HG)) cols <<= 1;
    p.tmem_cols = cols;
    const size_t smem = attn_tc_smem(c.dim, p.HG, &p.off_q, &p.off_misc);
    cudaError_t e = cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_attn_tc, dim3((unsigned)aw.nchunk, (unsigned)(c.batch * T), (unsigned)(H / p.HG)),
                      dim3(kThreads), smem, st, p);
}

}  // namespace csa2

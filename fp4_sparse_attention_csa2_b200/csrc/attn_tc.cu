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
// query token) and one group of HG heads (HG = H, or 32 or 16 when the
// (chunk, segment) grid would otherwise leave SMs idle) -- a top-k
// entry that is -1, beyond p or inside the window is masked, so the attended
// set is window ∪ top-k without double counting:
//   1. fetch each FP4 row with one bulk copy (TMA) into a staging area, and
//      dequantise exactly to fp16 into a 128 x D tile laid out K-major with
//      the 128-byte swizzle; while the rows are in flight, convert the
//      group's bf16 queries to fp16 scaled by a power of two per head (exact)
//      in the same layout;
//   2. S[pos, head] = V Q^T : tcgen05.mma M=128 (positions), N=HG, K=D;
//   3. softmax read straight from the tensor memory (thread = position):
//      per-head max and exp over the 128 positions; P (fp16) written K-major;
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
constexpr int kWorkers = 256;               // 8 warps: rows, queries, dequantisation, softmax, stores
constexpr int kThreads = kWorkers + 32;     // + the warp that allocates TMEM and issues the MMAs

struct Params {
    DevCache c;
    const __nv_bfloat16* q;   // [B*T][H][D]
    const int32_t* topk;      // [B*T][top_k]
    int T, H, HG, top_k, window, nchunk;
    float scale;
    float* part_o;            // [seg][chunk][D][H]
    float* part_ml;           // [seg][chunk][H][2]
    uint32_t* status;
    uint32_t row_bytes;       // bytes fetched per row: D/2 codes + D/16 scales, rounded up to 16
    uint32_t stage_stride;    // row pitch of the staging area: row_bytes, or + 16 to make it an odd multiple of 16
    uint32_t off_q, off_stage, off_misc, tmem_cols;
};

struct Misc {
    float fac[64];               // per head of the group: softmax scale * log2(e) / query scale
    float red[8][64];            // per head: the four warps' maxima (rows 0-3) and sums (rows 4-7)
    int32_t pos[kRows];
    uint64_t row_bar;            // the chunk's row copies (one arrival per row)
    uint64_t kb_bar[8];          // K block k of V written (one arrival per worker)
    uint64_t s_bar;              // S = V Q^T complete
    uint64_t p_bar;              // P written (one arrival per worker)
    uint64_t o_bar[4];           // slab s of O^T complete
    uint64_t drain_bar;          // every MMA of the CTA complete
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

// Named barrier of one worker warpgroup (128 threads; ids 2 and 3).
__device__ __forceinline__ void group_sync(int wgrp) {
    asm volatile("bar.sync %0, 128;" ::"r"(2 + wgrp) : "memory");
}

// The float an order-preserving key came from (-0 comes back as +0).
__device__ __forceinline__ float key_to_float(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Softmax, first half, for NV heads c0.. of this thread's position: the
// scaled logits (-inf where the position is empty) into z, and this warp's
// maximum of each head into red[quad][head].
template <int NV>
__device__ __forceinline__ void logits_max(uint32_t trow, int c0, bool valid, Misc* misc, int quad, int lane, float* z) {
    float v[NV];
    if constexpr (NV == 8) tc::tmem_ld8(trow + c0, v);
    else tc::tmem_ld16(trow + c0, v);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        z[i] = valid ? v[i] * misc->fac[c0 + i] : -INFINITY;
        const uint32_t mk = __reduce_max_sync(0xffffffffu, ordered_key(z[i]));
        if (lane == i) misc->red[quad][c0 + i] = key_to_float(mk);
    }
}

// Softmax, second half: p = 2^(z - m) per head, rounded to fp16 and stored in
// the K-major P operand (row = head, 64 positions per 128-byte row, chunk pc,
// element el); this warp's sum of the rounded values into red[4 + quad][head].
// The sums leave the warp by an exchange that halves the values a lane
// carries at each step (NV - 1 shuffles for NV heads, not 5 NV); lanes 2 j
// and 2 j + 1 end with head j mod NV.
template <int NV>
__device__ __forceinline__ void probs_sums(uint8_t* prow, int pc, int el, int c0, Misc* misc, int quad, int lane,
                                           const float* z) {
    float sv[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int h = c0 + i;
        const float m = fmaxf(fmaxf(misc->red[0][h], misc->red[1][h]), fmaxf(misc->red[2][h], misc->red[3][h]));
        const float e = m == -INFINITY ? 0.0f : exp2f(z[i] - m);
        const __half ph = __float2half_rn(e);
        *reinterpret_cast<__half*>(prow + tc::sw128_offset(h, pc) + 2 * el) = ph;
        sv[i] = __half2float(ph);
    }
#pragma unroll
    for (int w = NV / 2; w >= 1; w >>= 1) {
        const bool up = (lane & (2 * w)) != 0;
#pragma unroll
        for (int i = 0; i < w; ++i) {
            const float send = up ? sv[i] : sv[i + w];
            const float keep = up ? sv[i + w] : sv[i];
            sv[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2 * w);
        }
    }
    sv[0] += __shfl_xor_sync(0xffffffffu, sv[0], 1);
#pragma unroll
    for (int o = 2 * NV; o < 32; o <<= 1) sv[0] += __shfl_xor_sync(0xffffffffu, sv[0], o);
    if (lane < 2 * NV && (lane & 1) == 0) misc->red[4 + quad][c0 + (lane >> 1)] = sv[0];
}

// Named barrier of the kWorkers worker threads (the MMA warp is not part of it).
__device__ __forceinline__ void workers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kWorkers) : "memory"); }

__global__ void __launch_bounds__(kThreads, 1) k_attn_tc(const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int D = p.c.dim, H = p.H, HG = p.HG;
    const int nkb = D / 64;                     // 64-wide K blocks of the V tile
    uint8_t* sV = smem;                         // nkb x [128 rows x 128 B]
    uint8_t* sQ = smem + p.off_q;               // nkb x [HG rows x 128 B]; later P
    uint8_t* sP = sQ;                           // 2 x [HG rows x 128 B] (after S is computed)
    uint8_t* sStage = smem + p.off_stage;       // [128 rows][stage_stride]: the FP4 rows as fetched (inside sV)
    Misc* misc = reinterpret_cast<Misc*>(smem + p.off_misc);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int chunk = blockIdx.x, seg = blockIdx.y, h_base = blockIdx.z * HG;
    if (tid == 0) {
        tc::mbar_init(&misc->row_bar, kRows);
        for (int k = 0; k < 8; ++k) tc::mbar_init(&misc->kb_bar[k], kWorkers);
        tc::mbar_init(&misc->s_bar, 1);
        tc::mbar_init(&misc->p_bar, kWorkers);
        for (int s = 0; s < 4; ++s) tc::mbar_init(&misc->o_bar[s], 1);
        tc::mbar_init(&misc->drain_bar, 1);
        tc::fence_mbar_init();
    }
    __syncthreads();
    // everything below may read what the preceding kernel wrote (and the
    // tensor memory is allocated only once that kernel has released its own)
    pdl_begin();
    const int b = seg / p.T, j = seg % p.T;

    if (warp == kWorkers / 32) {
        // ================= MMA warp: TMEM, then both products as their operands arrive
        tc::tmem_alloc(&misc->tmem_base, p.tmem_cols);
        tc::fence_before_sync();
        __syncthreads();                                  // (1) operands staged, TMEM address published
        tc::fence_after_sync();
        const uint32_t tmem = misc->tmem_base;
        if (lane == 0) {
            bool ok = true;
            // S = V Q^T, one 64-wide K block at a time as the workers finish it
            const uint32_t idesc1 = tc::idesc_f16_f32(kRows, HG);
            const uint32_t v0 = tc::smem_u32(sV), q0 = tc::smem_u32(sQ), p0 = tc::smem_u32(sP);
            for (int kb = 0; kb < nkb; ++kb) {
                ok = ok && tc::mbar_wait(&misc->kb_bar[kb], 0);
                if (!ok) break;
                tc::fence_after_sync();
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    tc::mma_f16(tmem, tc::desc_sw128(v0 + kb * (kRows * 128) + 32 * k),
                                tc::desc_sw128(q0 + kb * (HG * 128) + 32 * k), idesc1, (kb | k) != 0);
            }
            tc::mma_commit(&misc->s_bar);                 // arrives once the issued MMAs are done
            // O^T = V^T P^T, one 128-wide slab of d per accumulator, each slab committed on its own
            ok = ok && tc::mbar_wait(&misc->p_bar, 0);
            if (ok) tc::fence_after_sync();
            const uint32_t idesc2 = tc::idesc_f16_f32(kRows, HG, /*a_mn=*/true, /*b_mn=*/false);
            for (int s = 0; s < D / 128; ++s) {
                if (ok)
                    for (int ks = 0; ks < kRows / 16; ++ks)
                        tc::mma_f16(tmem + (uint32_t)(HG + s * HG),
                                    tc::desc_mn_sw128(v0 + (2 * s) * (kRows * 128) + ks * 2048, kRows * 128, 1024),
                                    tc::desc_sw128(p0 + (ks >> 2) * (HG * 128) + 32 * (ks & 3)), idesc2, ks != 0);
                tc::mma_commit(&misc->o_bar[s]);
            }
            tc::mma_commit(&misc->drain_bar);
            ok = tc::mbar_wait(&misc->drain_bar, 0) && ok;   // nothing in flight when TMEM is freed
            if (!ok) flag(p.status, kStatusTimeout);
        }
        __syncwarp();
        tc::fence_before_sync();
        __syncthreads();                                  // (2) the workers are done with TMEM
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, p.tmem_cols);
        return;
    }

    // ================= workers (8 warps)
    // loads that do not depend on each other are issued together: this
    // thread's top-k entry, the group's queries, the sequence length
    const int v_entry = chunk * kRows + tid;
    const bool is_topk = tid < kRows && v_entry >= p.window && v_entry < p.window + p.top_k;
    int32_t t_raw = -1;
    if (is_topk) t_raw = __ldg(p.topk + (int64_t)seg * p.top_k + (v_entry - p.window));
    // queries: tph consecutive threads share one head, D / tph consecutive values each
    const int tph = kWorkers / HG;                   // 4, 8 or 16
    const int hl = tid / tph, part = tid % tph;
    const int span = D / tph;                        // a multiple of 8, at most 128
    uint4 qv[16];
    {
        const __nv_bfloat16* src = p.q + ((int64_t)seg * H + h_base + hl) * D + part * span;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (8 * i < span) qv[i] = __ldg(reinterpret_cast<const uint4*>(src + 8 * i));
    }
    const int64_t L = seq_len(p.c, b, p.status);
    const int64_t pq = L - p.T + j;

    // ---- rows: thread r < 128 resolves entry r of the chunk and fetches its
    // whole FP4 row (codes + scales) with one bulk copy into the staging area
    if (tid < kRows) {
        int32_t t = -1;
        if (pq >= 0 && v_entry < p.window + p.top_k) {
            if (v_entry < p.window) {
                t = pq - v_entry >= 0 ? (int32_t)(pq - v_entry) : -1;
            } else {
                t = t_raw;
                if (t < -1 || t >= L) { flag(p.status, kStatusBounds); t = -1; }
                else if (t > pq || t > pq - p.window) t = -1;   // future, or already in the window
            }
        }
        const int64_t slot = t >= 0 ? slot_of(p.c, b, t) : -1;
        if (t >= 0 && slot < 0) { flag(p.status, kStatusBounds); t = -1; }
        misc->pos[tid] = t;
        if (t >= 0) {
            tc::mbar_arrive_expect_tx(&misc->row_bar, p.row_bytes);
            tc::bulk_g2s(sStage + tid * p.stage_stride, p.c.rows + slot * p.c.row_stride, p.row_bytes,
                         &misc->row_bar);
        } else {
            tc::mbar_arrive(&misc->row_bar);
        }
    }

    // ---- queries to fp16 scaled by 2^e per head, the row maximum in
    // [2^14, 2^15) so that every bf16 value down to 2^-32 of it is exact
    {
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
    tc::fence_proxy_async_smem();                     // the queries are an MMA operand
    tc::fence_before_sync();
    __syncthreads();                                  // (1) pos[], queries, TMEM address
    tc::fence_after_sync();
    const uint32_t tmem = misc->tmem_base;

    // ---- dequantise: value(code) * value(scale), exact in fp16, into the
    // swizzled V tile.  Thread t owns row t % 128 and the 32-channel chunks
    // cc = 2k + t / 128 (k < D / 64), so a warp's 16-byte accesses walk 32
    // consecutive rows: conflict-free in the staging area (odd 16-byte row
    // stride) and in the 128-byte-swizzled tile.  The staging area overlaps the
    // tile, so every read is done before the first write; masked rows become 0.
    // K block k is handed to the MMA warp as soon as every worker has written it.
    bool ok = tc::mbar_wait(&misc->row_bar, 0);
    const bool rows_ok = ok;
    const int r = tid & (kRows - 1), half = tid >> 7;
    const int n_own = D / 64;                        // chunks per thread, at most 8
    const bool live = misc->pos[r] >= 0;
    uint4 code[8];
    uint16_t scl[8];
    {
        const uint8_t* row = sStage + r * p.stage_stride;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (k < n_own) {
                const int cc = 2 * k + half;
                code[k] = live ? *reinterpret_cast<const uint4*>(row + cc * 16) : make_uint4(0u, 0u, 0u, 0u);
                scl[k] = live ? *reinterpret_cast<const uint16_t*>(row + (D >> 1) + 2 * cc) : (uint16_t)0;
            }
        }
    }
    workers_sync();
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if (k < n_own) {
            uint32_t s2;
            asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(s2) : "h"(scl[k]));
            const uint32_t s_lo = (s2 & 0xFFFFu) * 0x10001u;            // (s0, s0)
            const uint32_t s_hi = (s2 >> 16) * 0x10001u;                // (s1, s1)
            const uint32_t cw[4] = {code[k].x, code[k].y, code[k].z, code[k].w};
            uint32_t hv[16];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int bb = 0; bb < 4; ++bb)
                    hv[4 * q + bb] = hmul2_u32(cvt_e2m1x2_f16x2(cw[q] >> (8 * bb)), q < 2 ? s_lo : s_hi);
            uint8_t* blk = sV + k * (kRows * 128);               // K block k = cc / 2
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<uint4*>(blk + tc::sw128_offset(r, 4 * half + q)) =
                    make_uint4(hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3]);
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(&misc->kb_bar[k]);
        }
    }

    // ---- softmax straight from the tensor memory.  Thread = position (the
    // TMEM lane of its warp's quarter); each warpgroup takes one half of the
    // group's heads.  Per head: the maximum over the 128 positions (a
    // warp-wide max of order-preserving integer keys, then the four warps'
    // through shared memory); p = 2^(z - m) in fp16, stored straight into the
    // K-major P operand; the sum of the fp16 values as the MMA will use them.
    ok = tc::mbar_wait(&misc->s_bar, 0) && ok;
    tc::fence_after_sync();
    const int wgrp = warp >> 2, quad = warp & 3;
    const int hc = HG / 2;                           // heads of a warpgroup: 8, 16 or 32
    ok = __all_sync(0xffffffffu, ok);                // warp-uniform from here on
    const int pos = quad * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const bool valid = misc->pos[pos] >= 0;
    float zz[32];
    if (ok) {
        if (hc == 8) {
            logits_max<8>(trow, wgrp * 8, valid, misc, quad, lane, zz);
        } else {
#pragma unroll
            for (int blk = 0; blk < 2; ++blk)
                if (blk * 16 < hc) logits_max<16>(trow, wgrp * hc + blk * 16, valid, misc, quad, lane, zz + 16 * blk);
        }
    }
    group_sync(wgrp);
    if (ok) {
        uint8_t* prow = sP + (pos >> 6) * (HG * 128);
        const int pc = (pos & 63) >> 3, el = pos & 7;
        if (hc == 8) {
            probs_sums<8>(prow, pc, el, wgrp * 8, misc, quad, lane, zz);
        } else {
#pragma unroll
            for (int blk = 0; blk < 2; ++blk)
                if (blk * 16 < hc) probs_sums<16>(prow, pc, el, wgrp * hc + blk * 16, misc, quad, lane, zz + 16 * blk);
        }
    }
    tc::fence_proxy_async_smem();                     // P is an MMA operand
    tc::mbar_arrive(&misc->p_bar);
    group_sync(wgrp);
    {
        const int t = tid & 127;                      // thread of the warpgroup
        if (ok && t < hc) {
            const int h = wgrp * hc + t;
            const float m = fmaxf(fmaxf(misc->red[0][h], misc->red[1][h]), fmaxf(misc->red[2][h], misc->red[3][h]));
            const float l = (misc->red[4][h] + misc->red[5][h]) + (misc->red[6][h] + misc->red[7][h]);
            float* ml = p.part_ml + (((int64_t)seg * p.nchunk + chunk) * H + h_base + h) * 2;
            ml[0] = m;
            ml[1] = l;
        }
    }

    // ---- unnormalised partial output, [d][head], slab by slab as the MMA warp
    // finishes them (lane = d within the slab; each warpgroup takes one half
    // of the group's heads; 16-byte stores)
    {
        float* po = p.part_o + ((int64_t)seg * p.nchunk + chunk) * H * D + h_base;
        for (int s2 = 0; s2 < D / 128; ++s2) {
            ok = tc::mbar_wait(&misc->o_bar[s2], 0) && ok;
            tc::fence_after_sync();
            if (!ok) continue;
            const int d = s2 * 128 + quad * 32 + lane;
            const uint32_t tcol = trow + (uint32_t)(HG + s2 * HG);
            if (hc == 8) {
                float v[8];
                tc::tmem_ld8(tcol + wgrp * 8, v);
                float4* dst = reinterpret_cast<float4*>(po + (int64_t)d * H + wgrp * 8);
                dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                dst[1] = make_float4(v[4], v[5], v[6], v[7]);
            } else {
                for (int c0 = wgrp * hc; c0 < (wgrp + 1) * hc; c0 += 16) {
                    float v[16];
                    tc::tmem_ld16(tcol + c0, v);
                    float4* dst = reinterpret_cast<float4*>(po + (int64_t)d * H + c0);
#pragma unroll
                    for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                }
            }
        }
    }
    if (!ok) flag(p.status, kStatusTimeout);
    if (!rows_ok) tc::mbar_wait(&misc->row_bar, 0);   // no row copy may land after the CTA has left
    tc::fence_before_sync();
    __syncthreads();                                  // (2) TMEM is released by the MMA warp
}

// Bytes of one row the kernel fetches: codes and scales, rounded up to the
// 16-byte granule of a bulk copy (never past the row: the stride is a
// multiple of 16 and at least D/2 + D/16).
int attn_tc_row_bytes(int D) { return (D / 2 + D / 16 + 15) & ~15; }

size_t attn_tc_smem(int D, int HG, uint32_t stage_bytes, uint32_t* off_q, uint32_t* off_stage, uint32_t* off_misc) {
    const uint32_t v = (uint32_t)(D / 64) * kRows * 128;
    const uint32_t qbytes = (uint32_t)(D / 64) * HG * 128;
    const uint32_t pbytes = 2u * HG * 128;     // P, in the query's place once S is computed
    const uint32_t qreg = ((qbytes > pbytes ? qbytes : pbytes) + 1023) & ~1023u;
    *off_q = v;
    *off_stage = (v - stage_bytes) & ~1023u;   // the tail of the V tile: rows land there before the tile is written
    *off_misc = v + qreg;
    return (size_t)v + qreg + sizeof(Misc) + 1024;
}

uint32_t attn_tc_stage_stride(int D) {
    const uint32_t rb = (uint32_t)attn_tc_row_bytes(D);
    return ((rb / 16) & 1) ? rb : rb + 16;
}

}  // namespace

bool attn_tc_supported(const DevCache& c, int H) {
    uint32_t a, b, d;
    return c.dim % 128 == 0 && c.dim <= 512 && (H == 16 || H == 32 || H == 64) &&
           attn_tc_smem(c.dim, H, kRows * attn_tc_stage_stride(c.dim), &a, &b, &d) <= 227 * 1024;
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
    p.row_bytes = (uint32_t)attn_tc_row_bytes(c.dim);
    p.stage_stride = attn_tc_stage_stride(c.dim);
    uint32_t cols = 32;
    while (cols < (uint32_t)(p.HG + (c.dim / 128) * p.HG)) cols <<= 1;
    p.tmem_cols = cols;
    const size_t smem = attn_tc_smem(c.dim, p.HG, kRows * p.stage_stride, &p.off_q, &p.off_stage, &p.off_misc);
    cudaError_t e = cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_attn_tc, dim3((unsigned)aw.nchunk, (unsigned)(c.batch * T), (unsigned)(H / p.HG)),
                      dim3(kThreads), smem, st, p);
}

}  // namespace csa2

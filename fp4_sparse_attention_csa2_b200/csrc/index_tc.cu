// Indexer scoring on the 5th-generation tensor cores (tcgen05) for E4M3 index
// keys:  s_t = sum_h w_h * max(0, q_h . k_t)  for every visible position.
//
// Role of the indexer: tldrocket.com, "DeepSeek AI Released DeepSeek-V4.1-Flash
// with 1M Context, FP4 KV Cache, and Cross-Layer Attention Reuse", paragraph 3
// (a Full layer scores the whole context into a candidate pool of <= 16,384
// positions); hackernews.kjhq.dev post 49735410, key point 3.
//
// The key stream is the HBM-bound hot loop (64 B per position, 2*H_I*64 flop
// per position per query token).  Per 128-position tile:
//   producer warp   : 1-D bulk copies (TMA engine, no multicast) of the raw
//                     E4M3 keys, 64 positions (one page run) per copy, into an
//                     8-stage ring;
//   converter warps : E4M3 -> fp16 (exact) into a 128-byte-swizzled K-major
//                     operand tile;
//   MMA thread      : 4 x tcgen05.mma kind::f16 (M=128 positions, N = T*H_I
//                     query heads padded to 16, K=16) into a double-buffered
//                     TMEM accumulator;
//   epilogue warps  : tcgen05.ld of each position's row, ReLU + head-weighted
//                     sum, fp32 score store, and the level-1 radix histogram
//                     of the top-K select in shared memory.
// Queries go in as fp16 scaled by a power of two per (token, head) so every
// bf16 query value down to 2^-32 of the row maximum is exact; the scale is
// folded back into the head weight (exact, a power of two).
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa2 {

namespace {

constexpr int kTile = 128;
constexpr int kItemTiles = 4;
constexpr int kRaw = 6;
constexpr int kA = 2;
constexpr int kRawBytes = kTile * 64;   // E4M3 keys of one tile
constexpr int kABytes = kTile * 128;    // 128 rows x 64 fp16
constexpr int kThreads = 320;
constexpr int kWarpProducer = 0, kWarpMma = 1, kWarpConv0 = 2, kWarpEpi0 = 6;
constexpr uint32_t kDrainLimit = 65536;   // tries of the drain waits (x kSuspendNs)

struct Params {
    DevCache c;
    const __nv_bfloat16* q;  // [B][T][H_I][64]
    const float* hw;         // [B][T][H_I]
    int T, H_I, HP, NP;      // HP: H_I rounded up to 16; NP = T * HP (MMA N)
    float* scores;           // [(b*T + j) * cap + t]
    uint32_t* hist;          // [(b*T + j)][3][kRadixBins], level-1 part accumulated; nullable
    uint32_t* status;
    int64_t items_per_seq, total_items;
    uint32_t tmem_cols;
    uint32_t off_b, off_raw, off_hist, off_wq, off_bar;
};

struct Item {
    int b;
    int64_t t0, L;
    int ntiles;
};

__device__ __forceinline__ bool get_item(const Params& p, int64_t item, Item& it) {
    const int b = (int)(item / p.items_per_seq);
    const int64_t k = item - (int64_t)b * p.items_per_seq;
    int64_t L = __ldg(p.c.seq_lens + b);
    L = L < 0 ? 0 : (L > p.c.cap ? p.c.cap : L);
    const int64_t tiles = (L + kTile - 1) / kTile;
    const int64_t tile0 = k * kItemTiles;
    if (tile0 >= tiles) return false;
    it.b = b;
    it.t0 = tile0 * kTile;
    it.L = L;
    it.ntiles = (int)(tiles - tile0 < kItemTiles ? tiles - tile0 : (int64_t)kItemTiles);
    return true;
}

struct Bars {
    uint64_t raw_full[kRaw], raw_empty[kRaw];
    uint64_t a_full[kA], a_empty[kA];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t b_free[2], wq_ready[2], wq_free[2];
    uint64_t hist_done, hist_clear;
    uint64_t drain;
    uint32_t tmem_base;
};

__device__ __forceinline__ uint32_t cvt_e4m3x2_f16x2(uint32_t two_bytes) {
    uint32_t r;
    const uint16_t in = (uint16_t)two_bytes;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(in));
    return r;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    uint32_t r;
    memcpy(&r, &h, 4);
    return r;
}

// Query operand of one sequence: NP rows (column c = token j * HP + head h) of
// 64 fp16 values, scaled by 2^e per row, and the folded weights w * 2^-e.
__device__ void prepare_queries(const Params& p, int b, uint8_t* bq, float* wq, int tid) {
    const int row_in_pass = tid >> 2, quarter = tid & 3;
    for (int r0 = 0; r0 < p.NP; r0 += 32) {
        const int c = r0 + row_in_pass;
        const int j = c / p.HP, h = c - j * p.HP;
        const bool real = c < p.NP && h < p.H_I;
        float v[16];
        if (real) {
            const uint4* src = reinterpret_cast<const uint4*>(
                p.q + ((((int64_t)b * p.T + j) * p.H_I + h) * 64 + quarter * 16));
            const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
            const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                v[2 * k] = __uint_as_float(w[k] << 16);
                v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
            }
        } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] = 0.0f;
        }
        float m = 0.0f;
#pragma unroll
        for (int k = 0; k < 16; ++k) m = fmaxf(m, fabsf(v[k]));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        int e = 0;
        if (m > 0.0f) {
            const int E = (int)((__float_as_uint(m) >> 23) & 0xFF) - 127;
            e = 14 - E;
            e = e < -100 ? -100 : (e > 100 ? 100 : e);
        }
        const float up = __uint_as_float((uint32_t)(127 + e) << 23);
        const float down = __uint_as_float((uint32_t)(127 - e) << 23);
        if (c < p.NP) {
            uint32_t hv[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) hv[k] = pack_half2(v[2 * k] * up, v[2 * k + 1] * up);
            *reinterpret_cast<uint4*>(bq + tc::sw128_offset(c, 2 * quarter)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
            *reinterpret_cast<uint4*>(bq + tc::sw128_offset(c, 2 * quarter + 1)) =
                make_uint4(hv[4], hv[5], hv[6], hv[7]);
            if (quarter == 0) wq[c] = real ? __ldg(p.hw + ((int64_t)b * p.T + j) * p.H_I + h) * down : 0.0f;
        }
    }
}

__global__ void __launch_bounds__(kThreads, 2) k_score_full_tc(const Params p) {
    extern __shared__ uint8_t smem_raw[];
    // operand tiles need 1024-byte alignment for the 128-byte swizzle
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + p.off_b;
    uint8_t* sRaw = smem + p.off_raw;
    uint32_t* sHist = reinterpret_cast<uint32_t*>(smem + p.off_hist);
    float* sWq = reinterpret_cast<float*>(smem + p.off_wq);
    Bars* bars = reinterpret_cast<Bars*>(smem + p.off_bar);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    for (int i = threadIdx.x; i < p.T * kRadixBins; i += kThreads) sHist[i] = 0;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kRaw; ++i) { tc::mbar_init(&bars->raw_full[i], 1); tc::mbar_init(&bars->raw_empty[i], 128); }
        for (int i = 0; i < kA; ++i) { tc::mbar_init(&bars->a_full[i], 128); tc::mbar_init(&bars->a_empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&bars->acc_full[i], 1);
            tc::mbar_init(&bars->acc_empty[i], 128);
            tc::mbar_init(&bars->b_free[i], 1);
            tc::mbar_init(&bars->wq_ready[i], 128);
            tc::mbar_init(&bars->wq_free[i], 128);
        }
        tc::mbar_init(&bars->hist_done, 128);
        tc::mbar_init(&bars->hist_clear, 128);
        tc::mbar_init(&bars->drain, 1);
        tc::fence_mbar_init();
    }
    if (warp == kWarpMma) tc::tmem_alloc(&bars->tmem_base, p.tmem_cols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = bars->tmem_base;

    if (warp == kWarpProducer) {
        if (lane == 0) {
            uint32_t g = 0;
            bool ok = true;
            for (int64_t item = blockIdx.x; item < p.total_items && ok; item += gridDim.x) {
                Item it;
                if (!get_item(p, item, it)) continue;
                for (int tl = 0; tl < it.ntiles; ++tl, ++g) {
                    const int s = g % kRaw;
                    if (!tc::mbar_wait(&bars->raw_empty[s], ((g / kRaw) & 1) ^ 1)) { ok = false; break; }
                    const int64_t t0 = it.t0 + (int64_t)tl * kTile;
                    int64_t slot[2] = {-1, -1};
                    int cnt[2] = {0, 0};
                    uint32_t bytes = 0;
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int64_t p0 = t0 + 64 * r;
                        { const int64_t rem = it.L - p0; cnt[r] = rem <= 0 ? 0 : (rem > 64 ? 64 : (int)rem); }
                        if (cnt[r] > 0) {
                            slot[r] = slot_of(p.c, it.b, p0);
                            if (slot[r] < 0) flag(p.status, kStatusBounds);
                            else bytes += (uint32_t)cnt[r] * 64u;
                        }
                    }
                    if (bytes == 0) {
                        tc::mbar_arrive(&bars->raw_full[s]);
                    } else {
                        tc::mbar_arrive_expect_tx(&bars->raw_full[s], bytes);
#pragma unroll
                        for (int r = 0; r < 2; ++r)
                            if (cnt[r] > 0 && slot[r] >= 0)
                                tc::bulk_g2s(sRaw + s * kRawBytes + r * 4096,
                                             static_cast<const uint8_t*>(p.c.keys) + slot[r] * 64,
                                             (uint32_t)cnt[r] * 64u, &bars->raw_full[s]);
                    }
                }
            }
            if (!ok) flag(p.status, kStatusTimeout);
            // copies still in flight must land before the CTA's shared memory goes away
            for (uint32_t k = g > (uint32_t)kRaw ? g - kRaw : 0; k < g; ++k)
                tc::mbar_wait(&bars->raw_full[k % kRaw], (k / kRaw) & 1, kDrainLimit);
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_f16_f32(kTile, p.NP);
            uint32_t g = 0, n = 0;
            int cur_b = -1;
            bool ok = true;
            for (int64_t item = blockIdx.x; item < p.total_items && ok; item += gridDim.x) {
                Item it;
                if (!get_item(p, item, it)) continue;
                if (it.b != cur_b) {
                    // the query buffer of the previous sequence is free once its MMAs are done
                    if (cur_b >= 0) { tc::mma_commit(&bars->b_free[n & 1]); ++n; }
                    cur_b = it.b;
                }
                const uint32_t bq = tc::smem_u32(sB + (n & 1) * (p.NP * 128));
                for (int tl = 0; tl < it.ntiles; ++tl, ++g) {
                    const int a = g % kA, acc = g & 1;
                    if (!tc::mbar_wait(&bars->a_full[a], (g / kA) & 1) ||
                        !tc::mbar_wait(&bars->acc_empty[acc], ((g >> 1) & 1) ^ 1)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t aa = tc::smem_u32(sA + a * kABytes);
                    const uint32_t d = tmem + (uint32_t)(acc * p.NP);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc::mma_f16(d, tc::desc_sw128(aa + 32 * k), tc::desc_sw128(bq + 32 * k), idesc, k > 0);
                    tc::mma_commit(&bars->a_empty[a]);
                    tc::mma_commit(&bars->acc_full[acc]);
                }
            }
            if (!ok) flag(p.status, kStatusTimeout);
            tc::mma_commit(&bars->drain);
            tc::mbar_wait(&bars->drain, 0, kDrainLimit);
        }
    } else if (warp < kWarpEpi0) {
        // converters: 128 threads
        const int tid = threadIdx.x - kWarpConv0 * 32;
        uint32_t g = 0, n = 0;
        int cur_b = -1;
        bool ok = true;
        for (int64_t item = blockIdx.x; item < p.total_items && ok; item += gridDim.x) {
            Item it;
            if (!get_item(p, item, it)) continue;
            if (it.b != cur_b) {
                // a new sequence: stage its queries in the other buffer
                if (cur_b >= 0) ++n;
                cur_b = it.b;
                const int qb = n & 1;
                if (!tc::mbar_wait(&bars->b_free[qb], ((n >> 1) & 1) ^ 1) ||
                    !tc::mbar_wait(&bars->wq_free[qb], ((n >> 1) & 1) ^ 1)) { ok = false; break; }
                prepare_queries(p, it.b, sB + qb * (p.NP * 128), sWq + qb * p.NP, tid);
                tc::fence_proxy_async_smem();
                tc::mbar_arrive(&bars->wq_ready[qb]);
            }
            for (int tl = 0; tl < it.ntiles; ++tl, ++g) {
                const int s = g % kRaw, a = g % kA;
                if (!tc::mbar_wait(&bars->raw_full[s], (g / kRaw) & 1) ||
                    !tc::mbar_wait(&bars->a_empty[a], ((g / kA) & 1) ^ 1)) { ok = false; break; }
                const uint8_t* rs = sRaw + s * kRawBytes;
                uint8_t* as = sA + a * kABytes;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int cidx = k * 128 + tid;            // 16-byte chunk of the raw tile
                    const int row = cidx >> 2, quarter = cidx & 3;
                    const uint4 v = *reinterpret_cast<const uint4*>(rs + cidx * 16);
                    const uint4 lo = make_uint4(cvt_e4m3x2_f16x2(v.x), cvt_e4m3x2_f16x2(v.x >> 16),
                                                cvt_e4m3x2_f16x2(v.y), cvt_e4m3x2_f16x2(v.y >> 16));
                    const uint4 hi = make_uint4(cvt_e4m3x2_f16x2(v.z), cvt_e4m3x2_f16x2(v.z >> 16),
                                                cvt_e4m3x2_f16x2(v.w), cvt_e4m3x2_f16x2(v.w >> 16));
                    *reinterpret_cast<uint4*>(as + tc::sw128_offset(row, 2 * quarter)) = lo;
                    *reinterpret_cast<uint4*>(as + tc::sw128_offset(row, 2 * quarter + 1)) = hi;
                }
                tc::fence_proxy_async_smem();
                tc::mbar_arrive(&bars->a_full[a]);
                tc::mbar_arrive(&bars->raw_empty[s]);
            }
        }
        if (!ok) flag(p.status, kStatusTimeout);
    } else {
        // epilogue: 128 threads, thread = TMEM lane = position in the tile
        const int tid = threadIdx.x - kWarpEpi0 * 32;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
        uint32_t g = 0, n = 0, nflush = 0;
        int cur_b = -1;
        bool ok = true;
        // Move the shared histogram of sequence b into the global one.  The
        // 128 epilogue threads meet on two mbarriers (bounded waits, so a
        // thread that gave up earlier cannot hang the others).
        auto flush = [&](int b) -> bool {
            tc::mbar_arrive(&bars->hist_done);
            if (!tc::mbar_wait(&bars->hist_done, nflush & 1)) return false;
            if (p.hist) {
                for (int j = 0; j < p.T; ++j) {
                    uint32_t* gh = p.hist + ((int64_t)b * p.T + j) * 3 * kRadixBins;
                    for (int i = tid; i < kRadixBins; i += 128) {
                        const uint32_t v = sHist[j * kRadixBins + i];
                        if (v) { atomicAdd(gh + i, v); sHist[j * kRadixBins + i] = 0; }
                    }
                }
            }
            tc::mbar_arrive(&bars->hist_clear);
            if (!tc::mbar_wait(&bars->hist_clear, nflush & 1)) return false;
            ++nflush;
            return true;
        };
        // all lanes of a warp take the same decision before tcgen05.ld (.aligned)
        auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
            const bool got = tc::mbar_wait(bar, parity);
            return __all_sync(0xffffffffu, got);
        };
        const float* wq = sWq;
        for (int64_t item = blockIdx.x; item < p.total_items && ok; item += gridDim.x) {
            Item it;
            if (!get_item(p, item, it)) continue;
            if (it.b != cur_b) {
                if (cur_b >= 0) {
                    if (!flush(cur_b)) { ok = false; break; }
                    tc::mbar_arrive(&bars->wq_free[n & 1]);
                    ++n;
                }
                cur_b = it.b;
                if (!warp_wait(&bars->wq_ready[n & 1], (n >> 1) & 1)) { ok = false; break; }
                wq = sWq + (n & 1) * p.NP;
            }
            for (int tl = 0; tl < it.ntiles; ++tl, ++g) {
                const int acc = g & 1;
                if (!warp_wait(&bars->acc_full[acc], (g >> 1) & 1)) { ok = false; break; }
                tc::fence_after_sync();
                const int64_t t = it.t0 + (int64_t)tl * kTile + row;
                for (int j = 0; j < p.T; ++j) {
                    float s0 = 0.0f, s1 = 0.0f;
                    for (int c0 = j * p.HP; c0 < (j + 1) * p.HP; c0 += 16) {
                        float v[16];
                        tc::tmem_ld16(lane_addr + (uint32_t)(acc * p.NP + c0), v);
                        const float4* w4 = reinterpret_cast<const float4*>(wq + c0);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float4 ww = w4[i];
                            s0 = fmaf(ww.x, fmaxf(v[4 * i], 0.0f), s0);
                            s1 = fmaf(ww.y, fmaxf(v[4 * i + 1], 0.0f), s1);
                            s0 = fmaf(ww.z, fmaxf(v[4 * i + 2], 0.0f), s0);
                            s1 = fmaf(ww.w, fmaxf(v[4 * i + 3], 0.0f), s1);
                        }
                    }
                    const float s = s0 + s1;
                    const bool vis = t <= it.L - p.T + j;
                    if (vis) p.scores[((int64_t)it.b * p.T + j) * p.c.cap + t] = s;
                    if (p.hist) {
                        // lanes that hit the same bin add once (scores crowd into few bins)
                        const uint32_t bin = vis ? (ordered_key(s) >> 21) : 0xFFFFFFFFu;
                        const uint32_t peers = __match_any_sync(0xffffffffu, bin);
                        if (vis && lane == __ffs(peers) - 1)
                            atomicAdd(&sHist[j * kRadixBins + bin], (uint32_t)__popc(peers));
                    }
                }
                tc::fence_before_sync();
                tc::mbar_arrive(&bars->acc_empty[acc]);
            }
        }
        if (ok && cur_b >= 0 && !flush(cur_b)) ok = false;
        if (!ok) flag(p.status, kStatusTimeout);
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == kWarpMma) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, p.tmem_cols);
    }
}

}  // namespace

namespace {

size_t smem_bytes(int T, int NP) {
    return (size_t)kA * kABytes + 2 * (size_t)NP * 128 + (size_t)kRaw * kRawBytes + (size_t)T * kRadixBins * 4 +
           2 * (size_t)NP * 4 + sizeof(Bars) + 16 + 1024;
}

}  // namespace

bool score_full_tc_supported(const DevCache& c, int T, int H_I) {
    const int HP = (H_I + 15) / 16 * 16;
    return c.key_dtype == 2 && c.idx_dim == 64 && T * HP <= 256 && smem_bytes(T, T * HP) <= 227 * 1024;
}

cudaError_t launch_score_full_tc(const DevCache& c, const void* q, const float* hw, int T, int H_I, float* scores,
                                 uint32_t* hist, uint32_t* status, cudaStream_t st, int num_sms) {
    Params p;
    p.c = c;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.hw = hw;
    p.T = T;
    p.H_I = H_I;
    p.HP = (H_I + 15) / 16 * 16;
    p.NP = T * p.HP;
    p.scores = scores;
    p.hist = hist;
    p.status = status;
    const int64_t tiles_cap = (c.cap + kTile - 1) / kTile;
    p.items_per_seq = (tiles_cap + kItemTiles - 1) / kItemTiles;
    p.total_items = p.items_per_seq * c.batch;
    uint32_t cols = 32;
    while (cols < (uint32_t)(2 * p.NP)) cols <<= 1;
    p.tmem_cols = cols;
    uint32_t off = kA * kABytes;
    p.off_b = off;
    off += 2 * p.NP * 128;
    p.off_raw = off;
    off += kRaw * kRawBytes;
    p.off_hist = off;
    off += T * kRadixBins * 4;
    p.off_wq = off;
    off += 2 * p.NP * 4;
    off = (off + 15) / 16 * 16;
    p.off_bar = off;
    off += sizeof(Bars);
    const size_t smem = off + 1024;  // room to align the base to 1024 B
    cudaError_t e = cudaFuncSetAttribute(k_score_full_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int64_t grid = 2 * (int64_t)num_sms;   // two CTAs per SM
    if (grid > p.total_items) grid = p.total_items;
    if (grid < 1) grid = 1;
    k_score_full_tc<<<(unsigned)grid, kThreads, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace csa2

// Sparse + sliding-window attention on the tcgen05 tensor cores.
//
// Method: hackernews.kjhq.dev post 49735410, key point 2 (local sliding windows
// plus global sparse retrieval over one shared main KV); tldrocket.com,
// "DeepSeek AI Released DeepSeek-V4.1-Flash with 1M Context, FP4 KV Cache, and
// Cross-Layer Attention Reuse", paragraphs 2-4 (128-token window in every
// layer; E2M1 values with one E4M3 scale per 16 channels, used as key and
// value of every head).
//
// The work of one layer is a few hundred kilobytes of rows and well under a
// GFLOP, so the kernel is built for latency: every CTA runs one short chain
// and the grid covers the GPU.  One CTA owns 64 entries of the (window ++
// top-k) list of one (sequence, query token) and a group of HG heads (a top-k
// entry that is -1, beyond p or inside the window is masked, so the attended
// set is window ∪ top-k without double counting):
//   1. 512 worker threads issue every load at once: the group's bf16 queries,
//      the top-k entries, then each row's codes and scales (8 threads per row,
//      64 channels each) straight into registers;
//   2. queries -> fp16 scaled by a power of two per head (exact), rows ->
//      fp16 by bit placement and two exact fp16 products (see
//      e2m1x8_to_f16x2_scaled), both stored K-major with the 128-byte swizzle;
//   3. S[pos, head] = V Q^T on the tensor core (M = 128: rows 64..127 of the
//      operand are the next K block's rows, their S rows are never used),
//      its K = D split over four accumulators issued by four warps at once
//      (one thread issues an MMA every ~70 cycles, and the 32 of one K = 512
//      product would otherwise be one chain), summed by the softmax;
//   4. softmax read from the tensor memory by 8 warps (thread = position,
//      2 warps' maxima and sums per head through shared memory); P in fp16;
//   5. O^T[d, head] = V^T P^T (K = the 64 positions), one M = 128 slab of d
//      per accumulator, the slabs issued by the same four warps;
//   6. the unnormalised partial output [head][d] and (max, sum) per head in
//      base-2 units to the workspace, merged by the split-softmax combine kernel.
// With a layer-local bf16 ring ([FANOUT] item 2: the sliding-window state stays
// with the layer) the window entries' rows are the ring's bf16 rows.  bf16
// reaches far outside the fp16 range, so a chunk that holds ring rows is scaled
// by one exact power of two 2^e (its largest magnitude lands in [2^14, 2^15)):
// e is uniform over the chunk, so it leaves the tensor-core products as they
// are and comes off as 2^-e on the logits and on the partial output.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa2 {

namespace {

constexpr int kRows = 64;                   // entries per CTA
constexpr int kWorkers = 512;               // 16 warps
constexpr int kThreads = kWorkers + 32;     // + the warp that allocates TMEM and issues the MMAs
constexpr int kBlkBytes = kRows * 128;      // one 64-channel K block of the V tile: 64 rows x 128 B
constexpr uint32_t kDrainLimit = 65536;
constexpr int kIssuers = 4;                 // warps 12..15 (lane 0) issue the MMAs, one accumulator each
constexpr int kIssuer0 = 12;

struct Params {
    DevCache c;
    const __nv_bfloat16* q;   // [B*T][H][D]
    const int32_t* topk;      // [B*T][top_k]
    int T, H, top_k, window, nchunk;
    float scale;
    float* part_o;            // [seg][chunk][H][D]
    float* part_ml;           // [seg][chunk][H][2]
    uint32_t* status;
    uint32_t wait_limit;      // tries of the waits that guard work (not of the drain)
    uint32_t off_q, off_p, off_misc, tmem_cols;
    const __nv_bfloat16* ring;   // [batch][ring_len][D] or nullptr (window rows from the FP4 cache)
    int64_t ring_len;
    // a context-parallel shard (T = 1): the cache holds positions [cp_pos0[b],
    // cp_pos0[b] + L) of a sequence of cp_glens[b] positions; window and top-k
    // are global positions and only the shard's are attended (nullptr: off)
    const int32_t* cp_pos0;
    const int32_t* cp_glens;
};

template <int HG>
struct Misc {
    float fac[HG];               // per head of the group: softmax scale * log2(e) / query scale
    float red[4][HG];            // per head: maxima of the two row halves (0, 1), sums (2, 3)
    uint64_t vq_bar;             // V and Q written (one arrival per worker)
    uint64_t s_bar;              // S = V Q^T complete (one commit per issuing warp)
    uint64_t p_bar;              // P written (one arrival per softmax thread)
    uint64_t o_bar;              // O^T complete (one commit per issuing warp)
    uint64_t drain_bar;          // every MMA of the CTA complete (one commit per issuing warp)
    uint32_t tmem_base;
    uint32_t vmax;               // bits of the largest row magnitude of a chunk with ring rows
};

// Eight E2M1 codes (one 32-bit word, channel 2j in the low nibble of byte j)
// to four fp16 pairs holding value(code) * 2^-14, by bit placement alone: an
// E2M1 code s.e1e0.m placed at fp16 bits 15 and 11..9 is the fp16 number
// 2^(e-15) (1 + m/2) = value * 2^-14 for e > 0, and the subnormal m * 2^-15 =
// value * 2^-14 for e = 0 (the sign is kept, so -0 stays -0).  Pair k holds
// channels 2k (low half) and 2k + 1 (high half).  Integer instructions only:
// several times the throughput of the E2M1 conversion instruction.
__device__ __forceinline__ void e2m1x8_to_f16x2_scaled(uint32_t w, uint32_t* out) {
    // per byte: sign << 7 | magnitude << 1 of the byte's low nibble (fe) and high nibble (fo)
    const uint32_t fe = ((w << 4) & 0x80808080u) | ((w << 1) & 0x0E0E0E0Eu);
    const uint32_t fo = (w & 0x80808080u) | ((w >> 3) & 0x0E0E0E0Eu);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint32_t r;
        // high byte of the low half <- byte k of fe, high byte of the high half <- byte k of fo
        asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(fe), "r"(fo), "r"((uint32_t)(k << 4) | ((uint32_t)(4 + k) << 12)));
        out[k] = r & 0xFF00FF00u;
    }
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

// The float an order-preserving key came from (-0 comes back as +0).
__device__ __forceinline__ float key_to_float(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Named barrier of the softmax warps (the 8 warps that can read TMEM lanes 0..63).
__device__ __forceinline__ void softmax_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Named barrier of the 16 worker warps.
__device__ __forceinline__ void workers_sync() { asm volatile("bar.sync 2, 512;" ::: "memory"); }

// 2^e as a float, e in [-126, 127].
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

// RING: the launch has a layer-local ring (the window entries' rows come from it).
template <int HG, bool RING>
__global__ void __launch_bounds__(kThreads, 1) k_attn_tc(const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int D = p.c.dim, H = p.H;
    const int nkb = D / 64;                     // 64-channel K blocks
    uint8_t* sV = smem;                         // (nkb + 1) x [64 rows x 128 B]: M = 128 reads one block past the last
    uint8_t* sQ = smem + p.off_q;               // nkb x [HG rows x 128 B]
    uint8_t* sP = smem + p.off_p;               // [HG rows x 128 B]: 64 positions per head
    Misc<HG>* misc = reinterpret_cast<Misc<HG>*>(smem + p.off_misc);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int chunk = blockIdx.x, seg = blockIdx.y, h_base = blockIdx.z * HG;
    if (tid == 0) {
        tc::mbar_init(&misc->vq_bar, kWorkers);
        tc::mbar_init(&misc->s_bar, kIssuers);
        tc::mbar_init(&misc->p_bar, 256);
        tc::mbar_init(&misc->o_bar, kIssuers);
        tc::mbar_init(&misc->drain_bar, kIssuers);
        misc->vmax = 0u;
        tc::fence_mbar_init();
    }
    if (warp == kWorkers / 32) tc::tmem_alloc(&misc->tmem_base, p.tmem_cols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = misc->tmem_base;
    // everything below may read what the preceding kernel wrote
    pdl_begin();
    const int b = seg / p.T, j = seg % p.T;

    if (warp == kWorkers / 32) {
        // ================= the warp that owns the tensor memory: once every
        // MMA the issuing warps started is complete, release it
        bool ok = true;
        if (lane == 0) ok = tc::mbar_wait(&misc->drain_bar, 0, kDrainLimit);
        if (!ok) flag(p.status, kStatusTimeout);
        __syncwarp();
        tc::fence_before_sync();
        __syncthreads();                                  // the workers are done with TMEM
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, p.tmem_cols);
        return;
    }

    // ================= workers (16 warps)
    // every load that does not depend on another is issued first: the
    // group's queries (tph threads per head, `span` channels each), the
    // sequence length, this thread's top-k entry
    // tph threads per head, at least 8 channels each (one 16-byte load)
    const int tph = (kWorkers / HG) < (D / 8) ? (kWorkers / HG) : (D / 8);
    const int hl = tid / tph, qpart = tid % tph;
    const bool q_thread = hl < HG;
    const int span = D / tph;                        // 8 .. 64 channels, a multiple of 8
    uint4 qv[8];
    if (q_thread) {
        const __nv_bfloat16* src = p.q + ((int64_t)seg * H + h_base + hl) * D + qpart * span;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (8 * i < span) qv[i] = __ldg(reinterpret_cast<const uint4*>(src + 8 * i));
    }
    // rows: thread t covers row r = t % 64, channels [64 kp, 64 kp + 64) (K block kp)
    const int r = tid & (kRows - 1), kp = tid >> 6;
    const bool row_thread = kp < nkb;
    const int v_entry = chunk * kRows + r;
    const bool is_topk = v_entry >= p.window && v_entry < p.window + p.top_k;
    int32_t t_raw = -1;
    if (is_topk) t_raw = __ldg(p.topk + (int64_t)seg * p.top_k + (v_entry - p.window));
    const int64_t L = seq_len(p.c, b, p.status);
    // on a context-parallel shard the query sits at the sequence's last
    // position and the entries are the sequence's positions; the shard's own
    // ones are mapped to its positions below, the others masked
    const bool cp = p.cp_pos0 != nullptr;
    const int64_t Lg = cp ? (int64_t)__ldg(p.cp_glens + b) : L;
    const int64_t pq = cp ? Lg - 1 : L - p.T + j;
    int32_t t = -1;
    if (pq >= 0 && v_entry < p.window + p.top_k) {
        if (!is_topk) {
            t = pq - v_entry >= 0 ? (int32_t)(pq - v_entry) : -1;
        } else {
            t = t_raw;
            if (t < -1 || t >= Lg) { if (kp == 0) flag(p.status, kStatusBounds); t = -1; }
            else if (t > pq || t > pq - p.window) t = -1;   // future, or already in the window
        }
    }
    if (cp && t >= 0) {
        const int64_t ts = (int64_t)t - __ldg(p.cp_pos0 + b);
        t = ts >= 0 && ts < L ? (int32_t)ts : -1;
    }
    // a window entry of a launch with a ring takes its row from the ring (CTA-uniform: ring_chunk)
    const bool ring_chunk = RING && chunk * kRows < p.window;
    const bool ring_row = ring_chunk && v_entry < p.window && t >= 0;
    const int64_t slot = t >= 0 && !ring_row ? slot_of(p.c, b, t) : -1;
    if (t >= 0 && !ring_row && slot < 0) { if (kp == 0) flag(p.status, kStatusBounds); t = -1; }
    uint4 cv[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
    uint32_t sv = 0;
    uint4 rv[RING ? 8 : 1];                          // this thread's 64 bf16 channels of a ring row
    if (RING && row_thread && ring_row) {
        const uint4* src = reinterpret_cast<const uint4*>(p.ring + ((int64_t)b * p.ring_len + t % p.ring_len) * D + 64 * kp);
#pragma unroll
        for (int i = 0; i < (RING ? 8 : 1); ++i) rv[i] = __ldg(src + i);
    } else if (row_thread && t >= 0) {
        const uint8_t* row = p.c.rows + slot * p.c.row_stride;
        cv[0] = __ldg(reinterpret_cast<const uint4*>(row + 32 * kp));
        cv[1] = __ldg(reinterpret_cast<const uint4*>(row + 32 * kp + 16));
        sv = __ldg(reinterpret_cast<const uint32_t*>(row + (D >> 1) + 4 * kp));
    }

    // ---- queries to fp16 scaled by 2^e per head, the head's maximum in
    // [2^14, 2^15) so that every bf16 value down to 2^-24 of it is exact
    if (q_thread) {
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (8 * i < span) {
                const uint32_t wv[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    m = fmaxf(m, fmaxf(fabsf(__uint_as_float(wv[k] << 16)), fabsf(__uint_as_float(wv[k] & 0xFFFF0000u))));
            }
        }
        // the tph threads of a head are consecutive lanes of one warp (tph a power of two, at most 32)
        for (int o = 1; o < tph; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        int e = 0;
        if (m > 0.0f) {
            e = 14 - ((int)((__float_as_uint(m) >> 23) & 0xFF) - 127);
            e = e < -100 ? -100 : (e > 100 ? 100 : e);
        }
        const float up = __uint_as_float((uint32_t)(127 + e) << 23);
        // logits in base-2 units: softmax_scale * log2(e) / 2^e
        if (qpart == 0) misc->fac[hl] = p.scale * 1.4426950408889634f * __uint_as_float((uint32_t)(127 - e) << 23);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (8 * i < span) {
                const uint32_t wv[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
                uint32_t hv[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    __half2 hh = __floats2half2_rn(__uint_as_float(wv[k] << 16) * up,
                                                   __uint_as_float(wv[k] & 0xFFFF0000u) * up);
                    memcpy(&hv[k], &hh, 4);
                }
                const int d = qpart * span + 8 * i;       // 8 values: one 16-byte chunk
                *reinterpret_cast<uint4*>(sQ + (d >> 6) * (HG * 128) + tc::sw128_offset(hl, (d & 63) >> 3)) =
                    make_uint4(hv[0], hv[1], hv[2], hv[3]);
            }
        }
    }

    // ---- the chunk scale of a chunk with ring rows: 2^ec with its largest
    // magnitude in [2^14, 2^15) (an FP4 row counts as 6 x 448, the largest
    // E2M1 x E4M3 product); every other chunk has ec = 0
    int ec = 0;
    if (RING && ring_chunk) {
        float am = 0.0f;
        if (row_thread && ring_row) {
#pragma unroll
            for (int i = 0; i < (RING ? 8 : 1); ++i) {
                const uint32_t wv[4] = {rv[i].x, rv[i].y, rv[i].z, rv[i].w};
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    am = fmaxf(am, fmaxf(fabsf(__uint_as_float(wv[k] << 16)), fabsf(__uint_as_float(wv[k] & 0xFFFF0000u))));
            }
        } else if (row_thread && t >= 0) {
            am = 2688.0f;
        }
        const uint32_t mk = __reduce_max_sync(0xffffffffu, __float_as_uint(am));   // non-negative floats order as integers
        if (lane == 0) atomicMax(&misc->vmax, mk);
        workers_sync();
        const uint32_t vm = *reinterpret_cast<volatile uint32_t*>(&misc->vmax);
        if (vm != 0u) {
            ec = 14 - ((int)((vm >> 23) & 0xFF) - 127);
            ec = ec < -100 ? -100 : (ec > 100 ? 100 : ec);
        }
    }
    const float cup = RING ? exp2i(ec) : 1.0f, cdown = RING ? exp2i(-ec) : 1.0f;

    // ---- dequantise this thread's 64 channels of its row: value(code) *
    // value(scale), exact in fp16, into K block kp of the swizzled V tile
    // (masked rows are 0).  A warp's 16-byte stores walk 32 consecutive rows
    // of one K block: conflict-free under the 128-byte swizzle.
    if (RING && row_thread && ring_row) {
        // a ring row: bf16 x 2^ec, rounded once to fp16
        uint8_t* blk = sV + kp * kBlkBytes;
#pragma unroll
        for (int c = 0; c < (RING ? 8 : 1); ++c) {
            const uint32_t wv[4] = {rv[c].x, rv[c].y, rv[c].z, rv[c].w};
            uint32_t hv[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const __half2 hh = __floats2half2_rn(__uint_as_float(wv[k] << 16) * cup,
                                                     __uint_as_float(wv[k] & 0xFFFF0000u) * cup);
                memcpy(&hv[k], &hh, 4);
            }
            *reinterpret_cast<uint4*>(blk + tc::sw128_offset(r, c)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        }
    } else if (row_thread) {
        uint32_t s2[2];
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(s2[0]) : "h"((uint16_t)(sv & 0xFFFFu)));
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(s2[1]) : "h"((uint16_t)(sv >> 16)));
        const uint32_t two14 = 0x74007400u;                      // (2^14, 2^14) in fp16
        const uint32_t cw[8] = {cv[0].x, cv[0].y, cv[0].z, cv[0].w, cv[1].x, cv[1].y, cv[1].z, cv[1].w};
        uint8_t* blk = sV + kp * kBlkBytes;
#pragma unroll
        for (int c = 0; c < 8; ++c) {                            // 8 channels per 16-byte chunk c
            const uint32_t sc = c < 4 ? (c < 2 ? (s2[0] & 0xFFFFu) : (s2[0] >> 16))
                                      : (c < 6 ? (s2[1] & 0xFFFFu) : (s2[1] >> 16));
            const uint32_t s_pair = sc * 0x10001u;               // (s, s): scale of channels 16 (c / 2) ..
            uint32_t hv[4];
            e2m1x8_to_f16x2_scaled(cw[c], hv);
            // value * 2^-14 -> value (exact, a normal fp16), then times the
            // block scale (exact: E2M1 x E4M3 products fit fp16)
#pragma unroll
            for (int k = 0; k < 4; ++k) hv[k] = hmul2_u32(hmul2_u32(hv[k], two14), s_pair);
            if (RING && ec != 0) {
                // an FP4 row in a chunk with ring rows: times 2^ec, rounded once
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    __half2 hh;
                    memcpy(&hh, &hv[k], 4);
                    const float2 f = __half22float2(hh);
                    hh = __floats2half2_rn(f.x * cup, f.y * cup);
                    memcpy(&hv[k], &hh, 4);
                }
            }
            *reinterpret_cast<uint4*>(blk + tc::sw128_offset(r, c)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        }
    }
    tc::fence_proxy_async_smem();                     // V and Q are MMA operands
    tc::mbar_arrive(&misc->vq_bar);
    // ---- S = V Q^T: M = 128 rows (64 real), N = HG, K = D split in kIssuers
    // parts; issuer i accumulates K blocks [i nkb / kIssuers, (i + 1) nkb / kIssuers)
    // into TMEM columns [i HG, (i + 1) HG)
    const int issuer = warp - kIssuer0;               // 0..3 on the issuing warps
    const int nacc = nkb < kIssuers ? nkb : kIssuers; // S accumulators in use (D / 64 of them when D < 256)
    const bool issues = issuer >= 0 && issuer < kIssuers && lane == 0;
    const uint32_t v0 = tc::smem_u32(sV), q0 = tc::smem_u32(sQ), p0 = tc::smem_u32(sP);
    bool iss_ok = true;
    if (issues) {
        iss_ok = tc::mbar_wait(&misc->vq_bar, 0, p.wait_limit);
        if (iss_ok) {
            tc::fence_after_sync();
            const uint32_t idesc1 = tc::idesc_f16_f32(128, HG);
            const uint64_t dv = tc::desc_sw128(v0), dq = tc::desc_sw128(q0);
            // issuer i < nacc takes K blocks [i nkb / nacc, (i + 1) nkb / nacc); the others none
            const int kb0 = issuer < nacc ? issuer * nkb / nacc : 0;
            const int kb1 = issuer < nacc ? (issuer + 1) * nkb / nacc : 0;
            for (int kb = kb0; kb < kb1; ++kb)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    tc::mma_f16(tmem + (uint32_t)(issuer * HG),
                                tc::desc_at(dv, (uint32_t)kb * kBlkBytes + 32u * k),
                                tc::desc_at(dq, (uint32_t)kb * (HG * 128) + 32u * k), idesc1, kb != kb0 || k != 0);
        }
        tc::mma_commit(&misc->s_bar);                 // arrives once this issuer's MMAs are done
    }

    // ---- softmax straight from the tensor memory.  The 8 warps that can read
    // TMEM lanes 0..63 (warp % 4 < 2): thread = position (lane group quad),
    // cg = warp / 4 takes HG / 4 heads.  Per head: the maximum over the 64
    // positions (a warp-wide max of order-preserving integer keys, then the
    // two row halves' through shared memory); p = 2^(z - m) in fp16, stored
    // straight into the K-major P operand; the sum of the fp16 values as the
    // MMA will use them.
    constexpr int NV = HG / 4;                       // 4, 8 or 16 heads per softmax thread
    const int quad = warp & 3, cg = warp >> 2;
    const bool smx = quad < 2;
    // (every worker's writes before its vq_bar arrival -- the per-head
    // factors among them -- are visible once that phase is seen complete)
    bool ok = tc::mbar_wait(&misc->vq_bar, 0, p.wait_limit);
    ok = tc::mbar_wait(&misc->s_bar, 0, p.wait_limit) && ok;
    tc::fence_after_sync();
    ok = __all_sync(0xffffffffu, ok);                // warp-uniform from here on
    if (smx) {
        // a softmax thread's position is the row r = tid % 64 it loaded: its t says whether it is attended
        const int pos = quad * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        const bool valid = t >= 0;
        const int c0 = cg * NV;
        float z[NV];
        if (ok) {
            // S = the sum of the issuers' partial products over K: every
            // accumulator's columns in flight at once, one wait
            uint32_t rr[kIssuers][NV];
#pragma unroll
            for (int a = 0; a < kIssuers; ++a) {
                if (a >= nacc) break;                    // nacc is uniform over the CTA
                const uint32_t col = trow + (uint32_t)(a * HG + c0);
                if constexpr (NV == 4) tc::tmem_ld4_nowait(col, rr[a]);
                else if constexpr (NV == 8) tc::tmem_ld8_nowait(col, rr[a]);
                else tc::tmem_ld16_nowait(col, rr[a]);
            }
            tc::tmem_ld_wait();
            float v[NV];
#pragma unroll
            for (int i = 0; i < NV; ++i) v[i] = 0.0f;
#pragma unroll
            for (int a = 0; a < kIssuers; ++a) {
                if (a >= nacc) break;
#pragma unroll
                for (int i = 0; i < NV; ++i) v[i] += __uint_as_float(rr[a][i]);
            }
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                // (the chunk scale comes off last: v * fac alone stays inside the fp32 range)
                z[i] = valid ? v[i] * misc->fac[c0 + i] * cdown : -INFINITY;
                const uint32_t mk = __reduce_max_sync(0xffffffffu, ordered_key(z[i]));
                if (lane == i) misc->red[quad][c0 + i] = key_to_float(mk);
            }
        }
        softmax_sync();
        float sums[NV];
        if (ok) {
            uint8_t* prow = sP;
            const int pc = pos >> 3, el = pos & 7;
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const int h = c0 + i;
                const float m = fmaxf(misc->red[0][h], misc->red[1][h]);
                const float e = m == -INFINITY ? 0.0f : exp2f(z[i] - m);
                const __half ph = __float2half_rn(e);
                *reinterpret_cast<__half*>(prow + tc::sw128_offset(h, pc) + 2 * el) = ph;
                sums[i] = __half2float(ph);
            }
        }
        tc::fence_proxy_async_smem();                 // P is an MMA operand
        tc::mbar_arrive(&misc->p_bar);
        if (ok) {
            // per-head warp sums: an exchange that halves the values a lane
            // carries at each step; lanes 2 j and 2 j + 1 end with head j mod NV
#pragma unroll
            for (int w = NV / 2; w >= 1; w >>= 1) {
                const bool up = (lane & (2 * w)) != 0;
#pragma unroll
                for (int i = 0; i < w; ++i) {
                    const float send = up ? sums[i] : sums[i + w];
                    const float keep = up ? sums[i + w] : sums[i];
                    sums[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2 * w);
                }
            }
            sums[0] += __shfl_xor_sync(0xffffffffu, sums[0], 1);
#pragma unroll
            for (int o = 2 * NV; o < 32; o <<= 1) sums[0] += __shfl_xor_sync(0xffffffffu, sums[0], o);
            if (lane < 2 * NV && (lane & 1) == 0) misc->red[2 + quad][c0 + (lane >> 1)] = sums[0];
        }
        softmax_sync();
        if (ok && quad == 0 && lane < NV) {
            const int h = c0 + lane;
            float* ml = p.part_ml + (((int64_t)seg * p.nchunk + chunk) * H + h_base + h) * 2;
            ml[0] = fmaxf(misc->red[0][h], misc->red[1][h]);
            ml[1] = misc->red[2][h] + misc->red[3][h];
        }
    }

    // ---- O^T = V^T P^T: M = 128 channels per slab (two K blocks, MN-major),
    // N = HG, K = 64 positions; issuer i takes slabs i, i + kIssuers, ..
    if (issues) {
        bool pok = iss_ok && tc::mbar_wait(&misc->p_bar, 0, p.wait_limit);
        if (pok) {
            tc::fence_after_sync();
            const uint32_t idesc2 = tc::idesc_f16_f32(128, HG, /*a_mn=*/true, /*b_mn=*/false);
            const uint64_t dvt = tc::desc_mn_sw128(v0, kBlkBytes, 1024), dp = tc::desc_sw128(p0);
            for (int s = issuer; s < D / 128; s += kIssuers)
#pragma unroll
                for (int ks = 0; ks < kRows / 16; ++ks)
                    tc::mma_f16(tmem + (uint32_t)(kIssuers * HG + s * HG),
                                tc::desc_at(dvt, (uint32_t)(2 * s) * kBlkBytes + ks * 2048u), tc::desc_at(dp, 32u * ks),
                                idesc2, ks != 0);
        }
        tc::mma_commit(&misc->o_bar);
        tc::mma_commit(&misc->drain_bar);
    }

    // ---- unnormalised partial output, [head][d]: warp w reads slab w / 4,
    // TMEM lanes of its quad (lane = d within the slab); a warp's stores of
    // one head are 32 consecutive floats
    {
        ok = tc::mbar_wait(&misc->o_bar, 0, p.wait_limit) && ok;
        tc::fence_after_sync();
        ok = __all_sync(0xffffffffu, ok);
        const int s2 = warp >> 2;
        if (ok && s2 < D / 128) {
            const int d = s2 * 128 + quad * 32 + lane;
            const uint32_t tcol = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(kIssuers * HG + s2 * HG);
            float* po = p.part_o + (((int64_t)seg * p.nchunk + chunk) * H + h_base) * D + d;
#pragma unroll
            for (int c0 = 0; c0 < HG; c0 += 16) {
                float v[16];
                tc::tmem_ld16(tcol + c0, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) po[(int64_t)(c0 + i) * D] = v[i] * cdown;
            }
        }
    }
    if (!ok) flag(p.status, kStatusTimeout);
    tc::fence_before_sync();
    __syncthreads();                                  // TMEM is released by the MMA warp
}

template <int HG>
size_t attn_tc_smem(int D, uint32_t* off_q, uint32_t* off_p, uint32_t* off_misc) {
    const uint32_t v = (uint32_t)(D / 64 + 1) * kBlkBytes;           // + one block read past the end by M = 128
    const uint32_t qbytes = ((uint32_t)(D / 64) * HG * 128 + 1023) & ~1023u;
    const uint32_t pbytes = ((uint32_t)HG * 128 + 1023) & ~1023u;
    *off_q = v;
    *off_p = v + qbytes;
    *off_misc = v + qbytes + pbytes;
    return (size_t)v + qbytes + pbytes + sizeof(Misc<HG>) + 1024;
}

template <int HG, bool RING>
cudaError_t launch_hg(const DevCache& c, const Params& p0, int nseg, cudaStream_t st) {
    Params p = p0;
    uint32_t cols = 32;
    while (cols < (uint32_t)(kIssuers * HG + (c.dim / 128) * HG)) cols <<= 1;
    p.tmem_cols = cols;
    const size_t smem = attn_tc_smem<HG>(c.dim, &p.off_q, &p.off_p, &p.off_misc);
    cudaError_t e = cudaFuncSetAttribute(k_attn_tc<HG, RING>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_attn_tc<HG, RING>, dim3((unsigned)p.nchunk, (unsigned)nseg, (unsigned)(p.H / HG)),
                      dim3(kThreads), smem, st, p);
}

}  // namespace

bool attn_tc_supported(const DevCache& c, int H) {
    uint32_t a, b, d;
    return c.dim % 128 == 0 && c.dim <= 512 && (H == 16 || H == 32 || H == 64) &&
           attn_tc_smem<64>(c.dim, &a, &b, &d) <= 227 * 1024;
}

int attn_tc_rows_per_chunk() { return kRows; }

int attn_tc_heads_per_cta(int H, int nchunk, int nseg, int num_sms) {
    int hg = H;
    while (hg > 16 && (int64_t)nchunk * nseg * (H / hg) < num_sms) hg >>= 1;
    return hg;
}

cudaError_t launch_attention_tc(const DevCache& c, const void* q, int T, int H, const int32_t* topk, int top_k,
                                int window, float sm_scale, const Ring& ring, const AttnWork& aw, uint32_t* status,
                                cudaStream_t st, int num_sms, const CpShard& cp) {
    if (cp.pos0 && (T != 1 || ring.rows)) return cudaErrorInvalidValue;
    Params p;
    p.cp_pos0 = cp.pos0;
    p.cp_glens = cp.glens;
    p.c = c;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.topk = topk;
    p.T = T;
    p.H = H;
    p.top_k = top_k;
    p.window = window;
    p.nchunk = aw.nchunk;
    p.scale = sm_scale;
    p.part_o = aw.part_o;
    p.part_ml = aw.part_ml;
    p.status = status;
    p.wait_limit = wait_limit();
    p.ring = ring.rows;
    p.ring_len = ring.len;
    const int nseg = c.batch * T;
    const int hg = attn_tc_heads_per_cta(H, aw.nchunk, nseg, num_sms);
    if (ring.rows) {
        if (hg == 16) return launch_hg<16, true>(c, p, nseg, st);
        if (hg == 32) return launch_hg<32, true>(c, p, nseg, st);
        return launch_hg<64, true>(c, p, nseg, st);
    }
    if (hg == 16) return launch_hg<16, false>(c, p, nseg, st);
    if (hg == 32) return launch_hg<32, false>(c, p, nseg, st);
    return launch_hg<64, false>(c, p, nseg, st);
}

}  // namespace csa2

// Quantise-on-append: bf16 latent rows -> FP4 rows (E2M1 codes + one E4M3
// scale per 16 channels, no global scale), and index keys -> E4M3 or fp32.
//
// Format: tldrocket.com, "DeepSeek AI Released DeepSeek-V4.1-Flash with 1M
// Context, FP4 KV Cache, and Cross-Layer Attention Reuse", paragraph 4.
// Per 16-channel block:  s = E4M3_rne_sat(amax / 6),  c = E2M1_rne_sat(x / s),
// both divisions IEEE binary32; s == 0 gives all-zero codes.
//
// One thread owns one 16-channel block: 32 B of bf16 in (two 16 B loads), 8 B
// of codes and 1 scale byte out.  Consecutive threads own consecutive blocks
// of a row, so a warp reads 1 KB and writes 256 + 32 contiguous bytes of a
// D = 512 row.  The kernel is a streaming HBM pass (read 2 B, write 0.5625 B
// per channel).
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

__global__ void __launch_bounds__(256)
k_append_quant(DevCache c, const __nv_bfloat16* __restrict__ x, const void* __restrict__ idx_new,
               int idx_new_f32, const int32_t* __restrict__ start_pos, int n_new, uint32_t* status) {
    pdl_begin();
    const int nblk = c.dim >> 4;
    const int64_t rows_total = (int64_t)c.batch * n_new;
    const int64_t n_row_work = rows_total * nblk;
    const int kblk = c.idx_dim >> 4;
    const int64_t n_key_work = idx_new ? rows_total * kblk : 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;

    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n_row_work + n_key_work; g += stride) {
        const bool is_row = g < n_row_work;
        const int64_t gg = is_row ? g : g - n_row_work;
        const int per = is_row ? nblk : kblk;
        const int blk = (int)(gg % per);
        const int64_t r = gg / per;
        const int b = (int)(r / n_new);
        const int64_t t = (int64_t)__ldg(start_pos + b) + (r - (int64_t)b * n_new);
        if (t < 0 || t >= c.cap) { flag(status, kStatusBounds); continue; }
        const int64_t slot = slot_of(c, b, t);
        if (slot < 0) { flag(status, kStatusBounds); continue; }

        if (is_row) {
            const uint4* src = reinterpret_cast<const uint4*>(x + r * c.dim + blk * 16);
            uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
            const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            float v[16];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                v[2 * k] = __uint_as_float(w[k] << 16);
                v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
            }
            float amax = 0.0f;
#pragma unroll
            for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(v[k]));
            const uint8_t sc = (uint8_t)(cvt_e4m3x2(0.0f, __fdiv_rn(amax, 6.0f)) & 0xFF);
            const float s = e4m3_to_float(sc);
            uint2 codes = make_uint2(0u, 0u);
            if (s != 0.0f) {
                float q[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) q[k] = __fdiv_rn(v[k], s);
                codes.x = cvt_e2m1x8(q);
                codes.y = cvt_e2m1x8(q + 8);
            }
            uint8_t* row = c.rows + slot * c.row_stride;
            *reinterpret_cast<uint2*>(row + blk * 8) = codes;
            row[(c.dim >> 1) + blk] = sc;
        } else {
            float v[16];
            const int64_t off = r * c.idx_dim + blk * 16;
            if (idx_new_f32) {
                const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(idx_new) + off);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float4 f = __ldg(src + k);
                    v[4 * k] = f.x; v[4 * k + 1] = f.y; v[4 * k + 2] = f.z; v[4 * k + 3] = f.w;
                }
            } else {
                const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(idx_new) + off);
                uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
                const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    v[2 * k] = __uint_as_float(w[k] << 16);
                    v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
                }
            }
            if (c.key_dtype == 2) {
                uint32_t o[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint32_t lo = cvt_e4m3x2(v[4 * k + 1], v[4 * k]);
                    uint32_t hi = cvt_e4m3x2(v[4 * k + 3], v[4 * k + 2]);
                    o[k] = lo | (hi << 16);
                }
                *reinterpret_cast<uint4*>(static_cast<uint8_t*>(c.keys) + slot * c.idx_dim + blk * 16) =
                    make_uint4(o[0], o[1], o[2], o[3]);
            } else {
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(c.keys) + slot * c.idx_dim + blk * 16);
#pragma unroll
                for (int k = 0; k < 4; ++k) dst[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
            }
        }
    }
}

namespace {

// Rows (codes then scales, dim / 2 + dim / 16 bytes) and index keys of
// positions start_pos[b] + i, between the cache and packed buffers
// [batch][n][...]: one warp per (sequence, position), 2-byte words for rows
// and 4-byte words for keys.  EXPORT: cache -> buffers (zeros and a bounds
// flag for a position outside the cache); otherwise buffers -> cache (the
// position skipped and flagged).
template <bool EXPORT>
__global__ void __launch_bounds__(256)
k_rows_io(DevCache c, const int32_t* __restrict__ start_pos, int n, uint8_t* rows, uint8_t* keys, uint32_t* status) {
    pdl_begin();
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= (int64_t)c.batch * n) return;
    const int lane = threadIdx.x & 31;
    const int b = (int)(r / n), i = (int)(r % n);
    const int64_t t = (int64_t)__ldg(start_pos + b) + i;
    const int64_t slot = t >= 0 && t < c.cap ? slot_of(c, b, t) : -1;
    if (slot < 0 && lane == 0) flag(status, kStatusBounds);
    const int row_bytes = c.dim / 2 + c.dim / 16;
    const int key_bytes = c.key_dtype == 2 ? c.idx_dim : 4 * c.idx_dim;
    uint16_t* brow = reinterpret_cast<uint16_t*>(rows + r * row_bytes);
    uint32_t* bkey = reinterpret_cast<uint32_t*>(keys + r * key_bytes);
    if (EXPORT) {
        const uint16_t* crow = slot >= 0 ? reinterpret_cast<const uint16_t*>(c.rows + slot * c.row_stride) : nullptr;
        const uint32_t* ckey = slot >= 0 ? reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(c.keys) +
                                                                             slot * key_bytes) : nullptr;
        for (int w = lane; w < row_bytes / 2; w += 32) brow[w] = crow ? crow[w] : 0;
        if (keys)
            for (int w = lane; w < key_bytes / 4; w += 32) bkey[w] = ckey ? ckey[w] : 0u;
    } else if (slot >= 0) {
        uint16_t* crow = reinterpret_cast<uint16_t*>(c.rows + slot * c.row_stride);
        uint32_t* ckey = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(c.keys) + slot * key_bytes);
        for (int w = lane; w < row_bytes / 2; w += 32) crow[w] = brow[w];
        if (keys)
            for (int w = lane; w < key_bytes / 4; w += 32) ckey[w] = bkey[w];
    }
}

// Diagnostic: the quantiser's own conversions (cvt_e2m1x8 for the codes,
// cvt_e4m3x2 for the scales and index keys) applied to arbitrary fp32 values,
// one code per output byte (E2M1 in the low nibble).  A thread takes 8
// consecutive values; a tail shorter than 8 is padded with zeros that are not
// written back.
__global__ void __launch_bounds__(256)
k_debug_encode(int format, const float* __restrict__ x, int64_t n, uint8_t* __restrict__ out) {
    pdl_begin();
    const int64_t groups = (n + 7) / 8;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i0 = g * 8;
        float v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = i0 + k < n ? x[i0 + k] : 0.0f;
        uint8_t c[8];
        if (format == 0) {
            const uint32_t w = cvt_e2m1x8(v);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                c[2 * k] = (uint8_t)((w >> (8 * k)) & 0xF);
                c[2 * k + 1] = (uint8_t)((w >> (8 * k + 4)) & 0xF);
            }
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint16_t h = cvt_e4m3x2(v[2 * k + 1], v[2 * k]);
                c[2 * k] = (uint8_t)(h & 0xFF);
                c[2 * k + 1] = (uint8_t)(h >> 8);
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (i0 + k < n) out[i0 + k] = c[k];
    }
}

}  // namespace

cudaError_t launch_debug_encode(int format, const float* x, int64_t n, uint8_t* out, cudaStream_t st, int num_sms) {
    int64_t blocks = (n / 8 + 255) / 256 + 1;
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    return launch_pdl(k_debug_encode, dim3((unsigned)blocks), dim3(256), 0, st, format, x, n, out);
}

cudaError_t launch_rows_io(const DevCache& c, bool to_buffers, const int32_t* start_pos, int n, void* rows, void* keys,
                           uint32_t* status, cudaStream_t st) {
    const int64_t r = (int64_t)c.batch * n;
    const dim3 grid((unsigned)((r + 7) / 8));
    uint8_t* rb = static_cast<uint8_t*>(rows);
    uint8_t* kb = static_cast<uint8_t*>(keys);
    return to_buffers ? launch_pdl(k_rows_io<true>, grid, dim3(256), 0, st, c, start_pos, n, rb, kb, status)
                      : launch_pdl(k_rows_io<false>, grid, dim3(256), 0, st, c, start_pos, n, rb, kb, status);
}

cudaError_t launch_append_quant(const DevCache& c, const void* x, const void* idx_new, int idx_new_f32,
                                const int32_t* start_pos, int n_new, uint32_t* status, cudaStream_t st,
                                int num_sms) {
    const int64_t work = (int64_t)c.batch * n_new * ((c.dim >> 4) + (idx_new ? (c.idx_dim >> 4) : 0));
    int64_t blocks = (work + 255) / 256;
    const int64_t max_blocks = (int64_t)num_sms * 8;
    if (blocks > max_blocks) blocks = max_blocks;
    if (blocks < 1) blocks = 1;
    return launch_pdl(k_append_quant, dim3((unsigned)blocks), dim3(256), 0, st, c, static_cast<const __nv_bfloat16*>(x), idx_new, idx_new_f32,
                                                      start_pos, n_new, status);
}

}  // namespace csa2

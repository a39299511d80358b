// Device-side helpers shared by the libcsa2 kernels (sm_100a).
#pragma once
#include <cstdint>
#include <utility>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace csa2 {

// Sticky status bits ORed into the workspace status word by kernels.
constexpr uint32_t kStatusBounds = 1u;
constexpr uint32_t kStatusTimeout = 2u;

// A by-value copy of csa2_cache plus the derived per-sequence capacity.
struct DevCache {
    uint8_t* rows;
    void* keys;
    const int32_t* page_table;
    const int32_t* seq_lens;
    int32_t batch, max_pages, page_size, dim, idx_dim, row_stride;
    int64_t seq_stride, n_slots, cap;
    int32_t key_dtype;  // 0 fp32, 2 e4m3
};

__device__ __forceinline__ void flag(uint32_t* status, uint32_t bit) {
    if (status) atomicOr(status, bit);
}

// The debug build (-DCSA2_DEBUG_BOUNDS) checks every position and page where
// it becomes a cache slot (slot_of, the one place all kernels translate
// positions): t outside [0, cap) and a contiguous slot beyond the cache give
// -1, which every caller flags in the status word and skips.  Indices taken
// from caller buffers (top-k, pool and candidate entries, page ids) are
// checked in every build.
#ifdef CSA2_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif

// Slot of position t of sequence b, or -1 when the page table points outside
// the cache.  The caller guarantees 0 <= t < cap (checked in the debug build).
__device__ __forceinline__ int64_t slot_of(const DevCache& c, int b, int64_t t) {
    if (kDebugBounds && (t < 0 || t >= c.cap || b < 0 || b >= c.batch)) return -1;
    if (c.page_table) {
        int64_t pg = t / c.page_size;
        int32_t phys = __ldg(c.page_table + (int64_t)b * c.max_pages + pg);
        int64_t s = (int64_t)phys * c.page_size + (t - pg * c.page_size);
        return (phys < 0 || s >= c.n_slots) ? -1 : s;
    }
    const int64_t s = (int64_t)b * c.seq_stride + t;
    return (kDebugBounds && s >= c.n_slots) ? -1 : s;
}

// Valid length of sequence b clamped to the capacity (flags a longer one).
__device__ __forceinline__ int64_t seq_len(const DevCache& c, int b, uint32_t* status) {
    int64_t L = __ldg(c.seq_lens + b);
    if (L > c.cap || L < 0) {
        flag(status, kStatusBounds);
        L = L < 0 ? 0 : c.cap;
    }
    return L;
}

// ---------------------------------------------------------------- conversions
// E4M3 round-to-nearest-even, saturating: `hi` lands in the upper byte.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float hi, float lo) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Four E2M1 pairs (round-to-nearest-even, saturating) packed into 32 bits:
// byte k holds x[2k] in its low nibble and x[2k+1] in its high nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float* x) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(x[0]), "f"(x[1]), "f"(x[2]), "f"(x[3]), "f"(x[4]), "f"(x[5]), "f"(x[6]), "f"(x[7]));
    return r;
}

// Two E4M3 bytes (low byte first) -> two halves; exact.
__device__ __forceinline__ __half2 e4m3x2_to_half2(uint16_t v) {
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
    __half2 h;
    memcpy(&h, &r, 4);
    return h;
}

__device__ __forceinline__ float e4m3_to_float(uint8_t v) {
    return __low2float(e4m3x2_to_half2((uint16_t)v));
}

// Two E2M1 codes (one byte, low nibble first) -> two halves; exact.
__device__ __forceinline__ __half2 e2m1x2_to_half2(uint8_t v) {
    uint32_t r;
    uint16_t in = v;
    asm("{\n\t.reg .b8 b, u;\n\tmov.b16 {b, u}, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(r) : "h"(in));
    __half2 h;
    memcpy(&h, &r, 4);
    return h;
}

// ---------------------------------------------------------------- launches
// Programmatic dependent launch: every kernel of the library is launched so
// that it may start while the previous kernel on the stream finishes; it calls
// pdl_begin() before touching global memory, which waits until the previous
// kernel has completed and its writes are visible, and then lets the next
// kernel launch early.
__device__ __forceinline__ void pdl_begin() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Monotone map of fp32 onto uint32 (larger float -> larger key); -0 == +0.
__device__ __forceinline__ uint32_t ordered_key(float f) {
    uint32_t u = __float_as_uint(f == 0.0f ? 0.0f : f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The score an ordered key came from (-0 comes back as +0).
__device__ __forceinline__ float key_score(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Selection key of a score: 0 (never selected) for an element that is not a
// candidate or whose score is NaN -- the mark a scorer leaves on a position it
// had to skip (a page id outside the cache) -- else the ordered key, which is
// never 0 for a non-NaN float.
__device__ __forceinline__ uint32_t select_key(float f, bool candidate) {
    return (candidate && !isnan(f)) ? ordered_key(f) : 0u;
}

}  // namespace csa2

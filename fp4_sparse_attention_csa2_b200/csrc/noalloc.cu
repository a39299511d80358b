// Reindex scoring + top-k for callers that cannot allocate device memory.
//
// csa2_index_reindex needs a caller-provided workspace.  Some callers have no
// way to provide one: code that runs while a framework is capturing a CUDA
// graph under a policy that forbids allocations during capture, plugins that
// are handed tensors but no allocator, and real-time paths that must not pay
// for cudaMalloc's implicit device synchronisation.  This variant keeps its
// scratch (the rescored pool and a status word) in a fixed array in device
// memory that is part of the library itself, so the caller passes only inputs
// and outputs.
#include <mutex>

#include <cuda.h>

#include "abi_checks.h"

namespace csa2 {
namespace {

// 4 MiB of scratch: 256 bytes of header (the status word), the per-segment
// arrival counters of the fused Reindex kernel (rounded up to 256 bytes),
// then the rescored pool: batch * T * pool_k floats.
constexpr size_t kScratchBytes = (size_t)4 << 20;
constexpr size_t kScratchHeader = 256;
constexpr int kMaxContexts = 64;

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_reindex_scratch[kScratchBytes];

// Device address of g_reindex_scratch per CUDA context, looked up once per
// context with that context current.  In host code the array's name is only a
// stand-in for the symbol, never a device address, so the address must come
// from cudaGetSymbolAddress.  The address belongs to the context it was looked
// up in (the module is loaded again into a new context, e.g. after
// cudaDeviceReset), so the cache is keyed on the current context's unique id
// (a new context gets a new id even where its handle value is reused).
using CtxGetCurrent = CUresult (*)(CUcontext*);
using CtxGetId = CUresult (*)(CUcontext, unsigned long long*);

void* driver_fn(const char* name) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &f, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return nullptr;
    return f;
}

std::mutex g_mu;
unsigned long long g_ctx[kMaxContexts] = {};
void* g_addr[kMaxContexts] = {};
int g_n = 0;

cudaError_t scratch_address(void** out) {
    static const CtxGetCurrent get = reinterpret_cast<CtxGetCurrent>(driver_fn("cuCtxGetCurrent"));
    static const CtxGetId get_id = reinterpret_cast<CtxGetId>(driver_fn("cuCtxGetId"));
    if (!get || !get_id) return cudaErrorNotSupported;
    CUcontext ctx = nullptr;
    if (get(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    if (!ctx) {
        // no context bound to this thread yet: bind the current device's
        // primary context (cudaSetDevice initialises it and makes it current)
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        e = cudaSetDevice(dev);
        if (e != cudaSuccess) return e;
        if (get(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
    }
    unsigned long long id = 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_n; ++i)
        if (g_ctx[i] == id) {
            *out = g_addr[i];
            return cudaSuccess;
        }
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_reindex_scratch);   // in the current context
    if (e != cudaSuccess) return e;
    if (g_n < kMaxContexts) {
        g_ctx[g_n] = id;
        g_addr[g_n] = p;
        ++g_n;
    }
    *out = p;
    return cudaSuccess;
}

}  // namespace
}  // namespace csa2

using namespace csa2;

extern "C" csa2_status csa2_index_reindex_noalloc(const csa2_cache* cache, const void* q_idx, csa2_dtype q_dtype,
                                                  const float* head_w, int T, int H_I, const int32_t* pool_idx,
                                                  int pool_k, int top_k, int32_t* topk_idx, void* stream) {
    CSA2_RANGE("csa2_index_reindex_noalloc");
    // the same checks, in the same order and with the same statuses, as
    // csa2_index_reindex; only then the bound of the fixed scratch
    csa2_status s = check_reindex_args(cache, q_idx, q_dtype, head_w, T, H_I, pool_idx, pool_k, top_k, topk_idx);
    if (s != CSA2_OK) return s;
    const size_t nseg = (size_t)cache->batch * T;
    const size_t cnt_bytes = (sizeof(uint32_t) * nseg + 255) / 256 * 256;
    const size_t need = kScratchHeader + cnt_bytes + sizeof(float) * nseg * pool_k;
    if (need > kScratchBytes) return CSA2_ERR_UNSUPPORTED;

    void* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return CSA2_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t* status = static_cast<uint32_t*>(scratch);
    uint32_t* counters = reinterpret_cast<uint32_t*>(static_cast<char*>(scratch) + kScratchHeader);
    float* scores = reinterpret_cast<float*>(static_cast<char*>(scratch) + kScratchHeader + cnt_bytes);
    // the status word and the counters must start at zero (a call cut short
    // could have left them set); the scorer writes a score for every pool
    // entry (a NaN marks one it rejected), so nothing stale from an earlier
    // call is read
    if (cudaMemsetAsync(status, 0, kScratchHeader + cnt_bytes, st) != cudaSuccess) return CSA2_ERR_CUDA;

    const DevCache d = dev_cache(cache);
    if (reindex_tc_supported(d, H_I)) {
        const cudaError_t e = launch_reindex_tc(d, q_idx, head_w, T, H_I, pool_idx, pool_k, top_k, topk_idx, scores,
                                                counters, nullptr, nullptr, status, st);
        return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
    }
    cudaError_t e = launch_score_pool(d, q_idx, q_dtype == CSA2_F32, head_w, T, H_I, pool_idx, pool_k, scores, status,
                                      st);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;
    SelSrc src;
    src.vals = scores;
    src.vals_stride = pool_k;
    src.ids = pool_idx;
    src.ids_stride = pool_k;
    src.gather = 0;
    src.n = pool_k;
    src.seq_lens = cache->seq_lens;
    src.T = T;
    src.cap = d.cap;
    // a pool-sized selection runs in one CTA per segment, in shared memory and registers
    e = launch_select_local(src, (int)nseg, top_k, topk_idx, nullptr, top_k, 0, nullptr, 0, st);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

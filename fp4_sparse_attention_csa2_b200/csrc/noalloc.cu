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

#include "../../include/csa2.h"
#include "kernels.h"

namespace csa2 {
namespace {

// 4 MiB of scratch: 256 bytes of header (status word) followed by the rescored
// pool, so batch * T * pool_k may not exceed (4 MiB - 256) / 4 = 1,048,512.
constexpr size_t kScratchBytes = (size_t)4 << 20;
constexpr size_t kScratchHeader = 256;
constexpr int kMaxDevices = 64;

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_reindex_scratch[kScratchBytes];

// Device address of g_reindex_scratch per device, looked up once per device.
// In host code the array's name is only a stand-in for the symbol, never a
// device address, so the address must come from cudaGetSymbolAddress.
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_reindex_scratch);   // with `dev` current
        if (e != cudaSuccess) return e;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace csa2

using namespace csa2;

extern "C" csa2_status csa2_index_reindex_noalloc(const csa2_cache* cache, const void* q_idx, csa2_dtype q_dtype,
                                                  const float* head_w, int T, int H_I, const int32_t* pool_idx,
                                                  int pool_k, int top_k, int32_t* topk_idx, void* stream) {
    if (!cache || !cache->kv_rows || !cache->idx_keys || !cache->seq_lens || !q_idx || !head_w || !pool_idx ||
        !topk_idx)
        return CSA2_ERR_INVALID_ARG;
    if (T < 1 || H_I < 1 || H_I > 64 || T * H_I > 256 || top_k < 1 || top_k > pool_k || pool_k > 16384 ||
        cache->batch < 1 || cache->idx_dim != 64)
        return CSA2_ERR_INVALID_ARG;
    if ((cache->idx_key_dtype == CSA2_E4M3 && q_dtype != CSA2_BF16) ||
        (cache->idx_key_dtype == CSA2_F32 && q_dtype != CSA2_F32))
        return CSA2_ERR_INVALID_ARG;
    // the fixed scratch bounds the problem size
    const size_t need = kScratchHeader + sizeof(float) * (size_t)cache->batch * T * pool_k;
    if (need > kScratchBytes) return CSA2_ERR_UNSUPPORTED;
    // the workspace-based entry point's validation covers the cache itself
    if (csa2_workspace_bytes(cache, T, 1, pool_k, top_k, 0) == 0) return CSA2_ERR_INVALID_ARG;

    void* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return CSA2_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t* status = static_cast<uint32_t*>(scratch);
    float* scores = reinterpret_cast<float*>(static_cast<char*>(scratch) + kScratchHeader);
    // the status word must start at zero; the scores are all written before they are read
    if (cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) return CSA2_ERR_CUDA;

    DevCache d;
    d.rows = cache->kv_rows;
    d.keys = cache->idx_keys;
    d.page_table = cache->page_table;
    d.seq_lens = cache->seq_lens;
    d.batch = cache->batch;
    d.max_pages = cache->max_pages;
    d.page_size = cache->page_size;
    d.dim = cache->dim;
    d.idx_dim = cache->idx_dim;
    d.row_stride = cache->row_stride;
    d.seq_stride = cache->seq_stride_slots;
    d.n_slots = cache->n_slots;
    d.cap = cache->page_table ? (int64_t)cache->max_pages * cache->page_size : cache->seq_stride_slots;
    d.key_dtype = cache->idx_key_dtype == CSA2_E4M3 ? 2 : 0;

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
    SelWork unused = {};   // a pool-sized selection runs in one CTA per segment, in shared memory
    e = launch_select(src, unused, cache->batch * T, top_k, topk_idx, top_k, st, false);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

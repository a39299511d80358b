// Host-side argument checks and cache conversion shared by the C-ABI entry
// points (api.cu, noalloc.cu), so that every entry point validates the same
// arguments the same way and returns the same status for the same fault.
#pragma once
#include "../../include/csa2.h"
#include "kernels.h"

// NVTX ranges, one per C-ABI call (built with -DCSA2_NVTX, the debug build):
// a profiler's timeline shows each call and the kernels it enqueued.  NVTX
// is header-only and costs a branch per call when no tool is attached.
#ifdef CSA2_NVTX
#include <nvtx3/nvToolsExt.h>
namespace csa2 {
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace csa2
#define CSA2_RANGE(name) ::csa2::NvtxRange csa2_nvtx_range_(name)
#else
#define CSA2_RANGE(name) ((void)0)
#endif

namespace csa2 {

// CSA2_OK, or the status csa2_index_reindex returns for these arguments
// before any launch: the cache, the query / weight / pool / top-k pointers
// (non-null, 16-byte aligned), the shape bounds and the dtype pairing.
csa2_status check_reindex_args(const csa2_cache* c, const void* q_idx, csa2_dtype q_dtype, const float* head_w,
                               int T, int H_I, const int32_t* pool_idx, int pool_k, int top_k,
                               const int32_t* topk_idx);

// The by-value device view of a validated cache.
DevCache dev_cache(const csa2_cache* c);

}  // namespace csa2

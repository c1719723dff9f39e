// zero_step_noalloc(): the full step for callers that cannot allocate device
// memory.
//
// zero_step() reports the gradient norm and overflow flag through a scratch
// workspace that the caller allocates.  Some callers cannot do that: a
// runtime whose device memory is carved up in advance by its own pool and that
// may not call cudaMalloc afterwards, a C program linking only this library
// without any allocator of its own, or code that must not allocate on the
// critical path.  For them this entry point keeps the scratch in a
// fixed-size array in device memory owned by the library.  The array lives on
// every GPU that loads the library until the process exits.
#include <cuda_runtime.h>

#include <map>
#include <mutex>
#include <string>

#include "zero_internal.h"

using zero_detail::set_error;

namespace {

// Largest scratch the no-allocation entry point can use: one fp64 partial and
// one u32 count per CTA slot of the step kernels, plus the guarded step's
// decision word (49,408 bytes).
constexpr uint64_t kNoAllocScratchBytes = zero_detail::kWorkspaceBytes;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side handle, so the address is looked up
// once per device (with that device current) and cached.
zero_status_t scratch_address(void **out) {
    static std::mutex mu;
    static std::map<int, void *> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return set_error(ZERO_ECUDA, std::string("zero_step_noalloc: cudaGetDevice: ") + cudaGetErrorString(e));
    std::lock_guard<std::mutex> g(mu);
    auto it = cache.find(dev);
    if (it != cache.end()) {
        *out = it->second;
        return ZERO_OK;
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
        return set_error(ZERO_ECUDA, std::string("zero_step_noalloc: cudaGetSymbolAddress: ") +
                                         cudaGetErrorString(e));
    cache[dev] = p;
    *out = p;
    return ZERO_OK;
}

}  // namespace

ZERO_API zero_status_t zero_step_noalloc(const zero_plan_t *plan, const zero_bufs_t *bufs,
                                         const zero_adam_t *adam, uint64_t t, void *stream) {
    zero_detail::clear_error();
    if (!plan || !bufs) return set_error(ZERO_EINVAL, "zero_step_noalloc: NULL argument");
    uint64_t need = 0;
    zero_status_t st = zero_plan_query(plan, ZERO_Q_WORKSPACE_BYTES, 0, &need);
    if (st != ZERO_OK) return st;
    if (need > kNoAllocScratchBytes)
        return set_error(ZERO_EINVAL, "zero_step_noalloc: the step needs " + std::to_string(need) +
                                          " bytes of scratch, more than the " +
                                          std::to_string(kNoAllocScratchBytes) +
                                          "-byte static array; use zero_step with a workspace");
    void *scratch = nullptr;
    st = scratch_address(&scratch);
    if (st != ZERO_OK) return st;
    // The step kernels add their per-CTA norm partials and non-finite counts
    // into this array.  zero_step() clears it with cudaMemsetAsync on the
    // stream before the first bucket's kernel, so whatever an earlier call
    // left in it does not reach this step's norm or overflow flag.
    zero_bufs_t local = *bufs;
    local.workspace = scratch;
    local.workspace_bytes = kNoAllocScratchBytes;
    return zero_step(plan, &local, adam, t, stream);
}

// Host-side helpers shared by the .cu files of the library (launch checks,
// alignment tests, the device's SM count).  Not part of the ABI.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <map>
#include <mutex>
#include <string>

#include "zero_internal.h"

namespace zero_host {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool mult8(int64_t x) { return (uint64_t(x) & 7u) == 0; }

// ZERO_ECUDA with `what` and the CUDA error text if the last launch failed.
inline zero_status_t check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return zero_detail::set_error(ZERO_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
    return ZERO_OK;
}

// ZERO_ECUDA if an earlier asynchronous CUDA error is pending.
inline zero_status_t check_pending(const char *what) {
    cudaError_t e = cudaPeekAtLastError();
    if (e != cudaSuccess)
        return zero_detail::set_error(ZERO_ECUDA, std::string("pending CUDA error before ") + what + ": " +
                                                      cudaGetErrorString(e));
    return ZERO_OK;
}

// Streaming multiprocessors of the current device (queried once per device).
inline zero_status_t sm_count(uint32_t *out) {
    static std::mutex mu;
    static std::map<int, uint32_t> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return zero_detail::set_error(ZERO_ECUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    std::lock_guard<std::mutex> g(mu);
    auto it = cache.find(dev);
    if (it == cache.end()) {
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess)
            return zero_detail::set_error(ZERO_ECUDA, std::string("device query: ") + cudaGetErrorString(e));
        it = cache.emplace(dev, uint32_t(sms > 0 ? sms : 1)).first;
    }
    *out = it->second;
    return ZERO_OK;
}

}  // namespace zero_host

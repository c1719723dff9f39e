// NVTX ranges around the library's host-side work: one range per call of a
// step, reshard or gather entry point, and nested ranges per bucket (and per
// pass of the guarded step), so a timeline tool shows which kernels belong to
// which bucket or layer.  All of them live in the NVTX domain "zero".
//
// Off unless the environment variable ZERO_NVTX is "1" when the library
// first asks (read once per process).  Off, a range costs one test of a
// static flag and formats nothing.  On, without a tool attached, NVTX itself
// returns at once; with one attached (NVTX_INJECTION64_PATH, or a profiler),
// the tool records the ranges.  No device work is added either way.
// Not part of the ABI.
#pragma once

#include <cstdarg>
#include <cstdio>
#include <cstdlib>

#include <nvtx3/nvToolsExt.h>

namespace zero_trace {

inline bool enabled() {
    static const bool on = [] {
        const char *e = std::getenv("ZERO_NVTX");
        return e != nullptr && e[0] == '1' && e[1] == '\0';
    }();
    return on;
}

inline nvtxDomainHandle_t domain() {
    static const nvtxDomainHandle_t d = nvtxDomainCreateA("zero");
    return d;
}

inline nvtxEventAttributes_t message(const char *text) {
    nvtxEventAttributes_t at{};
    at.version = NVTX_VERSION;
    at.size = NVTX_EVENT_ATTRIB_STRUCT_SIZE;
    at.messageType = NVTX_MESSAGE_TYPE_ASCII;
    at.message.ascii = text;
    return at;
}

// A range from construction to the end of the enclosing scope.
class Range {
   public:
    __attribute__((format(printf, 2, 3))) explicit Range(const char *fmt, ...) {
        if (!enabled()) return;
        char buf[128];
        va_list ap;
        va_start(ap, fmt);
        std::vsnprintf(buf, sizeof buf, fmt, ap);
        va_end(ap);
        const nvtxEventAttributes_t at = message(buf);
        nvtxDomainRangePushEx(domain(), &at);
        on_ = true;
    }
    ~Range() {
        if (on_) nvtxDomainRangePop(domain());
    }
    Range(const Range &) = delete;
    Range &operator=(const Range &) = delete;

   private:
    bool on_ = false;
};

// An instant event (a release has no duration on the device).
__attribute__((format(printf, 1, 2))) inline void mark(const char *fmt, ...) {
    if (!enabled()) return;
    char buf[128];
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    const nvtxEventAttributes_t at = message(buf);
    nvtxDomainMarkEx(domain(), &at);
}

}  // namespace zero_trace

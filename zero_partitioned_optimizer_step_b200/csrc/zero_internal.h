// Internal definitions shared by the planner (zero_plan.cpp) and the step
// kernels (zero_step.cu).  Not part of the ABI.
#pragma once

#include <cstdint>
#include <mutex>
#include <string>
#include <vector>

#include "zero.h"

#if defined(__GNUC__)
#define ZERO_API extern "C" __attribute__((visibility("default")))
#else
#define ZERO_API extern "C"
#endif

struct zero_plan {
    uint64_t psi = 0, psi_pad = 0, S = 0, bucket_elems = 0;
    uint32_t nd = 0, stage = 0, align = 0, k_bytes = 0, max_live = 0;
    std::vector<uint64_t> unit_len, unit_pad, unit_shard, unit_base, unit_offset;
    // bucket table, implicit: unit u holds buckets [unit_bucket0[u],
    // unit_bucket0[u+1]); bucket k of the unit covers
    // [U_u + k*bucket_elems, min(U_u + (k+1)*bucket_elems, U_u + P_u)).
    std::vector<uint64_t> unit_bucket0;
    uint64_t n_buckets = 0;

    // stage-3 live-layer bookkeeping (guarded by mu)
    mutable std::mutex mu;
    std::vector<uint8_t> live;
    uint32_t n_live = 0, peak_live = 0;
    uint64_t live_bytes = 0, peak_live_bytes = 0;
};

namespace zero_detail {

// Per-thread text of the last failure; set_error returns its status.
zero_status_t set_error(zero_status_t s, const std::string &msg);
void clear_error();

struct BucketRange {
    uint32_t unit;
    uint64_t begin, end;  // logical, [begin, end)
};
BucketRange bucket_range(const zero_plan_t &p, uint64_t b);

// Stage-3 liveness of the gathers; the caller holds p.mu.  live_check
// returns ZERO_ESTATE (message prefixed by `who`) if `unit` is live already
// or max_live units are live; live_mark records a successful gather.
zero_status_t live_check(const zero_plan_t &p, uint32_t unit, const char *who);
void live_mark(zero_plan_t &p, uint32_t unit);

// Device address of the current device's error word of the bulk-copy step
// kernel's bounded waits (what zero_stream_status() reports).
zero_status_t wait_error_word(int **out);

// Workspace layout for the gradient-norm / overflow reduction: one fp64
// partial and one u32 count per CTA slot, kMaxSlots slots, then 256 bytes
// for the guarded step's decision (clip coefficient and skip flag).
constexpr uint32_t kMaxSlots = 4096;
constexpr uint64_t kGuardOffset = uint64_t(kMaxSlots) * (8 + 4);
constexpr uint64_t kWorkspaceBytes = kGuardOffset + 256;

}  // namespace zero_detail

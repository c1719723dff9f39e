// Host-side shape of the bulk-copy step kernel's shared-memory ring: which
// ring a plan's buckets use (per Nd, measured on B200), the smaller ring of
// small buckets, and the environment switches that override both.  Shared by
// the one-GPU step and the ranks-as-devices step.  Not part of the ABI.
#pragma once

#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "zero_tma.cuh"

namespace zero_ring {

inline uint32_t align128(uint64_t x) { return uint32_t((x + 127) & ~uint64_t(127)); }

// Shared-memory ring of the bulk-copy kernel for Nd gradient rows.  Each
// tile pays a fixed synchronisation latency, so tiles are large; two consumer
// groups help where a tile is cheap to compute.  Shapes measured best on B200
// at 64 MB buckets (5e8 params), as (groups, tile, stages, elements/thread):
//   Nd <= 2: (2, 2048, 4, 8)     Nd <= 4: (1, 4096, 2, 8)     Nd <= 8: (1, 2048, 3, 8)
//   Nd <= 16: (1, 1024, 4, 4)    Nd <= 32: (1, 1024, 2, 8)
//   Nd <= 64: (1, 512, 3, 4)
// Read-heavy steps (parameters written once: stage 3 or one owner) do better
// with larger bulk copies, i.e. larger tiles: Nd <= 16 takes (1, 2048, 2, 8)
// (the stage-3 1.3B workload at Nd = 16).  Beyond 64 ranks the 16-byte-load
// kernel is used, and also for read-heavy steps with more than 32 ranks: there
// every gradient row of a 512-element tile is a 1 KB bulk copy, and the rate
// at which an SM completes such copies caps the read bandwidth (0.64 of copy
// bandwidth against 0.80 for the load kernel, one owner of 64 ranks).  With
// two groups the stage count is even (each group owns half the stages).
// ZERO_TMA_CW=16 runs 16 consumer warps instead of 8 (where the caller has
// such kernels; the per-thread vector width shrinks so every thread keeps
// work).  ZERO_TMA_TILE / ZERO_TMA_STAGES / ZERO_TMA_GROUPS / ZERO_TMA_VW override the
// shape (tuning; a tile must be a positive multiple of 256).  `err` is the
// device error word the kernel's bounded waits report to.
// Dynamic shared memory of a launch: the stages, then (bulk_p) two
// parameter tiles per consumer group.
inline size_t ring_smem_bytes(const zero_tma::Ring &r) {
    return size_t(r.stages) * r.stage_bytes + (r.bulk_p ? size_t(r.groups) * 2 * r.tile * 2 : 0);
}

inline zero_tma::Ring ring_for(uint32_t nd, uint64_t t, uint32_t stages, uint32_t groups) {
    zero_tma::Ring q{};
    q.cw = zero_tma::kConsumerWarps;
    q.tile = uint32_t(t);
    q.off_w = align128(uint64_t(nd) * t * 2);
    q.off_m = q.off_w + align128(4 * t);
    q.off_v = q.off_m + align128(4 * t);
    q.stage_bytes = q.off_v + align128(4 * t);
    q.stages = stages;
    q.groups = groups;
    return q;
}

// max_cw: the most consumer warps the caller has kernels for (8 or 16).
inline bool choose_ring(uint32_t nd, bool read_heavy, uint32_t budget, int *err, zero_tma::Ring *r,
                        uint32_t max_cw = zero_tma::kMaxConsumerWarps) {
    long force_t = 0, force_s = 0, force_g = 0, force_v = 0, force_c = 0;
    if (const char *e = std::getenv("ZERO_TMA_TILE")) force_t = std::strtol(e, nullptr, 10);
    if (const char *e = std::getenv("ZERO_TMA_STAGES")) force_s = std::strtol(e, nullptr, 10);
    if (const char *e = std::getenv("ZERO_TMA_GROUPS")) force_g = std::strtol(e, nullptr, 10);
    if (const char *e = std::getenv("ZERO_TMA_VW")) force_v = std::strtol(e, nullptr, 10);
    if (const char *e = std::getenv("ZERO_TMA_CW")) force_c = std::strtol(e, nullptr, 10);
    const uint32_t cw = (force_c == 16 && max_cw >= 16) ? 16u : uint32_t(zero_tma::kConsumerWarps);
    uint32_t groups, stages, vw;
    uint64_t tile;
    if (force_t >= 256 && force_t % 256 == 0 && force_t <= 16384) {
        tile = uint64_t(force_t);
        groups = force_g == 2 ? 2 : 1;
        stages = force_s >= 2 ? uint32_t(std::min<long>(force_s, zero_tma::kMaxStages)) : zero_tma::kMaxStages;
        const uint64_t busy = tile * groups / (32u * cw);  // keep a group's threads busy
        vw = busy >= 8 ? 8 : (busy >= 4 ? 4 : 2);
    } else if (nd <= 2) {
        groups = 2, tile = 2048, stages = 4, vw = 8;
    } else if (nd <= 4) {
        groups = 1, tile = 4096, stages = 2, vw = 8;
    } else if (nd <= 8) {
        groups = 1, tile = 2048, stages = 3, vw = 8;
    } else if (nd <= 16 && read_heavy) {
        groups = 1, tile = 2048, stages = 2, vw = 8;
    } else if (nd <= 16) {
        groups = 1, tile = 1024, stages = 4, vw = 4;
    } else if (nd <= 32) {
        groups = 1, tile = 1024, stages = 2, vw = 8;
    } else if (nd <= 64 && !read_heavy) {
        groups = 1, tile = 512, stages = 3, vw = 4;
    } else {
        return false;
    }
    if (force_t == 0 && cw > uint32_t(zero_tma::kConsumerWarps)) {
        // the table's shapes were sized for 8 consumer warps: keep every
        // thread of a group busy with twice as many
        const uint64_t busy = tile * groups / (32u * cw);
        vw = uint32_t(std::min<uint64_t>(vw, busy >= 8 ? 8 : (busy >= 4 ? 4 : 2)));
    }
    if (force_v == 2 || force_v == 4 || force_v == 8) vw = uint32_t(force_v);
    zero_tma::Ring q = ring_for(nd, tile, 0, groups);
    q.err = err;
    q.vw = vw;
    q.cw = cw;
    // ZERO_TEST_STALL_PRODUCER=<cta>: that CTA's producer issues nothing, so
    // its consumers' bounded waits run out (tests the ZERO_ETIMEOUT path)
    q.stall_cta = 0xffffffffu;
    if (const char *e = std::getenv("ZERO_TEST_STALL_PRODUCER")) {
        char *end = nullptr;
        const unsigned long v = std::strtoul(e, &end, 10);
        if (end != e && v < 0xffffffffu) q.stall_cta = uint32_t(v);
    }
    // Replica rows as bulk copies from shared memory at Nd <= 2, where a
    // tile's copies are few and large (2 per tile of 4 KB each): K1 went from
    // 0.950 to 0.979 of copy bandwidth at Nd = 2 (64 MB buckets, 5e8
    // params), was flat at Nd = 4, and lost 6 %, 3 % and 30 % at Nd = 8, 16
    // and 64, where one thread issues Nd small copies per tile.
    // ZERO_TMA_BULKP=0|1 overrides.
    q.bulk_p = (!read_heavy && nd <= 2) ? 1u : 0u;
    if (const char *e = std::getenv("ZERO_TMA_BULKP")) q.bulk_p = e[0] == '1' ? 1u : 0u;
    const uint64_t pbytes = q.bulk_p ? uint64_t(groups) * 2 * tile * 2 : 0;
    if (pbytes >= budget) return false;
    uint64_t ns = std::min<uint64_t>((budget - pbytes) / q.stage_bytes, stages);
    ns -= ns % groups;  // every stage belongs to one group
    if (ns < 2) return false;
    q.stages = uint32_t(ns);
    *r = q;
    return true;
}

// A small bucket is over soon after a CTA's ring has filled, and the next
// bucket's CTAs (launched early through programmatic dependent launch) cannot
// start on an SM while this ring takes most of its shared memory.  Below
// 32 x 2048 elements per SM the ring is cut to half of the SM's shared memory (tile
// halved while needed, at least 512, and as many stages as then fit), so two
// CTAs share an SM and the next bucket's loads overlap this one's tail.
// Measured on B200 (5e8 params): +50 % at 1-2 MB buckets for Nd <= 8 and
// +10-20 % up to 16 MB; from 32 MB up the full ring is faster.
// ZERO_TMA_ADAPT=0, or a forced ZERO_TMA_TILE, keeps the chosen ring;
// ZERO_TMA_ADAPT_TILES=<n> moves the threshold to n x 2048 elements per SM
// (tuning).
inline zero_tma::Ring ring_for_launch(const zero_tma::Ring &r, uint64_t n, uint32_t nd, uint32_t sms,
                               uint32_t budget) {
    static const bool off = [] {
        const char *e = std::getenv("ZERO_TMA_ADAPT");
        return (e && e[0] == '0') || std::getenv("ZERO_TMA_TILE") != nullptr;
    }();
    static const uint64_t per_sm = [] {
        const char *e = std::getenv("ZERO_TMA_ADAPT_TILES");
        const long v = e ? std::strtol(e, nullptr, 10) : 0;
        return uint64_t(v > 0 ? v : 32);
    }();
    if (off || n >= 2048ull * per_sm * sms) return r;
    const uint64_t half = budget / 2 - 1024;  // room for a second CTA's ring and static shared memory
    for (uint64_t tile = r.tile; tile >= 512; tile /= 2) {
        zero_tma::Ring q = ring_for(nd, tile, 0, r.groups);
        q.bulk_p = r.bulk_p;
        const uint64_t pbytes = q.bulk_p ? uint64_t(r.groups) * 2 * tile * 2 : 0;
        if (pbytes >= half) continue;
        uint64_t ns = std::min<uint64_t>((half - pbytes) / q.stage_bytes, zero_tma::kMaxStages);
        ns -= ns % r.groups;
        if (ns < 2 || ns < r.groups * 2) continue;
        q.err = r.err;
        q.stall_cta = r.stall_cta;
        q.cw = r.cw;
        const uint64_t busy = tile * r.groups / (32u * r.cw);
        q.vw = busy >= 8 ? 8 : (busy >= 4 ? 4 : 2);
        q.stages = uint32_t(ns);
        return q;
    }
    return r;
}

// ZERO_STEP_KERNEL=ldg|tma picks the vector kernel for aligned bucket bodies
// (default: the bulk-copy kernel whenever its ring fits).
inline int kernel_choice() {
    const char *s = std::getenv("ZERO_STEP_KERNEL");
    if (!s) return 0;
    if (std::strcmp(s, "ldg") == 0) return 1;
    if (std::strcmp(s, "tma") == 0) return 2;
    return 0;
}

}  // namespace zero_ring

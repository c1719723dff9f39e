// K1, bulk-copy path (sm_100a): the fused reduce-scatter + Adam + all-gather
// of one bucket with its operands staged through a shared-memory ring by the
// Tensor Memory Accelerator's 1-D bulk copies.
//
// Warp 0 is the producer.  Per tile of `tile` elements it issues one
// cp.async.bulk per gradient row (Nd rows, spread over its lanes) and one per
// state array and owner segment, all completing on the stage's `full`
// mbarrier.  Warps 1..CW are consumers (CW = 8 or 16, a template parameter): they read the stage from shared memory,
// sum the rows in rank order, run Adam, and write w, m, v and the bf16
// parameters (every replica row, or the owner shard) straight from registers
// with 16-byte streaming stores.  The stage is released through its `empty`
// mbarrier as soon as the consumers have read it, so the producer keeps
// (stages - 1) tiles of loads in flight per SM: registers no longer bound the
// bytes in flight.  No multicast is used.
//
// Every wait is bounded (kWaitLimitNs of %globaltimer).  A thread that gives
// up sets the CTA's abort flag and the device error word; the
// consumers leave the loop together (the decision is an OR-reduction over a
// barrier, so no consumer is left alone at a barrier), the producer waits a
// bounded time for the loads it issued, and the kernel returns.
// zero_stream_status() reports the error word (one word per device, owned by
// the library; its address travels in the Ring).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "zero_device.cuh"

namespace zero_tma {

using zero_dev::AdamConsts;
using zero_dev::StepArgs;

// Consumer warps: 8 by default (kThreads = 288 threads per CTA), or 16 (544),
// the kernel's CW template parameter; the ring records which.
constexpr int kConsumerWarps = 8;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kThreads = 32 + kConsumers;  // warp 0 produces
constexpr int kMaxConsumerWarps = 16;
// Consumers form GROUPS groups (a template parameter, 1 or 2) that take the
// CTA's tiles in turn.  Tile k goes to stage k % stages and to group
// k % GROUPS; the host makes `stages` a multiple of GROUPS, so every stage
// belongs to one group, which waits for its uses strictly in order.  (A group
// waiting on a stage that another group is still using could see the parity
// of an older, unfinished phase as "done": mbarrier parity waits only
// distinguish the current phase from the one before it.)
constexpr int kMaxStages = 8;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

// Shared-memory ring chosen on the host.  A stage holds Nd gradient rows of
// `tile` bf16 at offset 0, then w, m, v (fp32).  `vw` is the per-thread
// vector width the kernel was instantiated with.
struct Ring {
    int *err;            // device error word: 1 once a bounded wait has given up,
                         // 2 if a consumer found a stage holding another tile
                         // than the one it expected
    uint32_t stall_cta;  // test of the bounded waits: this CTA's producer issues
                         // nothing (0xffffffff: none)
    uint32_t vw;
    uint32_t cw;         // consumer warps the kernel was instantiated with
    uint32_t tile;
    uint32_t stages;  // a multiple of groups
    uint32_t groups;  // consumer groups the kernel was instantiated with
    uint32_t stage_bytes;
    uint32_t bulk_p;  // 1: with replica rows (fused step), the bf16 parameters
                      // go to two shared-memory tiles per group after the
                      // stages and out as one 1-D bulk copy per row and tile
    uint32_t off_w, off_m, off_v;
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase of `bar` with the given parity.  Gives up (returning
// false) when the CTA's abort flag is raised, or after kWaitLimitNs, in which
// case it raises the abort flag and sets the device error word *err to 1.
static __device__ __noinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                              int *err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                *abort_flag = 1;
                atomicExch(err, 1);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Named barrier `id` over `count` threads, returning the OR of `v` over them
// (the same value in every participating thread).  Ids: 1 + group for a
// consumer group, 1 + GROUPS for all consumers.
__device__ __forceinline__ bool barrier_or(uint32_t id, uint32_t count, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"(uint32_t(v)), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

// Calls f(j, count, state_shift, param_shift) for each piece of [jb, je) that
// has one owner: the state of element j sits at s_base + j + state_shift.
template <bool OWNER_MAP, typename F>
__device__ __forceinline__ void for_each_segment(const StepArgs &a, uint64_t jb, uint64_t je, F f) {
    if (!OWNER_MAP) {
        f(jb, je - jb, uint64_t(0), uint64_t(0));
        return;
    }
    uint64_t o = jb / a.shard;
    uint64_t j = jb;
    while (j < je) {
        const uint64_t e = min(je, (o + 1) * a.shard);
        f(j, e - j, o * a.jump, o * a.p_jump);
        j = e;
        ++o;
    }
}

__device__ __forceinline__ uint4 lds128(const unsigned char *p) {
    return *reinterpret_cast<const uint4 *>(p);
}

// Per-thread vector of VW consecutive elements (VW = 2, 4 or 8): bf16 rows
// read from shared memory as 4/8/16 bytes, fp32 state as 8/16/32 bytes, and
// streaming global stores of the same widths.  The host picks VW so that a
// tile keeps every consumer thread of a group busy.  The bf16 rows come in
// as VW / 2 fp32 pairs (exact), for the packed rank-order sum.
template <int VW>
__device__ __forceinline__ void lds_bf16x2(const unsigned char *p, uint64_t f[VW / 2]) {
    if constexpr (VW == 2) {
        f[0] = zero_dev::f2_bf16x2(*reinterpret_cast<const uint32_t *>(p));
    } else if constexpr (VW == 4) {
        const uint2 x = *reinterpret_cast<const uint2 *>(p);
        f[0] = zero_dev::f2_bf16x2(x.x);
        f[1] = zero_dev::f2_bf16x2(x.y);
    } else {
        const uint4 x = *reinterpret_cast<const uint4 *>(p);
        f[0] = zero_dev::f2_bf16x2(x.x);
        f[1] = zero_dev::f2_bf16x2(x.y);
        f[2] = zero_dev::f2_bf16x2(x.z);
        f[3] = zero_dev::f2_bf16x2(x.w);
    }
}

template <int VW>
__device__ __forceinline__ void lds_f32(const unsigned char *p, float f[VW]) {
    if constexpr (VW == 2) {
        const float2 x = *reinterpret_cast<const float2 *>(p);
        f[0] = x.x; f[1] = x.y;
    } else {
#pragma unroll
        for (int h = 0; h < VW / 4; ++h) {
            const float4 x = reinterpret_cast<const float4 *>(p)[h];
            f[4 * h] = x.x; f[4 * h + 1] = x.y; f[4 * h + 2] = x.z; f[4 * h + 3] = x.w;
        }
    }
}

template <int VW>
__device__ __forceinline__ void stg_f32(float *p, const float f[VW]) {
    if constexpr (VW == 2) {
        __stcs(reinterpret_cast<float2 *>(p), make_float2(f[0], f[1]));
    } else {
#pragma unroll
        for (int h = 0; h < VW / 4; ++h)
            __stcs(reinterpret_cast<float4 *>(p) + h, make_float4(f[4 * h], f[4 * h + 1], f[4 * h + 2], f[4 * h + 3]));
    }
}

// bf16(w) of VW elements to `rows` rows `stride` elements apart
template <int VW>
__device__ __forceinline__ void stg_bf16_rows(uint16_t *p, const float w[VW], uint32_t rows, uint64_t stride) {
    uint32_t pk[VW / 2];
#pragma unroll
    for (int h = 0; h < VW / 2; ++h) pk[h] = zero_dev::pack_bf16x2(w[2 * h], w[2 * h + 1]);
    for (uint32_t r = 0; r < rows; ++r) {
        uint16_t *q = p + uint64_t(r) * stride;
        if constexpr (VW == 2) {
            __stcs(reinterpret_cast<unsigned int *>(q), pk[0]);
        } else if constexpr (VW == 4) {
            __stcs(reinterpret_cast<uint2 *>(q), make_uint2(pk[0], pk[1]));
        } else {
            __stcs(reinterpret_cast<uint4 *>(q), make_uint4(pk[0], pk[1], pk[2], pk[3]));
        }
    }
}

// Where a tile's rows come from, and where the parameters go.
//   kGradRows: the Nd bf16 gradient rows at a.grads + r * a.grad_stride
//              (the fused step), parameters at a.params (+ row * param_stride);
//   kReduced:  one fp32 row, the reduced gradient at a.red in state order, and
//              g = (g_sum * grad_scale) * coef from the guarded step's decision,
//              nothing at all if that decision is to skip (its second pass);
//   kPeerRows: the Nd bf16 gradient rows at x.g[r] and the parameter rows at
//              x.p[q]: other ranks' buffers reached through their pointers.
enum RowSource { kGradRows = 0, kReduced = 1, kPeerRows = 2 };

struct NoExtra {};
struct ApplyExtra {
    const zero_dev::GuardWord *gw;
};

template <int SRC>
struct ExtraOf {
    using type = NoExtra;
};
template <>
struct ExtraOf<kReduced> {
    using type = ApplyExtra;
};
template <>
struct ExtraOf<kPeerRows> {
    using type = zero_dev::PeerTable;
};

// bf16(w) of VW elements into a shared-memory tile
template <int VW>
__device__ __forceinline__ void sts_bf16(uint16_t *p, const float w[VW]) {
    uint32_t pk[VW / 2];
#pragma unroll
    for (int h = 0; h < VW / 2; ++h) pk[h] = zero_dev::pack_bf16x2(w[2 * h], w[2 * h + 1]);
    if constexpr (VW == 2) {
        *reinterpret_cast<uint32_t *>(p) = pk[0];
    } else if constexpr (VW == 4) {
        *reinterpret_cast<uint2 *>(p) = make_uint2(pk[0], pk[1]);
    } else {
        *reinterpret_cast<uint4 *>(p) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
}

__device__ __forceinline__ void bulk_store(void *gdst, const void *ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(ssrc)),
                 "r"(bytes)
                 : "memory");
}

// bf16(w) of VW elements to `rows` parameter rows given by pointer
template <int VW>
__device__ __forceinline__ void stg_bf16_at(uint16_t *q, const uint32_t pk[VW / 2]) {
    if constexpr (VW == 2) {
        __stcs(reinterpret_cast<unsigned int *>(q), pk[0]);
    } else if constexpr (VW == 4) {
        __stcs(reinterpret_cast<uint2 *>(q), make_uint2(pk[0], pk[1]));
    } else {
        __stcs(reinterpret_cast<uint4 *>(q), make_uint4(pk[0], pk[1], pk[2], pk[3]));
    }
}

template <int VW>
__device__ __forceinline__ void stg_bf16_ptrs(uint16_t *const *rows, uint64_t off, const float w[VW], uint32_t n) {
    uint32_t pk[VW / 2];
#pragma unroll
    for (int h = 0; h < VW / 2; ++h) pk[h] = zero_dev::pack_bf16x2(w[2 * h], w[2 * h + 1]);
    if constexpr (VW == 8) {
        for (uint32_t r = 0; r < n; ++r) stg_bf16_at<VW>(rows[r] + off, pk);
    } else {
        // Four rows at a time, so that their pointers (in shared memory) are
        // loaded together instead of each store waiting for its own.  With
        // ranks as allocations on one B200, Psi = 5e8, Nd = 16, 64 MB buckets
        // (4 elements a thread): 0.886 -> 0.924 of copy bandwidth.  At 8
        // elements a thread it lost (Nd = 8: 0.927 -> 0.913), so that width
        // keeps the plain loop.
#pragma unroll 4
        for (uint32_t r = 0; r < n; ++r) stg_bf16_at<VW>(rows[r] + off, pk);
    }
}

// At most 96 registers a thread (which also fits 544 threads, CW = 16, in
// one CTA): for small buckets two CTAs share an SM
// (the cut ring), 18 warps, so one of the four schedulers holds 5 of them,
// and 5 x 96 x 32 registers is what one scheduler's share of the register
// file (16,384) holds; at 104 the second CTA did not fit and small buckets
// ran 20-40 % slower at Nd <= 8.
template <bool OWNER_MAP, int GROUPS, int VW, int SRC = kGradRows, int CW = kConsumerWarps>
__global__ void __maxnreg__(96)
    k_step_tma(const StepArgs a, const Ring ring, const typename ExtraOf<SRC>::type x) {
    constexpr uint32_t kCons = 32u * CW;
    constexpr uint32_t kGroupThreads = kCons / GROUPS;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full_bar[kMaxStages];
    __shared__ __align__(8) uint64_t empty_bar[kMaxStages];
    __shared__ uint64_t stage_tile[kMaxStages];  // tile a stage was filled with
    __shared__ int s_abort;
    __shared__ double s_norm[CW];
    __shared__ uint32_t s_bad[CW];
    __shared__ const uint16_t *s_rows[SRC == kPeerRows ? zero_dev::kMaxPeers : 1];
    __shared__ uint16_t *s_prow[SRC == kPeerRows ? zero_dev::kMaxPeers : 1];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t T = ring.tile;
    const uint32_t NS = ring.stages;
    const uint64_t n_tiles = (a.j1 - a.j0 + T - 1) / T;
    float coef = 1.0f;
    if constexpr (SRC == kReduced) {
        const zero_dev::GuardWord g = *x.gw;
        if (g.skip) {  // every thread, before any barrier
            zero_dev::pdl_wait();
            return;
        }
        coef = g.coef;
    }

    zero_dev::pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (uint32_t s = 0; s < NS; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        s_abort = 0;
        fence_barrier_init();
    }
    if constexpr (SRC == kPeerRows) {
        for (uint32_t i = threadIdx.x; i < a.nd; i += blockDim.x) s_rows[i] = x.g[i];
        for (uint32_t i = threadIdx.x; i < a.n_prow; i += blockDim.x) s_prow[i] = x.p[i];
    }
    __syncthreads();
    volatile int *abort_flag = &s_abort;

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (blockIdx.x == ring.stall_cta) return;  // consumers' waits run out
        constexpr uint32_t kRowBytes = SRC == kReduced ? 4u : 0u;
        uint32_t k = 0;
        for (uint64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++k) {
            const uint32_t s = k % NS;
            if (k >= NS) {
                int ok = 1;
                if (lane == 0) ok = mbar_wait(&empty_bar[s], ((k / NS) - 1) & 1u, abort_flag, ring.err);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
            const uint64_t jb = a.j0 + tile * T;
            const uint64_t je = min(jb + T, a.j1);
            const uint32_t n = uint32_t(je - jb);
            unsigned char *st = smem + size_t(s) * ring.stage_bytes;
            if (lane == 0) {
                stage_tile[s] = tile;  // published by the arrive below (release)
                const uint32_t per = SRC == kReduced ? 4u + 12u : 2u * a.nd + 12u;
                mbar_arrive_expect_tx(&full_bar[s], n * per);
            }
            __syncwarp();
            if constexpr (SRC != kReduced) {
                const int64_t gofs = a.g_base + int64_t(jb);
                for (uint32_t r = lane; r < a.nd; r += 32) {
                    const uint16_t *src = SRC == kPeerRows ? s_rows[r] + gofs
                                                           : a.grads + uint64_t(gofs) + uint64_t(r) * a.grad_stride;
                    bulk_load(st + size_t(r) * T * 2, src, n * 2u, &full_bar[s]);
                }
            }
            if (lane == 0) {
                for_each_segment<OWNER_MAP>(a, jb, je, [&](uint64_t js, uint64_t cnt, uint64_t so, uint64_t) {
                    const uint64_t off = js - jb;
                    const uint64_t si = uint64_t(a.s_base + int64_t(js)) + so;
                    if (kRowBytes) bulk_load(st + off * 4, a.red + si, uint32_t(cnt * 4), &full_bar[s]);
                    bulk_load(st + ring.off_w + off * 4, a.w + si, uint32_t(cnt * 4), &full_bar[s]);
                    bulk_load(st + ring.off_m + off * 4, a.m + si, uint32_t(cnt * 4), &full_bar[s]);
                    bulk_load(st + ring.off_v + off * 4, a.v + si, uint32_t(cnt * 4), &full_bar[s]);
                });
            }
        }
        if (*abort_flag && lane == 0) {
            // loads of the last tiles issued may still be landing: wait (bounded)
            int dummy = 0;
            volatile int *never = &dummy;
            for (uint32_t i = 0; i < NS && i < k; ++i) {
                const uint32_t kk = k - 1 - i;
                mbar_wait(&full_bar[kk % NS], (kk / NS) & 1u, never, ring.err);
            }
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    const AdamConsts C = zero_dev::consts_of(a);
    // Group g takes the CTA's tiles k = g, g + GROUPS, ..., so one group's
    // per-tile latency overlaps the other's.
    const int ct = threadIdx.x - 32;
    const uint32_t grp = uint32_t(ct) / kGroupThreads;
    const uint32_t gt = uint32_t(ct) % kGroupThreads;
    double acc = 0.0;
    uint32_t bad = 0;
    // Replica rows as bulk copies (ring.bulk_p): the group's two tiles of
    // parameters alternate; at the end of a tile the issuing thread (gt 0)
    // waits until the previous tile's copies have read the other one, the
    // group's barrier publishes that and this tile's writes, and then it
    // issues one copy per replica row.
    const bool bulkp = SRC == kGradRows && ring.bulk_p && a.n_prow > 1;
    uint16_t *ptile = reinterpret_cast<uint16_t *>(smem + size_t(NS) * ring.stage_bytes) + size_t(grp) * 2 * T;
    uint32_t pb = 0;
    uint32_t k = grp;
    for (uint64_t tile = blockIdx.x + uint64_t(grp) * gridDim.x; tile < n_tiles;
         tile += uint64_t(GROUPS) * gridDim.x, k += GROUPS) {
        const uint32_t s = k % NS;
        bool failed = !mbar_wait(&full_bar[s], (k / NS) & 1u, abort_flag, ring.err);
        if (!failed && stage_tile[s] != tile) {  // self-check of the ring protocol
            failed = true;
            *abort_flag = 1;
            atomicExch(ring.err, 2);
        }
        const uint64_t jb = a.j0 + tile * T;
        const uint32_t n = uint32_t(min(jb + T, a.j1) - jb);
        const unsigned char *st = smem + size_t(s) * ring.stage_bytes;
        if (!failed) {
            const uint32_t nv = n / VW;
            for (uint32_t vv = gt; vv < nv; vv += kGroupThreads) {
                // the rank-order sum, in fp32 pairs (each lane rounded as a
                // scalar add would be)
                float sum[VW];
                if constexpr (SRC == kReduced) {
                    lds_f32<VW>(st + size_t(vv) * (4 * VW), sum);
                } else {
                    const unsigned char *gp = st + size_t(vv) * (2 * VW);
                    uint64_t s2[VW / 2], f2[VW / 2];
                    lds_bf16x2<VW>(gp, s2);
#pragma unroll 4
                    for (uint32_t r = 1; r < a.nd; ++r) {
                        lds_bf16x2<VW>(gp + size_t(r) * T * 2, f2);
#pragma unroll
                        for (int h = 0; h < VW / 2; ++h) s2[h] = zero_dev::f2_add(s2[h], f2[h]);
                    }
#pragma unroll
                    for (int h = 0; h < VW / 2; ++h) zero_dev::f2_unpack(s2[h], sum[2 * h], sum[2 * h + 1]);
                }
                float wv[VW], mv[VW], vq[VW];
                lds_f32<VW>(st + ring.off_w + size_t(vv) * (4 * VW), wv);
                lds_f32<VW>(st + ring.off_m + size_t(vv) * (4 * VW), mv);
                lds_f32<VW>(st + ring.off_v + size_t(vv) * (4 * VW), vq);
                if (a.ws_mode) {
#pragma unroll
                    for (int e = 0; e < VW; ++e) {
                        acc += double(sum[e]) * double(sum[e]);
                        bad += zero_dev::not_finite(sum[e]);
                    }
                }
                const uint64_t j = jb + uint64_t(vv) * VW;
                const uint64_t o = OWNER_MAP ? j / a.shard : 0;
                const uint64_t si = uint64_t(a.s_base + int64_t(j)) + o * a.jump;
                const uint64_t pi = uint64_t(a.p_base + int64_t(j)) + o * a.p_jump;
                if (SRC != kReduced && a.red) stg_f32<VW>(a.red + si, sum);
#pragma unroll
                for (int e = 0; e < VW; ++e) zero_dev::adam1c(sum[e], coef, C, wv[e], mv[e], vq[e]);
                stg_f32<VW>(a.w + si, wv);
                stg_f32<VW>(a.m + si, mv);
                stg_f32<VW>(a.v + si, vq);
                if constexpr (SRC == kPeerRows) stg_bf16_ptrs<VW>(s_prow, pi, wv, a.n_prow);
                else if (bulkp) sts_bf16<VW>(ptile + size_t(pb) * T + size_t(vv) * VW, wv);
                else stg_bf16_rows<VW>(a.params + pi, wv, a.n_prow, a.param_stride);
            }
        }
        if (bulkp) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // this thread's tile writes
            if (gt == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        }
        // the whole group has read the stage (or the CTA is giving up): same
        // decision in all of its threads, then hand the stage back
        if (barrier_or(1 + grp, kGroupThreads, failed || *abort_flag)) break;
        if (bulkp && gt == 0) {
            // replica rows are contiguous in logical order (no owner jump)
            uint16_t *row = a.params + uint64_t(a.p_base + int64_t(jb));
            for (uint32_t r = 0; r < a.n_prow; ++r)
                bulk_store(row + uint64_t(r) * a.param_stride, ptile + size_t(pb) * T, n * 2u);
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
        pb ^= 1u;
        if (gt == 0) mbar_arrive(&empty_bar[s]);
    }
    // the parameter tiles must outlive their copies, which also complete the writes
    if (bulkp && gt == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");

    if constexpr (SRC == kPeerRows) {
        // every consumer's peer stores are performed before the kernel
        // completes: a consumer barrier, then one cumulative system fence
        barrier_or(1 + GROUPS, kCons, false);
        if (ct == 0) __threadfence_system();
    }
    zero_dev::pdl_wait();  // predecessor done: its norm slots are final
    if (a.ws_mode) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            acc += __shfl_down_sync(0xffffffffu, acc, off);
            bad += __shfl_down_sync(0xffffffffu, bad, off);
        }
        if (lane == 0) {
            s_norm[warp - 1] = acc;
            s_bad[warp - 1] = bad;
        }
        barrier_or(1 + GROUPS, kCons, false);
        if (ct == 0) {
            double t = 0.0;
            uint32_t b = 0;
            for (int i = 0; i < CW; ++i) {
                t += s_norm[i];
                b += s_bad[i];
            }
            a.ws_norm[blockIdx.x] += t;
            a.ws_bad[blockIdx.x] = min(a.ws_bad[blockIdx.x] + b, 0x7fffffffu);
        }
    }
}

}  // namespace zero_tma

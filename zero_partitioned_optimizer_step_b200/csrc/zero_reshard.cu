// Checkpoint resharding: one owner-storage state array from the layout of
// one plan (Nd ranks, its padding) to the layout of another plan with the
// same units.  The concept page "ZeRO" asks, in its "使用时应检查" list,
// whether a checkpoint can be restored after the parallelism changes; this
// is that step, as a device copy.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>

#include "zero_device.cuh"
#include "zero_host.cuh"
#include "zero_internal.h"
#include "zero_trace.h"

using zero_detail::set_error;

namespace {

using zero_dev::kThreads;

// K4: one unit of a state array, from owner storage under plan A to owner
// storage under plan B (same unit lengths, other Nd or padding).  The unit's
// logical element q sits under plan B at off_b + q + ob * jump_b, ob = q / s_b
// (jump = S - s_u), and under plan A at off_a + q + oa * jump_a, oa = q / s_a;
// q >= len is padding, written as zero.  A warp copies chunks of 32 * V * R
// consecutive q: lane l takes the groups of V elements at l*V, l*V + 32V, ...,
// so the warp's accesses are contiguous.  The two owners, found by one
// division per chunk, only advance within it.  A lane issues all R loads of
// its chunk before any of its stores, so R loads are in flight at once.
// V = 16 bytes of elements when every offset, shard and jump is a multiple of
// V, else 1 (a group of V then never straddles a shard boundary).
struct ReshardArgs {
    uint64_t off_a, jump_a, s_a;
    uint64_t off_b, jump_b, s_b;
    uint64_t n;    // nd_b * s_b, a multiple of V
    uint64_t len;  // real elements of the unit
};

template <typename T, int V>
struct Vec;
template <> struct Vec<uint32_t, 4> { using type = uint4; };
template <> struct Vec<uint16_t, 8> { using type = uint4; };
template <typename T> struct Vec<T, 1> { using type = T; };

template <typename T, int V, int R>
__global__ void __launch_bounds__(kThreads) k_reshard(const T *__restrict__ src, T *__restrict__ dst,
                                                     const ReshardArgs a) {
    zero_dev::pdl_launch_dependents();
    using VT = typename Vec<T, V>::type;
    constexpr uint64_t kChunk = 32ull * V * R;
    const uint32_t lane = threadIdx.x & 31u;
    const uint64_t warp = (uint64_t(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const uint64_t nwarps = (uint64_t(gridDim.x) * kThreads) >> 5;
    for (uint64_t c0 = warp * kChunk; c0 < a.n; c0 += nwarps * kChunk) {
        const uint64_t q0 = c0 + uint64_t(lane) * V;
        if (q0 >= a.n) continue;
        uint64_t oa = q0 / a.s_a, ob = q0 / a.s_b;
        uint64_t na = (oa + 1) * a.s_a, nb = (ob + 1) * a.s_b;  // next shard boundaries
        VT val[R];
        uint64_t sp[R], dp[R];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const uint64_t q = q0 + uint64_t(k) * 32 * V;
            sp[k] = dp[k] = ~uint64_t(0);
            if (q >= a.n) continue;
            while (q >= na) {
                ++oa;
                na += a.s_a;
            }
            while (q >= nb) {
                ++ob;
                nb += a.s_b;
            }
            sp[k] = a.off_a + q + oa * a.jump_a;
            dp[k] = a.off_b + q + ob * a.jump_b;
            if (q + V <= a.len) val[k] = __ldcs(reinterpret_cast<const VT *>(src + sp[k]));
        }
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const uint64_t q = q0 + uint64_t(k) * 32 * V;
            if (q >= a.n) continue;
            T *d = dst + dp[k];
            if (q + V <= a.len) {
                __stcs(reinterpret_cast<VT *>(d), val[k]);
            } else {  // the group holding the end of the unit, or padding
#pragma unroll
                for (int e = 0; e < V; ++e) d[e] = q + e < a.len ? src[sp[k] + e] : T(0);
            }
        }
    }
    // launched early behind the previous unit's copy (which touches other
    // bytes): complete only after it, so that completion stays in order
    zero_dev::pdl_wait();
}

}  // namespace

ZERO_API zero_status_t zero_reshard(const zero_plan_t *from, const void *src, const zero_plan_t *to, void *dst,
                                    uint32_t elem_bytes, void *stream_) {
    zero_detail::clear_error();
    const zero_trace::Range call("zero_reshard %u-byte elements", elem_bytes);
    if (!from || !to || !src || !dst) return set_error(ZERO_EINVAL, "zero_reshard: NULL argument");
    if (elem_bytes != 2 && elem_bytes != 4)
        return set_error(ZERO_EINVAL, "zero_reshard: elem_bytes must be 2 (bf16) or 4 (fp32)");
    if (from->unit_len != to->unit_len)
        return set_error(ZERO_EINVAL, "zero_reshard: the two plans must have the same unit lengths");
    if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) % elem_bytes)
        return set_error(ZERO_EINVAL, "zero_reshard: buffers must be aligned to the element size");
    zero_status_t st = zero_host::check_pending("zero_reshard");
    if (st != ZERO_OK) return st;
    uint32_t sms = 0;
    st = zero_host::sm_count(&sms);
    if (st != ZERO_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    // units after the first launch behind their predecessor (programmatic
    // dependent launch): they copy disjoint ranges; ZERO_PDL=0 turns it off
    const char *pdl_env = std::getenv("ZERO_PDL");
    const bool pdl = !(pdl_env && pdl_env[0] == '0');
    const int vec_bytes = ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15u) == 0;
    for (size_t u = 0; u < to->unit_len.size(); ++u) {
        ReshardArgs r;
        r.off_a = from->unit_offset[u];
        r.s_a = from->unit_shard[u];
        r.jump_a = from->S - r.s_a;
        r.off_b = to->unit_offset[u];
        r.s_b = to->unit_shard[u];
        r.jump_b = to->S - r.s_b;
        r.n = uint64_t(to->nd) * r.s_b;
        r.len = to->unit_len[u];
        const zero_trace::Range ru("reshard unit %zu", u);
        const uint64_t V = 16 / elem_bytes;
        const bool vec = vec_bytes && ((r.off_a | r.s_a | r.jump_a | r.off_b | r.s_b | r.jump_b) % V) == 0;
        constexpr int R = 8;
        const uint64_t per_thread = (vec ? V : 1) * R;
        const uint64_t blocks = (r.n + per_thread * kThreads - 1) / (per_thread * kThreads);
        const uint32_t grid = uint32_t(std::max<uint64_t>(1, std::min<uint64_t>(blocks, uint64_t(sms) * 8)));
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(kThreads);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = (pdl && u > 0) ? 1 : 0;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (elem_bytes == 4) {
            auto *s = static_cast<const uint32_t *>(src);
            auto *d = static_cast<uint32_t *>(dst);
            cudaLaunchKernelEx(&cfg, vec ? k_reshard<uint32_t, 4, R> : k_reshard<uint32_t, 1, R>, s, d, r);
        } else {
            auto *s = static_cast<const uint16_t *>(src);
            auto *d = static_cast<uint16_t *>(dst);
            cudaLaunchKernelEx(&cfg, vec ? k_reshard<uint16_t, 8, R> : k_reshard<uint16_t, 1, R>, s, d, r);
        }
        st = zero_host::check_launch("zero_reshard launch");
        if (st != ZERO_OK) return st;
    }
    return ZERO_OK;
}


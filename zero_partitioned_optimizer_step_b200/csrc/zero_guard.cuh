// Kernels of the guarded step (global-norm clipping, skip on non-finite
// gradients), which needs the whole step's gradient norm before any update:
//   k_reduce           pass 1: rank-order sum of the Nd bf16 rows into the
//                      fp32 reduced gradient, per-CTA sums of squares and
//                      non-finite counts (same arithmetic as the fused step);
//   k_guard_finalize   one CTA: the fixed-order total, the clip coefficient
//                      and the skip decision, written to the workspace;
//   k_apply            pass 2: Adam from the reduced gradient, with
//                      g = (g_sum * grad_scale) * coef, or nothing if skipped;
//   k_apply_bulk       pass 2 with Nd replica rows: the same update, the bf16
//                      parameters staged in shared memory and written to
//                      every replica row with 1-D bulk copies.
// HBM-bound streams; 16-byte accesses on the vector path (VEC = 8), any
// alignment on the scalar path (VEC = 1).
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "zero_device.cuh"

namespace zero_guarded {

using zero_dev::AdamConsts;
using zero_dev::StepArgs;
using zero_dev::kThreads;

using zero_dev::GuardWord;

__device__ __forceinline__ uint64_t owner_of(const StepArgs &a, uint64_t j, bool owner_map) {
    return owner_map ? j / a.shard : 0;
}

// 8 consecutive fp32 with one 32-byte access (sm_100 and later; the address
// must be 32-byte aligned), streaming cache hint.
__device__ __forceinline__ void ld8_cs(const float *p, float f[8]) {
    asm volatile("ld.global.cs.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=f"(f[0]), "=f"(f[1]), "=f"(f[2]), "=f"(f[3]), "=f"(f[4]), "=f"(f[5]), "=f"(f[6]), "=f"(f[7])
                 : "l"(p));
}

__device__ __forceinline__ void st8_cs(float *p, const float f[8]) {
    asm volatile("st.global.cs.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "f"(f[0]), "f"(f[1]),
                 "f"(f[2]), "f"(f[3]), "f"(f[4]), "f"(f[5]), "f"(f[6]), "f"(f[7])
                 : "memory");
}

// CTAs per SM the two passes are sized for (registers <= 64 per thread).
constexpr int kGuardMinB = 4;
// Gradient rows of pass 1 loaded together before their in-order adds.
constexpr int kGuardRB = 8;

// W32: the fp32 arrays are 32-byte aligned (one 32-byte access per 8 elements).
template <int VEC, bool OWNER_MAP, bool W32 = false>
__global__ void __launch_bounds__(kThreads, kGuardMinB) k_reduce(const StepArgs a) {
    zero_dev::pdl_launch_dependents();
    const uint64_t n = (a.j1 - a.j0) / VEC;
    const uint64_t stride = uint64_t(gridDim.x) * kThreads;
    double acc = 0.0;
    uint32_t bad = 0;
    for (uint64_t vi = uint64_t(blockIdx.x) * kThreads + threadIdx.x; vi < n; vi += stride) {
        const uint64_t j = a.j0 + vi * VEC;
        const uint64_t o = owner_of(a, j, OWNER_MAP);
        const uint64_t gi = uint64_t(a.g_base + int64_t(j));
        const uint64_t si = uint64_t(a.s_base + int64_t(j)) + o * a.jump;
        float s[VEC];
        if constexpr (VEC == 8) {
            const uint16_t *g = a.grads + gi;
            for (uint32_t r0 = 0; r0 < a.nd; r0 += kGuardRB) {
                uint4 x[kGuardRB];
#pragma unroll
                for (int k = 0; k < kGuardRB; ++k)
                    if (r0 + k < a.nd) x[k] = __ldcs(reinterpret_cast<const uint4 *>(g + uint64_t(r0 + k) * a.grad_stride));
#pragma unroll
                for (int k = 0; k < kGuardRB; ++k) {  // rank order, from rank 0's value
                    if (r0 + k >= a.nd) break;
                    if (r0 + k == 0) zero_dev::unpack8(x[0], s);
                    else zero_dev::add8(s, x[k]);
                }
            }
            if constexpr (W32) {
                st8_cs(a.red + si, s);
            } else {
                __stcs(reinterpret_cast<float4 *>(a.red + si), make_float4(s[0], s[1], s[2], s[3]));
                __stcs(reinterpret_cast<float4 *>(a.red + si + 4), make_float4(s[4], s[5], s[6], s[7]));
            }
        } else {
            s[0] = __uint_as_float(uint32_t(a.grads[gi]) << 16);
            for (uint32_t r = 1; r < a.nd; ++r)
                s[0] = __fadd_rn(s[0], __uint_as_float(uint32_t(a.grads[gi + uint64_t(r) * a.grad_stride]) << 16));
            a.red[si] = s[0];
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            acc += double(s[e]) * double(s[e]);
            bad += zero_dev::not_finite(s[e]);
        }
    }
    zero_dev::pdl_wait();  // predecessor done: its norm slots are final
    zero_dev::block_partials(acc, bad, a);
}

// One CTA: sum the partials in a fixed order, report them, and decide.
__global__ void __launch_bounds__(kThreads) k_guard_finalize(const double *ws_norm, const uint32_t *ws_bad,
                                                            uint32_t slots, double *norm_out,
                                                            int32_t *overflow_out, GuardWord *gw,
                                                            double max_norm, double grad_scale,
                                                            int skip_nonfinite) {
    __shared__ double sd[kThreads];
    __shared__ uint32_t sb[kThreads];
    double t = 0.0;
    uint32_t b = 0;
    for (uint32_t i = threadIdx.x; i < slots; i += kThreads) {
        t += ws_norm[i];
        b |= ws_bad[i] != 0;
    }
    sd[threadIdx.x] = t;
    sb[threadIdx.x] = b;
    __syncthreads();
    for (int s = kThreads / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) {
            sd[threadIdx.x] += sd[threadIdx.x + s];
            sb[threadIdx.x] |= sb[threadIdx.x + s];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const double norm_sq = sd[0];
        *norm_out = norm_sq;
        *overflow_out = sb[0] ? 1 : 0;
        float coef = 1.0f;
        if (max_norm > 0.0 && isfinite(norm_sq)) {
            const double total = fabs(grad_scale) * sqrt(norm_sq);
            coef = float(fmin(1.0, max_norm / (total + 1e-6)));
        }
        gw->coef = coef;
        gw->skip = (skip_nonfinite && sb[0]) ? 1 : 0;
    }
}

// Adam of 8 consecutive elements from the reduced gradient, g = (g_sum *
// grad_scale) * coef: loads the reduced gradient and w, m, v at state index
// si (32-byte accesses if W32, else 16-byte), stores w, m, v, and returns
// the new parameters packed as bf16.
template <bool W32>
__device__ __forceinline__ uint4 apply8(const StepArgs &a, const AdamConsts &C, float coef, uint64_t si) {
    float s[8], w[8], m[8], v[8];
    if constexpr (W32) {
        ld8_cs(a.red + si, s);
        ld8_cs(a.w + si, w);
        ld8_cs(a.m + si, m);
        ld8_cs(a.v + si, v);
    } else {
        const float4 *rp = reinterpret_cast<const float4 *>(a.red + si);
        const float4 *wp = reinterpret_cast<const float4 *>(a.w + si);
        const float4 *mp = reinterpret_cast<const float4 *>(a.m + si);
        const float4 *vp = reinterpret_cast<const float4 *>(a.v + si);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float4 r4 = __ldcs(rp + h), w4 = __ldcs(wp + h), m4 = __ldcs(mp + h), v4 = __ldcs(vp + h);
            s[4 * h] = r4.x; s[4 * h + 1] = r4.y; s[4 * h + 2] = r4.z; s[4 * h + 3] = r4.w;
            w[4 * h] = w4.x; w[4 * h + 1] = w4.y; w[4 * h + 2] = w4.z; w[4 * h + 3] = w4.w;
            m[4 * h] = m4.x; m[4 * h + 1] = m4.y; m[4 * h + 2] = m4.z; m[4 * h + 3] = m4.w;
            v[4 * h] = v4.x; v[4 * h + 1] = v4.y; v[4 * h + 2] = v4.z; v[4 * h + 3] = v4.w;
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) zero_dev::adam1c(s[e], coef, C, w[e], m[e], v[e]);
    if constexpr (W32) {
        st8_cs(a.w + si, w);
        st8_cs(a.m + si, m);
        st8_cs(a.v + si, v);
    } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            __stcs(reinterpret_cast<float4 *>(a.w + si) + h,
                   make_float4(w[4 * h], w[4 * h + 1], w[4 * h + 2], w[4 * h + 3]));
            __stcs(reinterpret_cast<float4 *>(a.m + si) + h,
                   make_float4(m[4 * h], m[4 * h + 1], m[4 * h + 2], m[4 * h + 3]));
            __stcs(reinterpret_cast<float4 *>(a.v + si) + h,
                   make_float4(v[4 * h], v[4 * h + 1], v[4 * h + 2], v[4 * h + 3]));
        }
    }
    uint4 pk;
    pk.x = zero_dev::pack_bf16x2(w[0], w[1]);
    pk.y = zero_dev::pack_bf16x2(w[2], w[3]);
    pk.z = zero_dev::pack_bf16x2(w[4], w[5]);
    pk.w = zero_dev::pack_bf16x2(w[6], w[7]);
    return pk;
}

template <int VEC, bool OWNER_MAP, bool W32 = false>
__global__ void __launch_bounds__(kThreads, kGuardMinB) k_apply(const StepArgs a, const GuardWord *gw) {
    // Launched early behind the previous bucket's apply, which itself started
    // only after the finalize completed, so the guard word is final here.
    zero_dev::pdl_launch_dependents();
    const GuardWord g = *gw;
    if (g.skip) {
        zero_dev::pdl_wait();
        return;
    }
    const AdamConsts C = zero_dev::consts_of(a);
    const uint64_t n = (a.j1 - a.j0) / VEC;
    const uint64_t stride = uint64_t(gridDim.x) * kThreads;
    for (uint64_t vi = uint64_t(blockIdx.x) * kThreads + threadIdx.x; vi < n; vi += stride) {
        const uint64_t j = a.j0 + vi * VEC;
        const uint64_t o = owner_of(a, j, OWNER_MAP);
        const uint64_t si = uint64_t(a.s_base + int64_t(j)) + o * a.jump;
        const uint64_t pi = uint64_t(a.p_base + int64_t(j)) + o * a.p_jump;
        if constexpr (VEC == 8) {
            const uint4 pk = apply8<W32>(a, C, g.coef, si);
            for (uint32_t r = 0; r < a.n_prow; ++r)
                __stcs(reinterpret_cast<uint4 *>(a.params + pi + uint64_t(r) * a.param_stride), pk);
        } else {
            float w = a.w[si], m = a.m[si], v = a.v[si];
            zero_dev::adam1c(a.red[si], g.coef, C, w, m, v);
            a.w[si] = w;
            a.m[si] = m;
            a.v[si] = v;
            __nv_bfloat16 h = __float2bfloat16_rn(w);
            const uint16_t bits = *reinterpret_cast<uint16_t *>(&h);
            for (uint32_t r = 0; r < a.n_prow; ++r) a.params[pi + uint64_t(r) * a.param_stride] = bits;
        }
    }
    zero_dev::pdl_wait();  // complete only after the predecessor, in stream order
}

// ---------------------------------------------------------------------------
// Pass 2 when the parameters go to Nd replica rows (stages 0-2), vector body
// only.  Each replica store of k_apply is one more 16-byte store per thread
// per 8 elements (8 of its 11-14 memory instructions at Nd = 8), and the
// load/store queue, not DRAM, held that pass back.  Here a CTA takes tiles
// of kApplyTile elements: every thread updates 8 of them as k_apply does,
// writes their bf16 to a shared-memory tile, and after a CTA barrier one
// thread copies the tile to every replica row with 1-D bulk copies
// (cp.async.bulk.global.shared::cta, no multicast), one per row.  Two tile
// buffers alternate; before one is rewritten, the issuing thread waits until
// the bulk copies of two tiles ago have read it.  Replica rows are contiguous
// in logical order (the parameter index has no owner jump), so a tile's row
// is one copy; the vector body starts and ends on multiples of 8 elements,
// so every copy is a multiple of 16 bytes at a 16-byte-aligned address.
constexpr uint32_t kApplyTile = kThreads * 8;

__device__ __forceinline__ void bulk_store_s2g(void *gdst, const void *ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
                 "r"(static_cast<uint32_t>(__cvta_generic_to_shared(ssrc))), "r"(bytes)
                 : "memory");
}

template <bool OWNER_MAP, bool W32>
__global__ void __launch_bounds__(kThreads, 3) k_apply_bulk(const StepArgs a, const GuardWord *gw) {
    __shared__ __align__(128) uint16_t tile_p[2][kApplyTile];
    zero_dev::pdl_launch_dependents();
    const GuardWord g = *gw;
    if (g.skip) {
        zero_dev::pdl_wait();
        return;
    }
    const AdamConsts C = zero_dev::consts_of(a);
    const uint64_t n_tiles = (a.j1 - a.j0 + kApplyTile - 1) / kApplyTile;
    uint32_t buf = 0;
    for (uint64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, buf ^= 1u) {
        // tile_p[buf] was last read by the copies of two tiles ago
        if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        __syncthreads();
        const uint64_t jt = a.j0 + tile * kApplyTile;
        const uint32_t cnt = uint32_t(min(uint64_t(kApplyTile), a.j1 - jt));  // a multiple of 8
        const uint32_t e0 = threadIdx.x * 8;
        if (e0 < cnt) {
            const uint64_t j = jt + e0;
            const uint64_t o = owner_of(a, j, OWNER_MAP);
            const uint64_t si = uint64_t(a.s_base + int64_t(j)) + o * a.jump;
            *reinterpret_cast<uint4 *>(&tile_p[buf][e0]) = apply8<W32>(a, C, g.coef, si);
        }
        // this thread's shared-memory writes, visible to the bulk copies
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        if (threadIdx.x == 0) {
            uint16_t *row = a.params + uint64_t(a.p_base + int64_t(jt));
            for (uint32_t r = 0; r < a.n_prow; ++r)
                bulk_store_s2g(row + uint64_t(r) * a.param_stride, &tile_p[buf][0], cnt * 2u);
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
    }
    // the shared tiles must outlive the copies, which also complete the writes
    if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    zero_dev::pdl_wait();
}

}  // namespace zero_guarded

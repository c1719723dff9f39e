// sm_100a kernels of the ZeRO partitioned mixed-precision Adam step, and the
// C-ABI entry points that launch them.  K1's default form, the bulk-copy
// (TMA) ring kernel k_step_tma, is in zero_tma.cuh and its ring shapes in
// zero_ring.cuh; this file holds K1's 16-byte-load and scalar forms, K2, the
// launch logic of the step, the guarded step and the layer gathers.
//
// K1 k_step_tma / k_step_vec8 / k_step_scalar -- one bucket of the step, fused:
//    reduce-scatter  : g_sum = sum over ranks r = 0..Nd-1 of float(G_r[j]),
//                      added in rank order from rank 0's value (fp32, RN);
//    owner Adam      : fp32 master w, first moment m, second moment v;
//    all-gather      : bf16(w) written to every replica row (stages 0-2) or
//                      to the owner's shard (stage 3 / one-owner view);
//    epilogue        : optional reduced-gradient store, and per-CTA partial
//                      sums of g_sum^2 and of non-finite g_sum for the
//                      gradient-norm / overflow check.
//    Sources: mind-map page "ZeRO 真正在做什么：长期分开存，计算时临时拼齐",
//    section "但 GPU 只存四分之一…" (gradients are split back to the owner of
//    each shard, which updates and keeps it) and glossary entries
//    "reduce-scatter" / "all-gather"; concept page "ZeRO", section
//    "为什么需要它" (mixed-precision Adam: low-precision parameters, fp32
//    master, two moments) and table "三个阶段".
// K2 k_gather -- stage-3 materialisation of one unit (glossary entry
//    "临时物化": the shards are briefly put together into the full layer).
// K3 k_finalize (zero_device.cuh) -- sums the per-CTA partials in a fixed order.
//
// Everything is HBM-bound streaming: per element K1 reads 2*Nd bytes of
// gradients and 12 bytes of state, writes 12 bytes of state and 2*Nd (or 2)
// bytes of parameters, for ~20 fp32 operations.  There is no contraction, so
// no tensor cores; the design goals are 16-byte coalesced accesses, enough
// bytes in flight per SM, streaming cache hints on one-touch data, and a
// persistent grid of (SM count x resident CTAs).
//
// Numerics: every Adam operation is an explicit round-to-nearest intrinsic
// (__fmul_rn, __fadd_rn, __fsqrt_rn, __fdiv_rn, which the compiler never
// contracts into FMA); the file is also built with -fmad=false.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <map>
#include <mutex>
#include <cstdlib>
#include <cstring>
#include <string>

#include "zero_device.cuh"
#include "zero_guard.cuh"
#include "zero_tma.cuh"
#include "zero_ring.cuh"
#include "zero_host.cuh"
#include "zero_internal.h"
#include "zero_trace.h"

using zero_detail::set_error;
using zero_host::aligned16;
using zero_host::check_launch;
using zero_host::mult8;
using zero_ring::choose_ring;
using zero_ring::kernel_choice;
using zero_ring::ring_for_launch;

namespace {

using namespace zero_dev;

// The bulk-copy kernels' device error word on each device (1: a bounded
// wait gave up; 2: a stage held another tile than expected).  Kernels get its
// address in their Ring; zero_stream_status() reads and clears it.
__device__ int g_wait_error;

// K1, vector path: 8 elements (16 B of bf16, 32 B of fp32) per thread and
// iteration.  Preconditions (checked on the host): j0, j1, all bases, strides,
// shard and jump are multiples of 8 and every pointer is 16-byte aligned.
// RB: gradient rows loaded together before their in-order adds; MINB: CTAs
// per SM the register budget is sized for.
template <bool OWNER_MAP, int RB, int MINB>
__global__ void __launch_bounds__(kThreads, MINB) k_step_vec8(const StepArgs a) {
    pdl_launch_dependents();
    const AdamConsts C = consts_of(a);
    const uint64_t nvec = (a.j1 - a.j0) >> 3;
    const uint64_t stride = uint64_t(gridDim.x) * kThreads;
    uint64_t vi = uint64_t(blockIdx.x) * kThreads + threadIdx.x;
    double acc = 0.0;
    uint32_t bad = 0;
    uint64_t owner = 0, next_b = 0;
    if (OWNER_MAP && vi < nvec) {
        owner = (a.j0 + (vi << 3)) / a.shard;
        next_b = (owner + 1) * a.shard;
    }
    for (; vi < nvec; vi += stride) {
        const uint64_t j = a.j0 + (vi << 3);
        uint64_t so = 0, po = 0;
        if (OWNER_MAP) {
            while (j >= next_b) {  // j only grows, so the owner only advances
                ++owner;
                next_b += a.shard;
            }
            so = owner * a.jump;
            po = owner * a.p_jump;
        }
        const uint64_t gi = uint64_t(a.g_base + int64_t(j));
        const uint64_t si = uint64_t(a.s_base + int64_t(j)) + so;
        const uint64_t pi = uint64_t(a.p_base + int64_t(j)) + po;

        // reduce-scatter: rank-order sum; RB rows in flight at a time
        const uint16_t *g = a.grads + gi;
        float s[8];
        {
            uint4 x[RB];
#pragma unroll
            for (int k = 0; k < RB; ++k)
                if (uint32_t(k) < a.nd)
                    x[k] = __ldcs(reinterpret_cast<const uint4 *>(g + uint64_t(k) * a.grad_stride));
            unpack8(x[0], s);
#pragma unroll
            for (int k = 1; k < RB; ++k)
                if (uint32_t(k) < a.nd) add8(s, x[k]);
        }
        for (uint32_t r0 = RB; r0 < a.nd; r0 += RB) {
            uint4 x[RB];
#pragma unroll
            for (int k = 0; k < RB; ++k)
                if (r0 + k < a.nd)
                    x[k] = __ldcs(reinterpret_cast<const uint4 *>(g + uint64_t(r0 + k) * a.grad_stride));
#pragma unroll
            for (int k = 0; k < RB; ++k)
                if (r0 + k < a.nd) add8(s, x[k]);
        }

        const float4 w0 = __ldcs(reinterpret_cast<const float4 *>(a.w + si));
        const float4 w1 = __ldcs(reinterpret_cast<const float4 *>(a.w + si + 4));
        const float4 m0 = __ldcs(reinterpret_cast<const float4 *>(a.m + si));
        const float4 m1 = __ldcs(reinterpret_cast<const float4 *>(a.m + si + 4));
        const float4 v0 = __ldcs(reinterpret_cast<const float4 *>(a.v + si));
        const float4 v1 = __ldcs(reinterpret_cast<const float4 *>(a.v + si + 4));

        if (a.ws_mode) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                acc += double(s[e]) * double(s[e]);
                bad += not_finite(s[e]);
            }
        }
        if (a.red) {
            __stcs(reinterpret_cast<float4 *>(a.red + si), make_float4(s[0], s[1], s[2], s[3]));
            __stcs(reinterpret_cast<float4 *>(a.red + si + 4), make_float4(s[4], s[5], s[6], s[7]));
        }

        float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        float mv[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
        float vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) adam1(s[e], C, wv[e], mv[e], vv[e]);

        __stcs(reinterpret_cast<float4 *>(a.w + si), make_float4(wv[0], wv[1], wv[2], wv[3]));
        __stcs(reinterpret_cast<float4 *>(a.w + si + 4), make_float4(wv[4], wv[5], wv[6], wv[7]));
        __stcs(reinterpret_cast<float4 *>(a.m + si), make_float4(mv[0], mv[1], mv[2], mv[3]));
        __stcs(reinterpret_cast<float4 *>(a.m + si + 4), make_float4(mv[4], mv[5], mv[6], mv[7]));
        __stcs(reinterpret_cast<float4 *>(a.v + si), make_float4(vv[0], vv[1], vv[2], vv[3]));
        __stcs(reinterpret_cast<float4 *>(a.v + si + 4), make_float4(vv[4], vv[5], vv[6], vv[7]));

        // all-gather: the same 16 bytes of bf16 to every parameter row
        uint4 pk;
        pk.x = pack_bf16x2(wv[0], wv[1]);
        pk.y = pack_bf16x2(wv[2], wv[3]);
        pk.z = pack_bf16x2(wv[4], wv[5]);
        pk.w = pack_bf16x2(wv[6], wv[7]);
        uint16_t *p = a.params + pi;
        for (uint32_t r = 0; r < a.n_prow; ++r)
            __stcs(reinterpret_cast<uint4 *>(p + uint64_t(r) * a.param_stride), pk);
    }
    pdl_wait();
    if (a.ws_mode) block_partials(acc, bad, a);
}

// K1, scalar path: any alignment (A not a multiple of 8, odd strides, bucket
// heads and tails).  Same arithmetic, one element per thread and iteration.
__global__ void __launch_bounds__(kThreads) k_step_scalar(const StepArgs a) {
    const AdamConsts C = consts_of(a);
    const uint64_t n = a.j1 - a.j0;
    const uint64_t stride = uint64_t(gridDim.x) * kThreads;
    double acc = 0.0;
    uint32_t bad = 0;
    for (uint64_t i = uint64_t(blockIdx.x) * kThreads + threadIdx.x; i < n; i += stride) {
        const uint64_t j = a.j0 + i;
        const uint64_t owner = a.shard ? j / a.shard : 0;
        const uint64_t gi = uint64_t(a.g_base + int64_t(j));
        const uint64_t si = uint64_t(a.s_base + int64_t(j)) + owner * a.jump;
        const uint64_t pi = uint64_t(a.p_base + int64_t(j)) + owner * a.p_jump;
        float s = __uint_as_float(uint32_t(a.grads[gi]) << 16);
        for (uint32_t r = 1; r < a.nd; ++r)
            s = __fadd_rn(s, __uint_as_float(uint32_t(a.grads[gi + uint64_t(r) * a.grad_stride]) << 16));
        if (a.ws_mode) {
            acc += double(s) * double(s);
            bad += not_finite(s);
        }
        if (a.red) a.red[si] = s;
        float w = a.w[si], m = a.m[si], v = a.v[si];
        adam1(s, C, w, m, v);
        a.w[si] = w;
        a.m[si] = m;
        a.v[si] = v;
        __nv_bfloat16 h = __float2bfloat16_rn(w);
        const uint16_t bits = *reinterpret_cast<uint16_t *>(&h);
        for (uint32_t r = 0; r < a.n_prow; ++r) a.params[pi + uint64_t(r) * a.param_stride] = bits;
    }
    if (a.ws_mode) block_partials(acc, bad, a);
}

// K2: full_layer[o*s_u + i] = owner_params[o*S + off_u + i] for the first
// len_u elements; `cpo` CTAs per owner, owners in rank order.  Each thread
// keeps four 16-byte loads in flight before it stores them.
__global__ void __launch_bounds__(kThreads) k_gather(const uint16_t *src, uint64_t S, uint64_t off_u,
                                                    uint64_t s_u, uint64_t len, uint16_t *dst,
                                                    uint32_t nd, uint32_t cpo, int vec_ok) {
    const uint32_t o = blockIdx.x / cpo, c = blockIdx.x % cpo;
    if (o >= nd) return;
    const uint64_t begin = uint64_t(o) * s_u;
    if (begin >= len) return;
    const uint64_t n = min(s_u, len - begin);
    const uint16_t *s = src + uint64_t(o) * S + off_u;
    uint16_t *d = dst + begin;
    const uint64_t stride = uint64_t(cpo) * kThreads;
    const uint64_t nv = vec_ok ? (n >> 3) : 0;
    const uint4 *s4 = reinterpret_cast<const uint4 *>(s);
    uint4 *d4 = reinterpret_cast<uint4 *>(d);
    uint64_t i = uint64_t(c) * kThreads + threadIdx.x;
    for (; i + 3 * stride < nv; i += 4 * stride) {
        const uint4 x0 = __ldcs(s4 + i), x1 = __ldcs(s4 + i + stride);
        const uint4 x2 = __ldcs(s4 + i + 2 * stride), x3 = __ldcs(s4 + i + 3 * stride);
        __stcs(d4 + i, x0);
        __stcs(d4 + i + stride, x1);
        __stcs(d4 + i + 2 * stride, x2);
        __stcs(d4 + i + 3 * stride, x3);
    }
    for (; i < nv; i += stride) __stcs(d4 + i, __ldcs(s4 + i));
    for (uint64_t q = (nv << 3) + uint64_t(c) * kThreads + threadIdx.x; q < n; q += stride) d[q] = s[q];
}

// ----------------------------------------------------------------- host side

// The bulk-copy kernel instantiations: owner map x consumer groups x vector
// width, for the fused step (rows = the Nd gradient rows) and for the guarded
// step's second pass (row = the reduced gradient).
template <int SRC>
using TmaKernelOf = void (*)(const StepArgs, const zero_tma::Ring, const typename zero_tma::ExtraOf<SRC>::type);
using TmaKernel = TmaKernelOf<zero_tma::kGradRows>;
using ApplyKernel = TmaKernelOf<zero_tma::kReduced>;

template <bool OM, int SRC, int CW>
TmaKernelOf<SRC> tma_kernel_cw(uint32_t groups, uint32_t vw) {
    using namespace zero_tma;
    if (groups == 2)
        return vw == 2 ? k_step_tma<OM, 2, 2, SRC, CW>
                       : (vw == 4 ? k_step_tma<OM, 2, 4, SRC, CW> : k_step_tma<OM, 2, 8, SRC, CW>);
    return vw == 2 ? k_step_tma<OM, 1, 2, SRC, CW>
                   : (vw == 4 ? k_step_tma<OM, 1, 4, SRC, CW> : k_step_tma<OM, 1, 8, SRC, CW>);
}

// ... and x consumer warps (8 or 16; a CTA has 32 + 32 * cw threads)
template <bool OM, int SRC = zero_tma::kGradRows>
TmaKernelOf<SRC> tma_kernel(uint32_t groups, uint32_t vw, uint32_t cw = zero_tma::kConsumerWarps) {
    return cw == 16 ? tma_kernel_cw<OM, SRC, 16>(groups, vw) : tma_kernel_cw<OM, SRC, zero_tma::kConsumerWarps>(groups, vw);
}

// Launch shapes of the step kernels on one device, computed once per device:
// the persistent grid of the vector kernel (SM count x resident CTAs, capped
// at the norm workspace's slot count), the SM count for the bulk-copy kernel
// (one CTA per SM: its ring takes most of shared memory), and the dynamic
// shared memory the bulk-copy kernel may use.
struct DeviceShapes {
    int *err = nullptr;       // g_wait_error on this device
    uint32_t grid_ldg = 0;
    uint32_t grid_guard = 0;  // the guarded step's two passes (fewer registers)
    uint32_t grid_apply_bulk = 0;  // the guarded step's second pass with bulk replica copies
    uint32_t sms = 0;
    uint32_t tma_smem = 0;
};

zero_status_t device_shapes(DeviceShapes *out) {
    static std::mutex mu;
    static std::map<int, DeviceShapes> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_error(ZERO_ECUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    std::lock_guard<std::mutex> g(mu);
    auto it = cache.find(dev);
    if (it != cache.end()) {
        *out = it->second;
        return ZERO_OK;
    }
    int sms = 0, occ = 0, optin = 0, occ_r = 0, occ_a = 0, occ_b = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_step_vec8<false, kRB, kMinB>, kThreads, 0);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_r, zero_guarded::k_reduce<8, true, true>, kThreads, 0);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_a, zero_guarded::k_apply<8, true, true>, kThreads, 0);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_b, zero_guarded::k_apply_bulk<true, true>, kThreads, 0);
    cudaFuncAttributes fa{}, fa16{};
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, tma_kernel<true>(2, 2));
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa16, tma_kernel<true>(2, 2, 16));
    DeviceShapes d;
    void *err = nullptr;
    if (e == cudaSuccess) e = cudaGetSymbolAddress(&err, g_wait_error);
    d.err = static_cast<int *>(err);
    d.sms = uint32_t(std::max(1, sms));
    d.grid_ldg = std::min(uint32_t(std::max(1, sms) * std::max(1, occ)), zero_detail::kMaxSlots);
    d.grid_guard = std::min(uint32_t(std::max(1, sms) * std::max(1, std::min(occ_r, occ_a))), zero_detail::kMaxSlots);
    // three CTAs per SM (24 warps): the pass is bound by load latency
    // (long-scoreboard stalls) at two; measured on B200 with the guarded
    // GPT-2-small step, 1 / 2 / 3 / 4 CTAs per SM gave 5.78 / 6.02 / 6.23 /
    // 5.99 TB/s; ZERO_APPLY_BULK_CTAS overrides (tuning)
    int per_sm = 3;
    if (const char *v = std::getenv("ZERO_APPLY_BULK_CTAS")) per_sm = std::max(1, std::atoi(v));
    d.grid_apply_bulk = uint32_t(std::max(1, sms) * std::max(1, std::min(occ_b, per_sm)));
    const int64_t budget = int64_t(optin) - int64_t(std::max(fa.sharedSizeBytes, fa16.sharedSizeBytes)) - 256;
    d.tma_smem = budget > 0 ? uint32_t(budget) : 0;
    if (d.tma_smem > 0) {
        for (uint32_t g : {1u, 2u})
            for (uint32_t vw : {2u, 4u, 8u})
            for (uint32_t cw : {8u, 16u}) {
                const void *fs[] = {reinterpret_cast<const void *>(tma_kernel<true>(g, vw, cw)),
                                    reinterpret_cast<const void *>(tma_kernel<false>(g, vw, cw)),
                                    reinterpret_cast<const void *>(tma_kernel<true, zero_tma::kReduced>(g, vw, cw)),
                                    reinterpret_cast<const void *>(tma_kernel<false, zero_tma::kReduced>(g, vw, cw))};
                for (const void *f : fs)
                    if (e == cudaSuccess)
                        e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, int(d.tma_smem));
            }
    }
    if (e != cudaSuccess) return set_error(ZERO_ECUDA, std::string("device query: ") + cudaGetErrorString(e));
    cache[dev] = d;
    *out = d;
    return ZERO_OK;
}

AdamConsts make_consts(const zero_adam_t &a, uint64_t t) {
    // double, then one rounding to float each (bias corrections by pow())
    const double bc1 = 1.0 - std::pow(a.beta1, double(t));
    const double bc2 = 1.0 - std::pow(a.beta2, double(t));
    AdamConsts c;
    c.grad_scale = float(a.grad_scale);
    c.beta1 = float(a.beta1);
    c.beta2 = float(a.beta2);
    c.eps = float(a.eps);
    c.omb1 = float(1.0 - a.beta1);
    c.omb2 = float(1.0 - a.beta2);
    c.step = float(a.lr / bc1);
    c.ibc2 = float(1.0 / std::sqrt(bc2));
    c.decay = float(1.0 - a.lr * a.weight_decay);
    return c;
}

// Launch with or without programmatic dependent launch on the stream.
template <typename... Params, typename... Args>
cudaError_t launch_ex(void (*kernel)(Params...), uint32_t grid, uint32_t block, size_t smem,
                      cudaStream_t stream, bool pdl, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ZERO_PDL=0 turns programmatic dependent launch off (for comparison).
bool pdl_enabled() {
    const char *s = std::getenv("ZERO_PDL");
    return !(s && s[0] == '0');
}

// Gradient rows a thread of the 16-byte-load kernel keeps in flight: 8 for
// more than 16 ranks (read-heavy), else 4.  ZERO_LDG_RB=4|8 overrides.
int ldg_rows(uint32_t nd) {
    if (const char *e = std::getenv("ZERO_LDG_RB")) {
        if (std::strcmp(e, "8") == 0) return 8;
        if (std::strcmp(e, "4") == 0) return 4;
    }
    return nd > 16 ? 8 : 4;
}

struct Launcher {
    DeviceShapes shapes;
    cudaStream_t stream;
    bool want_ws = false;
    bool use_tma = false;
    zero_tma::Ring ring{};
    uint32_t launches = 0;
    bool pdl = true;  // vector-kernel launches after the first may overlap their predecessor

    zero_status_t run(StepArgs a, bool owner_map, bool vec_ok) {
        if (a.j0 >= a.j1) return ZERO_OK;
        auto one = [&](uint64_t j0, uint64_t j1, bool vec) -> zero_status_t {
            if (j0 >= j1) return ZERO_OK;
            StepArgs b = a;
            b.j0 = j0;
            b.j1 = j1;
            b.ws_mode = want_ws ? 1 : 0;
            const bool dep = pdl && launches > 0;
            if (vec && use_tma) {
                const zero_tma::Ring rg = ring_for_launch(ring, j1 - j0, b.nd, shapes.sms, shapes.tma_smem);
                const uint64_t tiles = (j1 - j0 + rg.tile - 1) / rg.tile;
                const uint32_t grid = uint32_t(std::min<uint64_t>(tiles, shapes.sms));
                const size_t smem = zero_ring::ring_smem_bytes(rg);
                TmaKernel f = owner_map ? tma_kernel<true>(rg.groups, rg.vw, rg.cw)
                                        : tma_kernel<false>(rg.groups, rg.vw, rg.cw);
                launch_ex(f, grid, 32 + 32 * rg.cw, smem, stream, dep, b, rg, zero_tma::NoExtra{});
            } else if (vec) {
                const bool rb8 = ldg_rows(b.nd) == 8;
                auto f = owner_map ? (rb8 ? k_step_vec8<true, 8, kMinB> : k_step_vec8<true, kRB, kMinB>)
                                   : (rb8 ? k_step_vec8<false, 8, kMinB> : k_step_vec8<false, kRB, kMinB>);
                launch_ex(f, shapes.grid_ldg, kThreads, 0, stream, dep, b);
            } else {
                k_step_scalar<<<shapes.grid_ldg, kThreads, 0, stream>>>(b);
            }
            ++launches;
            return check_launch("zero_step kernel launch");
        };
        if (!vec_ok) return one(a.j0, a.j1, false);
        const uint64_t lo = (a.j0 + 7) & ~uint64_t(7), hi = a.j1 & ~uint64_t(7);
        if (lo >= hi) return one(a.j0, a.j1, false);
        zero_status_t s = one(a.j0, lo, false);
        if (s == ZERO_OK) s = one(lo, hi, true);
        if (s == ZERO_OK) s = one(hi, a.j1, false);
        return s;
    }
};

zero_status_t validate_step(const zero_plan_t *p, const zero_bufs_t *b, const zero_adam_t *adam,
                            uint64_t t) {
    if (!p || !b || !adam) return set_error(ZERO_EINVAL, "zero_step: NULL argument");
    if (t == 0) return set_error(ZERO_EINVAL, "zero_step: t must be >= 1");
    if (!(std::isfinite(adam->lr) && std::isfinite(adam->eps) && std::isfinite(adam->grad_scale) &&
          std::isfinite(adam->weight_decay)))
        return set_error(ZERO_EINVAL, "zero_step: lr, eps, grad_scale and weight_decay must be finite");
    if (!(adam->beta1 >= 0.0 && adam->beta1 < 1.0 && adam->beta2 >= 0.0 && adam->beta2 < 1.0))
        return set_error(ZERO_EINVAL, "zero_step: beta1 and beta2 must be in [0, 1)");
    if (b->owner_view < -1 || b->owner_view >= int64_t(p->nd))
        return set_error(ZERO_EINVAL, "zero_step: owner_view must be -1 or a rank in [0, nd)");
    const void *req[] = {b->grads, b->master, b->exp_avg, b->exp_avg_sq, b->params};
    for (const void *q : req) {
        if (!q) return set_error(ZERO_EINVAL, "zero_step: grads, master, exp_avg, exp_avg_sq and params are required");
        if (!aligned16(q)) return set_error(ZERO_EINVAL, "zero_step: device pointers must be 16-byte aligned");
    }
    const void *opt[] = {b->reduced_grad, b->grad_norm_sq, b->overflow, b->workspace, b->adam_consts};
    for (const void *q : opt)
        if (q && !aligned16(q)) return set_error(ZERO_EINVAL, "zero_step: device pointers must be 16-byte aligned");
    const bool owner = b->owner_view >= 0;
    if (b->grad_stride < (owner ? p->S : p->psi_pad))
        return set_error(ZERO_EINVAL, "zero_step: grad_stride is shorter than a rank's gradient");
    if (!owner && p->stage <= 2 && b->param_stride < p->psi_pad)
        return set_error(ZERO_EINVAL, "zero_step: param_stride is shorter than a replica");
    if ((b->grad_norm_sq || b->overflow) &&
        (!b->workspace || b->workspace_bytes < zero_detail::kWorkspaceBytes))
        return set_error(ZERO_EINVAL, "zero_step: norm/overflow output needs a workspace of ZERO_Q_WORKSPACE_BYTES");
    return ZERO_OK;
}

// Launch arguments shared by every bucket of one call.
StepArgs base_args(const zero_plan_t *p, const zero_bufs_t *b, const zero_adam_t *adam, uint64_t t) {
    const bool replicas = b->owner_view < 0 && p->stage <= 2;
    StepArgs a{};
    a.grads = static_cast<const uint16_t *>(b->grads);
    a.grad_stride = b->grad_stride;
    a.w = b->master;
    a.m = b->exp_avg;
    a.v = b->exp_avg_sq;
    a.red = b->reduced_grad;
    a.params = static_cast<uint16_t *>(b->params);
    a.param_stride = replicas ? b->param_stride : 0;
    a.n_prow = replicas ? p->nd : 1;
    a.nd = p->nd;
    a.c = make_consts(*adam, t);
    a.cdev = static_cast<const AdamConsts *>(b->adam_consts);
    auto *ws = static_cast<unsigned char *>(b->workspace);
    a.ws_norm = reinterpret_cast<double *>(ws);
    a.ws_bad = reinterpret_cast<uint32_t *>(ws + 8ull * zero_detail::kMaxSlots);
    return a;
}

// Arguments of bucket bk: its unit-local element range (the owner's part of
// it in the one-owner view) and the offsets that map it to gradients, state
// and parameters.  False if the bucket holds nothing for this view.
bool bucket_args(const zero_plan_t *p, const zero_bufs_t *b, const StepArgs &a, uint64_t bk,
                 StepArgs *out, bool *owner_map, bool *vec_ok) {
    const bool owner = b->owner_view >= 0;
    const bool replicas = !owner && p->stage <= 2;
    const bool multi = p->unit_len.size() > 1;
    const zero_detail::BucketRange br = zero_detail::bucket_range(*p, bk);
    const uint32_t u = br.unit;
    const uint64_t U = p->unit_base[u], s_u = p->unit_shard[u], O = p->unit_offset[u];
    StepArgs x = a;
    x.j0 = br.begin - U;
    x.j1 = br.end - U;
    *owner_map = false;
    if (owner) {
        const uint64_t lo = uint64_t(b->owner_view) * s_u, hi = lo + s_u;
        x.j0 = std::max(x.j0, lo);
        x.j1 = std::min(x.j1, hi);
        if (x.j0 >= x.j1) return false;
        x.g_base = x.s_base = x.p_base = int64_t(O) - int64_t(lo);
        x.shard = x.jump = x.p_jump = 0;
    } else {
        x.g_base = int64_t(U);
        x.s_base = int64_t(O);
        if (multi) {
            *owner_map = true;
            x.shard = s_u;
            x.jump = p->S - s_u;
        }
        x.p_base = replicas ? int64_t(U) : int64_t(O);
        x.p_jump = replicas ? 0 : x.jump;
    }
    const bool strides_ok = (b->grad_stride & 7u) == 0 && (!replicas || (b->param_stride & 7u) == 0);
    *vec_ok = strides_ok && mult8(x.g_base) && mult8(x.s_base) && mult8(x.p_base) &&
              (!*owner_map || ((x.shard & 7u) == 0 && (x.jump & 7u) == 0));
    *out = x;
    return true;
}

// Calls f(j0, j1, vec) for the unaligned head, the 8-aligned body and the
// unaligned tail of x's range (everything unaligned if !vec_ok).
template <typename F>
zero_status_t split_launch(const StepArgs &x, bool vec_ok, F f) {
    if (x.j0 >= x.j1) return ZERO_OK;
    if (!vec_ok) return f(x.j0, x.j1, false);
    const uint64_t lo = (x.j0 + 7) & ~uint64_t(7), hi = x.j1 & ~uint64_t(7);
    if (lo >= hi) return f(x.j0, x.j1, false);
    zero_status_t s = ZERO_OK;
    if (x.j0 < lo) s = f(x.j0, lo, false);
    if (s == ZERO_OK) s = f(lo, hi, true);
    if (s == ZERO_OK && hi < x.j1) s = f(hi, x.j1, false);
    return s;
}

}  // namespace

ZERO_API zero_status_t zero_step_buckets(const zero_plan_t *p, const zero_bufs_t *b,
                                         const zero_adam_t *adam, uint64_t t, uint64_t first,
                                         uint64_t count, void *stream_) {
    zero_detail::clear_error();
    const zero_trace::Range call("zero_step t=%llu buckets [%llu, %llu)", (unsigned long long)t,
                                 (unsigned long long)first, (unsigned long long)(first + count));
    zero_status_t st = validate_step(p, b, adam, t);
    if (st != ZERO_OK) return st;
    if (first > p->n_buckets || count > p->n_buckets - first)
        return set_error(ZERO_EINVAL, "zero_step_buckets: bucket range outside the plan");
    cudaError_t pre = cudaPeekAtLastError();
    if (pre != cudaSuccess)
        return set_error(ZERO_ECUDA, std::string("pending CUDA error before zero_step: ") + cudaGetErrorString(pre));
    DeviceShapes shapes;
    st = device_shapes(&shapes);
    if (st != ZERO_OK) return st;

    const StepArgs a = base_args(p, b, adam, t);

    Launcher L;
    L.shapes = shapes;
    L.stream = static_cast<cudaStream_t>(stream_);
    L.want_ws = b->grad_norm_sq || b->overflow;
    L.pdl = pdl_enabled();
    const int choice = kernel_choice();
    L.use_tma = choice == 2 ? choose_ring(p->nd, false, shapes.tma_smem, shapes.err, &L.ring)
                            : choice != 1 && choose_ring(p->nd, a.n_prow == 1, shapes.tma_smem, shapes.err, &L.ring);
    if (L.want_ws && first == 0) {
        // the step's first call zeroes the per-CTA norm slots
        cudaError_t e = cudaMemsetAsync(b->workspace, 0, zero_detail::kWorkspaceBytes, L.stream);
        if (e != cudaSuccess)
            return set_error(ZERO_ECUDA, std::string("zero_step workspace reset: ") + cudaGetErrorString(e));
    }

    for (uint64_t bk = first; bk < first + count; ++bk) {
        StepArgs x;
        bool owner_map, vec_ok;
        if (!bucket_args(p, b, a, bk, &x, &owner_map, &vec_ok)) continue;
        const zero_trace::Range r("bucket %llu", (unsigned long long)bk);
        st = L.run(x, owner_map, vec_ok);
        if (st != ZERO_OK) return st;
    }
    if (L.want_ws && first + count == p->n_buckets && count > 0) {
        const zero_trace::Range r("norm finalize");
        k_finalize<<<1, kThreads, 0, L.stream>>>(a.ws_norm, a.ws_bad, zero_detail::kMaxSlots, b->grad_norm_sq,
                                                 b->overflow);
        st = check_launch("zero_step finalize launch");
        if (st != ZERO_OK) return st;
    }
    return ZERO_OK;
}

ZERO_API zero_status_t zero_step(const zero_plan_t *p, const zero_bufs_t *b, const zero_adam_t *adam,
                                 uint64_t t, void *stream) {
    if (!p) {
        zero_detail::clear_error();
        return set_error(ZERO_EINVAL, "zero_step: NULL plan");
    }
    return zero_step_buckets(p, b, adam, t, 0, p->n_buckets, stream);
}

ZERO_API zero_status_t zero_gather_layer(zero_plan_t *p, uint32_t unit, const void *owner_params,
                                         void *full_layer, void *stream_) {
    zero_detail::clear_error();
    const zero_trace::Range call("zero_gather_layer unit %u", unit);
    if (!p) return set_error(ZERO_EINVAL, "zero_gather_layer: NULL plan");
    if (p->stage != 3) return set_error(ZERO_EINVAL, "zero_gather_layer: only stage 3 materialises layers");
    if (unit >= p->unit_len.size()) return set_error(ZERO_EINVAL, "zero_gather_layer: unit out of range");
    if (!owner_params || !full_layer) return set_error(ZERO_EINVAL, "zero_gather_layer: NULL buffer");
    if (!aligned16(owner_params) || !aligned16(full_layer))
        return set_error(ZERO_EINVAL, "zero_gather_layer: buffers must be 16-byte aligned");
    std::lock_guard<std::mutex> g(p->mu);
    zero_status_t st = zero_detail::live_check(*p, unit, "zero_gather_layer");
    if (st != ZERO_OK) return st;
    cudaError_t pre = cudaPeekAtLastError();
    if (pre != cudaSuccess)
        return set_error(ZERO_ECUDA, std::string("pending CUDA error before zero_gather_layer: ") +
                                         cudaGetErrorString(pre));
    DeviceShapes shapes;
    st = device_shapes(&shapes);
    if (st != ZERO_OK) return st;
    const uint64_t s_u = p->unit_shard[unit], off = p->unit_offset[unit], len = p->unit_len[unit];
    const int vec_ok = ((p->S | off | s_u) & 7u) == 0;
    const uint32_t cpo = std::max<uint32_t>(1, (shapes.sms * 8) / p->nd);  // 8 CTAs/SM
    const uint64_t blocks = uint64_t(cpo) * p->nd;
    if (blocks > 0x7fffffffull) return set_error(ZERO_EINVAL, "zero_gather_layer: nd too large for one launch");
    k_gather<<<uint32_t(blocks), kThreads, 0, static_cast<cudaStream_t>(stream_)>>>(
        static_cast<const uint16_t *>(owner_params), p->S, off, s_u, len, static_cast<uint16_t *>(full_layer),
        p->nd, cpo, vec_ok);
    st = check_launch("zero_gather_layer launch");
    if (st != ZERO_OK) return st;
    zero_detail::live_mark(*p, unit);
    return ZERO_OK;
}

zero_status_t zero_detail::wait_error_word(int **out) {
    DeviceShapes shapes;
    zero_status_t st = device_shapes(&shapes);
    if (st == ZERO_OK) *out = shapes.err;
    return st;
}

ZERO_API zero_status_t zero_stream_status(void *stream) {
    zero_detail::clear_error();
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return set_error(ZERO_ECUDA, std::string("zero_stream_status: ") + cudaGetErrorString(e));
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, g_wait_error, sizeof v);
    if (e != cudaSuccess) return set_error(ZERO_ECUDA, std::string("zero_stream_status: ") + cudaGetErrorString(e));
    if (v) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_wait_error, &zero, sizeof zero);
        return set_error(ZERO_ETIMEOUT,
                         v == 2 ? "zero_stream_status: the bulk-copy step kernel found a stage holding the wrong "
                                  "tile and gave up; the outputs of the steps since the last check are not valid"
                                : "zero_stream_status: a bounded wait in the bulk-copy step kernel gave up; the "
                                  "outputs of the steps since the last check are not valid");
    }
    return ZERO_OK;
}

ZERO_API zero_status_t zero_step_kernel(const zero_plan_t *p, int32_t owner_view, uint32_t *kind) {
    zero_detail::clear_error();
    if (!p || !kind) return set_error(ZERO_EINVAL, "zero_step_kernel: NULL argument");
    if (owner_view < -1 || owner_view >= int64_t(p->nd))
        return set_error(ZERO_EINVAL, "zero_step_kernel: owner_view must be -1 or a rank in [0, nd)");
    DeviceShapes shapes;
    zero_status_t st = device_shapes(&shapes);
    if (st != ZERO_OK) return st;
    const bool replicas = owner_view < 0 && p->stage <= 2;
    zero_tma::Ring ring{};
    const int choice = kernel_choice();
    const bool tma = choice == 2 ? choose_ring(p->nd, false, shapes.tma_smem, shapes.err, &ring)
                                 : choice != 1 && choose_ring(p->nd, !replicas || p->nd == 1,
                                                              shapes.tma_smem, shapes.err, &ring);
    *kind = tma ? ZERO_KERNEL_BULK_COPY : ZERO_KERNEL_VECTOR_LOAD;
    return ZERO_OK;
}

ZERO_API zero_status_t zero_step_guarded(const zero_plan_t *p, const zero_bufs_t *b, const zero_adam_t *adam,
                                         const zero_guard_t *guard, uint64_t t, void *stream_) {
    zero_detail::clear_error();
    const zero_trace::Range call("zero_step_guarded t=%llu", (unsigned long long)t);
    zero_status_t st = validate_step(p, b, adam, t);
    if (st != ZERO_OK) return st;
    if (!guard) return set_error(ZERO_EINVAL, "zero_step_guarded: NULL guard");
    if (!(std::isfinite(guard->max_grad_norm) && guard->max_grad_norm >= 0.0))
        return set_error(ZERO_EINVAL, "zero_step_guarded: max_grad_norm must be finite and >= 0");
    if (!b->reduced_grad || !b->grad_norm_sq || !b->overflow || !b->workspace)
        return set_error(ZERO_EINVAL,
                         "zero_step_guarded: reduced_grad, grad_norm_sq, overflow and workspace are required");
    cudaError_t pre = cudaPeekAtLastError();
    if (pre != cudaSuccess)
        return set_error(ZERO_ECUDA, std::string("pending CUDA error before zero_step_guarded: ") +
                                         cudaGetErrorString(pre));
    DeviceShapes shapes;
    st = device_shapes(&shapes);
    if (st != ZERO_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    StepArgs a = base_args(p, b, adam, t);
    a.ws_mode = 1;
    auto *gw = reinterpret_cast<zero_guarded::GuardWord *>(static_cast<unsigned char *>(b->workspace) +
                                                         zero_detail::kGuardOffset);
    cudaError_t e = cudaMemsetAsync(b->workspace, 0, zero_detail::kWorkspaceBytes, stream);
    if (e != cudaSuccess)
        return set_error(ZERO_ECUDA, std::string("zero_step_guarded workspace reset: ") + cudaGetErrorString(e));
    const uint32_t grid = shapes.grid_guard;
    // Within each pass, launches after the first use programmatic dependent
    // launch: pass-1 kernels share only the norm slots (added to after the
    // predecessor completes); a pass-2 kernel starts after its predecessor,
    // which started after the finalize completed, so the guard word is final.
    const bool pdl = pdl_enabled();
    uint32_t n1 = 0, n2 = 0;
    // fp32 arrays 32-byte aligned: 32-byte accesses on the vector path
    const bool w32 = ((reinterpret_cast<uintptr_t>(b->master) | reinterpret_cast<uintptr_t>(b->exp_avg) |
                       reinterpret_cast<uintptr_t>(b->exp_avg_sq) | reinterpret_cast<uintptr_t>(b->reduced_grad)) &
                      31u) == 0;
    // pass 1: reductions, sums of squares, non-finite counts
    for (uint64_t bk = 0; bk < p->n_buckets; ++bk) {
        StepArgs x;
        bool om, vec_ok;
        if (!bucket_args(p, b, a, bk, &x, &om, &vec_ok)) continue;
        const zero_trace::Range r("reduce bucket %llu", (unsigned long long)bk);
        st = split_launch(x, vec_ok, [&](uint64_t j0, uint64_t j1, bool vec) -> zero_status_t {
            StepArgs y = x;
            y.j0 = j0;
            y.j1 = j1;
            const bool dep = pdl && n1++ > 0;
            auto f = vec ? (w32 ? (om ? zero_guarded::k_reduce<8, true, true> : zero_guarded::k_reduce<8, false, true>)
                                : (om ? zero_guarded::k_reduce<8, true> : zero_guarded::k_reduce<8, false>))
                         : (om ? zero_guarded::k_reduce<1, true> : zero_guarded::k_reduce<1, false>);
            launch_ex(f, grid, kThreads, 0, stream, dep, y);
            return check_launch("zero_step_guarded reduce launch");
        });
        if (st != ZERO_OK) return st;
    }
    {
        const zero_trace::Range fin("guard finalize");
        zero_guarded::k_guard_finalize<<<1, kThreads, 0, stream>>>(a.ws_norm, a.ws_bad, zero_detail::kMaxSlots,
                                                                 b->grad_norm_sq, b->overflow, gw,
                                                                 guard->max_grad_norm, adam->grad_scale,
                                                                 guard->skip_nonfinite ? 1 : 0);
        st = check_launch("zero_step_guarded finalize launch");
        if (st != ZERO_OK) return st;
    }
    // pass 2: Adam from the reduced gradients (no-op when the step is skipped).
    // When the parameters are written once (stage 3), aligned bodies run in
    // the bulk-copy kernel with the reduced gradient as its one fp32 row (a
    // ring shaped as for two bf16 rows): 0.95 of copy bandwidth against 0.91
    // for k_apply on the stage-3 1.3B workload.  With Nd replicas to write
    // (28 B of stores per element at Nd = 8) k_apply with 32-byte accesses is
    // faster (189 us against 200 us per 25M-element bucket).
    // ZERO_STEP_KERNEL=tma|ldg forces either.
    zero_tma::Ring ring{};
    const int choice = kernel_choice();
    const bool tma = (choice == 2 || (choice == 0 && a.n_prow == 1)) &&
                     choose_ring(2, false, shapes.tma_smem, shapes.err, &ring);
    ring.bulk_p = 0;  // this pass's parameters: per-thread stores
    // With replica rows, the vector body's parameters go out as bulk copies
    // from shared memory (k_apply_bulk) unless ZERO_GUARD_APPLY=ldst asks for
    // k_apply's per-thread stores.
    const char *ga = std::getenv("ZERO_GUARD_APPLY");
    const bool bulk_replicas = a.n_prow > 1 && !(ga && std::strcmp(ga, "ldst") == 0);
    a.ws_mode = 0;
    for (uint64_t bk = 0; bk < p->n_buckets; ++bk) {
        StepArgs x;
        bool om, vec_ok;
        if (!bucket_args(p, b, a, bk, &x, &om, &vec_ok)) continue;
        const zero_trace::Range r("apply bucket %llu", (unsigned long long)bk);
        st = split_launch(x, vec_ok, [&](uint64_t j0, uint64_t j1, bool vec) -> zero_status_t {
            StepArgs y = x;
            y.j0 = j0;
            y.j1 = j1;
            const bool dep = pdl && n2++ > 0;
            if (vec && tma) {
                const zero_tma::Ring rg = ring_for_launch(ring, j1 - j0, 2, shapes.sms, shapes.tma_smem);
                const uint64_t tiles = (j1 - j0 + rg.tile - 1) / rg.tile;
                const uint32_t g = uint32_t(std::min<uint64_t>(tiles, shapes.sms));
                ApplyKernel f = om ? tma_kernel<true, zero_tma::kReduced>(rg.groups, rg.vw, rg.cw)
                                   : tma_kernel<false, zero_tma::kReduced>(rg.groups, rg.vw, rg.cw);
                launch_ex(f, g, 32 + 32 * rg.cw, zero_ring::ring_smem_bytes(rg), stream, dep, y, rg,
                          zero_tma::ApplyExtra{gw});
            } else if (vec && bulk_replicas) {
                auto f = w32 ? (om ? zero_guarded::k_apply_bulk<true, true> : zero_guarded::k_apply_bulk<false, true>)
                             : (om ? zero_guarded::k_apply_bulk<true, false> : zero_guarded::k_apply_bulk<false, false>);
                launch_ex(f, shapes.grid_apply_bulk, kThreads, 0, stream, dep, y,
                          static_cast<const zero_guarded::GuardWord *>(gw));
            } else {
                auto f = vec ? (w32 ? (om ? zero_guarded::k_apply<8, true, true> : zero_guarded::k_apply<8, false, true>)
                                    : (om ? zero_guarded::k_apply<8, true> : zero_guarded::k_apply<8, false>))
                             : (om ? zero_guarded::k_apply<1, true> : zero_guarded::k_apply<1, false>);
                launch_ex(f, grid, kThreads, 0, stream, dep, y, static_cast<const zero_guarded::GuardWord *>(gw));
            }
            return check_launch("zero_step_guarded apply launch");
        });
        if (st != ZERO_OK) return st;
    }
    return ZERO_OK;
}

ZERO_API zero_status_t zero_adam_consts(const zero_adam_t *adam, uint64_t t, float out[9]) {
    zero_detail::clear_error();
    if (!adam || !out) return set_error(ZERO_EINVAL, "zero_adam_consts: NULL argument");
    if (t == 0) return set_error(ZERO_EINVAL, "zero_adam_consts: t must be >= 1");
    static_assert(sizeof(AdamConsts) == 9 * sizeof(float), "nine packed fp32 constants");
    const AdamConsts c = make_consts(*adam, t);
    std::memcpy(out, &c, sizeof c);
    return ZERO_OK;
}

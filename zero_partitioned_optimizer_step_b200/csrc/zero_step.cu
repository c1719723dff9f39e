// sm_100a kernels of the ZeRO partitioned mixed-precision Adam step, and the
// C-ABI entry points that launch them.
//
// K1 k_step_vec8 / k_step_scalar -- one bucket of the step, fused:
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
// K3 k_finalize -- sums the per-CTA partials in a fixed order.
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
#include <string>

#include "zero_internal.h"

using zero_detail::set_error;

namespace {

constexpr int kThreads = 256;
constexpr int kRB = 4;    // gradient rows in flight per thread
constexpr int kMinB = 2;  // CTAs per SM the vector kernel is sized for

struct AdamConsts {
    float grad_scale, beta1, beta2, eps, omb1, omb2, step, ibc2;
};

// One launch: the unit-local element range [j0, j1) of one bucket.
// Element j reads gradients at  g_base + j           (+ r*grad_stride),
// state at                      s_base + j + o*jump,
// parameters at                 p_base + j + o*p_jump (+ row*param_stride),
// where o = j / shard is the owner (used only when the unit is one of several,
// so that owner storage and logical order differ).
struct StepArgs {
    const uint16_t *grads;
    uint64_t grad_stride;
    float *w, *m, *v, *red;
    uint16_t *params;
    uint64_t param_stride;
    uint32_t n_prow;
    uint32_t nd;
    int64_t g_base, s_base, p_base;
    uint64_t shard, jump, p_jump;
    uint64_t j0, j1;
    AdamConsts c;
    double *ws_norm;
    uint32_t *ws_bad;
    int ws_mode;  // 0: no norm; 1: store this launch's partials; 2: add them
};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4 x, float f[8]) {
    f[0] = bf16lo(x.x); f[1] = bf16hi(x.x);
    f[2] = bf16lo(x.y); f[3] = bf16hi(x.y);
    f[4] = bf16lo(x.z); f[5] = bf16hi(x.z);
    f[6] = bf16lo(x.w); f[7] = bf16hi(x.w);
}

__device__ __forceinline__ void add8(float s[8], const uint4 x) {
    float f[8];
    unpack8(x, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) s[e] = __fadd_rn(s[e], f[e]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ bool not_finite(float x) {
    return (__float_as_uint(x) & 0x7f800000u) == 0x7f800000u;
}

// Textbook Adam on one element, every operation rounded to nearest.
__device__ __forceinline__ void adam1(float g_sum, const AdamConsts &c, float &w, float &m,
                                      float &v) {
    const float g = __fmul_rn(g_sum, c.grad_scale);
    const float m_new = __fadd_rn(__fmul_rn(c.beta1, m), __fmul_rn(c.omb1, g));
    const float v_new = __fadd_rn(__fmul_rn(c.beta2, v), __fmul_rn(__fmul_rn(c.omb2, g), g));
    const float denom = __fadd_rn(__fmul_rn(__fsqrt_rn(v_new), c.ibc2), c.eps);
    const float delta = __fmul_rn(c.step, __fdiv_rn(m_new, denom));
    w = __fsub_rn(w, delta);
    m = m_new;
    v = v_new;
}

// Per-CTA partials of the gradient-norm / overflow reduction (fixed order,
// so the reported norm is the same on every run of the same launch shape).
__device__ __forceinline__ void block_partials(double acc, uint32_t bad, const StepArgs &a) {
    __shared__ double sd[kThreads / 32];
    __shared__ uint32_t sb[kThreads / 32];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        acc += __shfl_down_sync(0xffffffffu, acc, off);
        bad += __shfl_down_sync(0xffffffffu, bad, off);
    }
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (lane == 0) {
        sd[wid] = acc;
        sb[wid] = bad;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        uint32_t b = 0;
        for (int i = 0; i < kThreads / 32; ++i) {
            t += sd[i];
            b += sb[i];
        }
        if (a.ws_mode == 1) {
            a.ws_norm[blockIdx.x] = t;
            a.ws_bad[blockIdx.x] = b;
        } else {
            a.ws_norm[blockIdx.x] += t;
            a.ws_bad[blockIdx.x] = min(a.ws_bad[blockIdx.x] + b, 0x7fffffffu);
        }
    }
}

// K1, vector path: 8 elements (16 B of bf16, 32 B of fp32) per thread and
// iteration.  Preconditions (checked on the host): j0, j1, all bases, strides,
// shard and jump are multiples of 8 and every pointer is 16-byte aligned.
// RB: gradient rows loaded together before their in-order adds; MINB: CTAs
// per SM the register budget is sized for.
template <bool OWNER_MAP, int RB, int MINB>
__global__ void __launch_bounds__(kThreads, MINB) k_step_vec8(const StepArgs a) {
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
        for (int e = 0; e < 8; ++e) adam1(s[e], a.c, wv[e], mv[e], vv[e]);

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
    if (a.ws_mode) block_partials(acc, bad, a);
}

// K1, scalar path: any alignment (A not a multiple of 8, odd strides, bucket
// heads and tails).  Same arithmetic, one element per thread and iteration.
__global__ void __launch_bounds__(kThreads) k_step_scalar(const StepArgs a) {
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
        adam1(s, a.c, w, m, v);
        a.w[si] = w;
        a.m[si] = m;
        a.v[si] = v;
        __nv_bfloat16 h = __float2bfloat16_rn(w);
        const uint16_t bits = *reinterpret_cast<uint16_t *>(&h);
        for (uint32_t r = 0; r < a.n_prow; ++r) a.params[pi + uint64_t(r) * a.param_stride] = bits;
    }
    if (a.ws_mode) block_partials(acc, bad, a);
}

// K3: fixed-order sum of the per-CTA partials of one step.
__global__ void __launch_bounds__(kThreads) k_finalize(const double *ws_norm, const uint32_t *ws_bad,
                                                      uint32_t slots, double *norm_out,
                                                      int32_t *overflow_out) {
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
        if (norm_out) *norm_out = sd[0];
        if (overflow_out) *overflow_out = sb[0] ? 1 : 0;
    }
}

// K2: full_layer[o*s_u + i] = owner_params[o*S + off_u + i] for the first
// len_u elements; `cpo` CTAs per owner, owners in rank order.
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
    for (uint64_t i = uint64_t(c) * kThreads + threadIdx.x; i < nv; i += stride) __stcs(d4 + i, __ldcs(s4 + i));
    for (uint64_t i = (nv << 3) + uint64_t(c) * kThreads + threadIdx.x; i < n; i += stride) d[i] = s[i];
}

// ----------------------------------------------------------------- host side

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Grid of the step kernels on the current device: SM count x resident CTAs
// of the vector kernel, capped at the workspace's slot count.  Cached per
// device; all launches of a step use it, so the norm slots line up.
zero_status_t device_grid(uint32_t *grid) {
    static std::mutex mu;
    static std::map<int, uint32_t> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_error(ZERO_ECUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    std::lock_guard<std::mutex> g(mu);
    auto it = cache.find(dev);
    if (it != cache.end()) {
        *grid = it->second;
        return ZERO_OK;
    }
    int sms = 0, occ = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_step_vec8<false, kRB, kMinB>, kThreads, 0);
    if (e != cudaSuccess) return set_error(ZERO_ECUDA, std::string("device query: ") + cudaGetErrorString(e));
    uint32_t gsz = uint32_t(std::max(1, sms) * std::max(1, occ));
    gsz = std::min(gsz, zero_detail::kMaxSlots);
    cache[dev] = gsz;
    *grid = gsz;
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
    return c;
}

zero_status_t check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(ZERO_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
    return ZERO_OK;
}

bool mult8(int64_t x) { return (uint64_t(x) & 7u) == 0; }

struct Launcher {
    uint32_t grid;
    cudaStream_t stream;
    bool first = true;   // next launch stores (not adds) its norm partials
    bool want_ws = false;
    uint32_t launches = 0;

    zero_status_t run(StepArgs a, bool owner_map, bool vec_ok) {
        if (a.j0 >= a.j1) return ZERO_OK;
        auto one = [&](uint64_t j0, uint64_t j1, bool vec) -> zero_status_t {
            if (j0 >= j1) return ZERO_OK;
            StepArgs b = a;
            b.j0 = j0;
            b.j1 = j1;
            b.ws_mode = want_ws ? (first ? 1 : 2) : 0;
            if (vec) {
                if (owner_map)
                    k_step_vec8<true, kRB, kMinB><<<grid, kThreads, 0, stream>>>(b);
                else
                    k_step_vec8<false, kRB, kMinB><<<grid, kThreads, 0, stream>>>(b);
            } else {
                k_step_scalar<<<grid, kThreads, 0, stream>>>(b);
            }
            first = false;
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
    if (!(std::isfinite(adam->lr) && std::isfinite(adam->eps) && std::isfinite(adam->grad_scale)))
        return set_error(ZERO_EINVAL, "zero_step: lr, eps and grad_scale must be finite");
    if (!(adam->beta1 >= 0.0 && adam->beta1 < 1.0 && adam->beta2 >= 0.0 && adam->beta2 < 1.0))
        return set_error(ZERO_EINVAL, "zero_step: beta1 and beta2 must be in [0, 1)");
    if (b->owner_view < -1 || b->owner_view >= int64_t(p->nd))
        return set_error(ZERO_EINVAL, "zero_step: owner_view must be -1 or a rank in [0, nd)");
    const void *req[] = {b->grads, b->master, b->exp_avg, b->exp_avg_sq, b->params};
    for (const void *q : req) {
        if (!q) return set_error(ZERO_EINVAL, "zero_step: grads, master, exp_avg, exp_avg_sq and params are required");
        if (!aligned16(q)) return set_error(ZERO_EINVAL, "zero_step: device pointers must be 16-byte aligned");
    }
    const void *opt[] = {b->reduced_grad, b->grad_norm_sq, b->overflow, b->workspace};
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

}  // namespace

ZERO_API zero_status_t zero_step_buckets(const zero_plan_t *p, const zero_bufs_t *b,
                                         const zero_adam_t *adam, uint64_t t, uint64_t first,
                                         uint64_t count, void *stream_) {
    zero_detail::clear_error();
    zero_status_t st = validate_step(p, b, adam, t);
    if (st != ZERO_OK) return st;
    if (first > p->n_buckets || count > p->n_buckets - first)
        return set_error(ZERO_EINVAL, "zero_step_buckets: bucket range outside the plan");
    cudaError_t pre = cudaPeekAtLastError();
    if (pre != cudaSuccess)
        return set_error(ZERO_ECUDA, std::string("pending CUDA error before zero_step: ") + cudaGetErrorString(pre));
    uint32_t grid = 0;
    st = device_grid(&grid);
    if (st != ZERO_OK) return st;

    const bool owner = b->owner_view >= 0;
    const bool replicas = !owner && p->stage <= 2;
    const bool multi = p->unit_len.size() > 1;

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
    auto *ws = static_cast<unsigned char *>(b->workspace);
    a.ws_norm = reinterpret_cast<double *>(ws);
    a.ws_bad = reinterpret_cast<uint32_t *>(ws + 8ull * zero_detail::kMaxSlots);

    Launcher L;
    L.grid = grid;
    L.stream = static_cast<cudaStream_t>(stream_);
    L.want_ws = b->grad_norm_sq || b->overflow;
    L.first = (first == 0);

    const bool strides_ok = (b->grad_stride & 7u) == 0 && (!replicas || (b->param_stride & 7u) == 0);
    for (uint64_t bk = first; bk < first + count; ++bk) {
        const zero_detail::BucketRange br = zero_detail::bucket_range(*p, bk);
        const uint32_t u = br.unit;
        const uint64_t U = p->unit_base[u], s_u = p->unit_shard[u], O = p->unit_offset[u];
        StepArgs x = a;
        x.j0 = br.begin - U;
        x.j1 = br.end - U;
        bool owner_map = false;
        if (owner) {
            const uint64_t lo = uint64_t(b->owner_view) * s_u, hi = lo + s_u;
            x.j0 = std::max(x.j0, lo);
            x.j1 = std::min(x.j1, hi);
            if (x.j0 >= x.j1) continue;
            x.g_base = x.s_base = x.p_base = int64_t(O) - int64_t(lo);
            x.shard = x.jump = x.p_jump = 0;
        } else {
            x.g_base = int64_t(U);
            x.s_base = int64_t(O);
            if (multi) {
                owner_map = true;
                x.shard = s_u;
                x.jump = p->S - s_u;
            }
            x.p_base = replicas ? int64_t(U) : int64_t(O);
            x.p_jump = replicas ? 0 : x.jump;
        }
        const bool vec_ok = strides_ok && mult8(x.g_base) && mult8(x.s_base) && mult8(x.p_base) &&
                            (!owner_map || ((x.shard & 7u) == 0 && (x.jump & 7u) == 0));
        st = L.run(x, owner_map, vec_ok);
        if (st != ZERO_OK) return st;
    }
    if (L.want_ws && first + count == p->n_buckets && count > 0) {
        k_finalize<<<1, kThreads, 0, L.stream>>>(a.ws_norm, a.ws_bad, grid, b->grad_norm_sq, b->overflow);
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
    if (!p) return set_error(ZERO_EINVAL, "zero_gather_layer: NULL plan");
    if (p->stage != 3) return set_error(ZERO_EINVAL, "zero_gather_layer: only stage 3 materialises layers");
    if (unit >= p->unit_len.size()) return set_error(ZERO_EINVAL, "zero_gather_layer: unit out of range");
    if (!owner_params || !full_layer) return set_error(ZERO_EINVAL, "zero_gather_layer: NULL buffer");
    if (!aligned16(owner_params) || !aligned16(full_layer))
        return set_error(ZERO_EINVAL, "zero_gather_layer: buffers must be 16-byte aligned");
    std::lock_guard<std::mutex> g(p->mu);
    if (p->live[unit])
        return set_error(ZERO_ESTATE, "zero_gather_layer: unit " + std::to_string(unit) + " is already live");
    if (p->n_live >= p->max_live)
        return set_error(ZERO_ESTATE, "zero_gather_layer: max_live units are live; release one first");
    cudaError_t pre = cudaPeekAtLastError();
    if (pre != cudaSuccess)
        return set_error(ZERO_ECUDA, std::string("pending CUDA error before zero_gather_layer: ") +
                                         cudaGetErrorString(pre));
    uint32_t grid = 0;
    zero_status_t st = device_grid(&grid);
    if (st != ZERO_OK) return st;
    const uint64_t s_u = p->unit_shard[unit], off = p->unit_offset[unit], len = p->unit_len[unit];
    const int vec_ok = ((p->S | off | s_u) & 7u) == 0;
    const uint32_t cpo = std::max<uint32_t>(1, grid / p->nd);
    const uint64_t blocks = uint64_t(cpo) * p->nd;
    if (blocks > 0x7fffffffull) return set_error(ZERO_EINVAL, "zero_gather_layer: nd too large for one launch");
    k_gather<<<uint32_t(blocks), kThreads, 0, static_cast<cudaStream_t>(stream_)>>>(
        static_cast<const uint16_t *>(owner_params), p->S, off, s_u, len, static_cast<uint16_t *>(full_layer),
        p->nd, cpo, vec_ok);
    st = check_launch("zero_gather_layer launch");
    if (st != ZERO_OK) return st;
    p->live[unit] = 1;
    p->n_live += 1;
    p->live_bytes += 2 * len;
    p->peak_live = std::max(p->peak_live, p->n_live);
    p->peak_live_bytes = std::max(p->peak_live_bytes, p->live_bytes);
    return ZERO_OK;
}

// Device-side definitions shared by the step kernels: the launch arguments
// of one bucket, the Adam constants, bf16 packing and the per-element update.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace zero_dev {

constexpr int kThreads = 256;
constexpr int kRB = 4;    // gradient rows in flight per thread
constexpr int kMinB = 2;  // CTAs per SM the vector kernel is sized for

struct AdamConsts {
    float grad_scale, beta1, beta2, eps, omb1, omb2, step, ibc2;
    float decay;  // 1 - lr * weight_decay (AdamW); 1 for Adam
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
    const AdamConsts *cdev;  // if set, the constants are read from device memory
    double *ws_norm;
    uint32_t *ws_bad;
    int ws_mode;  // 0: no norm; 1: add this launch's per-CTA partials to the slots
};

// The guarded step's decision, written by its finalize kernel: the clip
// coefficient (<= 1) and whether to leave the state as it is.
struct GuardWord {
    float coef;
    int32_t skip;
};

// Device pointers of the Nd ranks when the ranks are devices, passed by
// value (2 KB of kernel parameters at ZERO_MAX_PEERS = 128).
constexpr int kMaxPeers = 128;
struct PeerTable {
    const uint16_t *g[kMaxPeers];  // rank q's gradient, logical order
    uint16_t *p[kMaxPeers];        // parameter rows: replicas, or the owner's shard
};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4 x, float f[8]) {
    f[0] = bf16lo(x.x); f[1] = bf16hi(x.x);
    f[2] = bf16lo(x.y); f[3] = bf16hi(x.y);
    f[4] = bf16lo(x.z); f[5] = bf16hi(x.z);
    f[6] = bf16lo(x.w); f[7] = bf16hi(x.w);
}


__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ bool not_finite(float x) {
    return (__float_as_uint(x) & 0x7f800000u) == 0x7f800000u;
}

// Programmatic dependent launch.  A bucket kernel lets the next one in the
// stream launch as soon as it starts, so that the next bucket's CTAs take
// each SM as this one's drain from it; the only memory consecutive bucket
// kernels share is the norm slots, so each waits for its predecessor to
// complete before adding to them.  Every CTA waits before it exits, so a
// kernel never completes before its predecessor.  Both are no-ops without
// the launch attribute.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// The Adam constants of a launch: from device memory when the caller
// supplied them there (so that a captured graph can be replayed for a new t),
// else the launch arguments.
__device__ __forceinline__ AdamConsts consts_of(const StepArgs &a) {
    return a.cdev ? *a.cdev : a.c;
}

// Textbook Adam on one element with decoupled weight decay, every operation
// rounded to nearest; g = (g_sum * grad_scale) * coef, where coef is the
// global-norm clip factor of the guarded step (1 elsewhere; a multiplication
// by 1, like the decay 1 of plain Adam, is exact).
__device__ __forceinline__ void adam1c(float g_sum, float coef, const AdamConsts &c, float &w,
                                       float &m, float &v) {
    const float g = __fmul_rn(__fmul_rn(g_sum, c.grad_scale), coef);
    const float m_new = __fadd_rn(__fmul_rn(c.beta1, m), __fmul_rn(c.omb1, g));
    const float v_new = __fadd_rn(__fmul_rn(c.beta2, v), __fmul_rn(__fmul_rn(c.omb2, g), g));
    const float denom = __fadd_rn(__fmul_rn(__fsqrt_rn(v_new), c.ibc2), c.eps);
    const float delta = __fmul_rn(c.step, __fdiv_rn(m_new, denom));
    w = __fsub_rn(__fmul_rn(w, c.decay), delta);
    m = m_new;
    v = v_new;
}

__device__ __forceinline__ void adam1(float g_sum, const AdamConsts &c, float &w, float &m,
                                      float &v) {
    adam1c(g_sum, 1.0f, c, w, m, v);
}

// ---------------------------------------------------------------------------
// Two fp32 lanes in one 64-bit register, for sm_100's packed fp32 add (one
// instruction per pair; each lane rounded to nearest exactly as the scalar
// add).  Used for the rank-order sum only, a chain of adds of loaded values
// (add8 below, and the bulk-copy kernel's consumers).
// The multiplications and additions of the Adam update stay scalar
// (__fmul_rn / __fadd_rn, never contracted): measured on B200 against them,
// packed multiplies and adds each matched bit for bit alone, but a packed
// multiply feeding a packed add differed in 19 % of pairs, as if fused into
// one rounding -- and so did the same pair written as packed fused
// multiply-adds with a -0 or 1 operand, once the constants were run-time
// values.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// Two bf16 (one 32-bit word, low half first) as an fp32 pair: exact.
__device__ __forceinline__ uint64_t f2_bf16x2(uint32_t w) { return f2_pack(bf16lo(w), bf16hi(w)); }

// s[e] += bf16 e of x for 8 consecutive elements, in four packed pairs
// (each lane rounded as __fadd_rn): one row of the rank-order sum.
__device__ __forceinline__ void add8(float s[8], const uint4 x) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int h = 0; h < 4; ++h)
        f2_unpack(f2_add(f2_pack(s[2 * h], s[2 * h + 1]), f2_bf16x2(w[h])), s[2 * h], s[2 * h + 1]);
}

// Per-CTA partials of the gradient-norm / overflow reduction, added to slot
// blockIdx.x (the slots are zeroed at the start of each step).  Fixed order,
// so the reported norm is the same on every run of the same launch shapes.
__device__ __forceinline__ void block_partials(double acc, uint32_t bad, double *ws_norm, uint32_t *ws_bad) {
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
        ws_norm[blockIdx.x] += t;
        ws_bad[blockIdx.x] = min(ws_bad[blockIdx.x] + b, 0x7fffffffu);
    }
}

__device__ __forceinline__ void block_partials(double acc, uint32_t bad, const StepArgs &a) {
    block_partials(acc, bad, a.ws_norm, a.ws_bad);
}

// K3: fixed-order sum of the per-CTA partials of one step (one block).  Each
// translation unit that includes this header has its own copy (static).
static __global__ void __launch_bounds__(kThreads) k_finalize(const double *ws_norm, const uint32_t *ws_bad,
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

}  // namespace zero_dev

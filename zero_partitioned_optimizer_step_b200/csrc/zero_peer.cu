// sm_100a kernels of one rank's share of the ZeRO step when the ranks have
// their own buffers (one GPU each, or separate allocations), and the CUDA IPC
// helpers that map another process's buffers into this one.
//
// K5 k_step_peer / k_step_peer_scalar -- rank r's part of one bucket, fused:
//    reduce-scatter : for each element p that r owns,
//                     g_sum = sum over q = 0..Nd-1 of float(G_q[p]), G_q read
//                     straight from rank q's memory (peer loads over
//                     NVLink/NVSwitch when q is another GPU), added in rank
//                     order from rank 0's value, fp32 round-to-nearest;
//    owner Adam     : r's fp32 w, m, v, which are local;
//    all-gather     : bf16(w) stored straight into every rank's replica
//                     (peer stores), or into r's own shard at stage 3;
//    epilogue       : optional reduced gradient, norm/overflow partials.
//    Source: mind-map page "ZeRO 真正在做什么：长期分开存，计算时临时拼齐",
//    section "但 GPU 只存四分之一…" (each GPU hands the gradient of a shard to
//    the GPU responsible for it, which updates and keeps it; the shards are
//    then exchanged) and glossary entries "reduce-scatter" / "all-gather".
//    The arithmetic is K1's, element for element, so every rank's results are
//    bit-identical to the one-GPU step on the same inputs.
// K6 k_gather_peer -- stage-3 materialisation of one unit, each owner's slice
//    read from that owner's memory (glossary entry "临时物化").
//
// The collective is inside the kernel: there is no separate reduce-scatter
// or all-gather launch and no staging buffer.  Per owned element a rank
// reads 2*Nd bytes of gradients (2*(Nd-1) across NVLink) and writes 2*Nd
// bytes of replicas (2*(Nd-1) across NVLink); on a node of B200s the NVLink
// traffic, not HBM, bounds it.  Ranks never wait for one another inside a
// kernel (each element has one owner, so no two ranks touch the same bytes);
// the caller orders whole steps across ranks on the host or with a stream
// collective.  Each CTA ends with a system-scope fence after a CTA barrier,
// so its peer stores are performed before the kernel counts as complete.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <unistd.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "zero_device.cuh"
#include "zero_host.cuh"
#include "zero_internal.h"
#include "zero_ring.cuh"
#include "zero_tma.cuh"
#include "zero_trace.h"

using zero_detail::set_error;
using zero_host::aligned16;
using zero_host::check_launch;
using zero_host::mult8;

namespace {

using namespace zero_dev;

constexpr int kPeerMinB = 2;  // CTAs per SM the vector kernel is sized for
constexpr int kPeerRB = 8;    // gradient rows in flight per thread

static_assert(kMaxPeers == ZERO_MAX_PEERS, "one peer table size");

// One launch: the logical range [p0, p1) of one unit that rank r owns.
// State index = p + s_shift; parameter index = p + q_shift (0 for replicas,
// s_shift for r's own stage-3 shard).
struct PeerArgs {
    uint64_t p0, p1;
    int64_t s_shift, q_shift;
    float *w, *m, *v, *red;
    uint32_t nd, n_prow;
    AdamConsts c;
    const AdamConsts *cdev;
    double *ws_norm;
    uint32_t *ws_bad;
    int ws_mode;
};

__device__ __forceinline__ AdamConsts peer_consts(const PeerArgs &a) { return a.cdev ? *a.cdev : a.c; }

// The CTA's stores (to peers included) are ordered before a system-scope
// fence: the barrier makes every thread's stores precede thread 0's fence,
// which is cumulative.  One fence per CTA instead of one per thread.
__device__ __forceinline__ void cta_release_system() {
    __syncthreads();
    if (threadIdx.x == 0) __threadfence_system();
}

// K5, vector path: 8 elements per thread and iteration, kPeerRB gradient rows
// loaded together (peer loads have a long latency) before their in-order
// adds.  Preconditions (host): p0, p1, s_shift, q_shift multiples of 8 and
// every pointer 16-byte aligned.
__global__ void __launch_bounds__(kThreads, kPeerMinB) k_step_peer(const PeerArgs a, const PeerTable T) {
    pdl_launch_dependents();
    __shared__ const uint16_t *sg[kMaxPeers];
    __shared__ uint16_t *sp[kMaxPeers];
    for (uint32_t i = threadIdx.x; i < a.nd; i += kThreads) sg[i] = T.g[i];
    for (uint32_t i = threadIdx.x; i < a.n_prow; i += kThreads) sp[i] = T.p[i];
    __syncthreads();
    const AdamConsts C = peer_consts(a);
    const uint64_t nvec = (a.p1 - a.p0) >> 3;
    const uint64_t stride = uint64_t(gridDim.x) * kThreads;
    double acc = 0.0;
    uint32_t bad = 0;
    for (uint64_t vi = uint64_t(blockIdx.x) * kThreads + threadIdx.x; vi < nvec; vi += stride) {
        const uint64_t p = a.p0 + (vi << 3);
        const uint64_t si = uint64_t(int64_t(p) + a.s_shift);
        const uint64_t pi = uint64_t(int64_t(p) + a.q_shift);

        // reduce-scatter: rank-order sum, kPeerRB rows in flight at a time
        float s[8];
        for (uint32_t r0 = 0; r0 < a.nd; r0 += kPeerRB) {
            uint4 x[kPeerRB];
#pragma unroll
            for (int k = 0; k < kPeerRB; ++k)
                if (r0 + k < a.nd) x[k] = __ldcs(reinterpret_cast<const uint4 *>(sg[r0 + k] + p));
#pragma unroll
            for (int k = 0; k < kPeerRB; ++k) {
                if (r0 + k >= a.nd) break;
                if (r0 + k == 0) unpack8(x[0], s);
                else add8(s, x[k]);
            }
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

        // all-gather: the same 16 bytes of bf16 into every parameter row
        uint4 pk;
        pk.x = pack_bf16x2(wv[0], wv[1]);
        pk.y = pack_bf16x2(wv[2], wv[3]);
        pk.z = pack_bf16x2(wv[4], wv[5]);
        pk.w = pack_bf16x2(wv[6], wv[7]);
        for (uint32_t q = 0; q < a.n_prow; ++q) __stcs(reinterpret_cast<uint4 *>(sp[q] + pi), pk);
    }
    cta_release_system();
    pdl_wait();  // predecessor done: its norm slots are final
    if (a.ws_mode) block_partials(acc, bad, a.ws_norm, a.ws_bad);
}

// K5, scalar path: any alignment (unit heads and tails, A not a multiple of 8).
__global__ void __launch_bounds__(kThreads) k_step_peer_scalar(const PeerArgs a, const PeerTable T) {
    __shared__ const uint16_t *sg[kMaxPeers];
    __shared__ uint16_t *sp[kMaxPeers];
    for (uint32_t i = threadIdx.x; i < a.nd; i += kThreads) sg[i] = T.g[i];
    for (uint32_t i = threadIdx.x; i < a.n_prow; i += kThreads) sp[i] = T.p[i];
    __syncthreads();
    const AdamConsts C = peer_consts(a);
    const uint64_t n = a.p1 - a.p0;
    const uint64_t stride = uint64_t(gridDim.x) * kThreads;
    double acc = 0.0;
    uint32_t bad = 0;
    for (uint64_t i = uint64_t(blockIdx.x) * kThreads + threadIdx.x; i < n; i += stride) {
        const uint64_t p = a.p0 + i;
        const uint64_t si = uint64_t(int64_t(p) + a.s_shift);
        const uint64_t pi = uint64_t(int64_t(p) + a.q_shift);
        float s = __uint_as_float(uint32_t(sg[0][p]) << 16);
        for (uint32_t q = 1; q < a.nd; ++q) s = __fadd_rn(s, __uint_as_float(uint32_t(sg[q][p]) << 16));
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
        for (uint32_t q = 0; q < a.n_prow; ++q) sp[q][pi] = bits;
    }
    cta_release_system();
    if (a.ws_mode) block_partials(acc, bad, a.ws_norm, a.ws_bad);
}

// K6: full_layer[o*s_u + i] = T.g[o][off_u + i] for the first len_u elements;
// `cpo` CTAs per owner, owners in rank order; four 16-byte loads in flight
// per thread.
__global__ void __launch_bounds__(kThreads) k_gather_peer(const PeerTable T, uint64_t off_u, uint64_t s_u,
                                                         uint64_t len, uint16_t *dst, uint32_t nd, uint32_t cpo,
                                                         int vec_ok) {
    const uint32_t o = blockIdx.x / cpo, c = blockIdx.x % cpo;
    if (o >= nd) return;
    const uint64_t begin = uint64_t(o) * s_u;
    if (begin >= len) return;
    const uint64_t n = min(s_u, len - begin);
    const uint16_t *s = T.g[o] + off_u;
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

// Launch shapes on the current device, computed once per device: the
// persistent grid of the peer step kernels (SM count x resident CTAs, capped
// at the norm workspace's slot count) and the SM count.
struct PeerShapes {
    uint32_t grid = 0, sms = 0;
    uint32_t tma_smem = 0;  // dynamic shared memory the bulk-copy kernel may use
};

// The bulk-copy kernel with the rows reached through the peer table.
using PeerTmaKernel = void (*)(const zero_dev::StepArgs, const zero_tma::Ring, const zero_dev::PeerTable);

PeerTmaKernel peer_tma_kernel(uint32_t groups, uint32_t vw) {
    using namespace zero_tma;
    if (groups == 2)
        return vw == 2 ? k_step_tma<false, 2, 2, kPeerRows>
                       : (vw == 4 ? k_step_tma<false, 2, 4, kPeerRows> : k_step_tma<false, 2, 8, kPeerRows>);
    return vw == 2 ? k_step_tma<false, 1, 2, kPeerRows>
                   : (vw == 4 ? k_step_tma<false, 1, 4, kPeerRows> : k_step_tma<false, 1, 8, kPeerRows>);
}

zero_status_t peer_shapes(PeerShapes *out) {
    static std::mutex mu;
    static std::map<int, PeerShapes> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_error(ZERO_ECUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    std::lock_guard<std::mutex> g(mu);
    auto it = cache.find(dev);
    if (it != cache.end()) {
        *out = it->second;
        return ZERO_OK;
    }
    int sms = 0, occ = 0, optin = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_step_peer, kThreads, 0);
    cudaFuncAttributes fa{};
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, peer_tma_kernel(2, 2));
    PeerShapes s;
    const int64_t budget = int64_t(optin) - int64_t(fa.sharedSizeBytes) - 256;
    s.tma_smem = budget > 0 ? uint32_t(budget) : 0;
    if (s.tma_smem > 0)
        for (uint32_t g : {1u, 2u})
            for (uint32_t vw : {2u, 4u, 8u})
                if (e == cudaSuccess)
                    e = cudaFuncSetAttribute(reinterpret_cast<const void *>(peer_tma_kernel(g, vw)),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(s.tma_smem));
    if (e != cudaSuccess) return set_error(ZERO_ECUDA, std::string("device query: ") + cudaGetErrorString(e));
    s.sms = uint32_t(std::max(1, sms));
    s.grid = std::min(uint32_t(std::max(1, sms) * std::max(1, occ)), zero_detail::kMaxSlots);
    cache[dev] = s;
    *out = s;
    return ZERO_OK;
}

// Launch with or without programmatic dependent launch on the stream.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), uint32_t grid, uint32_t block, size_t smem,
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

zero_status_t validate_peers(const zero_plan_t *p, const zero_peer_bufs_t *b, const zero_adam_t *adam,
                             uint64_t t) {
    if (!p || !b || !adam) return set_error(ZERO_EINVAL, "zero_step_peers: NULL argument");
    if (t == 0) return set_error(ZERO_EINVAL, "zero_step_peers: t must be >= 1");
    if (!(std::isfinite(adam->lr) && std::isfinite(adam->eps) && std::isfinite(adam->grad_scale) &&
          std::isfinite(adam->weight_decay)))
        return set_error(ZERO_EINVAL, "zero_step_peers: lr, eps, grad_scale and weight_decay must be finite");
    if (!(adam->beta1 >= 0.0 && adam->beta1 < 1.0 && adam->beta2 >= 0.0 && adam->beta2 < 1.0))
        return set_error(ZERO_EINVAL, "zero_step_peers: beta1 and beta2 must be in [0, 1)");
    if (p->stage == 0)
        return set_error(ZERO_EINVAL, "zero_step_peers: stage 0 keeps the full state on every rank; "
                                      "use a plan of stage 1, 2 or 3");
    if (p->nd > ZERO_MAX_PEERS) return set_error(ZERO_EINVAL, "zero_step_peers: nd exceeds ZERO_MAX_PEERS");
    if (b->rank >= p->nd) return set_error(ZERO_EINVAL, "zero_step_peers: rank must be in [0, nd)");
    if (!b->grads || !b->params) return set_error(ZERO_EINVAL, "zero_step_peers: NULL grads or params array");
    for (uint32_t q = 0; q < p->nd; ++q)
        if (!b->grads[q] || !aligned16(b->grads[q]))
            return set_error(ZERO_EINVAL, "zero_step_peers: grads[" + std::to_string(q) +
                                              "] is NULL or not 16-byte aligned");
    const bool replicas = p->stage <= 2;
    for (uint32_t q = 0; q < p->nd; ++q) {
        if (!replicas && q != b->rank) continue;
        if (!b->params[q] || !aligned16(b->params[q]))
            return set_error(ZERO_EINVAL, "zero_step_peers: params[" + std::to_string(q) +
                                              "] is NULL or not 16-byte aligned");
    }
    const void *req[] = {b->master, b->exp_avg, b->exp_avg_sq};
    for (const void *q : req)
        if (!q || !aligned16(q))
            return set_error(ZERO_EINVAL, "zero_step_peers: master, exp_avg and exp_avg_sq are required, "
                                          "16-byte aligned");
    const void *opt[] = {b->reduced_grad, b->grad_norm_sq, b->overflow, b->workspace, b->adam_consts};
    for (const void *q : opt)
        if (q && !aligned16(q)) return set_error(ZERO_EINVAL, "zero_step_peers: device pointers must be 16-byte aligned");
    if ((b->grad_norm_sq || b->overflow) &&
        (!b->workspace || b->workspace_bytes < zero_detail::kWorkspaceBytes))
        return set_error(ZERO_EINVAL, "zero_step_peers: norm/overflow output needs a workspace of "
                                      "ZERO_Q_WORKSPACE_BYTES");
    return ZERO_OK;
}

// Rank r's part of bucket bk: the logical range [p0, p1) and its 8-aligned
// body [vlo, vhi), which runs in a vector kernel when vec_ok.
struct PeerPart {
    uint64_t p0, p1, vlo, vhi;
    int64_t s_shift;  // state index = logical index + s_shift
    bool vec_ok;
};

PeerPart peer_part(const zero_plan_t &p, uint32_t r, uint64_t bk) {
    const zero_detail::BucketRange br = zero_detail::bucket_range(p, bk);
    const uint32_t u = br.unit;
    const uint64_t s_u = p.unit_shard[u];
    const uint64_t lo = p.unit_base[u] + uint64_t(r) * s_u;  // r's slice of unit u, logical
    PeerPart q{};
    q.p0 = std::max(br.begin, lo);
    q.p1 = std::min(br.end, lo + s_u);
    q.s_shift = int64_t(p.unit_offset[u]) - int64_t(lo);
    q.vlo = (q.p0 + 7) & ~uint64_t(7);
    q.vhi = q.p1 & ~uint64_t(7);
    q.vec_ok = q.p0 < q.p1 && mult8(q.s_shift) && q.vlo < q.vhi;
    return q;
}

// The kernel of rank r's call over buckets [first, first + count) for its
// aligned bodies: ZERO_KERNEL_BULK_COPY, ZERO_KERNEL_VECTOR_LOAD (K5), or
// ZERO_KERNEL_NONE when the call has none.  `ring` receives the bulk-copy
// ring (err: the device error word its waits report to; may be NULL for a
// query).
//
// Where the parameters are written once (stage 3), the bulk-copy kernel
// (rows pulled by 1-D bulk copies through the peer table, no multicast).
// With replicas to write, per call: the bulk-copy kernel when the call's
// aligned bodies average at least ring_min columns (32 x 2048 per SM, the
// size from which a launch keeps the full ring), else K5.  One kernel per
// call: choosing per launch by size, so that a call's chain mixed the two,
// ran below both kernels alone.  Measured with the ranks as allocations on
// one GPU, both with programmatic dependent launch, against K5 for every
// call (fraction of 6650 GB/s copy bandwidth):
//   stage 3 (1.3B, Nd = 16): 0.945 against 0.847;
//   Psi = 5e8, Nd = 8, one 62.5M-column launch a call: 0.950 against 0.892;
//   Psi = 5e8, Nd = 8, 64 MB buckets: 0.927 against 0.918;
//   Psi = 5e8, Nd = 32, 64 MB buckets (18 calls of 32 here): 0.885
//   against 0.855;
//   Psi = 5e8, Nd = 16, 64 MB buckets: 0.919 against 0.900;
//   GPT-2-small, Nd = 8, 25M-element buckets (4 calls of 8): 0.825
//   against 0.829 (a loss).
// The NVLink rate of either is not measured.  ZERO_STEP_KERNEL=tma|ldg
// forces either for every call; ZERO_PEER_RING_MIN=<columns> moves the
// threshold.  Unaligned edges always run in K5's scalar twin.
uint32_t peer_call_kernel(const zero_plan_t &p, uint32_t r, uint64_t first, uint64_t count,
                          const PeerShapes &shapes, int *err, zero_tma::Ring *ring) {
    const bool replicas = p.stage <= 2;
    const int choice = zero_ring::kernel_choice();
    const bool ring_ok = choice != 1 && zero_ring::choose_ring(p.nd, !replicas, shapes.tma_smem, err, ring,
                                                               zero_tma::kConsumerWarps);
    ring->bulk_p = 0;  // the peer rows are stored through their pointers
    uint64_t ring_min = replicas ? 32ull * 2048ull * shapes.sms : 0;
    if (const char *e = std::getenv("ZERO_PEER_RING_MIN")) {
        char *end = nullptr;
        const unsigned long long v = std::strtoull(e, &end, 10);
        if (end != e) ring_min = v;
    }
    if (choice == 2) ring_min = 0;
    uint64_t vec_cols = 0, vec_n = 0;
    for (uint64_t bk = first; bk < first + count; ++bk) {
        const PeerPart q = peer_part(p, r, bk);
        if (q.vec_ok) vec_cols += q.vhi - q.vlo, ++vec_n;
    }
    if (vec_n == 0) return ZERO_KERNEL_NONE;
    return ring_ok && vec_cols / vec_n >= ring_min ? ZERO_KERNEL_BULK_COPY : ZERO_KERNEL_VECTOR_LOAD;
}

}  // namespace

ZERO_API zero_status_t zero_step_peers(const zero_plan_t *p, const zero_peer_bufs_t *b, const zero_adam_t *adam,
                                       uint64_t t, uint64_t first, uint64_t count, void *stream_) {
    zero_detail::clear_error();
    const zero_trace::Range call("zero_step_peers t=%llu buckets [%llu, %llu)", (unsigned long long)t,
                                 (unsigned long long)first, (unsigned long long)(first + count));
    zero_status_t st = validate_peers(p, b, adam, t);
    if (st != ZERO_OK) return st;
    if (first > p->n_buckets || count > p->n_buckets - first)
        return set_error(ZERO_EINVAL, "zero_step_peers: bucket range outside the plan");
    cudaError_t pre = cudaPeekAtLastError();
    if (pre != cudaSuccess)
        return set_error(ZERO_ECUDA, std::string("pending CUDA error before zero_step_peers: ") +
                                         cudaGetErrorString(pre));
    PeerShapes shapes;
    st = peer_shapes(&shapes);
    if (st != ZERO_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const bool replicas = p->stage <= 2;
    const uint32_t r = b->rank;

    PeerTable tab;  // copied into the launch's parameters
    std::memset(&tab, 0, sizeof tab);
    for (uint32_t q = 0; q < p->nd; ++q) tab.g[q] = static_cast<const uint16_t *>(b->grads[q]);
    if (replicas)
        for (uint32_t q = 0; q < p->nd; ++q) tab.p[q] = static_cast<uint16_t *>(b->params[q]);
    else
        tab.p[0] = static_cast<uint16_t *>(b->params[r]);

    PeerArgs a{};
    a.w = b->master;
    a.m = b->exp_avg;
    a.v = b->exp_avg_sq;
    a.red = b->reduced_grad;
    a.nd = p->nd;
    a.n_prow = replicas ? p->nd : 1;
    float c9[9];
    st = zero_adam_consts(adam, t, c9);
    if (st != ZERO_OK) return st;
    static_assert(sizeof(AdamConsts) == sizeof c9, "nine packed fp32 constants");
    std::memcpy(&a.c, c9, sizeof c9);
    a.cdev = static_cast<const AdamConsts *>(b->adam_consts);
    const bool want_ws = b->grad_norm_sq || b->overflow;
    auto *ws = static_cast<unsigned char *>(b->workspace);
    a.ws_norm = reinterpret_cast<double *>(ws);
    a.ws_bad = reinterpret_cast<uint32_t *>(ws + 8ull * zero_detail::kMaxSlots);
    a.ws_mode = want_ws ? 1 : 0;
    if (want_ws && first == 0) {
        cudaError_t e = cudaMemsetAsync(b->workspace, 0, zero_detail::kWorkspaceBytes, stream);
        if (e != cudaSuccess)
            return set_error(ZERO_ECUDA, std::string("zero_step_peers workspace reset: ") + cudaGetErrorString(e));
    }

    zero_tma::Ring ring{};
    int *err = nullptr;
    st = zero_detail::wait_error_word(&err);
    if (st != ZERO_OK) return st;
    const bool use_ring = peer_call_kernel(*p, r, first, count, shapes, err, &ring) == ZERO_KERNEL_BULK_COPY;
    // Vector launches after the first of the call overlap their predecessor
    // (programmatic dependent launch): consecutive launches of one call share
    // only the norm slots, which every kernel adds to after its predecessor
    // has completed.  ZERO_PDL=0 turns it off.
    const char *pdl_env = std::getenv("ZERO_PDL");
    const bool pdl = !(pdl_env && pdl_env[0] == '0');
    uint32_t launches = 0;
    auto launch = [&](uint64_t p0, uint64_t p1, bool vec) -> zero_status_t {
        if (p0 >= p1) return ZERO_OK;
        PeerArgs x = a;
        x.p0 = p0;
        x.p1 = p1;
        const bool dep = pdl && launches++ > 0;
        if (vec && use_ring) {
            StepArgs sa{};
            sa.w = x.w;
            sa.m = x.m;
            sa.v = x.v;
            sa.red = x.red;
            sa.n_prow = x.n_prow;
            sa.nd = x.nd;
            sa.g_base = 0;  // the launch's element index is the logical index
            sa.s_base = x.s_shift;
            sa.p_base = x.q_shift;
            sa.j0 = p0;
            sa.j1 = p1;
            sa.c = x.c;
            sa.cdev = x.cdev;
            sa.ws_norm = x.ws_norm;
            sa.ws_bad = x.ws_bad;
            sa.ws_mode = x.ws_mode;
            const zero_tma::Ring rg = zero_ring::ring_for_launch(ring, p1 - p0, x.nd, shapes.sms, shapes.tma_smem);
            const uint64_t tiles = (p1 - p0 + rg.tile - 1) / rg.tile;
            const uint32_t grid = uint32_t(std::min<uint64_t>(tiles, shapes.sms));
            launch_pdl(peer_tma_kernel(rg.groups, rg.vw), grid, zero_tma::kThreads,
                       zero_ring::ring_smem_bytes(rg), stream, dep, sa, rg, tab);
        } else if (vec) {
            launch_pdl(k_step_peer, shapes.grid, kThreads, 0, stream, dep, x, tab);
        } else {
            k_step_peer_scalar<<<shapes.grid, kThreads, 0, stream>>>(x, tab);
        }
        return check_launch("zero_step_peers kernel launch");
    };
    for (uint64_t bk = first; bk < first + count; ++bk) {
        const PeerPart q = peer_part(*p, r, bk);
        const uint64_t p0 = q.p0, p1 = q.p1, vlo = q.vlo, vhi = q.vhi;
        if (p0 >= p1) continue;
        a.s_shift = q.s_shift;
        a.q_shift = replicas ? 0 : a.s_shift;
        const bool vec_ok = q.vec_ok;
        const zero_trace::Range rb("bucket %llu", (unsigned long long)bk);
        if (!vec_ok) {
            st = launch(p0, p1, false);
        } else {
            st = launch(p0, vlo, false);
            if (st == ZERO_OK) st = launch(vlo, vhi, true);
            if (st == ZERO_OK) st = launch(vhi, p1, false);
        }
        if (st != ZERO_OK) return st;
    }
    if (want_ws && first + count == p->n_buckets && count > 0) {
        const zero_trace::Range rf("norm finalize");
        k_finalize<<<1, kThreads, 0, stream>>>(a.ws_norm, a.ws_bad, zero_detail::kMaxSlots, b->grad_norm_sq,
                                               b->overflow);
        st = check_launch("zero_step_peers finalize launch");
        if (st != ZERO_OK) return st;
    }
    return ZERO_OK;
}

ZERO_API zero_status_t zero_step_peers_kernel(const zero_plan_t *p, uint32_t rank, uint64_t first,
                                              uint64_t count, uint32_t *kind) {
    zero_detail::clear_error();
    if (!p || !kind) return set_error(ZERO_EINVAL, "zero_step_peers_kernel: NULL argument");
    if (p->stage == 0) return set_error(ZERO_EINVAL, "zero_step_peers_kernel: stage 0 has no owners");
    if (p->nd > ZERO_MAX_PEERS) return set_error(ZERO_EINVAL, "zero_step_peers_kernel: nd exceeds ZERO_MAX_PEERS");
    if (rank >= p->nd) return set_error(ZERO_EINVAL, "zero_step_peers_kernel: rank out of range");
    if (first > p->n_buckets || count > p->n_buckets - first)
        return set_error(ZERO_EINVAL, "zero_step_peers_kernel: bucket range outside the plan");
    PeerShapes shapes;
    const zero_status_t st = peer_shapes(&shapes);
    if (st != ZERO_OK) return st;
    zero_tma::Ring ring{};
    *kind = peer_call_kernel(*p, rank, first, count, shapes, nullptr, &ring);
    return ZERO_OK;
}

ZERO_API zero_status_t zero_gather_layer_peers(zero_plan_t *p, uint32_t unit, const void *const *owner_params,
                                               void *full_layer, void *stream_) {
    zero_detail::clear_error();
    const zero_trace::Range call("zero_gather_layer_peers unit %u", unit);
    if (!p) return set_error(ZERO_EINVAL, "zero_gather_layer_peers: NULL plan");
    if (p->stage != 3) return set_error(ZERO_EINVAL, "zero_gather_layer_peers: only stage 3 materialises layers");
    if (p->nd > ZERO_MAX_PEERS) return set_error(ZERO_EINVAL, "zero_gather_layer_peers: nd exceeds ZERO_MAX_PEERS");
    if (unit >= p->unit_len.size()) return set_error(ZERO_EINVAL, "zero_gather_layer_peers: unit out of range");
    if (!owner_params || !full_layer || !aligned16(full_layer))
        return set_error(ZERO_EINVAL, "zero_gather_layer_peers: NULL or misaligned buffer");
    PeerTable tab;
    std::memset(&tab, 0, sizeof tab);
    for (uint32_t q = 0; q < p->nd; ++q) {
        if (!owner_params[q] || !aligned16(owner_params[q]))
            return set_error(ZERO_EINVAL, "zero_gather_layer_peers: owner_params[" + std::to_string(q) +
                                              "] is NULL or not 16-byte aligned");
        tab.g[q] = static_cast<const uint16_t *>(owner_params[q]);
    }
    std::lock_guard<std::mutex> g(p->mu);
    zero_status_t st = zero_detail::live_check(*p, unit, "zero_gather_layer_peers");
    if (st != ZERO_OK) return st;
    cudaError_t pre = cudaPeekAtLastError();
    if (pre != cudaSuccess)
        return set_error(ZERO_ECUDA, std::string("pending CUDA error before zero_gather_layer_peers: ") +
                                         cudaGetErrorString(pre));
    PeerShapes shapes;
    st = peer_shapes(&shapes);
    if (st != ZERO_OK) return st;
    const uint64_t s_u = p->unit_shard[unit], off = p->unit_offset[unit], len = p->unit_len[unit];
    const int vec_ok = ((off | s_u) & 7u) == 0;
    const uint32_t cpo = std::max<uint32_t>(1, (shapes.sms * 8) / p->nd);  // 8 CTAs/SM
    k_gather_peer<<<cpo * p->nd, kThreads, 0, static_cast<cudaStream_t>(stream_)>>>(
        tab, off, s_u, len, static_cast<uint16_t *>(full_layer), p->nd, cpo, vec_ok);
    st = check_launch("zero_gather_layer_peers launch");
    if (st != ZERO_OK) return st;
    zero_detail::live_mark(*p, unit);
    return ZERO_OK;
}

// ------------------------------------------------------------------- IPC
namespace {

// cuMemGetAddressRange from the driver, found through the runtime (no link
// against the driver library): the allocation that contains a pointer.
using GetRangeFn = CUresult (*)(CUdeviceptr *, size_t *, CUdeviceptr);

GetRangeFn get_range_fn() {
    static GetRangeFn fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return GetRangeFn(nullptr);
        return reinterpret_cast<GetRangeFn>(f);
    }();
    return fn;
}

// Mappings opened in this process: one per exported allocation
// (exporter pid, exporter address), reference-counted over the buffers
// opened in it; and, per address handed out, the allocation it belongs to.
struct Mapping {
    void *base = nullptr;  // local address of the allocation (nullptr: same process, not mapped)
    uint64_t refs = 0;
};
std::mutex g_ipc_mu;
std::map<std::pair<int32_t, uint64_t>, Mapping> g_maps;
std::multimap<uintptr_t, std::pair<int32_t, uint64_t>> g_opened;

}  // namespace

ZERO_API zero_status_t zero_ipc_export(const void *ptr, zero_ipc_handle_t *out) {
    zero_detail::clear_error();
    if (!ptr || !out) return set_error(ZERO_EINVAL, "zero_ipc_export: NULL argument");
    cudaPointerAttributes attr{};
    cudaError_t e = cudaPointerGetAttributes(&attr, ptr);
    if (e != cudaSuccess || attr.type != cudaMemoryTypeDevice) {
        cudaGetLastError();
        return set_error(ZERO_EINVAL, "zero_ipc_export: not a device-memory pointer");
    }
    GetRangeFn range = get_range_fn();
    if (!range) return set_error(ZERO_ECUDA, "zero_ipc_export: cuMemGetAddressRange is not available");
    int prev = 0;
    e = cudaGetDevice(&prev);
    if (e == cudaSuccess && prev != attr.device) e = cudaSetDevice(attr.device);
    if (e != cudaSuccess) return set_error(ZERO_ECUDA, std::string("zero_ipc_export: ") + cudaGetErrorString(e));
    CUdeviceptr base = 0;
    size_t bytes = 0;
    const CUresult cr = range(&base, &bytes, CUdeviceptr(reinterpret_cast<uintptr_t>(ptr)));
    cudaIpcMemHandle_t h;
    if (cr == CUDA_SUCCESS) e = cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(uintptr_t(base)));
    if (prev != attr.device) cudaSetDevice(prev);
    if (cr != CUDA_SUCCESS)
        return set_error(ZERO_ECUDA, "zero_ipc_export: cuMemGetAddressRange failed (" + std::to_string(int(cr)) + ")");
    if (e != cudaSuccess)
        return set_error(ZERO_ECUDA, std::string("zero_ipc_export: cudaIpcGetMemHandle: ") + cudaGetErrorString(e) +
                                         " (the buffer must come from cudaMalloc)");
    std::memset(out, 0, sizeof *out);
    static_assert(sizeof h == sizeof out->handle, "cudaIpcMemHandle_t is 64 bytes");
    std::memcpy(out->handle, &h, sizeof h);
    out->offset = uint64_t(reinterpret_cast<uintptr_t>(ptr) - uintptr_t(base));
    out->alloc_bytes = uint64_t(bytes);
    out->exporter_va = uint64_t(base);
    out->device = attr.device;
    out->exporter_pid = int32_t(getpid());
    return ZERO_OK;
}

ZERO_API zero_status_t zero_ipc_open(const zero_ipc_handle_t *h, void **ptr) {
    zero_detail::clear_error();
    if (!h || !ptr) return set_error(ZERO_EINVAL, "zero_ipc_open: NULL argument");
    if (h->offset >= h->alloc_bytes) return set_error(ZERO_EINVAL, "zero_ipc_open: offset outside the allocation");
    const auto key = std::make_pair(h->exporter_pid, h->exporter_va);
    std::lock_guard<std::mutex> g(g_ipc_mu);
    auto it = g_maps.find(key);
    if (it == g_maps.end()) {
        Mapping m;
        if (h->exporter_pid != int32_t(getpid())) {
            cudaIpcMemHandle_t ch;
            std::memcpy(&ch, h->handle, sizeof ch);
            cudaError_t e = cudaIpcOpenMemHandle(&m.base, ch, cudaIpcMemLazyEnablePeerAccess);
            if (e != cudaSuccess) {
                cudaGetLastError();
                return set_error(ZERO_ECUDA, std::string("zero_ipc_open: cudaIpcOpenMemHandle: ") +
                                                 cudaGetErrorString(e));
            }
        }
        it = g_maps.emplace(key, m).first;
    }
    const uintptr_t base = it->second.base ? reinterpret_cast<uintptr_t>(it->second.base) : uintptr_t(h->exporter_va);
    const uintptr_t addr = base + uintptr_t(h->offset);
    it->second.refs += 1;
    g_opened.emplace(addr, key);
    *ptr = reinterpret_cast<void *>(addr);
    return ZERO_OK;
}

ZERO_API zero_status_t zero_ipc_close(void *ptr) {
    zero_detail::clear_error();
    std::lock_guard<std::mutex> g(g_ipc_mu);
    auto o = g_opened.find(reinterpret_cast<uintptr_t>(ptr));
    if (!ptr || o == g_opened.end())
        return set_error(ZERO_EINVAL, "zero_ipc_close: the pointer was not returned by zero_ipc_open");
    const auto key = o->second;
    g_opened.erase(o);
    auto it = g_maps.find(key);
    if (it == g_maps.end()) return ZERO_OK;
    if (--it->second.refs > 0) return ZERO_OK;
    void *base = it->second.base;
    g_maps.erase(it);
    if (base) {
        cudaError_t e = cudaIpcCloseMemHandle(base);
        if (e != cudaSuccess)
            return set_error(ZERO_ECUDA, std::string("zero_ipc_close: cudaIpcCloseMemHandle: ") +
                                             cudaGetErrorString(e));
    }
    return ZERO_OK;
}

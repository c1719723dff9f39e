/*
 * zero.h -- C ABI of libzero.so, the B200 (sm_100a) ZeRO partitioned
 * mixed-precision Adam step.
 *
 * What the library computes.  Nd data-parallel ranks are simulated as slices
 * of one GPU's memory.  One step, per bucket of the flat parameter vector:
 *   1. reduce-scatter (ZeRO "Pg"): for every padded element, the fp32 sum of
 *      the Nd ranks' bf16 gradients, added in rank order 0, 1, ..., Nd-1
 *      starting from rank 0's value; only the owner of the element keeps it;
 *   2. owner Adam (ZeRO "Pos"): the owner updates its fp32 master weight and
 *      its fp32 first and second moments (K = 12 bytes of state per element);
 *   3. all-gather: the new bf16 parameter is written to every rank's full
 *      replica (stages 0-2), or to the owner's shard only (stage 3), from
 *      where zero_gather_layer() materialises one layer at a time.
 * All of it runs in hand-written CUDA kernels; there is no CPU path.
 * zero_step_peers() runs one rank's share of the same step when the ranks
 * have their own buffers (one GPU per rank; see "Ranks as devices" below).
 *
 * Sources (three web pages about ZeRO, arXiv 1910.02054):
 *  [MM] mind-map page "ZeRO 真正在做什么：长期分开存，计算时临时拼齐"
 *       (paperbridge.wiki): the four-GPU A/B/C/D example; the loop "store
 *       apart -> gather the current layer -> compute -> split again"; the
 *       stage list; the 7.5B / Nd=64 memory estimate; the 2 Psi / 3 Psi
 *       communication volumes; the glossary (all-gather, reduce-scatter,
 *       temporary materialisation).
 *  [CP] concept page "ZeRO" (papers.lqhl.me): "为什么需要它" (mixed-precision
 *       Adam state), table "三个阶段" (what each stage shards), "关键设计取舍"
 *       item 1 (bucket size versus launch latency), the remark that ZeRO-3
 *       still materialises layers and that unreleased layers make peaks.
 *  [GG] gptget.net summary page of arXiv 1910.02054: stages Pos, Pg, Pp.
 *
 * Layouts (element counts; A = align_elems; u = unit, r = rank):
 *   P_u = ceil(len_u / (Nd*A)) * Nd*A    padded unit length
 *   s_u = P_u / Nd                       elements of unit u each rank owns
 *   U_u = sum_{u'<u} P_u'                unit u's start in the logical vector
 *   O_u = sum_{u'<u} s_u'                unit u's start inside a rank's block
 *   psi_pad = sum P_u,  S = sum s_u      (one unit: S = psi_pad / Nd)
 *   logical order:  unit after unit, each padded with zeros.
 *   owner storage:  rank-major [Nd][S]; rank o's slice of unit u (logical
 *                   U_u + o*s_u + i, 0 <= i < s_u) sits at o*S + O_u + i.
 *   With one unit the two orders coincide.
 *
 * Ownership.  The caller allocates, owns and frees every device buffer and
 * the stream; the library keeps only the host-side plan (maps, bucket table,
 * live-layer bookkeeping).  Device scratch, when needed, is the caller's
 * `workspace` (size: zero_plan_query(ZERO_Q_WORKSPACE_BYTES)).
 *
 * Errors.  No call aborts or prints.  Every call returns a status; the text of
 * the last failure on the calling thread is zero_last_error().  Invalid
 * arguments (NULL or non-16-byte-aligned device pointers, bad descriptor,
 * t = 0, index out of range) give ZERO_EINVAL before anything is launched.
 * Liveness violations give ZERO_ESTATE.  A failed launch gives ZERO_ECUDA;
 * faults inside a kernel are asynchronous and surface on a later CUDA call.
 *
 * Streams.  `stream` is a cudaStream_t passed as void*; NULL is the legacy
 * default stream.  Launches are asynchronous; nothing synchronises except
 * zero_stream_status().
 *
 * Kernels.  Aligned bucket bodies run in the bulk-copy (TMA) kernel when its
 * shared-memory ring fits Nd rows, else in the 16-byte-vector load kernel;
 * unaligned heads and tails in a scalar kernel.  All give identical results.
 * The environment variable ZERO_STEP_KERNEL=ldg|tma overrides the choice.
 * The bulk-copy kernel's shared-memory ring is sized per Nd; for a bucket of
 * fewer than 32 x 2048 elements per SM it is cut to half of an SM's shared
 * memory, so that the next bucket's CTAs share the SM.  Bucket kernels after the first
 * of a call use programmatic dependent launch.  Tuning switches (results do
 * not change): ZERO_TMA_TILE, ZERO_TMA_STAGES, ZERO_TMA_GROUPS, ZERO_TMA_VW,
 * ZERO_TMA_ADAPT=0, ZERO_TMA_ADAPT_TILES, ZERO_LDG_RB=4|8, ZERO_PDL=0.
 * ZERO_TEST_STALL_PRODUCER=<cta> exists only to test failure detection: that
 * CTA of the bulk-copy kernel loads nothing, its waits run out after 2 s, and
 * zero_stream_status() reports ZERO_ETIMEOUT (outputs of that step invalid).
 * Threads.  A plan may be shared by threads for zero_step*() and queries;
 * zero_gather_layer()/zero_release_layer() serialise on the plan internally.
 */
#ifndef ZERO_H_
#define ZERO_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ZERO_ABI_VERSION 4

typedef enum zero_status {
    ZERO_OK = 0,
    ZERO_EINVAL = 1,   /* invalid argument */
    ZERO_ENOMEM = 2,   /* host allocation failed */
    ZERO_ECUDA = 3,    /* CUDA runtime or launch error */
    ZERO_ESTATE = 4,   /* not allowed in the current live-layer state */
    ZERO_ETIMEOUT = 5  /* a bounded device wait gave up */
} zero_status_t;

typedef struct zero_plan zero_plan_t;      /* opaque, host memory */

/* Partition descriptor.  Zero-valued optional fields take their default. */
typedef struct zero_plan_desc {
    uint64_t psi;          /* parameters; = sum(unit_elems) when units given */
    uint32_t nd;           /* logical data-parallel ranks, >= 1 */
    uint32_t stage;        /* 0 replicated DP, 1 Pos, 2 Pos+g, 3 Pos+g+p */
    uint64_t bucket_elems; /* padded elements per bucket, >= 1 */
    uint32_t align_elems;  /* A; each unit padded to a multiple of Nd*A; 0 -> 64 */
    uint32_t k_bytes;      /* optimizer bytes/param of the memory model; 0 -> 12 */
    uint32_t n_units;      /* 0 -> one unit of psi elements */
    uint32_t max_live;     /* stage 3: units gathered at once; 0 -> 1 */
    const uint64_t *unit_elems; /* n_units lengths (host; copied), or NULL */
} zero_plan_desc_t;

/* Build a plan: shard sizes, offsets, padding, bucket table, accounting.
 * Source: [MM] four-GPU example (GPU i keeps block i) and section "但 GPU
 * 只存四分之一…" (each card keeps a shard of the current layer); [CP] table
 * "三个阶段"; [CP] "关键设计取舍" item 1 (buckets).  Units are cut into Nd
 * equal contiguous shards in rank order, after zero padding to a multiple of
 * Nd*A; a bucket is a contiguous range of bucket_elems padded elements of the
 * logical vector, cut at unit boundaries (a unit's last bucket is short).
 * Host only.  *out receives a new plan owned by the caller (free with
 * zero_plan_destroy).  ZERO_EINVAL: NULL argument, psi/nd/bucket_elems = 0,
 * stage > 3, unit lengths that are zero or do not sum to psi, or sizes that
 * overflow 64 bits.  ZERO_ENOMEM: host allocation failed. */
zero_status_t zero_plan(const zero_plan_desc_t *desc, zero_plan_t **out);

/* Free a plan (NULL is ignored).  Device buffers are the caller's. */
void zero_plan_destroy(zero_plan_t *plan);

typedef enum zero_query {
    ZERO_Q_PSI = 0,          /* psi */
    ZERO_Q_PSI_PAD = 1,      /* psi_pad */
    ZERO_Q_S = 2,            /* S, elements one rank owns */
    ZERO_Q_ND = 3,
    ZERO_Q_STAGE = 4,
    ZERO_Q_N_UNITS = 5,
    ZERO_Q_UNIT_LEN = 6,     /* idx = u: len_u */
    ZERO_Q_UNIT_PAD = 7,     /* idx = u: P_u */
    ZERO_Q_UNIT_SHARD = 8,   /* idx = u: s_u */
    ZERO_Q_UNIT_BASE = 9,    /* idx = u: U_u */
    ZERO_Q_UNIT_OFFSET = 10, /* idx = u: O_u */
    ZERO_Q_N_BUCKETS = 11,
    ZERO_Q_BUCKET_UNIT = 12, /* idx = b: unit of bucket b */
    ZERO_Q_BUCKET_BEGIN = 13,/* idx = b: logical begin (inclusive) */
    ZERO_Q_BUCKET_END = 14,  /* idx = b: logical end (exclusive) */
    ZERO_Q_OWNER = 15,       /* idx = logical p: owner rank */
    ZERO_Q_OWNER_OFFSET = 16,/* idx = logical p: offset in the owner's S block */
    ZERO_Q_MEM_BYTES_PER_RANK = 17, /* idx = stage 0..3: resident model-state
                                bytes per rank with padded sizes:
                                (4+K)psi_pad, 4psi_pad+K S, 2psi_pad+(2+K)S,
                                (4+K)S.  With A = 1 and Nd | psi these are the
                                [MM] closed forms exactly. */
    ZERO_Q_WORKSPACE_BYTES = 18,/* device workspace zero_step needs when it
                                   reports the gradient norm or overflow */
    ZERO_Q_LIVE_UNITS = 19,     /* stage 3: units gathered and not released */
    ZERO_Q_PEAK_LIVE_UNITS = 20,
    ZERO_Q_PEAK_LIVE_BYTES = 21,/* bf16 bytes of the largest live set seen */
    ZERO_Q_IS_LIVE = 22,        /* idx = u: 1 if unit u is live */
    ZERO_Q_MAX_LIVE = 23,
    ZERO_Q_ALIGN = 24,
    ZERO_Q_BUCKET_ELEMS = 25,
    ZERO_Q_STATE_REPLICAS = 26, /* ranks holding each element's optimizer
                                   state: Nd at stage 0, else 1 */
    ZERO_Q_GRAD_REPLICAS = 27,  /* ... its reduced gradient: Nd at stages 0-1 */
    ZERO_Q_PARAM_REPLICAS = 28, /* ... its parameter: Nd at stages 0-2 */
    ZERO_Q_LOST_RANK_UNRECOVERABLE = 29 /* idx = rank r: parameters whose
                                   optimizer state is lost with no other copy
                                   if rank r is lost (its real, unpadded owned
                                   elements when state is sharded; 0 at
                                   stage 0) */
} zero_query_t;

/* Read one value of the plan into *out.  Host only.  ZERO_EINVAL: NULL
 * argument, unknown `what`, or `idx` out of range. */
zero_status_t zero_plan_query(const zero_plan_t *plan, zero_query_t what,
                              uint64_t idx, uint64_t *out);

/* Adam hyperparameters (double, as optimizer settings usually are).  Per
 * element, with constants rounded once to fp32 (b1, b2, eps, grad_scale,
 * 1-b1, 1-b2, step = lr/(1-b1^t), ibc2 = 1/sqrt(1-b2^t), decay = 1-lr*wd,
 * powers by pow()):
 *   g = (g_sum*grad_scale)*c;  m = b1*m + (1-b1)*g;  v = b2*v + ((1-b2)*g)*g;
 *   w = w*decay - step * (m / (sqrt(v)*ibc2 + eps));  p = bf16_rne(w)
 * each operation a separate round-to-nearest fp32 operation (no FMA); c is
 * 1 except in zero_step_guarded().  This is textbook Adam (bias-corrected,
 * eps outside the root) with optional decoupled weight decay (AdamW; wd = 0
 * gives plain Adam bit for bit); [CP] "为什么需要它" names the state, the
 * pages give no formula. */
typedef struct zero_adam {
    double lr, beta1, beta2, eps;
    double grad_scale;     /* 1/Nd averages the summed gradient */
    double weight_decay;   /* decoupled (AdamW); 0 = Adam */
} zero_adam_t;

/* Device buffers of one step (all device pointers, 16-byte aligned). */
typedef struct zero_bufs {
    const void *grads;     /* bf16 [Nd][grad_stride]; all-ranks view: rank r's
                              full gradient in logical order (padding zero);
                              owner view: rank r's gradient on the owner's
                              columns, in the owner's storage order */
    uint64_t grad_stride;  /* elements between ranks: >= psi_pad (all ranks)
                              or >= S (owner view) */
    float *master;         /* fp32 master weights: [Nd*S] owner storage
                              (all ranks) or [S] (owner view); in/out */
    float *exp_avg;        /* fp32 m, same layout; in/out */
    float *exp_avg_sq;     /* fp32 v, same layout; in/out */
    void *params;          /* bf16 out.  Stages 0-2, all ranks: Nd replica
                              rows [Nd][param_stride] in logical order; stage 3
                              or owner view: owner shards in storage order */
    uint64_t param_stride; /* replica rows only: >= psi_pad */
    float *reduced_grad;   /* optional fp32 out, layout of master: the
                              reduce-scatter result g_sum (before grad_scale) */
    double *grad_norm_sq;  /* optional device scalar out: sum of g_sum^2 over
                              the elements processed by the call */
    int32_t *overflow;     /* optional device scalar out: 1 if any g_sum is
                              inf or NaN, else 0 */
    void *workspace;       /* device scratch, needed iff grad_norm_sq or
                              overflow is set; caller-owned */
    uint64_t workspace_bytes;
    int32_t owner_view;    /* -1: all Nd ranks; o in [0,Nd): rank o only */
    const void *adam_consts; /* optional device pointer to the 9 fp32 step
                              constants of zero_adam_consts(); when set the
                              kernels read them from there instead of from
                              adam and t, so a step captured in a CUDA graph
                              can be replayed for a new t by refreshing this
                              buffer (e.g. by a captured copy from pinned
                              host memory).  16-byte aligned. */
} zero_bufs_t;

/* The nine fp32 constants one step uses, in this order: grad_scale, beta1,
 * beta2, eps, 1-beta1, 1-beta2, lr/(1-beta1^t), 1/sqrt(1-beta2^t),
 * 1-lr*weight_decay (each computed in double and rounded once).  Host only.
 * ZERO_EINVAL: NULL argument or t = 0. */
zero_status_t zero_adam_consts(const zero_adam_t *adam, uint64_t t, float out[9]);

/* One full step: every bucket in order, then (if asked) the norm/overflow.
 * Source: [MM] section "但 GPU 只存四分之一…" (gradients are split back to
 * the GPU responsible for the shard, which updates and keeps it; shards are
 * exchanged so each card briefly holds the full layer); [CP] table
 * "三个阶段" rows ZeRO-1/2/3; [MM] "ZeRO 改的是…不是模型的学习算法" (the
 * result equals replicated data-parallel Adam).  t is the 1-based step.
 * The padding of `grads` must be zero; the padding of the state then stays 0.
 * ZERO_EINVAL: NULL/misaligned pointer, short stride, t = 0, owner_view out
 * of range, norm or overflow without a big enough workspace, non-finite lr,
 * beta outside [0,1).  ZERO_ECUDA: launch failure. */
zero_status_t zero_step(const zero_plan_t *plan, const zero_bufs_t *bufs,
                        const zero_adam_t *adam, uint64_t t, void *stream);

/* Buckets [first_bucket, first_bucket + n_buckets) of a step, for callers
 * that launch each bucket as soon as its gradients exist ([CP] "关键设计取舍"
 * item 1).  The norm/overflow workspace is reset by the call that contains
 * bucket 0 and reported by the call that contains the last bucket; calls of
 * one step must run in bucket order on one stream.  In the owner view,
 * buckets the owner has no part of launch nothing.  Errors as zero_step,
 * plus ZERO_EINVAL for a bucket range outside the plan. */
zero_status_t zero_step_buckets(const zero_plan_t *plan,
                                 const zero_bufs_t *bufs,
                                 const zero_adam_t *adam, uint64_t t,
                                 uint64_t first_bucket, uint64_t n_buckets,
                                 void *stream);

/* zero_step() without a caller-provided workspace, for callers that cannot
 * allocate device memory (a runtime whose device memory is all handed out by
 * its own pool up front, a plain C caller with no allocator of its own, code
 * that must not allocate while it runs).  The paper has no counterpart: this
 * is a packaging choice of this library.  The norm/overflow scratch lives in a
 * 49,408-byte static array in device memory owned by the library, present on
 * every GPU that loads it until the process exits; bufs->workspace and
 * bufs->workspace_bytes are ignored, every other field is as for zero_step.
 * No cudaMalloc, cudaFree or other allocating call is made.  The first call on
 * a device looks up the array's device address (cudaGetSymbolAddress) and
 * caches it; make that first call before any stream capture.  The cached
 * address belongs to the device's current context: do not reset the device
 * (cudaDeviceReset) or tear down its primary context between calls, since the
 * library would keep using the old address.  All calls share the one array:
 * calls whose kernels overlap on the GPU (several streams or threads at once)
 * race on it and must be serialised by the caller.  Each step clears the
 * array on its stream before its kernels add into it, so stale contents are
 * harmless.
 * ZERO_EINVAL: as zero_step, or a plan whose scratch would exceed the static
 * array (the message says so).  ZERO_ECUDA: the address lookup or a launch
 * failed. */
zero_status_t zero_step_noalloc(const zero_plan_t *plan, const zero_bufs_t *bufs,
                                const zero_adam_t *adam, uint64_t t, void *stream);

/* Guards of zero_step_guarded(); the pages have no counterpart (these are
 * the usual mixed-precision guards around an optimizer step). */
typedef struct zero_guard {
    double max_grad_norm;  /* > 0: clip the global norm of g = g_sum*grad_scale
                              to this (c = min(1, max/(norm + 1e-6))); 0: off */
    int32_t skip_nonfinite;/* 1: if any g_sum is inf or NaN, change nothing */
} zero_guard_t;

/* The step with global-norm clipping and/or skipping on non-finite
 * gradients, in two passes: (1) every bucket's rank-order reduction into
 * bufs->reduced_grad with the sum of squares and the non-finite count; a
 * one-block kernel then forms norm = |grad_scale| * sqrt(sum g_sum^2) (double)
 * and c (fp32; 1 if the norm is not finite); (2) unless skipped, Adam from
 * the reduced gradients with g = (g_sum*grad_scale)*c.  reduced_grad,
 * grad_norm_sq, overflow and workspace are required (the norm reported is
 * sum g_sum^2).  A skipped step leaves master, m, v and params unchanged;
 * *overflow tells the caller.  Moves 2Nd + 8 + 24 + params bytes per element
 * (zero_bytes_moved(ZERO_BYTES_HBM_GUARDED_STEP)).  ZERO_EINVAL as zero_step,
 * or a missing required buffer, or max_grad_norm < 0 or not finite. */
zero_status_t zero_step_guarded(const zero_plan_t *plan, const zero_bufs_t *bufs,
                                const zero_adam_t *adam, const zero_guard_t *guard,
                                uint64_t t, void *stream);

/* Reshard a checkpoint: copy one state array (fp32 master, m, v: elem_bytes
 * 4; bf16 owner parameters: 2) from owner storage under plan `from`
 * ([from.Nd * from.S]) to owner storage under plan `to` ([to.Nd * to.S]),
 * element by element through the logical order; the destination's padding is
 * written as zero.  The two plans must have the same unit lengths (the same
 * model); Nd, alignment, stage and buckets may differ.  A checkpoint is then
 * the owner-storage arrays plus t; resuming with another Nd is one call per
 * array.  The concept page's "使用时应检查" list asks whether a checkpoint can
 * be restored after the parallelism changes; this is that step.
 * ZERO_EINVAL: NULL, elem_bytes not 2 or 4, different units, misaligned
 * buffers.  ZERO_ECUDA: launch failure.  The buffers must not overlap. */
zero_status_t zero_reshard(const zero_plan_t *from, const void *src, const zero_plan_t *to, void *dst,
                           uint32_t elem_bytes, void *stream);

/* Stage 3: materialise unit `unit` -- copy the Nd owners' bf16 slices of it,
 * in rank order, into full_layer[0 .. len_u) (padding dropped) -- and mark
 * it live.  Source: [MM] glossary "临时物化" and "all-gather" (shards are
 * briefly put together into the full parameters of the current layer);
 * [CP] table "三个阶段" row ZeRO-3 (all-gather in execution order, release
 * promptly).  owner_params: bf16 [Nd*S] owner storage (zero_step's params at
 * stage 3); full_layer: bf16 [len_u], caller-owned.  ZERO_EINVAL: stage != 3,
 * unit out of range, NULL/misaligned pointer.  ZERO_ESTATE: the unit is
 * already live, or max_live units are live.  ZERO_ECUDA: launch failure (the
 * unit is then not marked live). */
zero_status_t zero_gather_layer(zero_plan_t *plan, uint32_t unit,
                                const void *owner_params, void *full_layer,
                                void *stream);

/* Stage 3: release a live unit (its full_layer buffer may be reused once the
 * work queued on it is done).  Source: [MM] glossary "临时物化" (no extra copy
 * is kept after the computation); [CP] remark under "三个阶段" (unreleased
 * layers form memory peaks).  Host only.  ZERO_EINVAL: unit out of range.
 * ZERO_ESTATE: the unit is not live. */
zero_status_t zero_release_layer(zero_plan_t *plan, uint32_t unit);

/* ---------------------------------------------------------------------------
 * Ranks as devices.  The calls above hold all Nd ranks on one GPU.  The calls
 * below run one rank's share of the same step when each rank has its own
 * buffers, which is how ZeRO runs: rank r's process calls them on its own
 * GPU, and every other rank's gradient and parameter replica are reachable
 * from that GPU through plain device pointers.  On one node those are peer
 * mappings over NVLink/NVSwitch (zero_ipc_open() of another process's
 * buffer); the same calls also accept local buffers, so that Nd ranks can be
 * separate allocations on one GPU.
 *
 * Rank r's step, per bucket (stages 1-3; [MM] section "但 GPU 只存四分之一…":
 * each rank sends the gradient of a shard to the rank that owns it, which
 * updates it; the updated parameters are then exchanged):
 *   reduce-scatter: for every element p that r owns, read G_q[p] from every
 *     rank q directly from q's memory and add them in rank order 0..Nd-1
 *     from rank 0's value, in fp32 (the same sum as zero_step);
 *   owner Adam on r's fp32 state, which is local;
 *   all-gather: store bf16(w) straight into every rank's replica (stages 1-2)
 *     or into r's own parameter shard (stage 3).
 * The collective is inside the kernel: there is no separate reduce-scatter
 * or all-gather.  Every rank's results are bit-identical to zero_step's on
 * the same inputs.  Each element is read and written by exactly one rank (its
 * owner), so the ranks' kernels never wait for one another and share no
 * flags.  The caller orders the step against the other ranks: all ranks'
 * gradients must be complete before any rank's call runs, and no rank may
 * read its replica or overwrite a gradient until every rank's call has
 * finished (e.g. a one-element all-reduce on the stream before and after;
 * the kernels end with a system-scope fence so that their stores to peers
 * are performed when they complete).  Stage 0 keeps a full state on every
 * rank, which this layout does not describe: ZERO_EINVAL.
 * ------------------------------------------------------------------------- */
#define ZERO_MAX_PEERS 128u

typedef struct zero_peer_bufs {
    uint32_t rank;           /* r: the owner whose shard this call updates */
    uint32_t reserved;       /* 0 */
    const void *const *grads;/* HOST array [Nd] of device pointers: grads[q] =
                                rank q's bf16 gradient [psi_pad] in logical
                                order (padding zero), readable from this
                                device; 16-byte aligned */
    void *const *params;     /* HOST array [Nd].  Stages 1-2: params[q] = rank
                                q's bf16 replica [psi_pad], logical order,
                                writable from this device.  Stage 3: only
                                params[rank] is used: r's bf16 owner shard [S]
                                in storage order */
    float *master;           /* r's fp32 master shard [S], storage order; in/out */
    float *exp_avg;          /* r's fp32 m [S]; in/out */
    float *exp_avg_sq;       /* r's fp32 v [S]; in/out */
    float *reduced_grad;     /* optional fp32 [S] out: r's g_sum */
    double *grad_norm_sq;    /* optional device scalar out: sum of g_sum^2 over
                                r's shard (sum it over ranks for the global
                                norm) */
    int32_t *overflow;       /* optional device scalar out: 1 if a g_sum of
                                r's shard is inf or NaN */
    void *workspace;         /* needed iff grad_norm_sq or overflow is set */
    uint64_t workspace_bytes;
    const void *adam_consts; /* optional, as in zero_bufs_t */
} zero_peer_bufs_t;

/* Rank bufs->rank's part of buckets [first_bucket, first_bucket + n_buckets)
 * of a step (n_buckets = zero_plan_query(ZERO_Q_N_BUCKETS) for the whole
 * step), as described above; the norm workspace is reset by the call that
 * contains bucket 0 and reported by the call that contains the last.  The
 * grads and params arrays are read on the host during the call only.  Bytes
 * per owned element: 2Nd read from the ranks' gradients (2(Nd-1) of them
 * from peers), 12 read + 12 written of local state, 2Nd written to replicas
 * (2(Nd-1) to peers), or 2 at stage 3.  ZERO_EINVAL: as zero_step, or stage
 * 0, Nd > ZERO_MAX_PEERS, rank out of range, a NULL or misaligned entry of
 * grads or params.  ZERO_ECUDA: launch failure.  Aligned bodies run in the
 * bulk-copy kernel, rows pulled by 1-D bulk copies from the peers (never
 * multicast), at stage 3, and with replicas when the call's aligned bodies
 * average at least 32 x 2048 columns per SM (ZERO_PEER_RING_MIN=<columns>
 * moves the threshold); other calls run them in a 16-byte-load kernel.
 * One kernel per call; zero_step_peers_kernel() says which.
 * ZERO_STEP_KERNEL=tma|ldg forces either. */
zero_status_t zero_step_peers(const zero_plan_t *plan, const zero_peer_bufs_t *bufs,
                              const zero_adam_t *adam, uint64_t t, uint64_t first_bucket,
                              uint64_t n_buckets, void *stream);

/* Stage 3 with ranks as devices: materialise unit `unit` into full_layer
 * [len_u] by reading owner q's slice from owner_params[q] (a HOST array [Nd]
 * of device pointers to each rank's bf16 owner shard [S], readable from this
 * device), in rank order.  Liveness as zero_gather_layer (the plan counts
 * this rank's live units).  Errors as zero_gather_layer, plus ZERO_EINVAL
 * for a NULL or misaligned entry of owner_params. */
zero_status_t zero_gather_layer_peers(zero_plan_t *plan, uint32_t unit,
                                      const void *const *owner_params, void *full_layer,
                                      void *stream);

/* Sharing a buffer with another process on the same node (CUDA IPC).  The
 * handle names the buffer's whole allocation plus the buffer's offset in it,
 * so buffers carved out of a larger allocation (a caching allocator's) can be
 * shared; the allocation must come from cudaMalloc (not from a virtual-memory
 * or managed allocator).  A handle is plain bytes: send it to the other ranks
 * by any means. */
typedef struct zero_ipc_handle {
    unsigned char handle[64];/* cudaIpcMemHandle_t of the allocation */
    uint64_t offset;         /* buffer start - allocation start, bytes */
    uint64_t alloc_bytes;    /* size of the allocation */
    uint64_t exporter_va;    /* allocation start in the exporting process */
    int32_t device;          /* CUDA ordinal of the buffer in the exporter */
    int32_t exporter_pid;    /* process that exported it */
} zero_ipc_handle_t;

/* Describe the device buffer at ptr for zero_ipc_open() in another process.
 * ZERO_EINVAL: NULL, or ptr is not device memory from cudaMalloc.
 * ZERO_ECUDA: the CUDA call failed. */
zero_status_t zero_ipc_export(const void *ptr, zero_ipc_handle_t *out);

/* Map a buffer exported by zero_ipc_export() into this process on the current
 * CUDA device (peer access is enabled as needed) and return its address.  A
 * handle exported by this same process returns the original address without
 * a mapping.  Opening several buffers of one allocation maps it once
 * (reference-counted).  ZERO_EINVAL: NULL.  ZERO_ECUDA: the mapping failed
 * (no peer access between the two devices, or the exporter has freed it). */
zero_status_t zero_ipc_open(const zero_ipc_handle_t *h, void **ptr);

/* Undo one zero_ipc_open(); the mapping goes when its last buffer is closed.
 * ZERO_EINVAL: ptr was not returned by zero_ipc_open() (or already closed).
 * ZERO_ECUDA: unmapping failed. */
zero_status_t zero_ipc_close(void *ptr);

typedef enum zero_bytes_kind {
    ZERO_BYTES_COMM_ELEMS_PER_RANK = 0, /* ring model, elements one rank sends
                                           per step: 2(Nd-1)S at stages 0-2,
                                           3(Nd-1)S at stage 3 */
    ZERO_BYTES_COMM_PER_RANK = 1,       /* the same in bytes (bf16) */
    ZERO_BYTES_HBM_STEP = 2,            /* bytes zero_step moves in HBM */
    ZERO_BYTES_HBM_GATHER_STEP = 3,     /* bytes of the stage-3 gathers of one
                                           step (2 per unit: 4 B/element) */
    ZERO_BYTES_HBM_GUARDED_STEP = 4     /* bytes zero_step_guarded moves */
} zero_bytes_kind_t;

#define ZERO_BYTES_FLAG_OWNER_VIEW 1u    /* HBM_STEP of one owner's shard */
#define ZERO_BYTES_FLAG_REDUCED 2u       /* HBM_STEP incl. reduced_grad writes */

/* Accounting.  Source: [MM] "论文证据" (plain DP and gradient partitioning
 * move 2 Psi per step, parameter partitioning 3 Psi, about 1.5 times).
 * HBM_STEP = n*(2Nd + 24 + w) [+4n], n = psi_pad (S in the owner view),
 * w = 2Nd for replicas (stages 0-2, all ranks) else 2.  ZERO_EINVAL: NULL
 * argument or unknown kind. */
zero_status_t zero_bytes_moved(const zero_plan_t *plan, zero_bytes_kind_t kind,
                               uint32_t flags, uint64_t *out);

/* Wait for `stream` and report device-side failures of the step kernels:
 * ZERO_ETIMEOUT if a bounded wait inside the bulk-copy step kernel gave up
 * since the last call (the outputs of those steps are not valid; the flag is
 * cleared), ZERO_ECUDA if the stream reports a CUDA error, else ZERO_OK.
 * Synchronises the stream (and reads one device word), so call it between
 * steps, not inside a captured graph. */
zero_status_t zero_stream_status(void *stream);

#define ZERO_KERNEL_NONE 0u         /* no aligned body: only the scalar edge kernel runs */
#define ZERO_KERNEL_BULK_COPY 1u    /* k_step_tma: bulk-copy (TMA) shared-memory ring */
#define ZERO_KERNEL_VECTOR_LOAD 2u  /* k_step_vec8 / k_step_peer: 16-byte vector loads */

/* Which kernel zero_step() uses for the aligned bucket bodies of `plan` on
 * the current CUDA device (owner_view as in zero_bufs_t), written to *kind.
 * Queries the device once.  ZERO_EINVAL: NULL argument or owner_view out of
 * range.  ZERO_ECUDA: the device query failed. */
zero_status_t zero_step_kernel(const zero_plan_t *plan, int32_t owner_view, uint32_t *kind);

/* Which kernel zero_step_peers() uses for the aligned bodies of rank
 * `rank`'s call over buckets [first_bucket, first_bucket + n_buckets) on the
 * current CUDA device, written to *kind: ZERO_KERNEL_BULK_COPY,
 * ZERO_KERNEL_VECTOR_LOAD (k_step_peer), or ZERO_KERNEL_NONE when the call
 * has no aligned body.  Reads the same environment overrides as the call.
 * Queries the device once.  ZERO_EINVAL: NULL argument, stage 0,
 * Nd > ZERO_MAX_PEERS, rank out of range or buckets outside the plan.
 * ZERO_ECUDA: the device query failed. */
zero_status_t zero_step_peers_kernel(const zero_plan_t *plan, uint32_t rank, uint64_t first_bucket,
                                     uint64_t n_buckets, uint32_t *kind);

/* Static text of a status code. */
const char *zero_status_str(zero_status_t status);

/* Text of the last failure on the calling thread ("" if none).  Valid until
 * the next call on that thread. */
const char *zero_last_error(void);

/* ZERO_ABI_VERSION of the loaded library. */
uint32_t zero_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ZERO_H_ */

// Partition planner of the ZeRO step: shard / offset / padding maps, the
// bucket table, per-stage memory and communication accounting, stage-3
// live-layer bookkeeping.  Host only, all integer.
//
// Sharding follows the four-GPU example of the mind-map page "ZeRO 真正在做什么：
// 长期分开存，计算时临时拼齐" (GPU i keeps block i) and its section "但 GPU 只存
// 四分之一…" (each card keeps a shard of the current layer): every unit is
// zero-padded to a multiple of Nd*A and cut into Nd equal contiguous shards
// in rank order.  Buckets follow item 1 of "关键设计取舍" on the concept page
// "ZeRO": contiguous ranges of bucket_elems padded elements, cut at unit
// boundaries.
#include <algorithm>
#include <cstring>
#include <new>

#include "zero_internal.h"
#include "zero_trace.h"

using zero_detail::set_error;

namespace zero_detail {

namespace {
thread_local std::string g_last_error;
}

zero_status_t set_error(zero_status_t s, const std::string &msg) {
    g_last_error = msg;
    return s;
}

void clear_error() { g_last_error.clear(); }

BucketRange bucket_range(const zero_plan_t &p, uint64_t b) {
    // unit whose bucket block holds b: last u with unit_bucket0[u] <= b
    auto it = std::upper_bound(p.unit_bucket0.begin(), p.unit_bucket0.end() - 1, b);
    uint32_t u = uint32_t(it - p.unit_bucket0.begin()) - 1;
    uint64_t k = b - p.unit_bucket0[u];
    uint64_t lo = p.unit_base[u] + k * p.bucket_elems;
    uint64_t hi = std::min(lo + p.bucket_elems, p.unit_base[u] + p.unit_pad[u]);
    return {u, lo, hi};
}

}  // namespace zero_detail

namespace {

bool mul_overflows(uint64_t a, uint64_t b, uint64_t *out) {
    return __builtin_mul_overflow(a, b, out);
}
bool add_overflows(uint64_t a, uint64_t b, uint64_t *out) {
    return __builtin_add_overflow(a, b, out);
}

}  // namespace

ZERO_API zero_status_t zero_plan(const zero_plan_desc_t *desc, zero_plan_t **out) {
    zero_detail::clear_error();
    if (!desc || !out) return set_error(ZERO_EINVAL, "zero_plan: NULL argument");
    *out = nullptr;
    if (desc->psi == 0) return set_error(ZERO_EINVAL, "zero_plan: psi must be >= 1");
    if (desc->nd == 0) return set_error(ZERO_EINVAL, "zero_plan: nd must be >= 1");
    if (desc->stage > 3) return set_error(ZERO_EINVAL, "zero_plan: stage must be 0..3");
    if (desc->bucket_elems == 0)
        return set_error(ZERO_EINVAL, "zero_plan: bucket_elems must be >= 1");
    if (desc->n_units > 1 && !desc->unit_elems)
        return set_error(ZERO_EINVAL, "zero_plan: n_units > 1 needs unit_elems");

    zero_plan_t *p = new (std::nothrow) zero_plan_t();
    if (!p) return set_error(ZERO_ENOMEM, "zero_plan: out of host memory");
    try {
        p->psi = desc->psi;
        p->nd = desc->nd;
        p->stage = desc->stage;
        p->bucket_elems = desc->bucket_elems;
        p->align = desc->align_elems ? desc->align_elems : 64;
        p->k_bytes = desc->k_bytes ? desc->k_bytes : 12;
        p->max_live = desc->max_live ? desc->max_live : 1;

        if (desc->n_units >= 1 && desc->unit_elems) {
            p->unit_len.assign(desc->unit_elems, desc->unit_elems + desc->n_units);
        } else {
            p->unit_len.assign(1, desc->psi);
        }
        uint64_t sum = 0;
        for (uint64_t n : p->unit_len) {
            if (n == 0 || add_overflows(sum, n, &sum)) {
                delete p;
                return set_error(ZERO_EINVAL, "zero_plan: unit lengths must be >= 1 and fit 64 bits");
            }
        }
        if (sum != p->psi) {
            delete p;
            return set_error(ZERO_EINVAL, "zero_plan: unit lengths do not sum to psi");
        }

        uint64_t quantum;
        if (mul_overflows(uint64_t(p->nd), uint64_t(p->align), &quantum)) {
            delete p;
            return set_error(ZERO_EINVAL, "zero_plan: nd*align overflows");
        }
        uint64_t U = 0, O = 0, nb = 0;
        const size_t nu = p->unit_len.size();
        p->unit_pad.resize(nu);
        p->unit_shard.resize(nu);
        p->unit_base.resize(nu);
        p->unit_offset.resize(nu);
        p->unit_bucket0.resize(nu + 1);
        for (size_t u = 0; u < nu; ++u) {
            uint64_t chunks = p->unit_len[u] / quantum + (p->unit_len[u] % quantum != 0);
            uint64_t P;
            if (mul_overflows(chunks, quantum, &P)) {
                delete p;
                return set_error(ZERO_EINVAL, "zero_plan: padded size overflows");
            }
            p->unit_pad[u] = P;
            p->unit_shard[u] = P / p->nd;
            p->unit_base[u] = U;
            p->unit_offset[u] = O;
            p->unit_bucket0[u] = nb;
            if (add_overflows(U, P, &U)) {
                delete p;
                return set_error(ZERO_EINVAL, "zero_plan: padded size overflows");
            }
            O += P / p->nd;
            nb += P / p->bucket_elems + (P % p->bucket_elems != 0);
        }
        p->unit_bucket0[nu] = nb;
        p->psi_pad = U;
        p->S = O;
        p->n_buckets = nb;
        p->live.assign(nu, 0);
    } catch (const std::bad_alloc &) {
        delete p;
        return set_error(ZERO_ENOMEM, "zero_plan: out of host memory");
    }
    *out = p;
    return ZERO_OK;
}

ZERO_API void zero_plan_destroy(zero_plan_t *plan) { delete plan; }

ZERO_API zero_status_t zero_plan_query(const zero_plan_t *p, zero_query_t what,
                                       uint64_t idx, uint64_t *out) {
    zero_detail::clear_error();
    if (!p || !out) return set_error(ZERO_EINVAL, "zero_plan_query: NULL argument");
    const uint64_t nu = p->unit_len.size();
    auto need_unit = [&]() { return idx < nu; };
    switch (what) {
        case ZERO_Q_PSI: *out = p->psi; return ZERO_OK;
        case ZERO_Q_PSI_PAD: *out = p->psi_pad; return ZERO_OK;
        case ZERO_Q_S: *out = p->S; return ZERO_OK;
        case ZERO_Q_ND: *out = p->nd; return ZERO_OK;
        case ZERO_Q_STAGE: *out = p->stage; return ZERO_OK;
        case ZERO_Q_N_UNITS: *out = nu; return ZERO_OK;
        case ZERO_Q_N_BUCKETS: *out = p->n_buckets; return ZERO_OK;
        case ZERO_Q_WORKSPACE_BYTES: *out = zero_detail::kWorkspaceBytes; return ZERO_OK;
        case ZERO_Q_MAX_LIVE: *out = p->max_live; return ZERO_OK;
        case ZERO_Q_ALIGN: *out = p->align; return ZERO_OK;
        case ZERO_Q_BUCKET_ELEMS: *out = p->bucket_elems; return ZERO_OK;
        case ZERO_Q_STATE_REPLICAS: *out = p->stage == 0 ? p->nd : 1; return ZERO_OK;
        case ZERO_Q_GRAD_REPLICAS: *out = p->stage <= 1 ? p->nd : 1; return ZERO_OK;
        case ZERO_Q_PARAM_REPLICAS: *out = p->stage <= 2 ? p->nd : 1; return ZERO_OK;
        case ZERO_Q_LOST_RANK_UNRECOVERABLE: {
            if (idx >= p->nd) return set_error(ZERO_EINVAL, "zero_plan_query: rank out of range");
            uint64_t lost = 0;
            if (p->stage != 0 || p->nd == 1) {
                for (size_t u = 0; u < nu; ++u) {
                    const uint64_t lo = idx * p->unit_shard[u];
                    if (p->unit_len[u] > lo) lost += std::min(p->unit_shard[u], p->unit_len[u] - lo);
                }
            }
            *out = lost;
            return ZERO_OK;
        }
        case ZERO_Q_UNIT_LEN:
        case ZERO_Q_UNIT_PAD:
        case ZERO_Q_UNIT_SHARD:
        case ZERO_Q_UNIT_BASE:
        case ZERO_Q_UNIT_OFFSET:
        case ZERO_Q_IS_LIVE:
            if (!need_unit()) return set_error(ZERO_EINVAL, "zero_plan_query: unit out of range");
            switch (what) {
                case ZERO_Q_UNIT_LEN: *out = p->unit_len[idx]; break;
                case ZERO_Q_UNIT_PAD: *out = p->unit_pad[idx]; break;
                case ZERO_Q_UNIT_SHARD: *out = p->unit_shard[idx]; break;
                case ZERO_Q_UNIT_BASE: *out = p->unit_base[idx]; break;
                case ZERO_Q_UNIT_OFFSET: *out = p->unit_offset[idx]; break;
                default: {
                    std::lock_guard<std::mutex> g(p->mu);
                    *out = p->live[idx];
                }
            }
            return ZERO_OK;
        case ZERO_Q_BUCKET_UNIT:
        case ZERO_Q_BUCKET_BEGIN:
        case ZERO_Q_BUCKET_END: {
            if (idx >= p->n_buckets)
                return set_error(ZERO_EINVAL, "zero_plan_query: bucket out of range");
            zero_detail::BucketRange r = zero_detail::bucket_range(*p, idx);
            *out = what == ZERO_Q_BUCKET_UNIT ? r.unit
                   : what == ZERO_Q_BUCKET_BEGIN ? r.begin : r.end;
            return ZERO_OK;
        }
        case ZERO_Q_OWNER:
        case ZERO_Q_OWNER_OFFSET: {
            if (idx >= p->psi_pad)
                return set_error(ZERO_EINVAL, "zero_plan_query: element out of range");
            auto it = std::upper_bound(p->unit_base.begin(), p->unit_base.end(), idx);
            size_t u = size_t(it - p->unit_base.begin()) - 1;
            uint64_t j = idx - p->unit_base[u];
            uint64_t o = j / p->unit_shard[u];
            *out = what == ZERO_Q_OWNER ? o : p->unit_offset[u] + (j - o * p->unit_shard[u]);
            return ZERO_OK;
        }
        case ZERO_Q_MEM_BYTES_PER_RANK: {
            const uint64_t K = p->k_bytes;
            switch (idx) {
                case 0: *out = (4 + K) * p->psi_pad; return ZERO_OK;
                case 1: *out = 4 * p->psi_pad + K * p->S; return ZERO_OK;
                case 2: *out = 2 * p->psi_pad + (2 + K) * p->S; return ZERO_OK;
                case 3: *out = (4 + K) * p->S; return ZERO_OK;
                default:
                    return set_error(ZERO_EINVAL, "zero_plan_query: stage must be 0..3");
            }
        }
        case ZERO_Q_LIVE_UNITS:
        case ZERO_Q_PEAK_LIVE_UNITS:
        case ZERO_Q_PEAK_LIVE_BYTES: {
            std::lock_guard<std::mutex> g(p->mu);
            *out = what == ZERO_Q_LIVE_UNITS ? p->n_live
                   : what == ZERO_Q_PEAK_LIVE_UNITS ? p->peak_live : p->peak_live_bytes;
            return ZERO_OK;
        }
    }
    return set_error(ZERO_EINVAL, "zero_plan_query: unknown query");
}

ZERO_API zero_status_t zero_bytes_moved(const zero_plan_t *p, zero_bytes_kind_t kind,
                                        uint32_t flags, uint64_t *out) {
    zero_detail::clear_error();
    if (!p || !out) return set_error(ZERO_EINVAL, "zero_bytes_moved: NULL argument");
    const uint64_t one_collective = uint64_t(p->nd - 1) * p->S;  // ring RS or AG
    const uint64_t comm = (p->stage == 3 ? 3 : 2) * one_collective;
    switch (kind) {
        case ZERO_BYTES_COMM_ELEMS_PER_RANK: *out = comm; return ZERO_OK;
        case ZERO_BYTES_COMM_PER_RANK: *out = 2 * comm; return ZERO_OK;
        case ZERO_BYTES_HBM_STEP: {
            const bool owner = flags & ZERO_BYTES_FLAG_OWNER_VIEW;
            const uint64_t n = owner ? p->S : p->psi_pad;
            uint64_t per = 2ull * p->nd + 24;                 // grads in, w/m/v in+out
            per += (owner || p->stage == 3) ? 2 : 2ull * p->nd;  // bf16 params out
            if (flags & ZERO_BYTES_FLAG_REDUCED) per += 4;
            *out = n * per;
            return ZERO_OK;
        }
        case ZERO_BYTES_HBM_GUARDED_STEP: {
            // pass 1: Nd bf16 rows in, fp32 sum out; pass 2: fp32 sum and
            // w, m, v in, w, m, v and the parameters out
            const bool owner = flags & ZERO_BYTES_FLAG_OWNER_VIEW;
            const uint64_t n = owner ? p->S : p->psi_pad;
            uint64_t per = 2ull * p->nd + 4 + 4 + 24;
            per += (owner || p->stage == 3) ? 2 : 2ull * p->nd;
            *out = n * per;
            return ZERO_OK;
        }
        case ZERO_BYTES_HBM_GATHER_STEP: {
            uint64_t s = 0;
            for (uint64_t n : p->unit_len) s += 4 * n;
            *out = 2 * s;  // forward and backward materialisation
            return ZERO_OK;
        }
    }
    return set_error(ZERO_EINVAL, "zero_bytes_moved: unknown kind");
}

namespace zero_detail {

zero_status_t live_check(const zero_plan_t &p, uint32_t unit, const char *who) {
    if (p.live[unit])
        return set_error(ZERO_ESTATE, std::string(who) + ": unit " + std::to_string(unit) + " is already live");
    if (p.n_live >= p.max_live)
        return set_error(ZERO_ESTATE, std::string(who) + ": max_live units are live; release one first");
    return ZERO_OK;
}

void live_mark(zero_plan_t &p, uint32_t unit) {
    p.live[unit] = 1;
    p.n_live += 1;
    p.live_bytes += 2 * p.unit_len[unit];
    p.peak_live = std::max(p.peak_live, p.n_live);
    p.peak_live_bytes = std::max(p.peak_live_bytes, p.live_bytes);
}

}  // namespace zero_detail

ZERO_API zero_status_t zero_release_layer(zero_plan_t *p, uint32_t unit) {
    zero_detail::clear_error();
    if (!p) return set_error(ZERO_EINVAL, "zero_release_layer: NULL plan");
    if (unit >= p->unit_len.size())
        return set_error(ZERO_EINVAL, "zero_release_layer: unit out of range");
    std::lock_guard<std::mutex> g(p->mu);
    if (!p->live[unit])
        return set_error(ZERO_ESTATE, "zero_release_layer: unit " + std::to_string(unit) +
                                          " is not live");
    p->live[unit] = 0;
    p->n_live -= 1;
    p->live_bytes -= 2 * p->unit_len[unit];
    zero_trace::mark("zero_release_layer unit %u", unit);
    return ZERO_OK;
}

ZERO_API const char *zero_status_str(zero_status_t s) {
    switch (s) {
        case ZERO_OK: return "ZERO_OK";
        case ZERO_EINVAL: return "ZERO_EINVAL: invalid argument";
        case ZERO_ENOMEM: return "ZERO_ENOMEM: host allocation failed";
        case ZERO_ECUDA: return "ZERO_ECUDA: CUDA error";
        case ZERO_ESTATE: return "ZERO_ESTATE: not allowed in the current live-layer state";
        case ZERO_ETIMEOUT: return "ZERO_ETIMEOUT: a bounded device wait gave up";
    }
    return "unknown zero_status_t";
}

ZERO_API const char *zero_last_error(void) { return zero_detail::g_last_error.c_str(); }

ZERO_API uint32_t zero_abi_version(void) { return ZERO_ABI_VERSION; }

"""Oracle step drivers: replicated data parallelism (stage 0) and the ZeRO
partitioned step (stages 1-3), on the CPU, with numpy.  Test infrastructure.

Sources.  Mind-map page "ZeRO 真正在做什么：长期分开存，计算时临时拼齐":
  - section "但 GPU 只存四分之一…": gradients are split again and sent to the
    GPU responsible for each shard, which updates it and keeps it; before a
    layer is computed the shards are exchanged so that every card briefly
    holds the full layer, and the borrowed shards are dropped afterwards.
  - "ZeRO 改的是训练状态的保存与通信方式，不是模型的学习算法": ZeRO changes
    how state is stored and moved, not the learning algorithm.
Concept page "ZeRO", section "为什么需要它": an update only needs all ranks to
see one consistent full model logically; and table "三个阶段" (which states
stay replicated at each stage: parameters at ZeRO-1/2, none at ZeRO-3, where
parameters are all-gathered in execution order and released promptly).

So the replicated step is the definition, and the partitioned step must reach
exactly the same numbers: each owner runs the same elementwise core on its
shard's columns, written through the partition maps of ``oracle.plan``.
"""
import numpy as np

from . import core
from .plan import Plan


def step_replicated(nd, grads, w, m, v, adam, t, want_reduced=False):
    """Stage 0: every rank keeps the full state and runs the full update.

    grads: uint16 [nd, n] (rank r's bf16 gradient, logical order).
    w, m, v: fp32 [nd, n], rank r's own full copy, updated in place.
    Returns params uint16 [nd, n] (each rank's bf16 copy), reduced fp32 [n] of
    rank 0 (or None), norm_sq, nonfinite (of rank 0's view).
    """
    n = grads.shape[1]
    params = np.empty((nd, n), dtype=np.uint16)
    red0 = None
    norm0 = bad0 = None
    for r in range(nd):
        # all-reduce: every rank sums all ranks' gradients in rank order
        p, red, norm, bad = core.update(grads, w[r], m[r], v[r], adam, t,
                                        want_reduced=want_reduced)
        params[r] = p
        if r == 0:
            red0, norm0, bad0 = red, norm, bad
    return params, red0, norm0, bad0


def step_partitioned(pl: Plan, grads, master, m, v, params, adam, t,
                     reduced=None, clip_coef=1.0):
    """Stages 1-3 over all Nd logical ranks.

    grads: uint16 [nd, psi_pad], logical order (zero in the padding).
    master, m, v, reduced: fp32 [nd * S], rank-major owner storage
      (owner o's unit-u shard at o*S + O_u + [0, s_u)); updated in place.
    params: uint16; stages 0-2: [nd, psi_pad] replicas, every rank's copy
      rewritten with the owner's new values (the all-gather); stage 3:
      [nd * S] owner shards only.
    Returns (norm_sq, nonfinite) over all padded elements.
    """
    nd, S = pl.nd, pl.S
    norm = 0.0
    bad = 0
    for o in range(nd):
        for u in range(len(pl.unit_pad)):
            s = pl.unit_shard[u]
            lo = pl.unit_base[u] + o * s            # logical columns
            st = o * S + pl.unit_offset[u]          # owner storage
            cols = grads[:, lo:lo + s]
            w_ = master[st:st + s]
            m_ = m[st:st + s]
            v_ = v[st:st + s]
            p, red, nn, bb = core.update(cols, w_, m_, v_, adam, t,
                                         want_reduced=reduced is not None,
                                         clip_coef=clip_coef)
            norm += nn
            bad += bb
            if reduced is not None:
                reduced[st:st + s] = red
            if pl.stage == 3:
                params[st:st + s] = p
            else:
                params[:, lo:lo + s] = p[None, :]
    return norm, bad


def step_owner_view(pl: Plan, owner, grads_owner, master, m, v, adam, t,
                    want_reduced=False, clip_coef=1.0):
    """One owner's part of the step.

    grads_owner: uint16 [nd, S]: for every rank, its gradient on the columns
      that `owner` owns, in the owner's storage order.
    master, m, v: fp32 [S] (the owner's own state), updated in place.
    Returns (params uint16 [S], reduced fp32 [S] or None, norm_sq, nonfinite).
    """
    p, red, nn, bb = core.update(grads_owner, master, m, v, adam, t,
                                 want_reduced=want_reduced, clip_coef=clip_coef)
    return p, red, nn, bb


def owner_columns(pl: Plan, owner):
    """Logical column indices that `owner` owns, in its storage order."""
    parts = []
    for u in range(len(pl.unit_pad)):
        s = pl.unit_shard[u]
        lo = pl.unit_base[u] + owner * s
        parts.append(np.arange(lo, lo + s, dtype=np.int64))
    return np.concatenate(parts)


def gather_layer(pl: Plan, unit, owner_params):
    """Stage 3 materialisation of one unit: concatenate the Nd owners' slices
    of the unit in rank order and keep the first len_u (unpadded) elements.
    owner_params: uint16 [nd * S] -> uint16 [len_u]."""
    s = pl.unit_shard[unit]
    pieces = []
    for o in range(pl.nd):
        st = o * pl.S + pl.unit_offset[unit]
        pieces.append(owner_params[st:st + s])
    return np.concatenate(pieces)[:pl.unit_len[unit]].copy()


def logical_to_storage(pl: Plan, x_logical):
    """[psi_pad] in logical order -> [nd * S] in rank-major owner storage."""
    out = np.empty(pl.nd * pl.S, dtype=x_logical.dtype)
    for o in range(pl.nd):
        for u in range(len(pl.unit_pad)):
            s = pl.unit_shard[u]
            lo = pl.unit_base[u] + o * s
            st = o * pl.S + pl.unit_offset[u]
            out[st:st + s] = x_logical[lo:lo + s]
    return out


def storage_to_logical(pl: Plan, x_storage):
    out = np.empty(pl.psi_pad, dtype=x_storage.dtype)
    for o in range(pl.nd):
        for u in range(len(pl.unit_pad)):
            s = pl.unit_shard[u]
            lo = pl.unit_base[u] + o * s
            st = o * pl.S + pl.unit_offset[u]
            out[lo:lo + s] = x_storage[st:st + s]
    return out


# ------------------------------------------------------------- guarded step
# Not on the pages: the usual mixed-precision guards around an optimizer
# step, as torch.nn.utils.clip_grad_norm_ defines the clip and as dynamic
# loss scaling skips a step whose gradients overflowed.
CLIP_EPS = 1e-6


def guard_coef(norm_sq_gsum, grad_scale, max_norm):
    """Global-norm clip factor of the gradient Adam sees, g = g_sum*s:
    total = |s| * sqrt(sum g_sum^2) (double), c = max_norm / (total + 1e-6),
    clamped to at most 1 and rounded once to fp32.  max_norm <= 0: no clip.
    A non-finite norm leaves the gradient unscaled (c = 1): skip_nonfinite
    is the guard for that case."""
    if max_norm <= 0 or not np.isfinite(norm_sq_gsum):
        return np.float32(1.0)
    total = abs(grad_scale) * np.sqrt(norm_sq_gsum)
    return np.float32(min(1.0, max_norm / (total + CLIP_EPS)))


def step_guarded(pl: Plan, grads, master, m, v, params, adam, t, max_norm,
                 skip_nonfinite, reduced):
    """Two passes.  1: the rank-order reduction of every element into
    `reduced` (owner storage), its sum of squares and non-finite count.
    2: unless skip_nonfinite and some sum is not finite, the step of
    step_partitioned with g = (g_sum*s)*c.  Returns (norm_sq, nonfinite,
    coef, skipped)."""
    norm = 0.0
    bad = 0
    for o in range(pl.nd):
        for u in range(len(pl.unit_pad)):
            s = pl.unit_shard[u]
            lo = pl.unit_base[u] + o * s
            st = o * pl.S + pl.unit_offset[u]
            red = core.reduce(grads[:, lo:lo + s])
            reduced[st:st + s] = red
            r64 = red.astype(np.float64)
            norm += float(np.dot(r64, r64))
            bad += int((~np.isfinite(red)).sum())
    if skip_nonfinite and bad:
        return norm, bad, np.float32(1.0), True
    coef = guard_coef(norm, adam["grad_scale"], max_norm)
    step_partitioned(pl, grads, master, m, v, params, adam, t, clip_coef=coef)
    return norm, bad, coef, False


def reshard(pl_from: Plan, x, pl_to: Plan):
    """A checkpointed owner-storage array under `pl_from`, laid out for
    `pl_to` (same unit lengths): element (unit u, index j < len_u) keeps its
    value; the new padding is zero."""
    assert pl_from.unit_len == pl_to.unit_len
    logical_a = storage_to_logical(pl_from, x)
    logical_b = np.zeros(pl_to.psi_pad, dtype=x.dtype)
    for u, n in enumerate(pl_to.unit_len):
        a0, b0 = pl_from.unit_base[u], pl_to.unit_base[u]
        logical_b[b0:b0 + n] = logical_a[a0:a0 + n]
    return logical_to_storage(pl_to, logical_b)

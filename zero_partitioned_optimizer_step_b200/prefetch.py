"""Stage-3 layer walk with a prefetch window.

At stage 3 each layer is materialised (all-gathered) just before it is used
and released afterwards.  Collective buckets, the prefetch window,
communication buffers and layers not yet released are what make the
temporary memory peaks (concept page "ZeRO", remark under the table "三个阶段";
"使用时应检查" asks for them to be measured).  ``walk_layers`` gathers the next
``depth`` layers on a side stream while the current one is used on the
compute stream.  It releases each layer as soon as its use has been queued,
so at most ``depth + 1`` layers are live; the plan's ``max_live`` must allow
that, and ``ZERO_Q_PEAK_LIVE_*`` report what was reached.

Orchestration only: the gathers are the library's kernel, ordering is CUDA
events between the two streams.
"""
import torch

from . import ZERO_Q_MAX_LIVE, ZERO_Q_UNIT_LEN, zero_gather_layer, zero_release_layer


def walk_layers(plan, owner_params, order, use, depth=1, buffers=None, stream=None,
                side_stream=None):
    """Materialise the units of ``order`` one after the other.

    use(u, layer) is called with a bf16 view of unit u's full layer that is
    ready on ``stream`` (default: the current stream); it must queue its work
    on that stream.  A unit may appear again in ``order`` only after at least
    ``depth + 1`` other entries (walk forward and backward as two calls).
    Returns the ring of ``depth + 1`` layer buffers (reusable via ``buffers``).
    """
    if depth < 0:
        raise ValueError("depth must be >= 0")
    if depth + 1 > plan.query(ZERO_Q_MAX_LIVE):
        raise ValueError("the plan's max_live must be at least depth + 1")
    dev = owner_params.device
    stream = stream or torch.cuda.current_stream(dev)
    side = side_stream or torch.cuda.Stream(dev)
    lens = {u: plan.query(ZERO_Q_UNIT_LEN, u) for u in set(order)}
    nbuf = depth + 1
    if buffers is None:
        biggest = max(lens.values()) if lens else 0
        buffers = [torch.empty(biggest, dtype=torch.bfloat16, device=dev) for _ in range(nbuf)]
    if len(buffers) < nbuf:
        raise ValueError("need depth + 1 buffers")
    ready = [torch.cuda.Event() for _ in range(nbuf)]
    done = [torch.cuda.Event() for _ in range(nbuf)]
    used = [False] * nbuf
    side.wait_stream(stream)            # owner_params are final on `stream`

    def issue(i):
        u, slot = order[i], i % nbuf
        if used[slot]:
            side.wait_event(done[slot])  # the slot's previous layer is used up
        used[slot] = True
        zero_gather_layer(plan, u, owner_params, buffers[slot][:lens[u]], stream=side)
        ready[slot].record(side)

    for i in range(min(depth, len(order))):
        issue(i)
    for i, u in enumerate(order):
        if i + depth < len(order):
            issue(i + depth)
        slot = i % nbuf
        stream.wait_event(ready[slot])
        use(u, buffers[slot][:lens[u]])
        done[slot].record(stream)
        zero_release_layer(plan, u)
    stream.wait_stream(side)
    return buffers

"""The ZeRO step with one rank per GPU of a node.

Each process owns one GPU and one rank's buffers: its full bf16 gradient,
its bf16 parameter replica (stages 1-2) or parameter shard (stage 3), and the
fp32 master, m and v of the shard it owns.  ``PeerStep`` maps every other
rank's gradient and parameter buffer into this process (CUDA IPC; over
NVLink/NVSwitch on a B200 node) and runs the library's fused kernel
``zero_step_peers``: it reads the gradients of the owned shard straight from
the peers, adds them in rank order, runs Adam locally and stores the new
bf16 parameters straight into every peer's replica.  The reduce-scatter and
the all-gather are the kernel's peer loads and stores (mind-map page "ZeRO
真正在做什么：长期分开存，计算时临时拼齐", section "但 GPU 只存四分之一…"); no
collective library moves the data.

What this module adds is ordering between processes: before a step every
rank's gradients must be complete, and after it nobody may read a replica or
overwrite a gradient until every rank's kernel has finished.  With NCCL that
is a one-element all-reduce on the current stream before and after the
kernel (stream-ordered, the host does not block); with gloo the host
synchronises its stream and meets the others at a barrier.

Orchestration only: every byte of the step is moved by the library's kernel.
"""
import torch
import torch.distributed as dist

from . import (zero_gather_layer_peers, zero_ipc_close, zero_ipc_export, zero_ipc_open,
               zero_step_peers)


def _sync_stream():
    if torch.cuda.is_available() and torch.cuda.is_initialized():
        torch.cuda.current_stream().synchronize()


def exchange_handles(buffers, group=None, export=zero_ipc_export):
    """All-gather of IPC handles: returns, per rank, the list of handles of
    that rank's ``buffers`` (bytes each), in the same order."""
    mine = [export(b) for b in buffers]
    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, mine, group=group)
    return out


class PeerStep:
    """One rank of a ZeRO step whose Nd ranks are the Nd processes of `group`.

    plan: a plan of stage 1, 2 or 3 with nd = the group's size.
    grads: this rank's bf16 gradient [psi_pad] (logical order, padding zero).
    params: this rank's bf16 replica [psi_pad] (stages 1-2) or its owner
        shard [S] (stage 3).
    master, exp_avg, exp_avg_sq: this rank's fp32 shard [S].
    The buffers must stay allocated, at the same addresses, until close().
    """

    def __init__(self, plan, grads, params, master, exp_avg, exp_avg_sq, group=None,
                 ipc_open=zero_ipc_open, ipc_close=zero_ipc_close, ipc_export=zero_ipc_export):
        self.group = group
        self.rank = dist.get_rank(group)
        nd = dist.get_world_size(group)
        if plan.nd != nd:
            raise ValueError("the plan has nd=%d but the group has %d ranks" % (plan.nd, nd))
        if plan.stage == 0:
            raise ValueError("stage 0 keeps the full state on every rank; use stage 1, 2 or 3")
        self.plan = plan
        self.master, self.exp_avg, self.exp_avg_sq = master, exp_avg, exp_avg_sq
        self._close = ipc_close
        self.nccl = dist.get_backend(group) == "nccl"
        self._token = torch.zeros(1, dtype=torch.float32,
                                  device=grads.device if self.nccl else "cpu")
        handles = exchange_handles([grads, params], group, ipc_export)
        self.grads, self.params, self._opened = [], [], []
        for q in range(nd):
            if q == self.rank:
                g, p = grads, params
            else:
                g, p = ipc_open(handles[q][0]), ipc_open(handles[q][1])
                self._opened += [g, p]
            self.grads.append(g)
            self.params.append(p)

    def barrier(self):
        """Every rank's queued work up to here is complete before any rank's
        later work runs."""
        if self.nccl:
            dist.all_reduce(self._token, group=self.group)
        else:
            _sync_stream()
            dist.barrier(group=self.group)

    def step(self, adam, t, grad_norm_sq=None, overflow=None, workspace=None, reduced_grad=None,
             adam_consts=None, events=None):
        """Step t on this rank's shard.  If grad_norm_sq / overflow are given
        they hold the global values afterwards (summed / maxed over ranks).
        events: optional pair of CUDA events recorded just before and after
        the kernels (to time them without the barriers)."""
        self.barrier()
        if events is not None:
            events[0].record()
        zero_step_peers(self.plan, self.rank, self.grads, self.params, self.master, self.exp_avg,
                        self.exp_avg_sq, adam, t, reduced_grad=reduced_grad,
                        grad_norm_sq=grad_norm_sq, overflow=overflow, workspace=workspace,
                        adam_consts=adam_consts)
        if events is not None:
            events[1].record()
        self.barrier()
        for x, op in ((grad_norm_sq, dist.ReduceOp.SUM), (overflow, dist.ReduceOp.MAX)):
            if x is None:
                continue
            if self.nccl:
                dist.all_reduce(x, op=op, group=self.group)
            else:
                h = x.cpu()
                dist.all_reduce(h, op=op, group=self.group)
                x.copy_(h)

    def gather_layer(self, unit, full_layer):
        """Stage 3: materialise unit `unit` into full_layer (bf16 [len_u]) from
        every rank's shard; release it with zero_release_layer(plan, unit)."""
        zero_gather_layer_peers(self.plan, unit, self.params, full_layer)

    def close(self):
        """Unmap the peers' buffers; returns once every rank has done so, after
        which each rank may free its own buffers."""
        _sync_stream()
        for p in self._opened:
            self._close(p)
        self._opened = []
        self.grads, self.params = [], []
        if self.nccl:
            dist.all_reduce(self._token, group=self.group)
            _sync_stream()
        else:
            dist.barrier(group=self.group)

"""Replay the ZeRO step as a CUDA graph.

With small buckets the step is bound by launch latency (concept page "ZeRO",
"关键设计取舍" item 1): one launch per bucket.  Capturing the whole step
once and replaying it removes the CPU cost of every launch.  The step's fp32
constants depend on t, so the captured step reads them from a device buffer
(``adam_consts``), which a captured copy refreshes from pinned host memory at
each replay.  Two graphs alternate, so the host can fill the next step's
constants while the previous replay may still be reading its own.

Orchestration only: every kernel is the library's.
"""
import torch

from . import zero_adam_consts, zero_step, zero_step_kernel


class StepGraph:
    """zero_step(plan, ...) captured for replay with a new t each call.

    The tensors passed here are bound into the graph: later steps must write
    new gradients into the same ``grads`` tensor.
    """

    def __init__(self, plan, grads, master, exp_avg, exp_avg_sq, params, adam, **kw):
        dev = master.device
        self.adam = dict(adam)
        zero_step_kernel(plan, kw.get("owner_view", -1))  # per-device set-up, before capture
        self.host = [torch.zeros(16, dtype=torch.float32).pin_memory() for _ in range(2)]
        self.dconst = [torch.zeros(16, dtype=torch.float32, device=dev) for _ in range(2)]
        self.done = [torch.cuda.Event() for _ in range(2)]
        self.used = [False, False]
        self.graphs = []
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        for i in range(2):
            zero_adam_consts(self.adam, 1, self.host[i])
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                self.dconst[i][:9].copy_(self.host[i][:9], non_blocking=True)
                zero_step(plan, grads, master, exp_avg, exp_avg_sq, params, self.adam, 1,
                          stream=side, adam_consts=self.dconst[i], **kw)
            self.graphs.append(g)
        torch.cuda.current_stream(dev).wait_stream(side)
        self.k = 0

    def replay(self, t):
        """Run step t (>= 1) on the current stream."""
        i = self.k % 2
        if self.used[i]:
            self.done[i].synchronize()   # that replay has read its constants
        zero_adam_consts(self.adam, t, self.host[i])
        self.graphs[i].replay()
        self.done[i].record()
        self.used[i] = True
        self.k += 1

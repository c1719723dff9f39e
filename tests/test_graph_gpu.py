"""The step captured as a CUDA graph and replayed for t = 1, 2, 3 gives the
same bits as the eager step, and the oracle's."""
import pytest
import torch

import zero_partitioned_optimizer_step_b200 as Z
from zero_partitioned_optimizer_step_b200.graph import StepGraph
from zero_cases import Case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kernel", ["tma", "ldg"])
@pytest.mark.parametrize("psi,nd,stage,units,bucket", [(1_000_003, 8, 2, None, 1 << 17),
                                                       (400_000, 16, 3, [150_000, 250_000], 1 << 15)])
def test_graph_replay_matches_eager_and_oracle(kernel, psi, nd, stage, units, bucket, monkeypatch):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    monkeypatch.setenv("ZERO_STEP_KERNEL", kernel)
    adam = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.05)
    eager = Case(psi, nd, stage, bucket, units=units, config_id=22, adam=adam)
    graph = Case(psi, nd, stage, bucket, units=units, config_id=22, adam=adam)
    G = torch.empty_like(eager.grads(1))
    sg = StepGraph(graph.lp, G, graph.w, graph.m, graph.v, graph.params, graph.adam,
                   reduced_grad=graph.red, grad_norm_sq=graph.norm, overflow=graph.ovf,
                   workspace=graph.ws)
    for t in (1, 2, 3):
        Gt = eager.grads(t)
        G.copy_(Gt)
        diff = eager.step_and_compare(t, Gt)       # eager path vs oracle
        assert all(v == 0 for v in diff.values()), diff
        sg.replay(t)
        Z.zero_stream_status()
        for x, y in ((eager.w, graph.w), (eager.m, graph.m), (eager.v, graph.v), (eager.red, graph.red)):
            assert torch.equal(x.view(torch.int32), y.view(torch.int32))
        assert torch.equal(eager.params.view(torch.int16), graph.params.view(torch.int16))
        assert eager.norm.item() == graph.norm.item()

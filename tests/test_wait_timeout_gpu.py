"""Failure detection without a GPU fault: make the bulk-copy kernel's bounded
waits run out (one CTA's producer loads nothing, so nothing ever completes
its consumers' barrier) and check that the host reads ZERO_ETIMEOUT, that
the kernel returned on its own, and that the context stays usable."""
import time

import pytest
import torch

import zero_partitioned_optimizer_step_b200 as Z
from zero_cases import Case

pytestmark = pytest.mark.gpu


def test_wait_limit_reports_timeout_and_context_survives(monkeypatch):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    monkeypatch.setenv("ZERO_STEP_KERNEL", "tma")
    c = Case(600_000, 8, 2, 1 << 20, config_id=21)
    G = c.grads(1)
    Z.zero_stream_status()
    monkeypatch.setenv("ZERO_TEST_STALL_PRODUCER", "0")
    t0 = time.time()
    c.run_gpu(G, 1)
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_stream_status()
    waited = time.time() - t0
    assert e.value.status == Z.ZERO_ETIMEOUT
    assert 1.5 < waited < 30.0           # the 2 s limit, then the kernel returned
    # the error word is cleared by the report, and the context still works
    monkeypatch.delenv("ZERO_TEST_STALL_PRODUCER")
    Z.zero_stream_status()
    fresh = Case(600_000, 8, 2, 1 << 20, config_id=21)
    diff = fresh.step_and_compare(1, G)
    assert all(v == 0 for v in diff.values()), diff

"""Stage-3 layer walk with a prefetch window: every layer the user sees is the
oracle's gathered layer, and the live set never exceeds depth + 1."""
import numpy as np
import pytest
import torch

import zero_partitioned_optimizer_step_b200 as Z
from oracle import step as ST
from zero_partitioned_optimizer_step_b200.prefetch import walk_layers
from zero_cases import Case, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.empty_cache()


@pytest.mark.parametrize("depth", [0, 1, 2])
def test_walk_layers_forward_and_backward(depth):
    units = [300_001, 120_000, 5, 250_000, 64, 180_003]
    c = Case(sum(units), 8, 3, 1 << 16, units=units, config_id=19)
    c.step_and_compare(1)
    lp = Z.zero_plan(sum(units), 8, 3, 1 << 16, unit_elems=units, max_live=depth + 1)
    seen = {}
    side = torch.cuda.Stream()

    def use(u, layer):
        # some work on the compute stream that reads the layer
        seen.setdefault(u, []).append(layer.clone())

    n = len(units)
    walk_layers(lp, c.params, list(range(n)), use, depth=depth, side_stream=side)
    bufs = walk_layers(lp, c.params, list(reversed(range(n))), use, depth=depth, side_stream=side)
    torch.cuda.synchronize()
    assert len(bufs) == depth + 1
    for u in range(n):
        want = ST.gather_layer(c.op, u, c.hparams)
        assert len(seen[u]) == 2
        for got in seen[u]:
            assert np.array_equal(u16(got), want)
    assert lp.query(Z.ZERO_Q_LIVE_UNITS) == 0
    assert lp.query(Z.ZERO_Q_PEAK_LIVE_UNITS) == depth + 1
    assert lp.query(Z.ZERO_Q_PEAK_LIVE_BYTES) <= 2 * (depth + 1) * max(units)


def test_walk_layers_needs_max_live():
    units = [1000, 1000, 1000]
    lp = Z.zero_plan(3000, 4, 3, 1024, unit_elems=units, max_live=1)
    owner = torch.zeros(lp.nd * lp.S, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        walk_layers(lp, owner, [0, 1, 2], lambda u, x: None, depth=1)

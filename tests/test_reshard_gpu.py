"""GPU parity of checkpoint resharding (owner storage of one plan to owner
storage of another plan with the same units) against the oracle."""
import numpy as np
import pytest
import torch

import zero_partitioned_optimizer_step_b200 as Z
from oracle import plan as OP
from oracle import step as ST
from zero_cases import Case, f32, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.empty_cache()


PAIRS = [
    # units, (nd, stage, align) from, (nd, stage, align) to
    (None, (8, 2, 64), (3, 2, 64)),
    (None, (16, 2, 64), (64, 1, 8)),
    ([100_000, 7, 250_001], (16, 3, 64), (5, 3, 1)),
    ([100_000, 7, 250_001], (4, 3, 8), (12, 2, 64)),
]


@pytest.mark.parametrize("units,a,b", PAIRS)
def test_reshard_matches_oracle_and_round_trips(units, a, b):
    psi = sum(units) if units else 350_008
    pa_l = Z.zero_plan(psi, a[0], a[1], 1 << 16, align_elems=a[2], unit_elems=units)
    pb_l = Z.zero_plan(psi, b[0], b[1], 1 << 16, align_elems=b[2], unit_elems=units)
    pa = OP.make_plan(psi, a[0], a[1], 1 << 16, align=a[2], unit_elems=units)
    pb = OP.make_plan(psi, b[0], b[1], 1 << 16, align=b[2], unit_elems=units)
    # a state array after a few real steps, so it is not random noise
    c = Case(psi, a[0], a[1], 1 << 16, align=a[2], units=units, config_id=17)
    for t in (1, 2):
        c.step_and_compare(t)
    for src in (c.w, c.m, c.v):
        dst = torch.full((pb.nd * pb.S,), float("nan"), dtype=torch.float32, device="cuda")
        Z.zero_reshard(pa_l, src, pb_l, dst)
        Z.zero_stream_status()
        want = ST.reshard(pa, f32(src), pb)
        assert np.array_equal(f32(dst).view(np.uint32), want.view(np.uint32))
        back = torch.empty_like(src)
        Z.zero_reshard(pb_l, dst, pa_l, back)
        Z.zero_stream_status()
        assert torch.equal(back.view(torch.int32), src.view(torch.int32))
    if a[1] == 3:   # owner parameter shards (bf16) too
        dst = torch.zeros(pb.nd * pb.S, dtype=torch.bfloat16, device="cuda")
        Z.zero_reshard(pa_l, c.params, pb_l, dst)
        Z.zero_stream_status()
        assert np.array_equal(u16(dst), ST.reshard(pa, u16(c.params), pb))


def test_resume_after_reshard_matches_oracle():
    """Step on Nd = 8, reshard the state to Nd = 4, keep stepping there: the
    oracle, fed the same resharded state, agrees."""
    units = [200_000, 50_001]
    psi = sum(units)
    c8 = Case(psi, 8, 3, 1 << 16, units=units, config_id=18)
    c8.step_and_compare(1)
    c_to = Case(psi, 4, 3, 1 << 16, units=units, config_id=18)
    for src, dst in ((c8.w, c_to.w), (c8.m, c_to.m), (c8.v, c_to.v)):
        Z.zero_reshard(c8.lp, src, c_to.lp, dst)
    Z.zero_stream_status()
    c_to.hw, c_to.hm, c_to.hv = f32(c_to.w), f32(c_to.m), f32(c_to.v)
    for t in (2, 3):
        diff = c_to.step_and_compare(t)
        assert all(v == 0 for v in diff.values()), diff

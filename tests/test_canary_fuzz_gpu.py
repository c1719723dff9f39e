"""Memory safety and odd shapes on the GPU.

Canaries: every device buffer a call writes or reads is a slice in the middle
of a larger allocation whose guard zones hold a fixed byte pattern; after the
call the guards must be untouched (an out-of-bounds store would change them).
Fuzz: seeded random plans (units, Nd, alignment, bucket size, stage, one-owner
view) stepped through both K1 paths and compared with the oracle.
"""
import random

import numpy as np
import pytest
import torch

import zero_partitioned_optimizer_step_b200 as Z
from zero_partitioned_optimizer_step_b200 import inputs
from zero_partitioned_optimizer_step_b200.prefetch import walk_layers
from oracle import plan as OP
from oracle import step as ST
from zero_cases import Case, f32, u16

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side
PATTERN = 0xA5


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.empty_cache()


class Guarded:
    """A tensor of `shape`/`dtype` inside a byte buffer with guard zones."""

    def __init__(self, shape, dtype, fill=None):
        n = int(np.prod(shape)) if shape else 1
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.nbytes = nbytes
        self.t = self.raw[GUARD:GUARD + nbytes].view(dtype).view(shape)
        if fill is not None:
            self.t.copy_(fill)

    def intact(self):
        g = torch.cat([self.raw[:GUARD], self.raw[GUARD + self.nbytes:]])
        return bool((g == PATTERN).all())


def _guarded_case(psi, nd, stage, bucket, align, units, owner):
    c = Case(psi, nd, stage, bucket, align=align, units=units, owner_view=owner, config_id=23)
    bufs = {}
    for name in ("w", "m", "v", "red", "params", "norm", "ovf", "ws"):
        x = getattr(c, name)
        g = Guarded(tuple(x.shape), x.dtype, x)
        bufs[name] = g
        setattr(c, name, g.t)
    return c, bufs


SHAPES = [
    (65_536, 4, 2, 16_384, 64, None, -1),
    (100_003, 16, 3, 10_000, 64, [50_000, 3, 50_000], -1),
    (100_003, 7, 3, 999, 1, [10_001, 90_002], -1),
    (250_001, 64, 2, 1 << 14, 64, None, -1),
    (1_000_000, 64, 2, 100_000, 64, None, 63),
    (300_001, 16, 3, 20_000, 64, [100_000, 1, 200_000], 9),
    (77_777, 2, 2, 10_000, 8, None, -1),            # replica rows as bulk copies, ragged tail
    (90_001, 2, 1, 4096, 8, [30_000, 60_001], -1),  # the same, small buckets (cut ring), two units
]


@pytest.mark.parametrize("kernel", ["tma", "ldg"])
@pytest.mark.parametrize("psi,nd,stage,bucket,align,units,owner", SHAPES)
def test_step_writes_stay_inside_their_buffers(kernel, psi, nd, stage, bucket, align, units, owner,
                                               monkeypatch):
    monkeypatch.setenv("ZERO_STEP_KERNEL", kernel)
    c, bufs = _guarded_case(psi, nd, stage, bucket, align, units, owner)
    G = c.grads(1)
    gG = Guarded(tuple(G.shape), G.dtype, G)
    for t in (1, 2):
        c.step_and_compare(t, gG.t if t == 1 else None)
    for name, g in list(bufs.items()) + [("grads", gG)]:
        assert g.intact(), name
    if owner < 0:
        c.guarded_step_and_compare(3, 0.01, True)
        for name, g in bufs.items():
            assert g.intact(), "guarded " + name


def test_gather_reshard_prefetch_stay_inside_their_buffers():
    units = [100_000, 7, 250_001]
    psi = sum(units)
    c, bufs = _guarded_case(psi, 8, 3, 1 << 16, 8, units, -1)
    c.step_and_compare(1)
    layers = [Guarded((n,), torch.bfloat16) for n in units]
    for u in range(3):
        Z.zero_gather_layer(c.lp, u, c.params, layers[u].t)
        Z.zero_release_layer(c.lp, u)
    Z.zero_stream_status()
    for u in range(3):
        assert layers[u].intact()
        assert np.array_equal(u16(layers[u].t), ST.gather_layer(c.op, u, c.hparams))
    to = Z.zero_plan(psi, 5, 3, 1 << 16, align_elems=1, unit_elems=units)
    top = OP.make_plan(psi, 5, 3, 1 << 16, align=1, unit_elems=units)
    dst = Guarded((top.nd * top.S,), torch.float32)
    Z.zero_reshard(c.lp, c.w, to, dst.t)
    pdst = Guarded((top.nd * top.S,), torch.bfloat16)
    Z.zero_reshard(c.lp, c.params, to, pdst.t)
    Z.zero_stream_status()
    assert dst.intact() and pdst.intact()
    assert np.array_equal(f32(dst.t), ST.reshard(c.op, c.hw, top))
    lp2 = Z.zero_plan(psi, 8, 3, 1 << 16, align_elems=8, unit_elems=units, max_live=2)
    ring = [Guarded((max(units),), torch.bfloat16) for _ in range(2)]
    walk_layers(lp2, c.params, [0, 1, 2], lambda u, x: None, depth=1,
                buffers=[g.t for g in ring])
    Z.zero_stream_status()
    assert all(g.intact() for g in ring)
    for name, g in bufs.items():
        assert g.intact(), name


def _random_case(rnd):
    nd = rnd.choice([1, 2, 3, 4, 5, 7, 8, 12, 16, 24, 32, 48, 64, 80])
    align = rnd.choice([1, 2, 8, 64, 64, 64])
    n_units = rnd.choice([1, 1, 2, 3, 5])
    units = [rnd.randint(1, 120_000) for _ in range(n_units)]
    psi = sum(units)
    stage = rnd.randint(0, 3)
    bucket = rnd.choice([7, 1000, 4096, 33_333, 1 << 16, 1 << 20])
    owner = rnd.choice([-1, -1, -1, rnd.randrange(nd)])
    return psi, nd, stage, bucket, align, (units if n_units > 1 else None), owner


@pytest.mark.parametrize("seed", range(16))
def test_random_shapes_match_oracle(seed, monkeypatch):
    rnd = random.Random(1000 + seed)
    psi, nd, stage, bucket, align, units, owner = _random_case(rnd)
    for kernel in ("tma", "ldg"):
        monkeypatch.setenv("ZERO_STEP_KERNEL", kernel)
        c = Case(psi, nd, stage, bucket, align=align, units=units, owner_view=owner,
                 config_id=24 + seed)
        for t in (1, 2):
            diff = c.step_and_compare(t)
            assert all(v == 0 for v in diff.values()), (kernel, diff)


@pytest.mark.parametrize("seed", range(12))
def test_random_guarded_shapes_match_oracle(seed, monkeypatch):
    """The guarded step on seeded random plans (all ranks' view), with a clip
    threshold that clips, one that does not, or none, through every kernel
    its second pass can take: the bulk-copy ring (ZERO_STEP_KERNEL=tma), the
    replica rows as bulk copies from shared memory (ldg), and per-thread
    stores (ldst)."""
    rnd = random.Random(5000 + seed)
    psi, nd, stage, bucket, align, units, _ = _random_case(rnd)
    stage = max(stage, 1)   # the oracle's guarded step is the partitioned one
    bucket = max(bucket, 1000)   # two passes of 7-element buckets: too many launches for a test
    max_norm = rnd.choice([0.0, 1e-4, 1e-4, 1e9])
    for second in ("tma", "ldg", "ldst"):
        monkeypatch.setenv("ZERO_STEP_KERNEL", "ldg" if second == "ldst" else second)
        if second == "ldst":
            monkeypatch.setenv("ZERO_GUARD_APPLY", "ldst")
        else:
            monkeypatch.delenv("ZERO_GUARD_APPLY", raising=False)
        c = Case(psi, nd, stage, bucket, align=align, units=units, config_id=60 + seed)
        for t in (1, 2):
            diff, coef, skipped = c.guarded_step_and_compare(t, max_norm, True)   # tolerances
            assert not skipped
            if max_norm == 1e-4:
                assert coef < 1
            else:   # no clipping: the same bits as the definition
                assert coef == 1 and all(v == 0 for v in diff.values()), (second, diff)

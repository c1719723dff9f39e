"""GPU parity of the fused ZeRO step (CUDA path through the C ABI) against the
CPU oracle, element by element, on sizes the oracle finishes in seconds."""
import numpy as np
import pytest
import torch

import zero_partitioned_optimizer_step_b200 as Z
from oracle import step as ST
from zero_cases import Case, bf16_ulp_check, f32, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()
    yield
    torch.cuda.empty_cache()


@pytest.fixture(params=["tma", "ldg"])
def kernel(request, monkeypatch):
    """Run the test with the bulk-copy (TMA) kernel and with the 16-byte
    vector-load kernel for aligned bucket bodies."""
    monkeypatch.setenv("ZERO_STEP_KERNEL", request.param)
    yield request.param
    Z.zero_stream_status()


@pytest.mark.parametrize("stage", [0, 1, 2, 3])
def test_toy_four_ranks_bit_exact(stage, kernel):
    """The four-rank A/B/C/D toy, 3 steps: every output bit-identical to the
    oracle (which is itself pinned to equal replicated Adam)."""
    c = Case(65_536, 4, stage, 16_384, sigma=0.01, config_id=1)
    for t in (1, 2, 3):
        diff = c.step_and_compare(t)
        assert all(v == 0 for v in diff.values()), diff
    if stage <= 2:
        P = u16(c.params)
        for r in range(1, 4):
            assert np.array_equal(P[r], P[0])
    else:
        full = torch.empty(65_536, dtype=torch.bfloat16, device="cuda")
        Z.zero_gather_layer(c.lp, 0, c.params, full)
        torch.cuda.synchronize()
        assert np.array_equal(u16(full), ST.gather_layer(c.op, 0, c.hparams))
        Z.zero_release_layer(c.lp, 0)


RAGGED = [
    # psi, nd, stage, bucket, align, units
    (1, 1, 2, 8, 64, None),
    (7, 2, 2, 3, 1, None),
    (63, 3, 1, 8, 4, None),
    (65, 5, 0, 17, 1, None),
    (1000, 8, 2, 64, 8, None),
    (1000, 8, 3, 64, 8, [333, 667]),
    (100_003, 16, 2, 4_099, 64, None),
    (100_003, 16, 3, 10_000, 64, [50_000, 3, 50_000]),
    (100_003, 7, 3, 999, 1, [10_001, 90_002]),
    (250_001, 64, 2, 1 << 14, 64, None),
    (250_001, 64, 3, 1 << 20, 8, [1, 125_000, 125_000]),
    (1_234_567, 3, 2, 300_001, 8, None),
    (1_234_567, 8, 3, 1 << 18, 64, [1_000_000, 234_567]),
]


@pytest.mark.parametrize("psi,nd,stage,bucket,align,units", RAGGED)
def test_ragged_shapes(psi, nd, stage, bucket, align, units, kernel):
    """Odd sizes, scalar and vector paths, bucket heads and tails, several
    units (owner storage != logical order), Nd from 1 to 64."""
    c = Case(psi, nd, stage, bucket, align=align, units=units, config_id=7)
    for t in (1, 2):
        c.step_and_compare(t)


@pytest.mark.parametrize("owner", [0, 5, 63])
def test_owner_view(owner, kernel):
    """One owner's shard with its slices of all 64 ranks' gradients."""
    c = Case(1_000_000, 64, 2, 100_000, owner_view=owner, config_id=4)
    for t in (1, 2, 3):
        diff = c.step_and_compare(t)
        assert all(v == 0 for v in diff.values()), diff


def test_owner_view_multi_unit(kernel):
    c = Case(300_001, 16, 3, 20_000, units=[100_000, 1, 200_000], owner_view=9, config_id=4)
    for t in (1, 2):
        c.step_and_compare(t)


def test_bucket_calls_compose(kernel):
    """zero_step_buckets over pieces == zero_step in one call, norm included."""
    a = Case(500_000, 8, 2, 40_000, config_id=2)
    b = Case(500_000, 8, 2, 40_000, config_id=2)
    nb = a.lp.n_buckets
    for t in (1, 2):
        G = a.grads(t)
        a.run_gpu(G, t)
        cuts = [0, 1, 5, nb - 1, nb]
        for lo, hi in zip(cuts[:-1], cuts[1:]):
            Z.zero_step_buckets(b.lp, G, b.w, b.m, b.v, b.params, b.adam, t, lo, hi - lo,
                                grad_norm_sq=b.norm, overflow=b.ovf, workspace=b.ws,
                                reduced_grad=b.red)
        torch.cuda.synchronize()
        for x, y in ((a.w, b.w), (a.m, b.m), (a.v, b.v), (a.red, b.red)):
            assert torch.equal(x.view(torch.int32), y.view(torch.int32))
        assert torch.equal(a.params.view(torch.int16), b.params.view(torch.int16))
        assert a.norm.item() == b.norm.item()


def test_norm_and_overflow_flag(kernel):
    c = Case(200_000, 4, 2, 50_000, config_id=6)
    G = c.grads(1)
    G[1, 123] = float("inf")
    G[2, 777] = float("nan")
    diff = c.step_and_compare(1, G)
    assert int(c.ovf.item()) == 1
    assert np.isinf(f32(c.red)[123]) and np.isnan(f32(c.red)[777])
    G = c.grads(2)
    c.step_and_compare(2, G)
    # element 123 / 777 state is NaN from step 1 on; the flag follows step 2's
    # gradients only
    assert int(c.ovf.item()) == 0


@pytest.mark.parametrize("scale", [1e22, 1e-22, "mixed"])
def test_norm_at_extreme_magnitudes(scale, kernel):
    """Reduced gradients whose squares leave the fp32 range: all of them
    (|g_sum| near 1e19, squares past fp32's maximum; |g_sum| near 1e-25,
    squares below its smallest subnormal), or one column in 16 scaled up
    among ordinary values.  The norm is a double-precision sum of squares,
    so it must match the oracle's and stay finite: a square taken in fp32
    would overflow or vanish here."""
    c = Case(100_000, 4, 2, 30_000, config_id=7)
    G = c.grads(1).float()
    if scale == "mixed":
        G[:, ::16] *= 1e22
    else:
        G *= scale
    G = G.to(torch.bfloat16)
    c.step_and_compare(1, G)
    n = c.norm.item()
    assert np.isfinite(n) and n > 0 and int(c.ovf.item()) == 0


def test_subnormal_gradients(kernel):
    """bf16 subnormal gradients (exponent field 0): their fp32 sums, the
    gradient Adam sees and the first moment are fp32 subnormals, and the
    second moment underflows to zero.  Every operation must keep subnormals
    as IEEE arithmetic does (no flush to zero), packed pairs included."""
    c = Case(50_000, 4, 2, 16_384, config_id=8)
    gen = torch.Generator(device="cuda").manual_seed(8)
    n = c.op.psi_pad
    mant = torch.randint(1, 128, (4, n), generator=gen, device="cuda", dtype=torch.int32)
    sign = torch.randint(0, 2, (4, n), generator=gen, device="cuda", dtype=torch.int32) << 15
    G = (mant | sign).to(torch.int16).view(torch.bfloat16)
    G[:, 50_000:] = 0                     # padding
    for t in (1, 2):
        diff = c.step_and_compare(t, G)
        assert all(v == 0 for v in diff.values()), diff
    m = f32(c.m)[:50_000]
    assert np.count_nonzero((m != 0) & (np.abs(m) < np.finfo(np.float32).tiny)) > 1000


def test_norm_is_deterministic(kernel):
    c = Case(300_000, 8, 2, 30_000, config_id=6, with_reduced=False)
    G = c.grads(1)
    vals = set()
    for _ in range(3):
        c.run_gpu(G, 1)
        torch.cuda.synchronize()
        vals.add(c.norm.item())
    assert len(vals) == 1


def test_zero_gradient_keeps_state_and_padding(kernel):
    c = Case(10_001, 8, 2, 4096, config_id=5)
    G = torch.zeros((8, c.op.psi_pad), dtype=torch.bfloat16, device="cuda")
    w0 = f32(c.w).copy()
    c.step_and_compare(1, G)
    assert np.array_equal(f32(c.w), w0) and not f32(c.m).any() and not f32(c.v).any()
    pad = f32(c.w)[10_001:]
    assert not pad.any()


def test_gather_release_liveness():
    units = [5_000, 7_000, 3_000]
    c = Case(15_000, 4, 3, 2_048, units=units, config_id=3)
    c.step_and_compare(1)
    bufs = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for n in units]
    Z.zero_gather_layer(c.lp, 0, c.params, bufs[0])
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_gather_layer(c.lp, 1, c.params, bufs[1])   # max_live = 1
    assert e.value.status == Z.ZERO_ESTATE
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_gather_layer(c.lp, 0, c.params, bufs[0])   # already live
    assert e.value.status == Z.ZERO_ESTATE
    assert c.lp.query(Z.ZERO_Q_LIVE_UNITS) == 1
    Z.zero_release_layer(c.lp, 0)
    # forward order, then backward order
    for u in [0, 1, 2, 2, 1, 0]:
        Z.zero_gather_layer(c.lp, u, c.params, bufs[u])
        torch.cuda.synchronize()
        assert np.array_equal(u16(bufs[u]), ST.gather_layer(c.op, u, c.hparams))
        Z.zero_release_layer(c.lp, u)
    assert c.lp.query(Z.ZERO_Q_PEAK_LIVE_UNITS) == 1
    assert c.lp.query(Z.ZERO_Q_PEAK_LIVE_BYTES) == 2 * max(units)
    with pytest.raises(Z.ZeroError):
        Z.zero_release_layer(c.lp, 1)


def test_gather_max_live_two():
    units = [4_096, 4_096, 4_096]
    lp = Z.zero_plan(sum(units), 4, 3, 4096, unit_elems=units, max_live=2)
    owner = torch.arange(lp.nd * lp.S, dtype=torch.float32, device="cuda").to(torch.bfloat16)
    bufs = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for n in units]
    Z.zero_gather_layer(lp, 0, owner, bufs[0])
    Z.zero_gather_layer(lp, 1, owner, bufs[1])
    with pytest.raises(Z.ZeroError):
        Z.zero_gather_layer(lp, 2, owner, bufs[2])
    Z.zero_release_layer(lp, 0)
    Z.zero_gather_layer(lp, 2, owner, bufs[2])
    assert lp.query(Z.ZERO_Q_PEAK_LIVE_UNITS) == 2


def test_gather_odd_alignment_scalar_path():
    units = [1_001, 77, 5]
    lp = Z.zero_plan(sum(units), 3, 3, 100, align_elems=1, unit_elems=units)
    from oracle import plan as OP
    op = OP.make_plan(sum(units), 3, 3, 100, align=1, unit_elems=units)
    owner = (torch.randn(lp.nd * lp.S, device="cuda")).to(torch.bfloat16)
    host = u16(owner)
    for u, n in enumerate(units):
        buf = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        Z.zero_gather_layer(lp, u, owner, buf)
        torch.cuda.synchronize()
        assert np.array_equal(u16(buf), ST.gather_layer(op, u, host))
        Z.zero_release_layer(lp, u)


def test_library_errors_on_device_calls():
    c = Case(1000, 4, 2, 100, config_id=0)
    G = c.grads(1)
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_step(c.lp, G, c.w, c.m, c.v, c.params, c.adam, 0)
    assert e.value.status == Z.ZERO_EINVAL
    with pytest.raises(Z.ZeroError):
        Z.zero_step(c.lp, G[:, 1:], c.w, c.m, c.v, c.params, c.adam, 1)   # misaligned
    with pytest.raises(ValueError):
        Z.zero_step(c.lp, G.float(), c.w, c.m, c.v, c.params, c.adam, 1)


def test_kernels_agree_bitwise_large_nd():
    """Nd = 64 and Nd = 100 (ring of 3 and 2 stages): both vector kernels give
    the same bits."""
    import os
    for nd in (64, 100):
        outs = []
        for k in ("tma", "ldg"):
            os.environ["ZERO_STEP_KERNEL"] = k
            try:
                c = Case(300_000, nd, 2, 1 << 20, config_id=9, with_reduced=True)
                G = c.grads(1)
                c.run_gpu(G, 1)
                Z.zero_stream_status()
                outs.append([f32(c.w), f32(c.m), f32(c.v), f32(c.red), u16(c.params), c.norm.item()])
            finally:
                del os.environ["ZERO_STEP_KERNEL"]
        for x, y in zip(outs[0][:5], outs[1][:5]):
            assert np.array_equal(x, y)
        assert outs[0][5] == pytest.approx(outs[1][5], rel=1e-12)


@pytest.mark.parametrize("cw", ["8", "16"])
@pytest.mark.parametrize("vw", ["2", "4", "8"])
@pytest.mark.parametrize("psi,nd,stage,units,owner", [
    (700_001, 8, 2, None, -1), (600_000, 16, 3, [200_000, 1_000, 399_000], -1),
    (500_000, 64, 2, None, 7), (300_007, 2, 2, None, -1)])
def test_bulk_kernel_vector_widths(cw, vw, psi, nd, stage, units, owner, monkeypatch):
    """The bulk-copy kernel with 2, 4 and 8 elements per consumer thread, and
    8 or 16 consumer warps."""
    monkeypatch.setenv("ZERO_STEP_KERNEL", "tma")
    monkeypatch.setenv("ZERO_TMA_VW", vw)
    monkeypatch.setenv("ZERO_TMA_CW", cw)
    c = Case(psi, nd, stage, 1 << 18, units=units, owner_view=owner, config_id=11)
    for t in (1, 2):
        diff = c.step_and_compare(t)
        assert all(v == 0 for v in diff.values()), diff


@pytest.mark.parametrize("vw", ["2", "4", "8"])
@pytest.mark.parametrize("psi,nd,units,bucket", [
    (700_001, 8, None, 1 << 18), (300_007, 2, None, 1 << 18), (500_000, 64, None, 1 << 18),
    (600_000, 6, [200_000, 8, 399_992], 1 << 16), (50_000, 16, None, 4096)])
def test_bulk_kernel_replica_rows_as_bulk_copies(vw, psi, nd, units, bucket, monkeypatch):
    """The bulk-copy kernel with its replica rows written as 1-D bulk copies
    from shared memory (ZERO_TMA_BULKP=1), stage 2: the same bits as the
    oracle (several units: an owner map; small buckets: the cut ring)."""
    monkeypatch.setenv("ZERO_STEP_KERNEL", "tma")
    monkeypatch.setenv("ZERO_TMA_VW", vw)
    monkeypatch.setenv("ZERO_TMA_BULKP", "1")
    c = Case(psi, nd, 2, bucket, units=units, align=8 if units else 64, config_id=17)
    for t in (1, 2):
        diff = c.step_and_compare(t)
        assert all(v == 0 for v in diff.values()), diff

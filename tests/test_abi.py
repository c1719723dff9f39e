"""Host-side tests of libzero.so: it loads, exports every symbol the header
declares, and its planner / accounting is bit-exact to the oracle's maps.
No kernel is launched here."""
import ctypes
import os
import random
import re

import pytest
import torch

import zero_partitioned_optimizer_step_b200 as Z
from oracle import plan as OP

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zero.h")


def header_functions():
    src = open(HEADER, encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(zero_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_function():
    L = Z.lib()
    names = header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    assert L.zero_abi_version() == 4


def test_status_strings():
    L = Z.lib()
    for s in range(6):
        assert L.zero_status_str(s).decode().startswith("ZERO_")


def lib_plan_tables(pl):
    units = pl.units()
    return dict(psi=pl.psi, psi_pad=pl.psi_pad, S=pl.S,
                pad=[u[1] for u in units], shard=[u[2] for u in units],
                base=[u[3] for u in units], off=[u[4] for u in units],
                buckets=pl.buckets())


def check_against_oracle(psi, nd, stage, bucket, align, units, every_index=True):
    lp = Z.zero_plan(psi, nd, stage, bucket, align_elems=align, unit_elems=units)
    op = OP.make_plan(psi, nd, stage, bucket, align=align, unit_elems=units)
    t = lib_plan_tables(lp)
    assert (t["psi_pad"], t["S"]) == (op.psi_pad, op.S)
    assert t["pad"] == op.unit_pad and t["shard"] == op.unit_shard
    assert t["base"] == op.unit_base and t["off"] == op.unit_offset
    assert t["buckets"] == op.buckets
    idx = range(op.psi_pad) if every_index else \
        sorted({0, op.psi_pad - 1, *random.Random(psi).sample(range(op.psi_pad), min(200, op.psi_pad))})
    for p in idx:
        _, o, off, _ = OP.locate(op, p)
        assert lp.query(Z.ZERO_Q_OWNER, p) == o
        assert lp.query(Z.ZERO_Q_OWNER_OFFSET, p) == off
    for s in range(4):
        assert lp.query(Z.ZERO_Q_MEM_BYTES_PER_RANK, s) == OP.memory_bytes_per_rank_padded(op, s)
    assert Z.zero_bytes_moved(lp, Z.ZERO_BYTES_COMM_ELEMS_PER_RANK) == OP.comm_elems_per_rank(op)
    assert Z.zero_bytes_moved(lp, Z.ZERO_BYTES_COMM_PER_RANK) == OP.comm_bytes_per_rank(op)
    assert Z.zero_bytes_moved(lp, Z.ZERO_BYTES_HBM_STEP) == OP.hbm_step_bytes(op)
    assert Z.zero_bytes_moved(lp, Z.ZERO_BYTES_HBM_STEP, Z.ZERO_BYTES_FLAG_OWNER_VIEW) == \
        OP.hbm_step_bytes(op, owner_view=True)
    assert Z.zero_bytes_moved(lp, Z.ZERO_BYTES_HBM_STEP, Z.ZERO_BYTES_FLAG_REDUCED) == \
        OP.hbm_step_bytes(op, with_reduced=True)
    assert Z.zero_bytes_moved(lp, Z.ZERO_BYTES_HBM_GATHER_STEP) == OP.hbm_gather_bytes(op)
    for q, what in ((Z.ZERO_Q_STATE_REPLICAS, "state"), (Z.ZERO_Q_GRAD_REPLICAS, "grad"),
                    (Z.ZERO_Q_PARAM_REPLICAS, "param")):
        assert lp.query(q) == OP.replicas(op, what)
    if every_index:
        for r in range(nd):
            assert lp.query(Z.ZERO_Q_LOST_RANK_UNRECOVERABLE, r) == OP.lost_rank_unrecoverable(op, r)
    assert Z.zero_bytes_moved(lp, Z.ZERO_BYTES_HBM_GUARDED_STEP) == OP.hbm_guarded_step_bytes(op)
    assert Z.zero_bytes_moved(lp, Z.ZERO_BYTES_HBM_GUARDED_STEP, Z.ZERO_BYTES_FLAG_OWNER_VIEW) == \
        OP.hbm_guarded_step_bytes(op, owner_view=True)


def test_plan_bit_exact_to_oracle_bruteforce():
    rnd = random.Random(11)
    n = 0
    for psi in range(1, 65):
        for nd in (1, 2, 3, 5, 8, 16, 64):
            for align in (1, 4, 64):
                k = rnd.randint(1, min(4, psi))
                cuts = sorted(rnd.sample(range(1, psi), k - 1)) if k > 1 else []
                units = [b - a for a, b in zip([0] + cuts, cuts + [psi])]
                check_against_oracle(psi, nd, rnd.randint(0, 3), rnd.choice([1, 5, 8, 100]),
                                     align, units)
                n += 1
    assert n == 64 * 7 * 3


@pytest.mark.parametrize("name", ["toy", "gpt2_small", "stage3_1p3b", "owner_7p5b", "sweep"])
def test_plan_bit_exact_to_oracle_configs(name):
    if name == "toy":
        check_against_oracle(65536, 4, 2, 4096, 64, None)
    elif name == "gpt2_small":
        check_against_oracle(124_439_808, 8, 2, 25_000_000, 64, None, every_index=False)
    elif name == "stage3_1p3b":
        units = [107_120_640] + [50_358_272] * 24 + [4096]
        check_against_oracle(sum(units), 16, 3, 1 << 27, 64, units, every_index=False)
    elif name == "owner_7p5b":
        check_against_oracle(7_500_000_000, 64, 2, 25_000_000, 64, None, every_index=False)
    else:
        for nd in (2, 4, 8, 16, 64):
            for mb in (1, 64, 512):
                check_against_oracle(500_000_000, nd, 2, mb << 19, 64, None, every_index=False)


def test_memory_table_from_library_matches_pages():
    pl = Z.zero_plan(7_500_000_000, 64, 2, 25_000_000, align_elems=1)
    got = [pl.query(Z.ZERO_Q_MEM_BYTES_PER_RANK, s) for s in range(4)]
    assert got == [120_000_000_000, 31_406_250_000, 16_640_625_000, 1_875_000_000]


def test_invalid_plans_are_rejected():
    bad = [dict(psi=0, nd=4, stage=2, bucket_elems=8),
           dict(psi=10, nd=0, stage=2, bucket_elems=8),
           dict(psi=10, nd=4, stage=4, bucket_elems=8),
           dict(psi=10, nd=4, stage=2, bucket_elems=0),
           dict(psi=10, nd=4, stage=3, bucket_elems=8, unit_elems=[3, 3]),
           dict(psi=10, nd=4, stage=3, bucket_elems=8, unit_elems=[10, 0]),
           dict(psi=(1 << 64) - 1, nd=1 << 20, stage=2, bucket_elems=8, align_elems=1 << 20)]
    for kw in bad:
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_plan(**kw)
        assert e.value.status == Z.ZERO_EINVAL, kw


def test_query_out_of_range():
    pl = Z.zero_plan(1000, 4, 3, 100, unit_elems=[600, 400])
    for what, idx in ((Z.ZERO_Q_UNIT_LEN, 2), (Z.ZERO_Q_BUCKET_BEGIN, pl.n_buckets),
                      (Z.ZERO_Q_OWNER, pl.psi_pad), (Z.ZERO_Q_MEM_BYTES_PER_RANK, 4),
                      (999, 0)):
        with pytest.raises(Z.ZeroError) as e:
            pl.query(what, idx)
        assert e.value.status == Z.ZERO_EINVAL


def test_release_and_gather_state_errors_on_host():
    pl = Z.zero_plan(1000, 4, 3, 100, unit_elems=[600, 400])
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_release_layer(pl, 0)
    assert e.value.status == Z.ZERO_ESTATE
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_release_layer(pl, 2)
    assert e.value.status == Z.ZERO_EINVAL
    L = Z.lib()
    # gather argument checks run before any CUDA call
    assert L.zero_gather_layer(pl.handle, 5, ctypes.c_void_p(256), ctypes.c_void_p(512), None) == Z.ZERO_EINVAL
    assert L.zero_gather_layer(pl.handle, 0, None, ctypes.c_void_p(512), None) == Z.ZERO_EINVAL
    assert L.zero_gather_layer(pl.handle, 0, ctypes.c_void_p(258), ctypes.c_void_p(512), None) == Z.ZERO_EINVAL
    pl2 = Z.zero_plan(1000, 4, 2, 100)
    assert L.zero_gather_layer(pl2.handle, 0, ctypes.c_void_p(256), ctypes.c_void_p(512), None) == Z.ZERO_EINVAL
    assert pl.query(Z.ZERO_Q_LIVE_UNITS) == 0


def _fake_bufs(pl, **over):
    b = Z._Bufs()
    b.grads, b.master, b.exp_avg, b.exp_avg_sq, b.params = 4096, 8192, 12288, 16384, 20480
    b.grad_stride = pl.psi_pad
    b.param_stride = pl.psi_pad
    b.owner_view = -1
    for k, v in over.items():
        setattr(b, k, v)
    return b


def test_step_argument_checks_on_host():
    """Invalid arguments are rejected before anything touches the device."""
    L = Z.lib()
    pl = Z.zero_plan(1000, 4, 2, 100)
    adam = Z.make_adam(dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, grad_scale=0.25))

    def call(b, t=1, a=adam, first=0, count=None):
        count = pl.n_buckets if count is None else count
        return L.zero_step_buckets(pl.handle, ctypes.byref(b), ctypes.byref(a), t, first, count, None)

    assert call(_fake_bufs(pl), t=0) == Z.ZERO_EINVAL
    assert call(_fake_bufs(pl, grads=None)) == Z.ZERO_EINVAL
    assert call(_fake_bufs(pl, master=8200)) == Z.ZERO_EINVAL          # misaligned
    assert call(_fake_bufs(pl, grad_stride=pl.psi_pad - 8)) == Z.ZERO_EINVAL
    assert call(_fake_bufs(pl, param_stride=8)) == Z.ZERO_EINVAL
    assert call(_fake_bufs(pl, owner_view=4)) == Z.ZERO_EINVAL
    assert call(_fake_bufs(pl, grad_norm_sq=24576)) == Z.ZERO_EINVAL    # no workspace
    assert call(_fake_bufs(pl), first=1, count=pl.n_buckets) == Z.ZERO_EINVAL
    bad = Z.make_adam(dict(lr=1e-3, beta1=1.0, beta2=0.999, eps=1e-8, grad_scale=1.0))
    assert call(_fake_bufs(pl), a=bad) == Z.ZERO_EINVAL
    bad = Z.make_adam(dict(lr=float("nan"), beta1=0.9, beta2=0.999, eps=1e-8, grad_scale=1.0))
    assert call(_fake_bufs(pl), a=bad) == Z.ZERO_EINVAL
    assert L.zero_step(None, ctypes.byref(_fake_bufs(pl)), ctypes.byref(adam), 1, None) == Z.ZERO_EINVAL
    assert "t must be" in (call(_fake_bufs(pl), t=0) and L.zero_last_error().decode())


@pytest.mark.skipif(torch.cuda.is_available(), reason="needs a machine without a CUDA device")
def test_valid_step_without_device_reports_ecuda():
    L = Z.lib()
    pl = Z.zero_plan(1000, 4, 2, 100)
    adam = Z.make_adam(dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, grad_scale=0.25))
    assert L.zero_step(pl.handle, ctypes.byref(_fake_bufs(pl)), ctypes.byref(adam), 1, None) == Z.ZERO_ECUDA


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "zero_partitioned_optimizer_step_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cpp", ".h")):
                src = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"\boracle\b\s*(import|\.)|from\s+oracle|liboracle", src), f


def test_reshard_argument_checks_on_host():
    L = Z.lib()
    a = Z.zero_plan(1000, 4, 2, 100, unit_elems=[400, 600])
    b = Z.zero_plan(1000, 3, 3, 100, unit_elems=[400, 600])
    c = Z.zero_plan(1000, 3, 3, 100, unit_elems=[500, 500])
    ok = ctypes.c_void_p(4096)
    assert L.zero_reshard(a.handle, ok, c.handle, ctypes.c_void_p(8192), 4, None) == Z.ZERO_EINVAL
    assert L.zero_reshard(a.handle, ok, b.handle, ctypes.c_void_p(8192), 8, None) == Z.ZERO_EINVAL
    assert L.zero_reshard(a.handle, None, b.handle, ctypes.c_void_p(8192), 4, None) == Z.ZERO_EINVAL
    assert L.zero_reshard(a.handle, ctypes.c_void_p(4098), b.handle, ctypes.c_void_p(8192), 4,
                          None) == Z.ZERO_EINVAL


def test_plain_c_caller(tmp_path):
    """A C program (tests/c/plan_example.c) compiled against include/zero.h
    and linked to libzero.so gets the oracle's plan through the C ABI."""
    lib_dir = os.path.dirname(Z.LIB_PATH)
    exe = tmp_path / "plan_example"
    import subprocess
    subprocess.run(["gcc", "-std=c99", "-O1", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "plan_example.c"), "-L", lib_dir, "-lzero",
                    "-Wl,-rpath," + lib_dir, "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    got = {}
    for line in out.splitlines():
        k, v = line.split(" ", 1)
        got[k] = v
    op = OP.make_plan(124_439_808, 8, 2, 25_000_000)
    assert int(got["gpt2.psi_pad"]) == op.psi_pad and int(got["gpt2.S"]) == op.S
    assert int(got["gpt2.n_buckets"]) == len(op.buckets)
    assert int(got["gpt2.comm_elems"]) == OP.comm_elems_per_rank(op)
    assert int(got["gpt2.hbm_step"]) == OP.hbm_step_bytes(op, False, False)
    for st in range(4):
        assert int(got["gpt2.mem_stage%d" % st]) == OP.memory_bytes_per_rank_padded(op, st)
    assert int(got["gpt2.owner_of_77777777"]) == OP.locate(op, 77_777_777)[1]
    o3 = OP.make_plan(350_008, 5, 3, 65_536, align=8, unit_elems=[100_000, 7, 250_001])
    for u in range(3):
        assert got["st3.unit%d" % u] == "%d %d %d" % (o3.unit_pad[u], o3.unit_shard[u], o3.unit_offset[u])
    assert got["st3.release_unheld"] == "%d ESTATE" % Z.ZERO_ESTATE
    assert got["abi"] == "4"


try:
    from hypothesis import HealthCheck, given, settings, strategies as st
except ImportError:  # pragma: no cover
    given = None


if given is not None:
    @settings(max_examples=120, deadline=None, suppress_health_check=[HealthCheck.too_slow])
    @given(nd=st.integers(1, 300), stage=st.integers(0, 3), align=st.sampled_from([1, 2, 3, 8, 64, 100]),
           units=st.lists(st.integers(1, 5_000_000), min_size=1, max_size=6), data=st.data())
    def test_plan_matches_oracle_on_random_plans(nd, stage, align, units, data):
        """Random plans (up to 300 ranks, 6 units, odd alignments and bucket
        sizes, at most ~2000 buckets each): every table, sampled owners and
        every byte count as the oracle's maps give them."""
        psi = sum(units)
        bucket = data.draw(st.integers(max(1, psi // 2000), max(1, psi + 1000)))
        check_against_oracle(psi, nd, stage, bucket, align, units if len(units) > 1 else None,
                             every_index=False)

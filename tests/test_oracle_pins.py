"""Pins of the CPU oracle against things other than itself.

Each test ties an oracle function to a value the pages print, a closed form,
an independent library routine (torch's Adam, torch's bf16 conversion), exact
rational arithmetic, or brute force on tiny inputs.  None of them needs a GPU.
"""
import math
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import read_golden
from oracle import core
from oracle import plan as P
from oracle import step as ST
from oracle.adam_fp64 import adam_fp64

ADAM = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, grad_scale=0.25)


def f32_ulp(x):
    x = np.abs(np.asarray(x, dtype=np.float32))
    return np.spacing(np.maximum(x, np.float32(np.finfo(np.float32).tiny)))


def rand_bf16(rng, shape, sigma):
    x = (rng.standard_normal(shape) * sigma).astype(np.float32)
    return core.bf16_rne(x)


# ---------------------------------------------------------------- memory
def test_memory_table_matches_printed_values():
    rows = {r[0]: r[1] for r in read_golden("memory_table_7p5b_nd64.txt")}
    psi, nd = int(rows["psi"]), int(rows["nd"])
    for st in range(4):
        gb = P.memory_bytes_per_rank(st, psi, nd, 12) / Fraction(10 ** 9)
        assert round(float(gb), 1) == float(rows["stage%d_gb" % st]), st


def test_memory_table_exact_values_and_padded_plan():
    psi, nd = 7_500_000_000, 64
    exact = [Fraction(120), Fraction(3140625, 100000), Fraction(16640625, 1000000),
             Fraction(1875, 1000)]
    for st in range(4):
        assert P.memory_bytes_per_rank(st, psi, nd) == exact[st] * 10 ** 9
    # Nd divides Psi, so with A = 1 the padded plan allocates exactly that.
    pl = P.make_plan(psi, nd, 2, 25_000_000, align=1)
    assert pl.psi_pad == psi and pl.S == psi // nd
    for st in range(4):
        assert P.memory_bytes_per_rank_padded(pl, st) == exact[st] * 10 ** 9
    # With A = 64 the padding adds < Nd*A elements.
    pl64 = P.make_plan(psi, nd, 2, 25_000_000, align=64)
    assert pl64.psi_pad == 7_500_001_280 and pl64.S == 117_187_520


# ---------------------------------------------------------- communication
def test_comm_volume_limits_and_ratio():
    rows = {r[0]: Fraction(r[1]) for r in read_golden("comm_volume.txt")}
    psi = 2 ** 40
    for nd in (2, 4, 64, 1024, 2 ** 16):
        per_stage = {}
        for st in range(4):
            pl = P.make_plan(psi, nd, st, 2 ** 30, align=1)
            c = P.comm_elems_per_rank(pl)
            per_stage[st] = c
            want = rows["stage%d_psi" % st]
            # ring: the printed multiple of Psi times (Nd-1)/Nd, exactly
            assert Fraction(c, psi) == want * Fraction(nd - 1, nd)
        assert Fraction(per_stage[3], per_stage[0]) == rows["ratio_stage3_over_stage0"]
    # the printed 2 Psi / 3 Psi are the limit as Nd grows
    pl = P.make_plan(psi, 2 ** 20, 3, 2 ** 30, align=1)
    assert abs(Fraction(P.comm_elems_per_rank(pl), psi) - 3) < Fraction(1, 10 ** 5)


# ------------------------------------------------------------ ownership
def test_toy_four_rank_ownership():
    rows = read_golden("toy_ownership.txt")
    psi = int(rows[0][1])
    nd = int(rows[1][1])
    for stage in range(4):
        pl = P.make_plan(psi, nd, stage, 4096, align=64)
        assert pl.psi_pad == psi and pl.S == psi // nd
        for r, _name, b, e in rows[2:]:
            assert P.owner_ranges(pl, int(r)) == [(int(b), int(e))]
        for p in (0, 16383, 16384, 40000, 65535):
            assert P.locate(pl, p)[1] == p // 16384


def _brute_layout(units, nd, align, bucket):
    """Enumerate the padded layout element by element (independent of the
    closed forms): returns per-logical-index (unit, j, owner, storage offset),
    S, and the bucket list."""
    logical = []          # (unit, j)
    for u, n in enumerate(units):
        m = n
        while m % (nd * align) != 0:
            m += 1
        logical += [(u, j) for j in range(m)]
    # split each unit's padded run into nd equal consecutive groups
    by_unit = {}
    for p, (u, j) in enumerate(logical):
        by_unit.setdefault(u, []).append(p)
    owner_of = {}
    for u, ps in by_unit.items():
        g = len(ps) // nd
        for k, p in enumerate(ps):
            owner_of[p] = k // g
    blocks = {o: [] for o in range(nd)}
    for u in sorted(by_unit):
        for p in by_unit[u]:
            blocks[owner_of[p]].append(p)
    sizes = {len(b) for b in blocks.values()}
    assert len(sizes) == 1
    S = sizes.pop()
    where = {}
    for o, b in blocks.items():
        for off, p in enumerate(b):
            where[p] = (o, off)
    buckets = []
    for u in sorted(by_unit):
        ps = by_unit[u]
        for k in range(0, len(ps), bucket):
            chunk = ps[k:k + bucket]
            buckets.append((u, chunk[0], chunk[-1] + 1))
    return logical, where, S, buckets


def test_maps_brute_force_small():
    rnd = random.Random(7)
    cases = 0
    for psi in list(range(1, 65)):
        for nd in (1, 2, 3, 4, 5, 8, 16, 64):
            for align in (1, 4, 64):
                if nd * align > 256 and psi % 3:
                    continue
                n_units = rnd.randint(1, min(4, psi))
                cuts = sorted(rnd.sample(range(1, psi), n_units - 1)) if n_units > 1 else []
                units = [b - a for a, b in zip([0] + cuts, cuts + [psi])]
                bucket = rnd.choice([1, 3, 8, 64, 1000])
                stage = rnd.randint(0, 3)
                pl = P.make_plan(psi, nd, stage, bucket, align=align,
                                 unit_elems=units)
                logical, where, S, buckets = _brute_layout(units, nd, align, bucket)
                assert pl.psi_pad == len(logical) and pl.S == S
                for p, (u, j) in enumerate(logical):
                    lu, o, off, lj = P.locate(pl, p)
                    assert (lu, lj) == (u, j)
                    assert (o, off) == where[p]
                    assert P.is_padding(pl, p) == (j >= units[u])
                for u, n in enumerate(units):
                    assert 0 <= pl.unit_pad[u] - n < nd * align
                assert pl.buckets == buckets
                sidx = P.storage_index(pl, range(len(logical)))
                assert [int(x) for x in sidx] == [where[p][0] * S + where[p][1]
                                                  for p in range(len(logical))]
                cases += 1
    assert cases > 1000


def test_gpt2_small_and_owner_7p5b_plans():
    # GPT-2-small-shaped flat vector: 12 blocks of (12 h^2 + 13 h), token and
    # position tables, final norm (h = 768, 3072 MLP, 50257 x 768 tokens).
    h = 768
    psi = 12 * (12 * h * h + 13 * h) + 50257 * h + 1024 * h + 2 * h
    assert psi == 124_439_808
    pl = P.make_plan(psi, 8, 2, 25_000_000, align=64)
    assert pl.psi_pad == 124_440_064 and pl.S == 15_555_008
    assert [e - b for _, b, e in pl.buckets] == [25_000_000] * 4 + [24_440_064]
    # 7.5B at Nd = 64: owner 0's part of each 25M bucket
    pl = P.make_plan(7_500_000_000, 64, 2, 25_000_000, align=64)
    lo, hi = P.owner_ranges(pl, 0)[0]
    parts = [min(e, hi) - max(b, lo) for _, b, e in pl.buckets if b < hi and e > lo]
    assert parts == [25_000_000] * 4 + [17_187_520]


# ------------------------------------------------------------------ bf16
def test_bf16_rne_matches_torch():
    hi = np.arange(1 << 16, dtype=np.uint32) << 16
    lows = np.array([0, 1, 0x3FFF, 0x7FFF, 0x8000, 0x8001, 0xC000, 0xFFFF],
                    dtype=np.uint32)
    bits = (hi[:, None] | lows[None, :]).ravel()
    rng = np.random.default_rng(1)
    bits = np.concatenate([bits, rng.integers(0, 1 << 32, 1 << 20,
                                              dtype=np.uint64).astype(np.uint32)])
    x = bits.view(np.float32)
    ours = core.bf16_rne(x)
    theirs = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16)
    theirs = theirs.numpy().view(np.uint16)
    nan = np.isnan(x)
    assert np.array_equal(ours[~nan], theirs[~nan])
    # NaN: still NaN, quiet, sign kept
    q = ours[nan]
    assert np.all((q & 0x7F80) == 0x7F80) and np.all((q & 0x0040) != 0)
    assert np.array_equal(q >> 15, (bits[nan] >> 31).astype(np.uint16))
    # round trip is exact for values already in bf16
    back = core.bf16_to_f32(ours[~nan])
    assert np.array_equal(core.bf16_rne(back), ours[~nan])


def test_bf16_rne_matches_torch_on_every_pattern():
    """All 2^32 fp32 bit patterns, in chunks of 2^24: the same bf16 as
    torch's conversion for every non-NaN input; every NaN stays a quiet NaN
    with its sign."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    chunk = 1 << 22

    def check(c):
        bits = np.arange(c * chunk, (c + 1) * chunk, dtype=np.uint64).astype(np.uint32)
        x = bits.view(np.float32)
        ours = core.bf16_rne(x)
        theirs = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        nan = np.isnan(x)
        if nan.any():
            q = ours[nan]
            if not (np.all((q & 0x7F80) == 0x7F80) and np.all((q & 0x0040) != 0)
                    and np.array_equal(q >> 15, (bits[nan] >> 31).astype(np.uint16))):
                return c
            ours, theirs = ours[~nan], theirs[~nan]
        return None if np.array_equal(ours, theirs) else c

    threads = torch.get_num_threads()
    torch.set_num_threads(1)          # the chunks run side by side instead
    try:
        with ThreadPoolExecutor(max_workers=max(1, len(os.sched_getaffinity(0)))) as ex:
            bad = [c for c in ex.map(check, range(1 << 10)) if c is not None]
    finally:
        torch.set_num_threads(threads)
    assert not bad, bad


# ------------------------------------------------------------ reduction
def test_reduce_rank_order_cancellation():
    two25 = np.float32(2.0 ** 25)
    g = core.bf16_rne(np.array([[two25], [1.0], [-two25]], dtype=np.float32))
    # (2^25 + 1) rounds to 2^25 in fp32, so the rank-order sum is 0, not 1
    assert core.reduce(g)[0] == 0.0
    # the same three values with the cancelling pair first give 1
    g = core.bf16_rne(np.array([[two25], [-two25], [1.0]], dtype=np.float32))
    assert core.reduce(g)[0] == 1.0
    # the sum starts from rank 0's value: -0 + -0 keeps the sign
    g = core.bf16_rne(np.array([[-0.0], [-0.0]], dtype=np.float32))
    assert math.copysign(1.0, core.reduce(g)[0]) == -1.0


def test_reduce_within_rational_error_bound():
    rng = np.random.default_rng(2)
    for nd in (1, 2, 3, 8, 16, 64):
        g = rand_bf16(rng, (nd, 300), 1.0)
        # cancellation-heavy columns too
        g[:, :50] = rand_bf16(rng, (nd, 50), 1e3)
        got = core.reduce(g)
        vals = core.bf16_to_f32(g.ravel()).reshape(nd, -1)
        u = Fraction(1, 2 ** 24)
        gamma = (nd - 1) * u / (1 - (nd - 1) * u)
        for e in range(g.shape[1]):
            exact = sum(Fraction(float(vals[r, e])) for r in range(nd))
            bound = gamma * sum(abs(Fraction(float(vals[r, e]))) for r in range(nd))
            assert abs(Fraction(float(got[e])) - exact) <= bound


# ------------------------------------------------------------------ Adam
def test_nd1_stage0_matches_torch_adam():
    """Nd = 1 replicated step vs torch.optim.Adam (single-tensor path) on CPU.
    Each step starts both from torch's state, so the bound is one step's
    rounding: a few ulp of w plus a few ulp of the size of the update's terms."""
    rng = np.random.default_rng(3)
    n, T = 4096, 8
    a = dict(ADAM)
    w0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    prm = torch.nn.Parameter(torch.from_numpy(w0.copy()))
    opt = torch.optim.Adam([prm], lr=a["lr"], betas=(a["beta1"], a["beta2"]),
                           eps=a["eps"], foreach=False, fused=False)
    m_t = np.zeros(n, np.float32)
    v_t = np.zeros(n, np.float32)
    for t in range(1, T + 1):
        G = rand_bf16(rng, (1, n), 1e-3 * (1 + t % 3))
        g = core.bf16_to_f32(G[0]) * np.float32(a["grad_scale"])
        w_in = prm.detach().numpy().copy()
        ww, m, v = w_in.copy(), m_t.copy(), v_t.copy()
        p, _, _, _ = core.update(G, ww, m, v, a, t)
        prm.grad = torch.from_numpy(g.copy())
        opt.step()
        st = opt.state[prm]
        tw = prm.detach().numpy().astype(np.float64)
        tm = st["exp_avg"].numpy().astype(np.float64)
        tv = st["exp_avg_sq"].numpy().astype(np.float64)
        scale_m = a["beta1"] * np.abs(m_t) + (1 - a["beta1"]) * np.abs(g)
        assert np.all(np.abs(m - tm) <= 2e-6 * scale_m)
        np.testing.assert_allclose(v, tv, rtol=2e-6, atol=0)
        bc1 = 1 - a["beta1"] ** t
        bc2 = 1 - a["beta2"] ** t
        size = a["lr"] / bc1 * scale_m / (np.sqrt(tv / bc2) + a["eps"])
        assert np.all(np.abs(ww - tw) <= 2 * f32_ulp(w_in) + 4e-6 * size)
        assert np.array_equal(p, core.bf16_rne(ww))
        m_t = st["exp_avg"].numpy().copy()
        v_t = st["exp_avg_sq"].numpy().copy()


def test_fp32_core_within_error_of_fp64_textbook():
    rng = np.random.default_rng(4)
    n = 6000
    a = dict(ADAM)
    # magnitudes from eps-dominated (1e-9) to large (1e2)
    mags = 10.0 ** rng.uniform(-9, 2, n)
    g32 = (rng.standard_normal(n) * mags).astype(np.float32)
    gb = core.bf16_rne(g32)[None, :]
    for t in (1, 2, 7, 100, 5000):
        w = (rng.standard_normal(n) * 0.02).astype(np.float32)
        m = (rng.standard_normal(n) * mags * 0.1).astype(np.float32)
        v = ((rng.standard_normal(n) * mags) ** 2 * 1e-2).astype(np.float32)
        w64, m64, v64 = (x.astype(np.float64) for x in (w, m, v))
        g64 = core.bf16_to_f32(gb[0]).astype(np.float64) * float(np.float32(a["grad_scale"]))
        ew, em, ev = adam_fp64(g64, w64, m64, v64, a["lr"], a["beta1"],
                               a["beta2"], a["eps"], t)
        core.update(gb, w, m, v, a, t)
        # errors bounded by a few ulp of the size of each sum's terms
        scale_m = a["beta1"] * np.abs(m64) + (1 - a["beta1"]) * np.abs(g64)
        assert np.all(np.abs(m - em) <= 4e-7 * scale_m)
        np.testing.assert_allclose(v, ev, rtol=4e-7, atol=1e-45)
        bc1 = 1 - a["beta1"] ** t
        bc2 = 1 - a["beta2"] ** t
        size = a["lr"] / bc1 * scale_m / (np.sqrt(ev / bc2) + a["eps"])
        assert np.all(np.abs(w - ew) <= f32_ulp(ew) + 2e-6 * size)


def test_closed_form_first_step():
    rng = np.random.default_rng(5)
    n = 5000
    a = dict(ADAM, grad_scale=1.0)
    gb = rand_bf16(rng, (1, n), 1e-3)
    g = core.bf16_to_f32(gb[0]).astype(np.float64)
    w0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    w, m, v = w0.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    core.update(gb, w, m, v, a, 1)
    lr, eps = a["lr"], a["eps"]
    want = w0.astype(np.float64) - lr * g / (np.abs(g) + eps)
    assert np.all(np.abs(w - want) <= 2 * f32_ulp(want) + 1e-6 * lr)


def test_constant_gradient_moves_by_lr_each_step():
    n = 64
    a = dict(ADAM, grad_scale=1.0)
    gvals = np.linspace(-1e-2, 1e-2, n).astype(np.float32)
    gvals[gvals == 0] = 1e-3
    gb = core.bf16_rne(gvals)[None, :]
    g = core.bf16_to_f32(gb[0]).astype(np.float64)
    w, m, v = np.zeros(n, np.float32), np.zeros(n, np.float32), np.zeros(n, np.float32)
    lr, eps = a["lr"], a["eps"]
    for t in range(1, 21):
        w_prev = w.astype(np.float64)
        core.update(gb, w, m, v, a, t)
        step = w.astype(np.float64) - w_prev
        # bias-corrected moments are exactly g and g^2 for a constant gradient
        want = -lr * g / (np.abs(g) + eps)
        assert np.all(np.abs(step - want) <= 1e-5 * np.abs(want) + 2 * f32_ulp(w))


def test_zero_gradient_leaves_state_unchanged():
    rng = np.random.default_rng(6)
    n = 1000
    w0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    w, m, v = w0.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    gb = np.zeros((3, n), np.uint16)
    for t in (1, 2, 3):
        p, red, norm, bad = core.update(gb, w, m, v, ADAM, t, want_reduced=True)
        assert np.array_equal(w, w0) and not m.any() and not v.any()
        assert np.array_equal(p, core.bf16_rne(w0)) and not red.any()
        assert norm == 0.0 and bad == 0


def test_norm_and_nonfinite_count():
    rng = np.random.default_rng(8)
    nd, n = 4, 2000
    gb = rand_bf16(rng, (nd, n), 1e-1)
    w, m, v = (np.zeros(n, np.float32) for _ in range(3))
    _, red, norm, bad = core.update(gb, w, m, v, ADAM, 1, want_reduced=True)
    exact = math.fsum(float(x) * float(x) for x in red.astype(np.float64))
    assert abs(norm - exact) <= 1e-12 * exact and bad == 0
    gb[1, 5] = core.bf16_rne(np.array([np.inf], np.float32))[0]
    gb[2, 9] = core.bf16_rne(np.array([np.nan], np.float32))[0]
    gb[0, 11] = core.bf16_rne(np.array([3e38], np.float32))[0]
    gb[1, 11] = gb[0, 11]                     # the sum overflows to inf
    w, m, v = (np.zeros(n, np.float32) for _ in range(3))
    _, red, norm, bad = core.update(gb, w, m, v, ADAM, 1, want_reduced=True)
    assert bad == 3 and not np.isfinite(norm)
    assert np.isinf(red[5]) and np.isnan(red[9]) and np.isinf(red[11])


# ------------------------------------------ partitioned == replicated
def _random_units(rnd, psi, k):
    if k == 1:
        return [psi]
    cuts = sorted(rnd.sample(range(1, psi), k - 1))
    return [b - a for a, b in zip([0] + cuts, cuts + [psi])]


@pytest.mark.parametrize("psi,nd,align,n_units", [
    (65536, 4, 64, 1), (1000, 3, 1, 1), (777, 8, 4, 5), (4097, 16, 8, 3),
    (50, 64, 1, 2), (1, 2, 64, 1)])
def test_partitioned_equals_replicated(psi, nd, align, n_units):
    rnd = random.Random(psi * 31 + nd)
    rng = np.random.default_rng(psi + nd)
    units = _random_units(rnd, psi, n_units)
    a = dict(ADAM, grad_scale=1.0 / nd)
    pl0 = P.make_plan(psi, nd, 0, 1 << 20, align=align, unit_elems=units)
    pad = np.array([P.is_padding(pl0, p) for p in range(pl0.psi_pad)])
    w_log = (rng.standard_normal(pl0.psi_pad) * 0.02).astype(np.float32)
    w_log[pad] = 0.0
    # stage 0 reference: every rank keeps and updates the full state
    W = np.tile(w_log, (nd, 1))
    M = np.zeros_like(W)
    V = np.zeros_like(W)
    stages = {}
    for stage in (1, 2, 3):
        pl = P.make_plan(psi, nd, stage, 1 << 20, align=align, unit_elems=units)
        st = dict(w=ST.logical_to_storage(pl, w_log),
                  m=np.zeros(nd * pl.S, np.float32), v=np.zeros(nd * pl.S, np.float32),
                  p=(np.zeros(nd * pl.S, np.uint16) if stage == 3
                     else np.zeros((nd, pl.psi_pad), np.uint16)),
                  red=np.zeros(nd * pl.S, np.float32))
        stages[stage] = (pl, st)
    for t in (1, 2, 3):
        G = rand_bf16(rng, (nd, pl0.psi_pad), 0.01)
        G[:, pad] = 0
        params0, red0, norm0, bad0 = ST.step_replicated(nd, G, W, M, V, a, t,
                                                        want_reduced=True)
        for r in range(1, nd):
            assert np.array_equal(params0[r], params0[0])
            assert np.array_equal(W[r], W[0])
        for stage, (pl, st) in stages.items():
            norm, bad = ST.step_partitioned(pl, G, st["w"], st["m"], st["v"],
                                            st["p"], a, t, reduced=st["red"])
            assert np.array_equal(ST.storage_to_logical(pl, st["w"]), W[0])
            assert np.array_equal(ST.storage_to_logical(pl, st["m"]), M[0])
            assert np.array_equal(ST.storage_to_logical(pl, st["v"]), V[0])
            assert np.array_equal(ST.storage_to_logical(pl, st["red"]), red0)
            assert norm == pytest.approx(norm0, rel=1e-12) and bad == bad0
            if stage == 3:
                assert np.array_equal(ST.storage_to_logical(pl, st["p"]), params0[0])
                for u in range(len(units)):
                    full = ST.gather_layer(pl, u, st["p"])
                    b = pl.unit_base[u]
                    assert np.array_equal(full, params0[0][b:b + units[u]])
            else:
                for r in range(nd):
                    assert np.array_equal(st["p"][r], params0[0])
        # padding state stays exactly zero
        assert not W[0][pad].any() and not M[0][pad].any() and not V[0][pad].any()


def test_owner_view_equals_partitioned_slice():
    rng = np.random.default_rng(9)
    psi, nd = 10_000, 8
    pl = P.make_plan(psi, nd, 2, 3000, align=64)
    G = rand_bf16(rng, (nd, pl.psi_pad), 1e-3)
    w_log = (rng.standard_normal(pl.psi_pad) * 0.02).astype(np.float32)
    w_st = ST.logical_to_storage(pl, w_log)
    m = np.zeros(nd * pl.S, np.float32)
    v = np.zeros(nd * pl.S, np.float32)
    params = np.zeros((nd, pl.psi_pad), np.uint16)
    ST.step_partitioned(pl, G, w_st.copy(), m, v, params, ADAM, 1)
    w_full = w_st.copy()
    ST.step_partitioned(pl, G, w_full, np.zeros_like(m), np.zeros_like(v), params, ADAM, 1)
    for o in (0, 3, nd - 1):
        cols = ST.owner_columns(pl, o)
        w_o = w_st[o * pl.S:(o + 1) * pl.S].copy()
        p, _, _, _ = ST.step_owner_view(pl, o, G[:, cols], w_o,
                                        np.zeros(pl.S, np.float32),
                                        np.zeros(pl.S, np.float32), ADAM, 1)
        assert np.array_equal(w_o, w_full[o * pl.S:(o + 1) * pl.S])
        assert np.array_equal(p, params[0][cols])


def test_hbm_bytes_per_param():
    pl = P.make_plan(124_439_808, 8, 2, 25_000_000)
    assert P.hbm_step_bytes(pl) == pl.psi_pad * (4 * 8 + 24)
    units = [107_120_640] + [50_358_272] * 24 + [4096]
    pl3 = P.make_plan(sum(units), 16, 3, 1 << 28, unit_elems=units)
    assert pl3.psi_pad == sum(units) and pl3.S == 82_232_704
    assert P.hbm_step_bytes(pl3) == pl3.psi_pad * (2 * 16 + 24 + 2)
    pl4 = P.make_plan(7_500_000_000, 64, 2, 25_000_000)
    assert P.hbm_step_bytes(pl4, owner_view=True) == pl4.S * (2 * 64 + 24 + 2)


def _ring_reduce_scatter(chunks):
    """Brute-force ring reduce-scatter.  chunks[r][c]: rank r's piece c (a
    bf16 tensor).  At step k rank r sends its piece (r-k-1) mod Nd to rank
    r+1, which adds it to its own; after Nd-1 steps rank r holds the sum of
    piece r.  Returns (bytes each rank sent, elements each rank sent)."""
    nd = len(chunks)
    sent_b, sent_e = [0] * nd, [0] * nd
    for k in range(nd - 1):
        msgs = [(r, (r - k - 1) % nd, chunks[r][(r - k - 1) % nd].clone()) for r in range(nd)]
        for r, c, msg in msgs:
            sent_b[r] += msg.numel() * msg.element_size()
            sent_e[r] += msg.numel()
            chunks[(r + 1) % nd][c] += msg
    return sent_b, sent_e


def _ring_all_gather(chunks):
    """Brute-force ring all-gather: rank r starts with its piece r valid; at
    step k it forwards piece (r-k) mod Nd to rank r+1."""
    nd = len(chunks)
    sent_b, sent_e = [0] * nd, [0] * nd
    for k in range(nd - 1):
        msgs = [(r, (r - k) % nd, chunks[r][(r - k) % nd].clone()) for r in range(nd)]
        for r, c, msg in msgs:
            sent_b[r] += msg.numel() * msg.element_size()
            sent_e[r] += msg.numel()
            chunks[(r + 1) % nd][c] = msg
    return sent_b, sent_e


@pytest.mark.parametrize("stage", [0, 1, 2, 3])
@pytest.mark.parametrize("nd,align,units", [(1, 1, [10]), (3, 4, [37, 63, 5]),
                                            (4, 1, [64]), (5, 2, [3, 1, 40])])
def test_comm_bytes_equal_bytes_a_brute_force_ring_sends(stage, nd, align, units):
    """Run the ring collectives of one step on bf16 buffers (per unit: a
    reduce-scatter of the gradients, then one all-gather of the parameters,
    or two at stage 3, forward and backward) and count what every rank
    sends.  The sums and the gathered copies are checked too, with small
    integers that bf16 holds exactly, so the simulated ring is the real
    collective."""
    pl = P.make_plan(sum(units), nd, stage, 1 << 20, align=align, unit_elems=units)
    sent_b, sent_e = [0] * nd, [0] * nd
    gen = torch.Generator().manual_seed(nd * 100 + stage)
    for u, s in enumerate(pl.unit_shard):
        grads = torch.randint(0, 5, (nd, nd * s), generator=gen).to(torch.bfloat16)
        chunks = [[grads[r, c * s:(c + 1) * s].clone() for c in range(nd)] for r in range(nd)]
        b, e = _ring_reduce_scatter(chunks)
        for r in range(nd):
            assert torch.equal(chunks[r][r], grads[:, r * s:(r + 1) * s].sum(0))
            sent_b[r] += b[r]
            sent_e[r] += e[r]
        for _ in range(2 if stage == 3 else 1):
            owned = torch.randint(0, 100, (nd, s), generator=gen).to(torch.bfloat16)
            chunks = [[owned[c].clone() if c == r else torch.zeros(s, dtype=torch.bfloat16)
                       for c in range(nd)] for r in range(nd)]
            b, e = _ring_all_gather(chunks)
            for r in range(nd):
                assert all(torch.equal(chunks[r][c], owned[c]) for c in range(nd))
                sent_b[r] += b[r]
                sent_e[r] += e[r]
    assert len(set(sent_b)) == 1 and len(set(sent_e)) == 1
    assert P.comm_elems_per_rank(pl) == sent_e[0]
    assert P.comm_bytes_per_rank(pl) == sent_b[0]


@pytest.mark.parametrize("nd,align,units", [(3, 4, [37, 63, 5]), (4, 8, [100, 7]),
                                            (2, 1, [9, 1, 4])])
def test_gather_bytes_equal_bytes_the_gathers_move(nd, align, units):
    """Materialise every unit forward, then in reverse, through
    oracle.step.gather_layer on owner storage filled with distinct ids, and
    count the bf16 elements each gather reads from the owners' slices (the
    distinct ids in its output) and writes (its output).  The plans have
    padding, so counting padded lengths would fail."""
    pl = P.make_plan(sum(units), nd, 3, 1 << 20, align=align, unit_elems=units)
    assert pl.psi_pad > sum(units)
    owner_params = np.arange(nd * pl.S, dtype=np.uint16)
    moved = 0
    for u in list(range(len(units))) + list(reversed(range(len(units)))):
        out = ST.gather_layer(pl, u, owner_params)
        read = np.unique(out)
        assert read.size == out.size
        moved += read.size * owner_params.itemsize + out.nbytes
    assert P.hbm_gather_bytes(pl) == moved


def test_oracle_never_imports_the_product():
    import os
    import re
    here = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle")
    for name in os.listdir(here):
        if name.endswith((".py", ".c")):
            with open(os.path.join(here, name), encoding="utf-8") as f:
                src = f.read()
            assert not re.search(r"zero_partitioned_optimizer_step_b200|libzero", src), name


@pytest.mark.parametrize("stage,owner", [(2, None), (3, None), (2, 3)])
def test_hbm_bytes_equal_bytes_of_buffers_the_step_touches(stage, owner):
    """The accounting equals the sizes of the arrays one oracle step reads
    (gradients, w, m, v) and writes (w, m, v, parameters, reduced gradient)."""
    rng = np.random.default_rng(10)
    units = [3000, 5000] if stage == 3 else None
    pl = P.make_plan(8000, 8, stage, 2048, align=8, unit_elems=units)
    G = rand_bf16(rng, (8, pl.psi_pad), 1e-3)
    if owner is None:
        w = np.zeros(8 * pl.S, np.float32)
        m, v, red = w.copy(), w.copy(), w.copy()
        params = (np.zeros(8 * pl.S, np.uint16) if stage == 3
                  else np.zeros((8, pl.psi_pad), np.uint16))
        ST.step_partitioned(pl, G, w, m, v, params, ADAM, 1, reduced=red)
        reads = G.nbytes + w.nbytes + m.nbytes + v.nbytes
    else:
        Go = G[:, ST.owner_columns(pl, owner)]
        w = np.zeros(pl.S, np.float32)
        m, v = w.copy(), w.copy()
        params, red, _, _ = ST.step_owner_view(pl, owner, Go, w, m, v, ADAM, 1, want_reduced=True)
        reads = Go.nbytes + w.nbytes + m.nbytes + v.nbytes
    writes = w.nbytes + m.nbytes + v.nbytes + params.nbytes
    view = owner is not None
    assert P.hbm_step_bytes(pl, owner_view=view) == reads + writes
    assert P.hbm_step_bytes(pl, owner_view=view, with_reduced=True) == reads + writes + red.nbytes


def test_replicas_follow_the_stage_table():
    rows = read_golden("stage_table.txt")
    for st, state, grad, param in rows:
        pl = P.make_plan(1000, 8, int(st), 100)
        for what, mark in (("state", state), ("grad", grad), ("param", param)):
            assert P.replicas(pl, what) == (1 if mark == "S" else 8), (st, what)
    # the memory model agrees: a replicated state costs its full size per rank
    for st, state, grad, param in rows:
        pl = P.make_plan(64_000, 8, int(st), 100, align=1)
        want = sum(b * (pl.psi if mark == "R" else pl.psi // 8)
                   for b, mark in ((12, state), (2, grad), (2, param)))
        assert P.memory_bytes_per_rank_padded(pl, int(st)) == want


def test_lost_rank_counts_owned_real_elements():
    pl = P.make_plan(100, 3, 2, 10, align=4, unit_elems=[37, 63])
    counts = [P.lost_rank_unrecoverable(pl, r) for r in range(3)]
    assert sum(counts) == 100
    assert counts == [sum(1 for p in range(pl.psi_pad)
                          if P.locate(pl, p)[1] == r and not P.is_padding(pl, p))
                      for r in range(3)]
    assert P.lost_rank_unrecoverable(P.make_plan(100, 3, 0, 10), 1) == 0


def test_reshard_keeps_every_real_element():
    rng = np.random.default_rng(30)
    units = [37, 63, 5]
    a = P.make_plan(105, 3, 3, 10, align=4, unit_elems=units)
    b = P.make_plan(105, 8, 1, 7, align=1, unit_elems=units)
    x = rng.standard_normal(a.nd * a.S).astype(np.float32)
    pad_a = np.array([P.is_padding(a, p) for p in range(a.psi_pad)])
    x[ST.logical_to_storage(a, pad_a.astype(np.float32)) > 0] = 0
    y = ST.reshard(a, x, b)
    for p in range(b.psi_pad):
        u, o, off, j = P.locate(b, p)
        if j < units[u]:
            pa = a.unit_base[u] + j          # same unit, same index under plan a
            _, oa, offa, _ = P.locate(a, pa)
            assert y[o * b.S + off] == x[oa * a.S + offa]
        else:
            assert y[o * b.S + off] == 0
    assert np.array_equal(ST.reshard(b, y, a), x)


try:
    from hypothesis import given, settings, strategies as hst
except ImportError:  # pragma: no cover
    given = None

if given is not None:
    @settings(max_examples=60, deadline=None)
    @given(units=hst.lists(hst.integers(1, 300), min_size=1, max_size=5),
           a=hst.tuples(hst.integers(1, 12), hst.integers(0, 3), hst.sampled_from([1, 2, 4, 8])),
           b=hst.tuples(hst.integers(1, 12), hst.integers(0, 3), hst.sampled_from([1, 2, 4, 8])),
           seed=hst.integers(0, 2 ** 31))
    def test_reshard_property_random_plans(units, a, b, seed):
        """For random unit lists and any two plans of them: every real element
        lands where the destination plan's map puts it, the new padding is
        zero, and resharding back gives the source bytes."""
        psi = sum(units)
        pa = P.make_plan(psi, a[0], a[1], 97, align=a[2], unit_elems=units)
        pb = P.make_plan(psi, b[0], b[1], 53, align=b[2], unit_elems=units)
        rng = np.random.default_rng(seed)
        logical = np.zeros(pa.psi_pad, np.float32)
        for u, n in enumerate(units):
            logical[pa.unit_base[u]:pa.unit_base[u] + n] = rng.standard_normal(n)
        x = ST.logical_to_storage(pa, logical)
        y = ST.reshard(pa, x, pb)
        for p in range(pb.psi_pad):
            u, o, off, j = P.locate(pb, p)
            want = logical[pa.unit_base[u] + j] if j < units[u] else 0.0
            assert y[o * pb.S + off] == want
        assert np.array_equal(ST.reshard(pb, y, pa), x)

"""Pins of the oracle's AdamW decay and guarded step (global-norm clip,
skip on non-finite gradients) against torch's own AdamW and
clip_grad_norm_, and against the plain step."""
import numpy as np
import pytest
import torch

from oracle import core
from oracle import plan as P
from oracle import step as ST
from test_oracle_pins import ADAM, f32_ulp, rand_bf16


def _torch_vs_oracle(opt_cls, a, T, rng, clip=None, n=4096):
    """Stepwise comparison with torch: each step starts both from torch's
    state; returns nothing, asserts one step's rounding bound."""
    w0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    prm = torch.nn.Parameter(torch.from_numpy(w0.copy()))
    kw = dict(lr=a["lr"], betas=(a["beta1"], a["beta2"]), eps=a["eps"], foreach=False)
    if "weight_decay" in a:
        kw["weight_decay"] = a["weight_decay"]
    opt = opt_cls([prm], **kw)
    m_t = np.zeros(n, np.float32)
    v_t = np.zeros(n, np.float32)
    for t in range(1, T + 1):
        G = rand_bf16(rng, (1, n), 1e-2 * (1 + t % 3))
        g = core.bf16_to_f32(G[0]) * np.float32(a["grad_scale"])
        coef = np.float32(1.0)
        if clip is not None:
            norm_sq = float(np.dot(core.bf16_to_f32(G[0]).astype(np.float64),
                                   core.bf16_to_f32(G[0]).astype(np.float64)))
            coef = ST.guard_coef(norm_sq, a["grad_scale"], clip)
        w_in = prm.detach().numpy().copy()
        ww, m, v = w_in.copy(), m_t.copy(), v_t.copy()
        p, _, _, _ = core.update(G, ww, m, v, a, t, clip_coef=coef)
        prm.grad = torch.from_numpy(g.copy())
        if clip is not None:
            total = torch.nn.utils.clip_grad_norm_([prm], clip)
            # torch's norm is fp32; the oracle's coefficient agrees to rounding
            want = min(1.0, clip / (float(total) + 1e-6))
            assert abs(float(coef) - want) <= 1e-6 * want
        opt.step()
        st = opt.state[prm]
        tw = prm.detach().numpy().astype(np.float64)
        tm = st["exp_avg"].numpy().astype(np.float64)
        tv = st["exp_avg_sq"].numpy().astype(np.float64)
        gc = np.abs(g.astype(np.float64) * float(coef))
        scale_m = a["beta1"] * np.abs(m_t) + (1 - a["beta1"]) * gc
        assert np.all(np.abs(m - tm) <= 4e-6 * scale_m + 1e-30)
        np.testing.assert_allclose(v, tv, rtol=4e-6, atol=1e-30)
        bc1 = 1 - a["beta1"] ** t
        bc2 = 1 - a["beta2"] ** t
        size = a["lr"] / bc1 * scale_m / (np.sqrt(tv / bc2) + a["eps"])
        decay_part = a["lr"] * a.get("weight_decay", 0.0) * np.abs(w_in)
        assert np.all(np.abs(ww - tw) <= 2 * f32_ulp(w_in) + 6e-6 * size + 1e-6 * decay_part)
        assert np.array_equal(p, core.bf16_rne(ww))
        m_t = st["exp_avg"].numpy().copy()
        v_t = st["exp_avg_sq"].numpy().copy()


def test_adamw_matches_torch_adamw():
    a = dict(ADAM, weight_decay=0.1)
    _torch_vs_oracle(torch.optim.AdamW, a, 8, np.random.default_rng(20))


def test_global_norm_clip_matches_torch_clip_grad_norm():
    a = dict(ADAM, grad_scale=1.0)
    # 4096 entries of ~1e-2: norm ~0.6-2, so 0.05 always clips, 1e3 never does
    for clip in (0.05, 0.3, 1e3):
        _torch_vs_oracle(torch.optim.Adam, a, 6, np.random.default_rng(21), clip=clip)


def test_weight_decay_zero_and_unit_coefficient_are_bitwise_plain_adam():
    rng = np.random.default_rng(22)
    G = rand_bf16(rng, (4, 3000), 1e-2)
    base = [(rng.standard_normal(3000) * 0.02).astype(np.float32), np.zeros(3000, np.float32),
            np.zeros(3000, np.float32)]
    w1, m1, v1 = (x.copy() for x in base)
    w2, m2, v2 = (x.copy() for x in base)
    p1, _, _, _ = core.update(G, w1, m1, v1, ADAM, 1)
    p2, _, _, _ = core.update(G, w2, m2, v2, dict(ADAM, weight_decay=0.0), 1, clip_coef=1.0)
    for x, y in ((w1, w2), (m1, m2), (v1, v2)):
        assert np.array_equal(x.view(np.uint32), y.view(np.uint32))
    assert np.array_equal(p1, p2)
    # a clipped gradient moves m by exactly the clipped amount at t = 1
    w3, m3, v3 = (x.copy() for x in base)
    core.update(G, w3, m3, v3, ADAM, 1, clip_coef=0.5)
    g = core.reduce(G) * np.float32(ADAM["grad_scale"])
    want_m = np.float32(1 - 0.9) * (g * np.float32(0.5))
    np.testing.assert_allclose(m3, want_m, rtol=1e-6, atol=0)


def _guarded_case(stage, units, nd=4, psi=5000):
    pl = P.make_plan(psi, nd, stage, 1024, align=8, unit_elems=units)
    rng = np.random.default_rng(23)
    G = rand_bf16(rng, (nd, pl.psi_pad), 1e-2)
    pad = np.array([P.is_padding(pl, q) for q in range(pl.psi_pad)])
    G[:, pad] = 0
    w = ST.logical_to_storage(pl, (rng.standard_normal(pl.psi_pad) * 0.02).astype(np.float32))
    w[ST.logical_to_storage(pl, pad.astype(np.float32)) > 0] = 0
    return pl, G, w


@pytest.mark.parametrize("stage,units", [(2, None), (3, [2000, 3000])])
def test_guarded_step_equals_plain_step_when_nothing_triggers(stage, units):
    pl, G, w0 = _guarded_case(stage, units)
    a = dict(ADAM, grad_scale=0.25)
    outs = []
    for guarded in (False, True):
        w, m, v = w0.copy(), np.zeros_like(w0), np.zeros_like(w0)
        red = np.zeros_like(w0)
        params = (np.zeros(pl.nd * pl.S, np.uint16) if stage == 3
                  else np.zeros((pl.nd, pl.psi_pad), np.uint16))
        if guarded:
            norm, bad, coef, skipped = ST.step_guarded(pl, G, w, m, v, params, a, 1, 1e9, True, red)
            assert coef == 1.0 and not skipped and bad == 0
        else:
            ST.step_partitioned(pl, G, w, m, v, params, a, 1, reduced=red)
        outs.append((w, m, v, red, params))
    for x, y in zip(*outs):
        assert np.array_equal(x, y)


def test_guarded_step_clips_and_skips():
    pl, G, w0 = _guarded_case(2, None)
    a = dict(ADAM, grad_scale=0.25)
    w, m, v, red = w0.copy(), np.zeros_like(w0), np.zeros_like(w0), np.zeros_like(w0)
    params = np.zeros((pl.nd, pl.psi_pad), np.uint16)
    norm, bad, coef, skipped = ST.step_guarded(pl, G, w, m, v, params, a, 1, 1e-3, True, red)
    total = 0.25 * np.sqrt(norm)
    assert not skipped and 0 < coef < 1
    assert abs(float(coef) - 1e-3 / (total + 1e-6)) <= 1e-7 * float(coef)
    np.testing.assert_allclose(m, np.float32(0.1) * ((red * np.float32(0.25)) * coef), rtol=1e-6)
    # a NaN anywhere: nothing changes, the reduction still shows it
    G2 = G.copy()
    G2[1, 17] = core.bf16_rne(np.array([np.nan], np.float32))[0]
    w2, m2, v2, red2 = w.copy(), m.copy(), v.copy(), np.zeros_like(w0)
    p2 = params.copy()
    norm2, bad2, coef2, skipped2 = ST.step_guarded(pl, G2, w2, m2, v2, p2, a, 2, 1e-3, True, red2)
    assert skipped2 and bad2 == 1 and np.isnan(red2[17])
    for x, y in ((w, w2), (m, m2), (v, v2)):
        assert np.array_equal(x.view(np.uint32), y.view(np.uint32))
    assert np.array_equal(params, p2)


@pytest.mark.parametrize("stage", [2, 3])
def test_guarded_hbm_bytes_equal_buffers_the_two_passes_touch(stage):
    """Pass 1 reads the gradients and writes the reduced sum; pass 2 reads
    the sum and w, m, v and writes w, m, v and the parameters."""
    units = [2000, 3000] if stage == 3 else None
    pl, G, w = _guarded_case(stage, units)
    red = np.zeros_like(w)
    params = (np.zeros(pl.nd * pl.S, np.uint16) if stage == 3
              else np.zeros((pl.nd, pl.psi_pad), np.uint16))
    pass1 = G.nbytes + red.nbytes
    pass2 = red.nbytes + 2 * 3 * w.nbytes + params.nbytes
    assert P.hbm_guarded_step_bytes(pl) == pass1 + pass2

"""Shared helpers of the GPU parity tests: build one case's device buffers
from the seeded generators, run the CUDA step through the C ABI, run the
oracle on host copies of the same bytes, compare."""
import numpy as np
import torch

import zero_partitioned_optimizer_step_b200 as Z
from zero_partitioned_optimizer_step_b200 import inputs
from oracle import core
from oracle import plan as OP
from oracle import step as ST

FLT_MIN = np.float32(np.finfo(np.float32).tiny)

# parity tolerances: reduced sums, fp32 state, bf16 parameters, norm
RTOL_REDUCED = 1e-6
RTOL_STATE = 1e-5
BF16_ULP = 1
RTOL_NORM = 1e-5


def u16(t):
    """bf16 torch tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f32(t):
    return t.detach().contiguous().cpu().numpy()


def f32_rel_check(got, want, rtol, what):
    """Max relative error |a-b|/max(|b|, FLT_MIN), +-0 equal, NaN == NaN.
    Returns the number of elements that are not bit-identical."""
    got = np.asarray(got, dtype=np.float32)
    want = np.asarray(want, dtype=np.float32)
    assert got.shape == want.shape, what
    both_nan = np.isnan(got) & np.isnan(want)
    same = (got == want) | both_nan
    g = got.astype(np.float64)
    w = want.astype(np.float64)
    with np.errstate(invalid="ignore"):
        rel = np.abs(g - w) / np.maximum(np.abs(w), float(FLT_MIN))
    rel = np.where(same, 0.0, rel)
    rel = np.where(np.isnan(rel), np.inf, rel)
    worst = float(rel.max()) if rel.size else 0.0
    assert worst <= rtol, "%s: max rel err %g > %g" % (what, worst, rtol)
    return int((got.view(np.uint32) != want.view(np.uint32)).sum() - both_nan.sum())


def _bf16_key(b):
    b = b.astype(np.int32)
    return np.where(b & 0x8000, 0x8000 - (b & 0x7FFF), 0x8000 + b)


def bf16_ulp_check(got, want, max_ulp, what):
    got = np.asarray(got, dtype=np.uint16)
    want = np.asarray(want, dtype=np.uint16)
    assert got.shape == want.shape, what
    nan_g = ((got & 0x7F80) == 0x7F80) & ((got & 0x7F) != 0)
    nan_w = ((want & 0x7F80) == 0x7F80) & ((want & 0x7F) != 0)
    assert np.array_equal(nan_g, nan_w), "%s: NaN pattern differs" % what
    d = np.abs(_bf16_key(got) - _bf16_key(want))
    d = np.where(nan_g, 0, d)
    worst = int(d.max()) if d.size else 0
    assert worst <= max_ulp, "%s: %d ulp apart" % (what, worst)
    return int((d != 0).sum())


class Case:
    """A full-compare case: every element checked against the oracle."""

    def __init__(self, psi, nd, stage, bucket, align=64, units=None, owner_view=-1,
                 sigma=1e-3, outlier_frac=0.0, config_id=0, with_reduced=True,
                 with_norm=True, adam=None, device="cuda"):
        self.lp = Z.zero_plan(psi, nd, stage, bucket, align_elems=align, unit_elems=units)
        self.op = OP.make_plan(psi, nd, stage, bucket, align=align, unit_elems=units)
        self.nd, self.stage, self.owner = nd, stage, owner_view
        self.sigma, self.outlier, self.cfg = sigma, outlier_frac, config_id
        self.adam = dict(adam or dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8),
                         grad_scale=1.0 / nd)
        self.dev = device
        op = self.op
        S = op.S
        w_log = inputs.master_logical(op.unit_len, op.unit_pad, config_id, device)
        w_st = self.logical_to_storage(w_log)
        if owner_view >= 0:
            w_st = w_st[owner_view * S:(owner_view + 1) * S].clone()
        n = w_st.numel()
        self.w = w_st.contiguous()
        self.m = torch.zeros(n, dtype=torch.float32, device=device)
        self.v = torch.zeros(n, dtype=torch.float32, device=device)
        self.red = torch.zeros(n, dtype=torch.float32, device=device) if with_reduced else None
        if owner_view < 0 and stage <= 2:
            self.params = torch.zeros((nd, op.psi_pad), dtype=torch.bfloat16, device=device)
        else:
            self.params = torch.zeros(n, dtype=torch.bfloat16, device=device)
        self.norm = torch.zeros(1, dtype=torch.float64, device=device) if with_norm else None
        self.ovf = torch.zeros(1, dtype=torch.int32, device=device) if with_norm else None
        self.ws = Z.workspace_for(self.lp, device) if with_norm else None
        # host mirror for the oracle
        self.hw, self.hm, self.hv = f32(self.w), f32(self.m), f32(self.v)
        self.hred = np.zeros(n, np.float32) if with_reduced else None
        self.hparams = u16(self.params)

    # layout helpers (plain slicing with the plan's unit tables)
    def logical_to_storage(self, x):
        op = self.op
        out = torch.empty(op.nd * op.S, dtype=x.dtype, device=x.device)
        for o in range(op.nd):
            for u in range(len(op.unit_pad)):
                s = op.unit_shard[u]
                lo = op.unit_base[u] + o * s
                st = o * op.S + op.unit_offset[u]
                out[st:st + s] = x[lo:lo + s]
        return out

    def owner_grads(self, G):
        op, o = self.op, self.owner
        parts = [G[:, op.unit_base[u] + o * op.unit_shard[u]:
                   op.unit_base[u] + (o + 1) * op.unit_shard[u]] for u in range(len(op.unit_pad))]
        return torch.cat(parts, dim=1).contiguous()

    def grads(self, t):
        G = inputs.grads(self.nd, self.op.unit_len, self.op.unit_pad, self.sigma, self.cfg, t,
                         self.dev, outlier_frac=self.outlier)
        return self.owner_grads(G) if self.owner >= 0 else G

    def run_gpu(self, G, t, **kw):
        Z.zero_step(self.lp, G, self.w, self.m, self.v, self.params, self.adam, t,
                    reduced_grad=self.red, grad_norm_sq=self.norm, overflow=self.ovf,
                    workspace=self.ws, owner_view=self.owner, **kw)

    def run_gpu_guarded(self, G, t, max_norm, skip):
        Z.zero_step_guarded(self.lp, G, self.w, self.m, self.v, self.params, self.adam, t,
                            max_grad_norm=max_norm, skip_nonfinite=skip,
                            reduced_grad=self.red, grad_norm_sq=self.norm, overflow=self.ovf,
                            workspace=self.ws, owner_view=self.owner)

    def guarded_step_and_compare(self, t, max_norm, skip, G=None):
        """Two-pass guarded step against oracle.step.step_guarded."""
        assert self.owner < 0 and self.red is not None and self.norm is not None
        G = self.grads(t) if G is None else G
        Gh = u16(G)
        self.run_gpu_guarded(G, t, max_norm, skip)
        norm, bad, coef, skipped = ST.step_guarded(self.op, Gh, self.hw, self.hm, self.hv,
                                                   self.hparams, self.adam, t, max_norm, skip,
                                                   self.hred)
        Z.zero_stream_status()
        return self.compare(norm, bad), coef, skipped

    def run_oracle(self, Gh, t):
        if self.owner >= 0:
            p, red, norm, bad = ST.step_owner_view(self.op, self.owner, Gh, self.hw, self.hm,
                                                   self.hv, self.adam, t,
                                                   want_reduced=self.hred is not None)
            self.hparams[:] = p
            if self.hred is not None:
                self.hred[:] = red
            return norm, bad
        return ST.step_partitioned(self.op, Gh, self.hw, self.hm, self.hv, self.hparams,
                                   self.adam, t, reduced=self.hred)

    def step_and_compare(self, t, G=None):
        G = self.grads(t) if G is None else G
        Gh = u16(G)
        self.run_gpu(G, t)
        norm, bad = self.run_oracle(Gh, t)
        Z.zero_stream_status()          # synchronises; raises if a wait gave up
        return self.compare(norm, bad)

    def compare(self, norm, bad):
        diff = {}
        diff["master"] = f32_rel_check(f32(self.w), self.hw, RTOL_STATE, "master")
        diff["exp_avg"] = f32_rel_check(f32(self.m), self.hm, RTOL_STATE, "exp_avg")
        diff["exp_avg_sq"] = f32_rel_check(f32(self.v), self.hv, RTOL_STATE, "exp_avg_sq")
        if self.red is not None:
            diff["reduced"] = f32_rel_check(f32(self.red), self.hred, RTOL_REDUCED, "reduced")
        diff["params"] = bf16_ulp_check(u16(self.params), self.hparams, BF16_ULP, "params")
        if self.norm is not None:
            got = float(self.norm.item())
            if np.isfinite(norm):
                assert abs(got - norm) <= RTOL_NORM * max(abs(norm), 1e-300), (got, norm)
            else:
                assert not np.isfinite(got)
            assert int(self.ovf.item()) == (1 if bad else 0)
        return diff

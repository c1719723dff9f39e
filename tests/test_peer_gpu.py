"""GPU parity of the ranks-as-devices step (zero_step_peers, one rank's
share of the step, reading the other ranks' gradients and writing their
replicas through plain device pointers).

1. One process, Nd ranks as Nd separate allocations on one GPU: each rank's
   call in turn.  Every rank's outputs are bit-identical to the one-GPU step
   (zero_step over the same bytes), which the same test checks against the
   oracle; the norm, summed over ranks, within the norm tolerance.
2. Stage 3: the layers materialised from the Nd shards equal the oracle's.
3. Two processes on one GPU, each holding one rank's buffers in its own
   allocations, the other's mapped through CUDA IPC, ordered by gloo
   barriers (PeerStep).  The ranks' kernels never wait for one another.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import zero_partitioned_optimizer_step_b200 as Z
from oracle import plan as OP
from oracle import step as ST
from zero_cases import RTOL_NORM, Case, f32, u16

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.synchronize()


class Ranks:
    """Nd ranks' own buffers, each a separate allocation, initialised from a
    Case (the one-GPU layout) so that both paths start from the same bytes."""

    def __init__(self, c: Case):
        op = c.op
        S, nd = op.S, c.nd
        self.c, self.nd, self.S = c, nd, S
        self.master = [c.w[q * S:(q + 1) * S].clone() for q in range(nd)]
        self.m = [c.m[q * S:(q + 1) * S].clone() for q in range(nd)]
        self.v = [c.v[q * S:(q + 1) * S].clone() for q in range(nd)]
        self.red = [torch.zeros(S, dtype=torch.float32, device="cuda") for _ in range(nd)]
        if c.stage <= 2:
            self.params = [torch.zeros(op.psi_pad, dtype=torch.bfloat16, device="cuda") for _ in range(nd)]
        else:
            self.params = [torch.zeros(S, dtype=torch.bfloat16, device="cuda") for _ in range(nd)]
        self.norm = [torch.zeros(1, dtype=torch.float64, device="cuda") for _ in range(nd)]
        self.ovf = [torch.zeros(1, dtype=torch.int32, device="cuda") for _ in range(nd)]
        self.ws = [Z.workspace_for(c.lp) for _ in range(nd)]

    def step(self, G, t):
        grads = [G[q].clone() for q in range(self.nd)]
        for r in range(self.nd):
            Z.zero_step_peers(self.c.lp, r, grads, self.params, self.master[r], self.m[r], self.v[r],
                              self.c.adam, t, reduced_grad=self.red[r], grad_norm_sq=self.norm[r],
                              overflow=self.ovf[r], workspace=self.ws[r])
        Z.zero_stream_status()

    def compare_with_one_gpu_step(self):
        c, S = self.c, self.S
        for q in range(self.nd):
            sl = slice(q * S, (q + 1) * S)
            for mine, theirs, what in ((self.master[q], c.w[sl], "master"), (self.m[q], c.m[sl], "m"),
                                       (self.v[q], c.v[sl], "v"), (self.red[q], c.red[sl], "reduced")):
                assert torch.equal(mine.view(torch.int32), theirs.view(torch.int32)), (what, q)
            want = c.params[q] if c.stage <= 2 else c.params[sl]
            assert torch.equal(self.params[q].view(torch.int16), want.view(torch.int16)), ("params", q)
        total = sum(float(x.item()) for x in self.norm)
        ref = float(c.norm.item())
        assert abs(total - ref) <= RTOL_NORM * max(abs(ref), 1e-300), (total, ref)
        assert max(int(x.item()) for x in self.ovf) == int(c.ovf.item())


PEER_CASES = [
    # psi, nd, stage, bucket, align, units
    (65_536, 4, 2, 16_384, 64, None),
    (100_003, 7, 1, 999, 1, [10_001, 90_002]),
    (300_001, 16, 3, 20_000, 64, [100_000, 1, 200_000]),
    (250_001, 3, 2, 1 << 14, 8, None),
    (1_000_000, 8, 3, 100_000, 64, [400_000, 600_000]),
    (54_290, 1, 2, 1 << 20, 64, None),
    (128 * 64 * 3 + 5, 128, 2, 4096, 64, None),
]
GUARD_CASE = (100_003, 7, 3, 999, 1, [10_001, 90_002])


def call_means(lp):
    """Per rank: the mean size of the aligned bodies its zero_step_peers
    call launches (None for a rank whose parts are all scalar), from the
    plan's bucket and unit queries."""
    units = lp.units()
    out = []
    for r in range(lp.nd):
        cols = n = 0
        for b in range(lp.n_buckets):
            u = lp.query(Z.ZERO_Q_BUCKET_UNIT, b)
            lo_b, hi_b = lp.query(Z.ZERO_Q_BUCKET_BEGIN, b), lp.query(Z.ZERO_Q_BUCKET_END, b)
            _, _, s, U, O = units[u]
            lo = U + r * s
            p0, p1 = max(lo_b, lo), min(hi_b, lo + s)
            vlo, vhi = (p0 + 7) // 8 * 8, p1 // 8 * 8
            if p0 < p1 and (O - lo) % 8 == 0 and vlo < vhi:
                cols += vhi - vlo
                n += 1
        out.append(cols // n if n else None)
    return out


def use_kernel(monkeypatch, kernel, lp):
    """tma / ldg: every aligned body in the bulk-copy kernel or in K5.
    mixed: the library's per-call choice, with its threshold at the middle
    of the ranks' mean body sizes, so that where those differ some ranks'
    calls run the bulk-copy kernel and the others K5 in the same step."""
    if kernel == "mixed":
        means = sorted({m for m in call_means(lp) if m is not None})
        monkeypatch.delenv("ZERO_STEP_KERNEL", raising=False)
        monkeypatch.setenv("ZERO_PEER_RING_MIN", str(means[len(means) // 2] if means else 0))
    else:
        monkeypatch.delenv("ZERO_PEER_RING_MIN", raising=False)
        monkeypatch.setenv("ZERO_STEP_KERNEL", kernel)


@pytest.mark.parametrize("kernel", ["tma", "ldg", "mixed"])
@pytest.mark.parametrize("psi,nd,stage,bucket,align,units", PEER_CASES)
def test_ranks_as_allocations_equal_the_one_gpu_step(psi, nd, stage, bucket, align, units, kernel,
                                                     monkeypatch):
    """Aligned bodies in the bulk-copy kernel (rows through the peer table),
    in K5, or each launch in the kernel its size picks; all against the
    one-GPU step."""
    c = Case(psi, nd, stage, bucket, align=align, units=units, config_id=31)
    use_kernel(monkeypatch, kernel, c.lp)
    kinds = {Z.zero_step_peers_kernel(c.lp, r) for r in range(nd)} - {None}
    if kernel == "ldg" or nd > 64:
        assert kinds <= {"k_step_peer"}
    elif kernel == "tma":
        assert kinds <= {"k_step_tma"}
    elif len({m for m in call_means(c.lp) if m is not None}) > 1:
        assert kinds == {"k_step_tma", "k_step_peer"}, kinds   # both kernels in one step
    R = Ranks(c)
    for t in (1, 2, 3):
        G = c.grads(t)
        R.step(G, t)
        c.step_and_compare(t, G)          # the one-GPU step against the oracle
        R.compare_with_one_gpu_step()


def test_stage3_layers_from_the_ranks_shards():
    units = [100_000, 7, 250_001, 4096]
    c = Case(sum(units), 5, 3, 1 << 16, align=8, units=units, config_id=32)
    R = Ranks(c)
    for t in (1, 2):
        G = c.grads(t)
        R.step(G, t)
        c.step_and_compare(t, G)
    R.compare_with_one_gpu_step()
    lp = Z.zero_plan(sum(units), 5, 3, 1 << 16, align_elems=8, unit_elems=units, max_live=2)
    for u in list(range(len(units))) + list(reversed(range(len(units)))):
        buf = torch.empty(units[u], dtype=torch.bfloat16, device="cuda")
        Z.zero_gather_layer_peers(lp, u, R.params, buf)
        Z.zero_stream_status()
        assert np.array_equal(u16(buf), ST.gather_layer(c.op, u, c.hparams)), u
        Z.zero_release_layer(lp, u)
    assert lp.query(Z.ZERO_Q_PEAK_LIVE_UNITS) == 1


# ---------------------------------------------------- two processes, IPC
IPC_CASES = {
    "stage2": dict(psi=200_003, stage=2, bucket=50_000, align=64, units=None),
    "stage3": dict(psi=150_007, stage=3, bucket=1 << 16, align=8, units=[100_000, 7, 50_000]),
}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ipc_worker(rank, world, port, case, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import zero_partitioned_optimizer_step_b200 as Zw
    from zero_partitioned_optimizer_step_b200 import inputs
    from zero_partitioned_optimizer_step_b200.peer import PeerStep
    from oracle import plan as OPw
    from oracle import step as STw
    limit = datetime.timedelta(seconds=120)
    store = dist.TCPStore("127.0.0.1", port, world, rank == 0, timeout=limit)
    dist.init_process_group("gloo", store=store, rank=rank, world_size=world, timeout=limit)
    msg = "ok"
    try:
        torch.cuda.set_device(0)
        cfg = IPC_CASES[case]
        lp = Zw.zero_plan(cfg["psi"], world, cfg["stage"], cfg["bucket"], align_elems=cfg["align"],
                          unit_elems=cfg["units"], max_live=1)
        op = OPw.make_plan(cfg["psi"], world, cfg["stage"], cfg["bucket"], align=cfg["align"],
                           unit_elems=cfg["units"])
        S = op.S
        adam = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, grad_scale=1.0 / world)
        w_st = STw.logical_to_storage(op, inputs.master_logical(op.unit_len, op.unit_pad, 33, "cpu").numpy())
        # the oracle's copy of the whole job, and this rank's own buffers
        hw, hm, hv = w_st.copy(), np.zeros_like(w_st), np.zeros_like(w_st)
        hp = np.zeros((world, op.psi_pad) if op.stage <= 2 else world * S, np.uint16)
        master = torch.from_numpy(w_st[rank * S:(rank + 1) * S].copy()).cuda()
        m = torch.zeros(S, dtype=torch.float32, device="cuda")
        v = torch.zeros(S, dtype=torch.float32, device="cuda")
        # gradient and parameters inside one allocation, at offsets: the IPC
        # handles carry the offsets, and the peer maps the allocation once
        n_p = op.psi_pad if op.stage <= 2 else S
        g0 = 64 * (1 + rank)
        p0 = g0 + (op.psi_pad + 63) // 64 * 64
        arena = torch.zeros(p0 + n_p + 64, dtype=torch.bfloat16, device="cuda")
        grads, params = arena[g0:g0 + op.psi_pad], arena[p0:p0 + n_p]
        norm = torch.zeros(1, dtype=torch.float64, device="cuda")
        ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
        ws = Zw.workspace_for(lp)
        ps = PeerStep(lp, grads, params, master, m, v)
        for t in (1, 2):
            G = inputs.grads(world, op.unit_len, op.unit_pad, 1e-3, 33, t, "cuda")
            grads.copy_(G[rank])
            ps.step(adam, t, grad_norm_sq=norm, overflow=ovf, workspace=ws)
            Gh = u16(G)
            h_norm, h_bad = STw.step_partitioned(op, Gh, hw, hm, hv, hp, adam, t)
            torch.cuda.synchronize()
            sl = slice(rank * S, (rank + 1) * S)
            assert np.array_equal(f32(master).view(np.uint32), hw[sl].view(np.uint32)), "master"
            assert np.array_equal(f32(m).view(np.uint32), hm[sl].view(np.uint32)), "m"
            assert np.array_equal(f32(v).view(np.uint32), hv[sl].view(np.uint32)), "v"
            want_p = hp[rank] if op.stage <= 2 else hp[sl]
            assert np.array_equal(u16(params), want_p), "params"
            assert abs(norm.item() - h_norm) <= RTOL_NORM * h_norm, (norm.item(), h_norm)
            assert int(ovf.item()) == int(h_bad)
        if op.stage == 3:
            for u, n in enumerate(op.unit_len):
                buf = torch.empty(n, dtype=torch.bfloat16, device="cuda")
                ps.gather_layer(u, buf)
                torch.cuda.synchronize()
                assert np.array_equal(u16(buf), STw.gather_layer(op, u, hp)), "layer %d" % u
                Zw.zero_release_layer(lp, u)
        Zw.zero_stream_status()
        ps.barrier()
        ps.close()
    except Exception as e:  # reported to the parent, which fails the test
        msg = "%s: %s" % (type(e).__name__, e)
    finally:
        # A rank frees its buffers only after every rank has finished all of
        # its kernels (which may read them): each synchronises, says so in the
        # store, and waits for the others.  A rank stuck at a barrier its peer
        # never reaches gets there through the process group's timeout.
        try:
            torch.cuda.synchronize()
            store.set("done%d" % rank, "1")
            store.wait(["done%d" % q for q in range(world)], limit)
        except Exception as e:
            msg += "; exit handshake: %s" % e
        out.put((rank, msg))
        dist.destroy_process_group()


@pytest.mark.parametrize("case", sorted(IPC_CASES))
def test_two_processes_share_buffers_through_ipc(case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_worker, args=(r, 2, port, case, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=600) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=120)
            if p.exitcode is None:
                p.kill()
    assert res == [(0, "ok"), (1, "ok")], res
    assert all(p.exitcode == 0 for p in procs)


@pytest.mark.parametrize("kernel", ["tma", "ldg", "mixed"])
def test_peer_step_writes_stay_inside_their_buffers(kernel, monkeypatch):
    """Every rank's buffers inside guard zones of a fixed byte pattern."""
    from test_canary_fuzz_gpu import Guarded
    psi, nd, stage, bucket, align, units = GUARD_CASE
    c = Case(psi, nd, stage, bucket, align=align, units=units, config_id=34)
    use_kernel(monkeypatch, kernel, c.lp)
    R = Ranks(c)
    guarded = []
    for name in ("master", "m", "v", "red", "params", "norm", "ovf", "ws"):
        bufs = getattr(R, name)
        gs = [Guarded(tuple(x.shape), x.dtype, x) for x in bufs]
        guarded += gs
        setattr(R, name, [g.t for g in gs])
    for t in (1, 2):
        G = c.grads(t)
        gG = [Guarded(tuple(G[q].shape), G.dtype, G[q]) for q in range(c.nd)]
        grads = [g.t for g in gG]
        for r in range(c.nd):
            Z.zero_step_peers(c.lp, r, grads, R.params, R.master[r], R.m[r], R.v[r], c.adam, t,
                              reduced_grad=R.red[r], grad_norm_sq=R.norm[r], overflow=R.ovf[r],
                              workspace=R.ws[r])
        Z.zero_stream_status()
        c.step_and_compare(t, G)
        R.compare_with_one_gpu_step()
        assert all(g.intact() for g in gG + guarded)

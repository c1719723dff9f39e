"""Host-side tests of the ranks-as-devices calls (no kernel is launched):
struct layouts against the C header, argument checks, the IPC bookkeeping
that needs no device, and PeerStep's handle exchange over two gloo ranks."""
import ctypes
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

import zero_partitioned_optimizer_step_b200 as Z

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

LAYOUT_C = r"""
#include <stddef.h>
#include <stdio.h>
#include "zero.h"
#define F(T, m) printf("%s.%s %zu\n", #T, #m, offsetof(T, m))
#define S(T) printf("%s %zu\n", #T, sizeof(T))
int main(void) {
    S(zero_peer_bufs_t); S(zero_ipc_handle_t); S(zero_bufs_t); S(zero_adam_t);
    S(zero_plan_desc_t); S(zero_guard_t);
    F(zero_peer_bufs_t, rank); F(zero_peer_bufs_t, grads); F(zero_peer_bufs_t, params);
    F(zero_peer_bufs_t, master); F(zero_peer_bufs_t, reduced_grad);
    F(zero_peer_bufs_t, workspace_bytes); F(zero_peer_bufs_t, adam_consts);
    F(zero_ipc_handle_t, offset); F(zero_ipc_handle_t, exporter_va);
    F(zero_ipc_handle_t, device); F(zero_ipc_handle_t, exporter_pid);
    F(zero_bufs_t, owner_view); F(zero_bufs_t, adam_consts);
    F(zero_plan_desc_t, unit_elems);
    printf("ZERO_MAX_PEERS %u\n", ZERO_MAX_PEERS);
    return 0;
}
"""


def test_struct_layouts_match_the_header(tmp_path):
    src = tmp_path / "layout.c"
    src.write_text(LAYOUT_C)
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    got = dict(line.rsplit(" ", 1) for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                              check=True).stdout.splitlines())
    got = {k: int(v) for k, v in got.items()}
    want = {
        "zero_peer_bufs_t": ctypes.sizeof(Z._PeerBufs), "zero_ipc_handle_t": ctypes.sizeof(Z._IpcHandle),
        "zero_bufs_t": ctypes.sizeof(Z._Bufs), "zero_adam_t": ctypes.sizeof(Z._Adam),
        "zero_plan_desc_t": ctypes.sizeof(Z._PlanDesc), "zero_guard_t": ctypes.sizeof(Z._Guard),
        "ZERO_MAX_PEERS": Z.ZERO_MAX_PEERS,
    }
    for name, cls in (("zero_peer_bufs_t", Z._PeerBufs), ("zero_ipc_handle_t", Z._IpcHandle),
                      ("zero_bufs_t", Z._Bufs), ("zero_plan_desc_t", Z._PlanDesc)):
        for k in got:
            if k.startswith(name + "."):
                want[k] = getattr(cls, k.split(".", 1)[1]).offset
    assert got == want


def _peer_bufs(nd, rank=0, **kw):
    grads = (ctypes.c_void_p * nd)(*[4096 * (q + 1) for q in range(nd)])
    params = (ctypes.c_void_p * nd)(*[1 << 20 | 4096 * q for q in range(nd)])
    b = Z._PeerBufs()
    b.rank = rank
    b.grads = ctypes.cast(grads, ctypes.POINTER(ctypes.c_void_p))
    b.params = ctypes.cast(params, ctypes.POINTER(ctypes.c_void_p))
    b.master, b.exp_avg, b.exp_avg_sq = 1 << 24, 2 << 24, 3 << 24
    for k, v in kw.items():
        setattr(b, k, v)
    b._keep = (grads, params)
    return b, grads, params


def test_step_peers_argument_checks():
    L = Z.lib()
    adam = Z.make_adam(dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, grad_scale=0.25))
    pl = Z.zero_plan(1000, 4, 2, 100)

    def call(b, plan=pl, t=1, first=0, count=None):
        count = plan.n_buckets if count is None else count
        return L.zero_step_peers(plan.handle, ctypes.byref(b), ctypes.byref(adam), t, first, count, None)

    b, g, p = _peer_bufs(4)
    assert call(b, t=0) == Z.ZERO_EINVAL
    assert call(_peer_bufs(4, rank=4)[0]) == Z.ZERO_EINVAL
    assert "rank" in L.zero_last_error().decode()
    assert call(b, plan=Z.zero_plan(1000, 4, 0, 100)) == Z.ZERO_EINVAL
    assert "stage 0" in L.zero_last_error().decode()
    g[2] = 4096 + 8                                   # misaligned peer gradient
    assert call(b) == Z.ZERO_EINVAL and "grads[2]" in L.zero_last_error().decode()
    g[2] = None
    assert call(b) == Z.ZERO_EINVAL and "grads[2]" in L.zero_last_error().decode()
    b, g, p = _peer_bufs(4)
    p[3] = None                                       # a replica is missing at stage 2
    assert call(b) == Z.ZERO_EINVAL and "params[3]" in L.zero_last_error().decode()
    pl3 = Z.zero_plan(1000, 4, 3, 100)
    b, g, p = _peer_bufs(4, rank=1)
    p[0] = p[2] = p[3] = None                         # stage 3 needs only params[rank]
    b.master = 0
    assert call(b, plan=pl3) == Z.ZERO_EINVAL and "master" in L.zero_last_error().decode()
    b, g, p = _peer_bufs(4, grad_norm_sq=1 << 26)
    assert call(b) == Z.ZERO_EINVAL and "workspace" in L.zero_last_error().decode()
    b, g, p = _peer_bufs(4)
    assert call(b, first=1, count=pl.n_buckets) == Z.ZERO_EINVAL
    big = Z.zero_plan(129 * 64, 129, 2, 1000)
    assert call(_peer_bufs(129)[0], plan=big) == Z.ZERO_EINVAL
    assert "ZERO_MAX_PEERS" in L.zero_last_error().decode()
    assert L.zero_step_peers(pl.handle, None, ctypes.byref(adam), 1, 0, 1, None) == Z.ZERO_EINVAL


@pytest.mark.skipif(torch.cuda.is_available(), reason="needs a machine without a CUDA device")
def test_valid_peer_step_without_device_reports_ecuda():
    L = Z.lib()
    adam = Z.make_adam(dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, grad_scale=0.25))
    pl = Z.zero_plan(1000, 4, 2, 100)
    b, g, p = _peer_bufs(4)
    assert L.zero_step_peers(pl.handle, ctypes.byref(b), ctypes.byref(adam), 1, 0, pl.n_buckets,
                             None) == Z.ZERO_ECUDA


def test_step_peers_kernel_argument_checks():
    """The kernel query checks its arguments before it looks at the device."""
    L = Z.lib()
    out = ctypes.c_uint32()
    pl = Z.zero_plan(1000, 4, 2, 100)
    assert L.zero_step_peers_kernel(None, 0, 0, 1, ctypes.byref(out)) == Z.ZERO_EINVAL
    assert L.zero_step_peers_kernel(pl.handle, 0, 0, 1, None) == Z.ZERO_EINVAL
    assert L.zero_step_peers_kernel(pl.handle, 4, 0, 1, ctypes.byref(out)) == Z.ZERO_EINVAL
    assert "rank" in L.zero_last_error().decode()
    assert L.zero_step_peers_kernel(pl.handle, 0, 1, pl.n_buckets, ctypes.byref(out)) == Z.ZERO_EINVAL
    assert "bucket" in L.zero_last_error().decode()
    pl0 = Z.zero_plan(1000, 4, 0, 100)
    assert L.zero_step_peers_kernel(pl0.handle, 0, 0, 1, ctypes.byref(out)) == Z.ZERO_EINVAL
    big = Z.zero_plan(129 * 64, 129, 2, 1000)
    assert L.zero_step_peers_kernel(big.handle, 0, 0, 1, ctypes.byref(out)) == Z.ZERO_EINVAL
    assert "ZERO_MAX_PEERS" in L.zero_last_error().decode()


@pytest.mark.skipif(torch.cuda.is_available(), reason="needs a machine without a CUDA device")
def test_step_peers_kernel_without_device_reports_ecuda():
    out = ctypes.c_uint32()
    pl = Z.zero_plan(1000, 4, 2, 100)
    assert Z.lib().zero_step_peers_kernel(pl.handle, 0, 0, pl.n_buckets, ctypes.byref(out)) == Z.ZERO_ECUDA


def test_gather_layer_peers_argument_checks():
    L = Z.lib()
    pl = Z.zero_plan(1000, 4, 3, 100, unit_elems=[400, 600])
    arr = (ctypes.c_void_p * 4)(4096, 8192, 12288, 16384)
    ptrs = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    dst = ctypes.c_void_p(1 << 20)
    assert L.zero_gather_layer_peers(pl.handle, 2, ptrs, dst, None) == Z.ZERO_EINVAL      # unit
    assert L.zero_gather_layer_peers(pl.handle, 0, None, dst, None) == Z.ZERO_EINVAL
    assert L.zero_gather_layer_peers(pl.handle, 0, ptrs, ctypes.c_void_p((1 << 20) + 2), None) == Z.ZERO_EINVAL
    arr[1] = 8200
    assert L.zero_gather_layer_peers(pl.handle, 0, ptrs, dst, None) == Z.ZERO_EINVAL
    assert "owner_params[1]" in L.zero_last_error().decode()
    pl2 = Z.zero_plan(1000, 4, 2, 100)
    arr[1] = 8192
    assert L.zero_gather_layer_peers(pl2.handle, 0, ptrs, dst, None) == Z.ZERO_EINVAL
    assert pl.query(Z.ZERO_Q_LIVE_UNITS) == 0


def _handle(pid, va, offset, alloc=1 << 20):
    h = Z._IpcHandle()
    h.exporter_pid, h.exporter_va, h.offset, h.alloc_bytes, h.device = pid, va, offset, alloc, 0
    return bytes(h)


def test_ipc_open_of_own_handle_maps_nothing_and_counts_references():
    va = 1 << 40
    a = Z.zero_ipc_open(_handle(os.getpid(), va, 256))
    b = Z.zero_ipc_open(_handle(os.getpid(), va, 4096))
    assert (a, b) == (va + 256, va + 4096)
    Z.zero_ipc_close(a)
    Z.zero_ipc_close(b)
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_ipc_close(b)
    assert e.value.status == Z.ZERO_EINVAL
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_ipc_open(_handle(os.getpid(), va, 1 << 20))     # offset outside the allocation
    assert e.value.status == Z.ZERO_EINVAL
    with pytest.raises(ValueError):
        Z.zero_ipc_open(b"short")


@pytest.mark.skipif(torch.cuda.is_available(), reason="needs a machine without a CUDA device")
def test_ipc_without_device_fails_cleanly():
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_ipc_open(_handle(os.getpid() + 1, 1 << 40, 0))
    assert e.value.status == Z.ZERO_ECUDA
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_ipc_export(1 << 20)
    assert e.value.status == Z.ZERO_EINVAL


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _exchange_worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import zero_partitioned_optimizer_step_b200 as Zw
    from zero_partitioned_optimizer_step_b200.peer import PeerStep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        opened, closed = [], []

        def fake_export(t):
            return ("r%d:%s" % (rank, t.tag)).encode()

        def fake_open(h):
            opened.append(h.decode())
            return 1000 * (len(opened))

        class Buf:
            def __init__(self, tag):
                self.tag, self.device = tag, "cpu"

        plan = Zw.zero_plan(1000, world, 2, 100)
        ps = PeerStep(plan, Buf("g"), Buf("p"), None, None, None, ipc_open=fake_open,
                      ipc_close=closed.append, ipc_export=fake_export)
        kinds = [(x.tag if isinstance(x, Buf) else x) for x in ps.grads + ps.params]
        ps.barrier()
        ps.close()
        out.put((rank, opened, kinds, closed))
    finally:
        dist.destroy_process_group()


def test_peer_step_maps_every_other_rank_and_unmaps_on_close():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 3
    procs = [ctx.Process(target=_exchange_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, opened, kinds, closed in res:
        others = [o for o in range(world) if o != rank]
        assert opened == [s for o in others for s in ("r%d:g" % o, "r%d:p" % o)]
        # own buffers in place, the peers' as the addresses ipc_open returned
        g, p = kinds[:world], kinds[world:]
        assert g[rank] == "g" and p[rank] == "p"
        assert [g[o] for o in others] == [1000 * (2 * i + 1) for i in range(len(others))]
        assert [p[o] for o in others] == [1000 * (2 * i + 2) for i in range(len(others))]
        assert sorted(closed) == sorted([g[o] for o in others] + [p[o] for o in others])


def _dropout_worker(rank, world, port, out):
    """Rank 1 builds its PeerStep and then leaves without stepping; rank 0's
    step must end with an error from the process group's timeout, not hang."""
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import zero_partitioned_optimizer_step_b200 as Zw
    from zero_partitioned_optimizer_step_b200.peer import PeerStep
    store = dist.TCPStore("127.0.0.1", port, world, rank == 0, timeout=datetime.timedelta(seconds=30))
    dist.init_process_group("gloo", store=store, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=3))

    class Buf:
        def __init__(self, tag):
            self.tag, self.device = tag, "cpu"

    calls = []
    plan = Zw.zero_plan(1000, world, 2, 100)
    ps = PeerStep(plan, Buf("g"), Buf("p"), None, None, None, ipc_open=lambda h: 4096,
                  ipc_close=lambda p: None, ipc_export=lambda t: b"x")
    if rank == 1:
        out.put((rank, "left"))
        out.close()
        out.join_thread()   # the message is out before the process is
        os._exit(0)   # gone between steps: no kernel or collective of it in flight
    import zero_partitioned_optimizer_step_b200.peer as P
    P.zero_step_peers = lambda *a, **k: calls.append("kernel")   # the barrier decides
    try:
        ps.step(dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, grad_scale=0.5), 1)
        out.put((rank, "stepped"))
    except Exception as e:  # the expected path
        out.put((rank, "error:" + type(e).__name__ + ":" + ("kernel" if calls else "no-kernel")))


def test_a_rank_that_leaves_makes_the_next_step_fail_not_hang():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dropout_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = dict(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.exitcode is None:
                p.kill()
    assert res[1] == "left"
    assert res[0].startswith("error:") and res[0].endswith(":no-kernel"), res


def test_header_compiles_as_c_and_cpp(tmp_path):
    """include/zero.h is plain C99 and also valid C++ (extern "C")."""
    src = tmp_path / "h.c"
    src.write_text('#include "zero.h"\nint main(void) { return (int)sizeof(zero_peer_bufs_t) == 0; }\n')
    for cc, std, name in (("gcc", "-std=c99", "h.c"), ("g++", "-std=c++17", "h.cpp")):
        f = tmp_path / name
        f.write_text(src.read_text())
        subprocess.run([cc, std, "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"), "-c",
                        str(f), "-o", str(tmp_path / (name + ".o"))], check=True)


def test_mixed_mode_splits_the_calls():
    """The GPU parity tests' mixed mode sets the per-call threshold so that
    some ranks' calls fall on each side of it wherever their mean body
    sizes differ."""
    from test_peer_gpu import GUARD_CASE, PEER_CASES, call_means

    split = 0
    for psi, nd, stage, bucket, align, units in PEER_CASES + [GUARD_CASE]:
        lp = Z.zero_plan(psi, nd, stage, bucket, align_elems=align, unit_elems=units)
        means = sorted({m for m in call_means(lp) if m is not None})
        if len(means) > 1:
            thr = means[len(means) // 2]
            assert min(means) < thr <= max(means)
            split += 1
    assert split >= 3

"""NVTX ranges of the library (host side), recorded by a minimal NVTX tool.

tests/c/nvtx_recorder.c is built here with gcc and loaded by NVTX through
NVTX_INJECTION64_PATH; it writes every push, pop and mark of the domain API
to a file.  Each case runs in a child process, since NVTX reads its
environment once per process.

CPU: with ZERO_NVTX=1 a zero_step call opens and closes its range even when
it fails (no GPU here: the call returns ZERO_ECUDA after the range opened);
without ZERO_NVTX the library makes no NVTX call at all, so the tool is never
loaded.  GPU: a stage-3 step shows one range per bucket inside the call's
range, the finalize, a range per layer gather and a mark per release, and
every push is popped.
"""
import os
import subprocess
import sys
import textwrap

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = "/usr/local/cuda/include"


@pytest.fixture(scope="module")
def recorder(tmp_path_factory):
    if not os.path.exists(os.path.join(CUDA_INC, "nvtx3", "nvToolsExt.h")):
        pytest.skip("NVTX headers not found")
    out = str(tmp_path_factory.mktemp("nvtx") / "libnvtx_recorder.so")
    subprocess.run(["gcc", "-O1", "-std=c99", "-fPIC", "-shared", "-Wall", "-Wextra", "-I", CUDA_INC,
                    os.path.join(ROOT, "tests", "c", "nvtx_recorder.c"), "-o", out], check=True)
    return out


def _run(script, recorder, log, nvtx_on):
    env = dict(os.environ, NVTX_INJECTION64_PATH=recorder, ZERO_NVTX_LOG=str(log))
    env.pop("ZERO_NVTX", None)
    if nvtx_on:
        env["ZERO_NVTX"] = "1"
    r = subprocess.run([sys.executable, "-c", textwrap.dedent(script)], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-3000:]
    return r.stdout


def _events(log):
    if not os.path.exists(log):
        return []
    with open(log) as f:
        return [ln.rstrip("\n") for ln in f if ln.strip()]


def _balanced(ev):
    depth = 0
    for e in ev:
        if e.startswith("push "):
            depth += 1
        elif e == "pop":
            depth -= 1
            assert depth >= 0, ev
    assert depth == 0, ev


CPU_CALL = """
    import ctypes
    import zero_partitioned_optimizer_step_b200 as Z
    lp = Z.zero_plan(4096, 4, 2, 2048)
    b = Z._Bufs()
    for f in ("grads", "master", "exp_avg", "exp_avg_sq", "params"):
        setattr(b, f, 0x1000)          # never dereferenced: the call stops before any launch
    b.grad_stride = b.param_stride = lp.psi_pad
    b.owner_view = -1
    adam = Z.make_adam(dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, grad_scale=0.25))
    st = Z.lib().zero_step(lp.handle, ctypes.byref(b), ctypes.byref(adam), 1, None)
    print(st)
"""


@pytest.mark.skipif(torch.cuda.is_available(), reason="the call must fail for lack of a GPU")
def test_nvtx_range_on_a_failed_call_without_gpu(recorder, tmp_path):
    log = tmp_path / "on.log"
    out = _run(CPU_CALL, recorder, log, True)
    import zero_partitioned_optimizer_step_b200 as Z
    assert int(out.split()[-1]) == Z.ZERO_ECUDA
    ev = _events(log)
    assert ev[0] == "domain zero"
    assert ev[1:] == ["push zero_step t=1 buckets [0, 2)", "pop"], ev


def test_nvtx_off_makes_no_nvtx_call(recorder, tmp_path):
    log = tmp_path / "off.log"
    _run(CPU_CALL, recorder, log, False)
    assert _events(log) == []


GPU_STEP = """
    import torch
    import zero_partitioned_optimizer_step_b200 as Z
    from zero_partitioned_optimizer_step_b200 import inputs
    units = [3000, 5000, 700]
    lp = Z.zero_plan(sum(units), 4, 3, 2048, unit_elems=units)
    n = lp.nd * lp.S
    G = inputs.grads(4, units, [u[1] for u in lp.units()], 1e-3, 9, 1, "cuda")
    w = torch.zeros(n, device="cuda"); m = torch.zeros_like(w); v = torch.zeros_like(w)
    p = torch.zeros(n, dtype=torch.bfloat16, device="cuda")
    norm = torch.zeros(1, dtype=torch.float64, device="cuda")
    ovf = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = Z.workspace_for(lp, "cuda")
    adam = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, grad_scale=0.25)
    Z.zero_step(lp, G, w, m, v, p, adam, 1, grad_norm_sq=norm, overflow=ovf, workspace=ws)
    buf = torch.empty(max(units), dtype=torch.bfloat16, device="cuda")
    for u in range(len(units)):
        Z.zero_gather_layer(lp, u, p, buf[:units[u]])
        Z.zero_release_layer(lp, u)
    Z.zero_stream_status()
    print(lp.n_buckets)
"""


@pytest.mark.gpu
def test_nvtx_ranges_of_a_stage3_step_and_its_gathers(recorder, tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    log = tmp_path / "gpu.log"
    nb = int(_run(GPU_STEP, recorder, log, True).split()[-1])
    ev = _events(log)
    _balanced(ev)
    assert ev[0] == "domain zero"
    pushes = [e[5:] for e in ev if e.startswith("push ")]
    assert pushes[:1 + nb + 1] == (["zero_step t=1 buckets [0, %d)" % nb] +
                                   ["bucket %d" % k for k in range(nb)] + ["norm finalize"])
    for u in range(3):
        assert "zero_gather_layer unit %d" % u in pushes
        assert "mark zero_release_layer unit %d" % u in ev
    # each release comes after its gather's range closed
    for u in range(3):
        g = ev.index("push zero_gather_layer unit %d" % u)
        assert ev[g + 1] == "pop" and ev[g + 2] == "mark zero_release_layer unit %d" % u

"""A plain C program (tests/c/step_example.c) drives two ZeRO steps on the
GPU through the C ABI alone (device memory from the CUDA runtime, no Python
in the loop); its inputs and outputs are compared with the oracle here."""
import os
import subprocess

import numpy as np
import pytest
import torch

import zero_partitioned_optimizer_step_b200 as Z
from oracle import plan as OP
from oracle import step as ST
from zero_cases import RTOL_NORM

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def test_c_program_steps_match_oracle(tmp_path):
    lib_dir = os.path.dirname(Z.LIB_PATH)
    exe = tmp_path / "step_example"
    subprocess.run(["gcc", "-std=c99", "-O1", "-I", os.path.join(ROOT, "include"), "-I",
                    os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c", "step_example.c"),
                    "-L", lib_dir, "-lzero", "-Wl,-rpath," + lib_dir, "-L", os.path.join(CUDA, "lib64"),
                    "-lcudart", "-Wl,-rpath," + os.path.join(CUDA, "lib64"), "-o", str(exe)], check=True)
    out = tmp_path / "out.bin"
    r = subprocess.run([str(exe), str(out)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr
    raw = out.read_bytes()
    nd, psi_pad, S = np.frombuffer(raw, np.uint64, 3)
    nd, psi_pad, S = int(nd), int(psi_pad), int(S)
    off = 24
    def take(dtype, count):
        nonlocal off
        a = np.frombuffer(raw, dtype, count, off)
        off += a.nbytes
        return a
    g = take(np.uint16, 2 * nd * psi_pad).reshape(2, nd, psi_pad)
    w0 = take(np.float32, nd * S).copy()
    got = take(np.float32, 4 * nd * S).reshape(4, nd * S)
    params = take(np.uint16, nd * psi_pad).reshape(nd, psi_pad)
    norms = take(np.float64, 2)
    ovfs = take(np.int32, 2)
    assert off == len(raw)

    op = OP.make_plan(65_536, 4, 2, 16_384)
    assert (op.psi_pad, op.S) == (psi_pad, S)
    adam = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, grad_scale=0.25, weight_decay=0.01)
    w, m, v = w0, np.zeros_like(w0), np.zeros_like(w0)
    red = np.zeros_like(w0)
    hp = np.zeros((nd, psi_pad), np.uint16)
    for t in (1, 2):
        norm, bad = ST.step_partitioned(op, np.ascontiguousarray(g[t - 1]), w, m, v, hp, adam, t, reduced=red)
        assert abs(norms[t - 1] - norm) <= RTOL_NORM * norm and int(ovfs[t - 1]) == int(bad > 0)
    for i, (want, name) in enumerate(((w, "master"), (m, "exp_avg"), (v, "exp_avg_sq"), (red, "reduced"))):
        assert np.array_equal(got[i].view(np.uint32), want.view(np.uint32)), name
    assert np.array_equal(params, hp)

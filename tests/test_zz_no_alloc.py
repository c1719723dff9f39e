"""zero_step_noalloc() gives the same step as zero_step().

zero_step_noalloc() serves callers that cannot allocate device memory -- for
example a runtime whose device memory is all handed out by its own pool up
front, or a plain C caller without an allocator: instead of a caller-provided
workspace, the gradient-norm / overflow scratch is the library's own static
device array.  This test calls it through the C ABI twice in a row and
checks every output against zero_step() with a caller-provided workspace on
the same inputs: replicas at stage 2, owner shards of several layers at
stage 3, and the one-owner view.  Free device memory is read around the
second call, after the first has loaded the library's static array: an
allocation of any size inside the call would reserve at least one page of it.
The file is named to run last.
"""
import ctypes
import gc

import pytest
import torch

import zero_partitioned_optimizer_step_b200 as Z
from zero_cases import (BF16_ULP, RTOL_NORM, RTOL_REDUCED, RTOL_STATE, Case, bf16_ulp_check,
                        f32, f32_rel_check, u16)

pytestmark = pytest.mark.gpu

CASES = {
    "stage2_replicas": dict(psi=1_000_003, nd=8, stage=2, bucket=100_000),
    "stage3_layers": dict(psi=3 * 70_001 + 999, nd=5, stage=3, bucket=50_000,
                          units=[70_001, 70_001, 70_001, 999]),
    "owner_view": dict(psi=64 * 20_000, nd=64, stage=2, bucket=300_000, owner_view=5),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_step_matches_zero_step_on_two_calls(name):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kw = dict(CASES[name])
    args = (kw.pop("psi"), kw.pop("nd"), kw.pop("stage"), kw.pop("bucket"))
    ref = Case(*args, config_id=2, **kw)   # zero_step + workspace
    new = Case(*args, config_id=2, **kw)   # zero_step_noalloc
    L = Z.lib()
    for t in (1, 2):
        G = ref.grads(t)
        ref.run_gpu(G, t)
        bufs = Z.make_bufs(new.lp, G, new.w, new.m, new.v, new.params, reduced_grad=new.red,
                           grad_norm_sq=new.norm, overflow=new.ovf, owner_view=new.owner)
        adam = Z.make_adam(new.adam)
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        # no garbage collection inside the measured window: a collection
        # there would free tensors of earlier tests and move the counters
        gc.collect()
        gc.disable()
        try:
            before = torch.cuda.memory_allocated()
            free_before = torch.cuda.mem_get_info()[0]
            st = L.zero_step_noalloc(new.lp.handle, ctypes.byref(bufs), ctypes.byref(adam), t, stream)
            torch.cuda.synchronize()
            after = torch.cuda.memory_allocated()
            free_after = torch.cuda.mem_get_info()[0]
        finally:
            gc.enable()
        assert st == Z.ZERO_OK, L.zero_last_error().decode()
        assert after == before
        if t == 2:
            assert free_after == free_before
        f32_rel_check(f32(new.w), f32(ref.w), RTOL_STATE, "master")
        f32_rel_check(f32(new.m), f32(ref.m), RTOL_STATE, "exp_avg")
        f32_rel_check(f32(new.v), f32(ref.v), RTOL_STATE, "exp_avg_sq")
        f32_rel_check(f32(new.red), f32(ref.red), RTOL_REDUCED, "reduced")
        bf16_ulp_check(u16(new.params), u16(ref.params), BF16_ULP, "params")
        n_ref, n_new = ref.norm.item(), new.norm.item()
        assert n_ref > 0
        assert abs(n_new - n_ref) <= RTOL_NORM * n_ref
        assert int(new.ovf.item()) == int(ref.ovf.item()) == 0


def test_noalloc_rejects_bad_arguments():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    c = Case(4096, 4, 2, 1024, config_id=2)
    G = c.grads(1)
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_step_noalloc(c.lp, G, c.w, c.m, c.v, c.params, c.adam, 0,
                            grad_norm_sq=c.norm, overflow=c.ovf)
    assert e.value.status == Z.ZERO_EINVAL

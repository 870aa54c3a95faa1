"""dfssm_linear_fwd_noalloc: the entry point that allocates nothing.

It is there for callers that cannot call cudaMalloc, for instance an embedder
whose device allocator must not be re-entered from inside the layer, or a host
with a fixed device memory budget: the kernel's only scratch (its error word)
is a fixed device array inside the library. This test calls it through the C
ABI and checks its output bit for bit against dfssm_linear_fwd (the same
kernel on the same inputs) and against the oracle, on two calls in a row with
different shapes and tokens, so the second call also shows that what the first
left in the shared scratch does not leak into its result. The file is named to
be collected last.
"""
import numpy as np
import pytest
import torch

import bit_gemv_gemm_dfssm_b200 as dfssm
from gpu_util import Linear, check_linear_full

pytestmark = pytest.mark.gpu


def run_plan(lin):
    lin.dy.fill_(float("nan"))
    plan = dfssm.dfssm_linear_plan([lin.desc()])
    try:
        dfssm.dfssm_linear_fwd(plan, 0, lin.weights(), lin.dx.data_ptr(), lin.m, lin.dy.data_ptr(), None,
                               torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        return lin.y_host().copy()
    finally:
        dfssm.dfssm_plan_destroy(plan)


def run_noalloc(lin):
    lin.dy.fill_(float("nan"))
    desc = dfssm.LinearDesc(lin.d_in, lin.d_out, dfssm.RANK, lin.m, lin.y_dtype, 0)
    st = dfssm.lib().dfssm_linear_fwd_noalloc(desc, lin.weights(), lin.dx.data_ptr(), lin.m, lin.dy.data_ptr(),
                                              torch.cuda.current_stream().cuda_stream)
    assert st == dfssm.DFSSM_OK, dfssm.dfssm_status_string(st)
    torch.cuda.synchronize()
    return lin.y_host().copy()


def test_noalloc_matches_plan_entry_point_twice():
    cases = [(4096, 2048, 1, dfssm.DFSSM_BF16), (2048, 1000, 5, dfssm.DFSSM_F32)]
    for i, (d_in, d_out, m, y_dtype) in enumerate(cases):
        lin = Linear(0x5EED + i, 9, 500 + i, d_in, d_out, m, y_dtype, dbg=False)
        ref = run_plan(lin)
        got = run_noalloc(lin)
        assert np.array_equal(got.view(np.uint8), ref.view(np.uint8)), "outputs differ from dfssm_linear_fwd"
        check_linear_full(lin)          # lin.dy holds the no-allocation call's output


def test_noalloc_allocates_no_device_memory():
    # after the first call (the per-device set-up), repeated calls leave the device's free memory
    # unchanged
    lin = Linear(0x5EED, 9, 600, 2048, 640, 3, dfssm.DFSSM_BF16, dbg=False)
    run_noalloc(lin)
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        run_noalloc(lin)
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_refuses_sizes_beyond_its_limits():
    lin = Linear(7, 9, 1, 256, 64, 1, dfssm.DFSSM_F32, dbg=False)
    too_many = dfssm.LinearDesc(256, 64, dfssm.RANK, 32, dfssm.DFSSM_F32, 0)
    st = dfssm.lib().dfssm_linear_fwd_noalloc(too_many, lin.weights(), lin.dx.data_ptr(),
                                              dfssm.DFSSM_NOALLOC_MAX_M + 1, lin.dy.data_ptr(), None)
    assert st == dfssm.DFSSM_ERR_UNSUPPORTED_SHAPE
    wide = dfssm.LinearDesc(16384, 64, dfssm.RANK, 1, dfssm.DFSSM_F32, 0)
    st = dfssm.lib().dfssm_linear_fwd_noalloc(wide, lin.weights(), lin.dx.data_ptr(), 1, lin.dy.data_ptr(), None)
    assert st == dfssm.DFSSM_ERR_UNSUPPORTED_SHAPE

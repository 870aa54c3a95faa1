"""Residual add + RMS norm (dfssm_add_rmsnorm) on the GPU against the oracle, through the C ABI.

The residual is one fp32 addition per element: bit for bit. The output carries a relative
error below 1e-6 (fp32 sum of squares in a fixed order, correctly rounded square root and
division, two products): fp32 outputs within 2^-18 |ref| (and 1e-3 normwise); bf16 outputs
equal the nearest bf16 of the oracle's value, or either neighbour where that value lies within
2^-18 |ref| of a rounding midpoint.
"""
import numpy as np
import pytest
import torch

import bit_gemv_gemm_dfssm_b200 as dfssm
import oracle
from gpu_util import check_y

pytestmark = pytest.mark.gpu
BF16, F32 = dfssm.DFSSM_BF16, dfssm.DFSSM_F32


def run(r, delta, w, eps, out_dtype, in_place=False):
    m, d = r.shape
    dr = torch.from_numpy(r.copy()).cuda()
    dd = None
    if delta is not None:
        dd = torch.from_numpy(delta.view(np.int16).copy() if delta.dtype == np.uint16 else delta.copy()).cuda()
    dw = torch.from_numpy(w.copy()).cuda()
    ro = dr if in_place else torch.full((m, d), float("nan"), dtype=torch.float32, device="cuda")
    out = torch.full((m, d), float("nan"), dtype=torch.bfloat16 if out_dtype == BF16 else torch.float32,
                     device="cuda")
    ddt = BF16 if delta is not None and delta.dtype == np.uint16 else F32
    dfssm.dfssm_add_rmsnorm(dw.data_ptr(), d, eps, dr.data_ptr(), dd.data_ptr() if dd is not None else 0, ddt, m,
                            ro.data_ptr(), out.data_ptr(), out_dtype, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    o = out.view(torch.int16).cpu().numpy().view(np.uint16) if out_dtype == BF16 else out.cpu().numpy()
    return ro.cpu().numpy(), o


def inputs(seed, m, d, delta_kind):
    rng = np.random.default_rng(seed)
    r = (rng.standard_normal((m, d)) * rng.uniform(0.05, 20, (m, 1))).astype(np.float32)
    w = rng.uniform(0.5, 1.5, d).astype(np.float32)
    delta = None
    if delta_kind == "f32":
        delta = rng.standard_normal((m, d)).astype(np.float32)
    elif delta_kind == "bf16":
        delta = oracle.f64_to_bf16(rng.standard_normal((m, d)))
    return r, delta, w


@pytest.mark.parametrize("m,d,delta_kind,out_dtype", [(1, 2048, "bf16", BF16), (3, 8, None, F32),
                                                     (5, 8192, "f32", BF16), (2, 2056, "bf16", F32),
                                                     (16, 512, None, BF16)])
def test_add_rmsnorm_parity(m, d, delta_kind, out_dtype):
    r, delta, w = inputs(m * 1000 + d, m, d, delta_kind)
    ro, o = run(r, delta, w, 1e-5, out_dtype)
    ref = oracle.add_rmsnorm(r, delta, w, 1e-5)
    np.testing.assert_array_equal(ro, ref["resid"])
    check_y(o, ref["out"], 2.0 ** -18 * np.abs(ref["out"]), out_dtype)


def test_add_rmsnorm_in_place_and_zero_rows():
    r, delta, w = inputs(9, 4, 1024, "bf16")
    r[1] = 0.0
    delta[1] = 0
    ro, o = run(r, delta, w, 0.25, BF16, in_place=True)
    ref = oracle.add_rmsnorm(r, delta, w, 0.25)
    np.testing.assert_array_equal(ro, ref["resid"])
    assert (o[1] == 0).all()
    check_y(o, ref["out"], 2.0 ** -18 * np.abs(ref["out"]), BF16)

"""Helpers for the GPU parity tests: device buffers, library calls, comparisons.

Tolerance (the layer's floating-point output): the oracle computes y in float64
from the exact int32 sums; the CUDA epilogue computes it in fp32 in a fixed
order. For every element the fp32 rounding error is bounded by a few units of
2^-24 times the magnitudes of the two terms,
    T_i = |s_x alpha acc| + |s_x s_A| * sum_k |W_A[o,k] s_B[k] h[t,k]|,
and the checks use eb_i = 2^-16 * T_i (about 250x that bound):
  * fp32 output: |y_gpu - y_ref| <= eb_i elementwise, and the normwise
    max-abs-rel error max|y_gpu - y_ref| / max|y_ref| <= 1e-3;
  * bf16 output: y_gpu equals bf16_RNE(y_ref), except where bf16_RNE(y_ref - eb_i)
    and bf16_RNE(y_ref + eb_i) differ (y_ref near a rounding midpoint), where any
    bf16 value between those two is accepted; the normwise error against
    bf16_RNE(y_ref) over the other elements is 0.
Integer results (q, s_x, sum terms acc and h) must match bit for bit.
"""
from __future__ import annotations

import numpy as np
import torch

import bit_gemv_gemm_dfssm_b200 as dfssm
import dfssm_synth as synth
import oracle

TOL_NORMWISE = 1e-3


def dev(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


class Linear:
    """One linear's host inputs, device copies and output buffers."""

    def __init__(self, seed, cfg, index, d_in, d_out, m, y_dtype=dfssm.DFSSM_BF16, x=None, w=None, dbg=True):
        self.d_in, self.d_out, self.m, self.y_dtype = d_in, d_out, m, y_dtype
        self.w = w if w is not None else synth.linear_weights(seed, synth.weight_cfg(cfg), index, d_in, d_out)
        self.x = x if x is not None else synth.activations(seed, cfg, index, m, d_in)
        self.dw = {k: dev(v) for k, v in self.w.items()}
        self.dx = dev(self.x)
        tdt = torch.bfloat16 if y_dtype == dfssm.DFSSM_BF16 else torch.float32
        self.dy = torch.full((m, d_out), float("nan"), dtype=tdt, device="cuda")
        self.dbg = None
        if dbg:
            self.dq = torch.zeros((m, d_in), dtype=torch.int8, device="cuda")
            self.dsx = torch.zeros(m, dtype=torch.float32, device="cuda")
            self.dacc = torch.zeros((m, d_out), dtype=torch.int32, device="cuda")
            self.dh = torch.zeros((m, 16), dtype=torch.int32, device="cuda")
            self.dbg = dfssm.Debug(self.dq.data_ptr(), self.dsx.data_ptr(), self.dacc.data_ptr(),
                                   self.dh.data_ptr())

    def weights(self):
        d = self.dw
        return dfssm.weights_struct(d["sign"], d["alpha"], d["wa"], d["sa"], d["wb"], d["sb"])

    def entry(self, index, with_dbg=True):
        dbg = self.dbg if (self.dbg is not None and with_dbg) else dfssm.Debug(0, 0, 0, 0)
        return dfssm.StackEntry(self.weights(), self.dx.data_ptr(), self.dy.data_ptr(), dbg, index, 0)

    def desc(self, max_m=None):
        return (self.d_in, self.d_out, max_m or self.m, self.y_dtype)

    def y_host(self):
        if self.y_dtype == dfssm.DFSSM_BF16:
            return self.dy.view(torch.int16).cpu().numpy().view(np.uint16)
        return self.dy.cpu().numpy()


def mapped_address(host_ptr: int) -> int:
    """The device address of pinned host memory; raises before any launch if it is not mapped."""
    from cuda.bindings import runtime as rt
    err, attr = rt.cudaPointerGetAttributes(host_ptr)
    assert err == rt.cudaError_t.cudaSuccess and attr.type == rt.cudaMemoryType.cudaMemoryTypeHost, err
    assert attr.devicePointer
    return int(attr.devicePointer)


def entries_device(entries) -> torch.Tensor:
    raw = dfssm.stack_entries_bytes(entries)
    return torch.frombuffer(bytearray(raw), dtype=torch.uint8).cuda()


def term_bound(ref, w, rows=None):
    """eb = 2^-16 * (|s_x alpha acc| + |s_x s_A| sum_k |W_A s_B h|) per element."""
    sx = ref["sx"].astype(np.float64)[:, None]
    alpha = w["alpha"].astype(np.float64)
    sa = w["sa"].astype(np.float64)
    wa = w["wa"].astype(np.float64)
    if rows is not None:
        alpha, sa, wa = alpha[rows], sa[rows], wa[rows]
    t1 = np.abs(sx * alpha[None, :] * ref["acc"])
    lora_abs = np.abs(ref["h"].astype(np.float64) * w["sb"].astype(np.float64)[None, :]) @ np.abs(wa).T
    t2 = np.abs(sx * sa[None, :]) * lora_abs
    return 2.0 ** -16 * (t1 + t2)


def check_y(y_gpu, y_ref, eb, y_dtype):
    """Raise AssertionError unless y_gpu meets the tolerance above. Returns stats."""
    y_ref = np.asarray(y_ref, np.float64)
    scale = max(np.abs(y_ref).max(), 1e-300)
    if y_dtype == dfssm.DFSSM_F32:
        err = np.abs(y_gpu.astype(np.float64) - y_ref)
        bad = err > eb
        assert not bad.any(), f"{bad.sum()} fp32 outputs outside the element bound; worst {err.max():.3e}"
        e = err.max() / scale
        assert e <= TOL_NORMWISE, e
        return dict(normwise=e, ambiguous=0)
    ref_b = oracle.f64_to_bf16(y_ref)
    exact = y_gpu == ref_b
    # The kernel rounds an fp32 value within eb of y_ref, and rounding is monotone, so its
    # bf16 result lies between bf16(y_ref - eb) and bf16(y_ref + eb). Where those differ
    # (y_ref near a midpoint, or eb wider than an ulp after cancellation) any value in
    # that range is correct.
    lo = oracle.bf16_bits_to_f64(oracle.f64_to_bf16(y_ref - eb))
    hi = oracle.bf16_bits_to_f64(oracle.f64_to_bf16(y_ref + eb))
    amb = lo != hi
    got = oracle.bf16_bits_to_f64(y_gpu)
    ok_amb = amb & (got >= lo) & (got <= hi)
    bad = ~(exact | ok_amb)
    assert not bad.any(), (f"{bad.sum()} bf16 outputs differ from bf16(y_ref) "
                           f"(first at {np.argwhere(bad)[0]}: got {got[bad][0]!r}, "
                           f"ref {y_ref[bad][0]!r})")
    e = np.abs(got - oracle.bf16_bits_to_f64(ref_b))[~amb].max(initial=0.0) / scale
    assert e <= TOL_NORMWISE
    return dict(normwise=e, ambiguous=int(amb.sum()))


def check_linear_full(lin: Linear, ref=None, ints: bool = True):
    """Compare every output of one linear with the full oracle (ints=False: y only)."""
    if ref is None:
        ref = oracle.linear(lin.x, lin.w, lin.m, lin.d_in, lin.d_out)
    if lin.dbg is not None and ints:
        np.testing.assert_array_equal(lin.dq.cpu().numpy(), ref["q"])
        np.testing.assert_array_equal(lin.dsx.cpu().numpy(), ref["sx"])
        np.testing.assert_array_equal(lin.dh.cpu().numpy(), ref["h"])
        np.testing.assert_array_equal(lin.dacc.cpu().numpy(), ref["acc"])
    return check_y(lin.y_host(), ref["y"], term_bound(ref, lin.w), lin.y_dtype)


def check_linear_sampled(lin: Linear, n_samples: int, rng, ints: bool = True):
    """Compare sampled outputs with the oracle computed one by one (full-size workloads).

    ints=False checks y only (a call made without the debug exports)."""
    t = np.sort(rng.integers(0, lin.m, n_samples)).astype(np.int32)
    o = rng.integers(0, lin.d_out, n_samples).astype(np.int32)
    s = oracle.linear_sampled(lin.x, lin.w, lin.m, lin.d_in, lin.d_out, t, o)
    # per-token quantities of the sampled tokens: q, s_x, h from the oracle (one output row suffices)
    tok, inv = np.unique(t, return_inverse=True)
    w1 = {k: (v[:1] if k in ("sign", "alpha", "wa", "sa") else v) for k, v in lin.w.items()}
    tref = oracle.linear(np.ascontiguousarray(lin.x[tok]), w1, len(tok), lin.d_in, 1)
    if lin.dbg is not None and ints:
        np.testing.assert_array_equal(lin.dacc.cpu().numpy()[t, o], s["acc"])
        np.testing.assert_array_equal(lin.dq.cpu().numpy()[tok], tref["q"])
        np.testing.assert_array_equal(lin.dsx.cpu().numpy()[tok], tref["sx"])
        np.testing.assert_array_equal(lin.dh.cpu().numpy()[tok], tref["h"])
    y = lin.y_host()[t, o]
    sxt = tref["sx"].astype(np.float64)[inv]
    ht = tref["h"].astype(np.float64)[inv]
    t1 = np.abs(sxt * lin.w["alpha"].astype(np.float64)[o] * s["acc"])
    lora_abs = np.sum(np.abs(lin.w["wa"].astype(np.float64)[o] * lin.w["sb"].astype(np.float64)[None, :] * ht),
                      axis=1)
    t2 = np.abs(sxt * lin.w["sa"].astype(np.float64)[o]) * lora_abs
    return check_y(y, s["y"], 2.0 ** -16 * (t1 + t2), lin.y_dtype)

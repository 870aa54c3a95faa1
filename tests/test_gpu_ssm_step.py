"""The decode step of the Mamba-2 state operations on the GPU against the oracle, through the C ABI.

"Density Field State Space Models" (gist.science technical summary), §2.C, state
operations: shift register (causal convolution) and SSM recurrence. The shift register is
compared bit for bit. The state and the output follow per-element bounds derived from the
fp32 arithmetic and the oracle's own term magnitudes (float64):
  * xc: e_x = 2^-20 (sum_k |w_k win_k| + |b|) + 2^-22 |xc|   (four fp32 fmas, expf, one division)
  * dt: e_dt = 2^-21 dt;  dA: e_dA = dA (|A| e_dt + 2^-21 (1 + |dt A|))
  * S:  e_S = |S0| e_dA + dt (|x| e_B + |B| e_x) + |x B| e_dt + 2^-22 (|S0| dA + dt |x B|)
  * out (fp32): 2^-12 (sum_n |S C| + |D x|) |silu(z)| r |w| + 2^-12 |out|, and the normwise
    max-abs-rel error <= 1e-3 (the stated output bound); bf16 out: the nearest bf16 of the
    oracle's value, or either neighbour within that bound of a midpoint.
Each bound is checked with a margin of 4.
"""
import numpy as np
import pytest
import torch

import bit_gemv_gemm_dfssm_b200 as dfssm
import dfssm_synth as synth
import oracle
from gpu_util import check_y

pytestmark = pytest.mark.gpu
BF16, F32 = dfssm.DFSSM_BF16, dfssm.DFSSM_F32


def dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).cuda()
    return torch.from_numpy(a.copy()).cuda()


class Layers:
    """n layers' inputs on the host and the device, the layer array and a workspace."""

    def __init__(self, dims, n, m, out_dtype, seed=5):
        self.dims, self.n, self.m, self.out_dtype = dims, n, m, out_dtype
        self.inp = [synth.ssm_layer_inputs(seed, 8, i, m, dims) for i in range(n)]
        self.d = [{k: dev(v) for k, v in x.items()} for x in self.inp]
        odt = torch.bfloat16 if out_dtype == BF16 else torch.float32
        self.out = [torch.full((m, dims["d_inner"]), float("nan"), dtype=odt, device="cuda") for _ in range(n)]
        self.c = dfssm.SsmDims(dims["d_inner"], dims["headdim"], dims["d_state"], dims["d_conv"], dims["eps"],
                               out_dtype)
        self.layers = [self.layer(i) for i in range(n)]
        self.ldev = torch.frombuffer(bytearray(dfssm.ssm_layers_bytes(self.layers)), dtype=torch.uint8).cuda()
        self.ws_bytes = dfssm.dfssm_ssm_workspace_bytes(self.c, n, m)
        self.ws = torch.zeros(self.ws_bytes // 4 + 64, dtype=torch.int32, device="cuda")
        assert self.ws.data_ptr() % 256 == 0

    def layer(self, i):
        d = self.d[i]
        return dfssm.SsmLayer(*[d[k].data_ptr() for k in ("zxbcdt", "conv_state", "ssm_state", "conv_w", "conv_b",
                                                            "dt_bias", "a_log", "d_skip", "norm_w")],
                              self.out[i].data_ptr())

    def step(self):
        stream = torch.cuda.current_stream().cuda_stream
        dfssm.dfssm_ssm_step(self.c, self.ldev.data_ptr(), self.n, self.m, self.ws.data_ptr(), self.ws_bytes, stream)
        return dfssm.dfssm_ssm_read_error(self.ws.data_ptr(), stream)

    def state(self, i):
        return (self.d[i]["conv_state"].cpu().numpy().view(np.uint16), self.d[i]["ssm_state"].cpu().numpy())

    def out_host(self, i):
        if self.out_dtype == BF16:
            return self.out[i].view(torch.int16).cpu().numpy().view(np.uint16)
        return self.out[i].cpu().numpy()


def bounds(dims, inp, ref):
    """Per-element bounds of the state and the fp32 output (module docstring)."""
    d_inner, P, N = dims["d_inner"], dims["headdim"], dims["d_state"]
    nheads = d_inner // P
    conv_dim = d_inner + 2 * N
    m = inp["zxbcdt"].shape[0]
    win = np.concatenate([inp["conv_state"][:, :, 1:], inp["zxbcdt"][:, d_inner:d_inner + conv_dim, None]], axis=2)
    winf = (win.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    tc = np.abs(winf * inp["conv_w"].astype(np.float64)[None]).sum(axis=2) + np.abs(inp["conv_b"].astype(np.float64))
    e_xc = 2.0 ** -20 * tc + 2.0 ** -22 * np.abs(ref["xc"])
    x, B, C = ref["xc"][:, :d_inner], ref["xc"][:, d_inner:d_inner + N], ref["xc"][:, d_inner + N:]
    ex, eB = e_xc[:, :d_inner], e_xc[:, d_inner:d_inner + N]
    dt, dA = ref["dt"], ref["dA"]
    A = -np.exp(inp["a_log"].astype(np.float64))[None, :]
    e_dt = 2.0 ** -21 * dt
    e_dA = dA * (np.abs(A) * e_dt + 2.0 ** -21 * (1 + np.abs(dt * A)))
    s0 = np.abs(inp["ssm_state"].astype(np.float64))
    xh = np.abs(x).reshape(m, nheads, P)[..., None]
    exh = ex.reshape(m, nheads, P)[..., None]
    Bn, eBn = np.abs(B)[:, None, None, :], eB[:, None, None, :]
    dth, e_dth, dAh, e_dAh = (v[:, :, None, None] for v in (dt, e_dt, dA, e_dA))
    e_S = s0 * e_dAh + dth * (xh * eBn + Bn * exh) + xh * Bn * e_dth + 2.0 ** -22 * (s0 * dAh + dth * xh * Bn)
    # output
    z = (inp["zxbcdt"][:, :d_inner].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    silu_z = np.abs(z / (1 + np.exp(-z)))
    ty = (np.abs(ref["ssm_state"]) * np.abs(C)[:, None, None, :]).sum(axis=3).reshape(m, d_inner) + \
        np.abs(np.repeat(inp["d_skip"].astype(np.float64), P)[None, :] * x)
    e_out = 2.0 ** -12 * ty * silu_z * ref["r"][:, None] * np.abs(inp["norm_w"].astype(np.float64))[None, :] + \
        2.0 ** -12 * np.abs(ref["out"])
    return e_S, e_out


def check_layer(L, i, ref, e_S, e_out):
    cs, ss = L.state(i)
    np.testing.assert_array_equal(cs, ref["conv_state"])
    err = np.abs(ss.astype(np.float64) - ref["ssm_state"])
    bad = err > 4 * e_S + 1e-30
    assert not bad.any(), f"layer {i}: {bad.sum()} state elements outside the bound; worst {err.max():.3e}"
    out = L.out_host(i)
    if L.out_dtype == F32:
        err = np.abs(out.astype(np.float64) - ref["out"])
        bad = err > 4 * e_out
        assert not bad.any(), f"layer {i}: {bad.sum()} outputs outside the bound; worst {err.max():.3e}"
        assert err.max() / np.abs(ref["out"]).max() <= 1e-3
    else:
        check_y(out, ref["out"], 4 * e_out, BF16)


@pytest.mark.parametrize("d_inner,n,m,out_dtype", [(64, 1, 1, F32), (256, 3, 3, BF16), (4096, 2, 16, F32),
                                                   (1024, 5, 2, BF16), (4096, 1, 1, BF16)])
def test_ssm_step_parity(d_inner, n, m, out_dtype):
    dims = dict(synth.SSM_DIMS, d_inner=d_inner)
    L = Layers(dims, n, m, out_dtype)
    st, bits = L.step()
    assert st == dfssm.DFSSM_OK, hex(bits)
    for i in range(n):
        ref = oracle.ssm_step(dims, L.inp[i])
        e_S, e_out = bounds(dims, L.inp[i], ref)
        check_layer(L, i, ref, e_S, e_out)


def test_ssm_steps_in_a_row_update_the_state_in_place():
    # three steps on the GPU with the states fed back in place; the oracle steps from the GPU's own
    # previous state each time (so each step is held to its own bound)
    dims = dict(synth.SSM_DIMS, d_inner=512)
    L = Layers(dims, 2, 2, F32, seed=11)
    for k in range(3):
        prev = [L.state(i) for i in range(L.n)]
        for i in range(L.n):
            L.inp[i]["zxbcdt"] = synth.ssm_layer_inputs(100 + k, 8, i, L.m, dims)["zxbcdt"]
            L.d[i]["zxbcdt"].copy_(dev(L.inp[i]["zxbcdt"]))
        st, bits = L.step()
        assert st == dfssm.DFSSM_OK, hex(bits)
        for i in range(L.n):
            inp = dict(L.inp[i], conv_state=prev[i][0], ssm_state=prev[i][1])
            ref = oracle.ssm_step(dims, inp)
            e_S, e_out = bounds(dims, inp, ref)
            check_layer(L, i, ref, e_S, e_out)


def test_ssm_step_full_size_stack():
    # the bench's workload: the 48 layers of Mamba-2 1.3B at one token, bf16 out
    dims = synth.SSM_DIMS
    L = Layers(dims, 48, 1, BF16, seed=21)
    st, bits = L.step()
    assert st == dfssm.DFSSM_OK, hex(bits)
    for i in range(L.n):
        ref = oracle.ssm_step(dims, L.inp[i])
        e_S, e_out = bounds(dims, L.inp[i], ref)
        check_layer(L, i, ref, e_S, e_out)


def test_ssm_step_bad_layer_pointer_is_skipped_and_reported():
    dims = dict(synth.SSM_DIMS, d_inner=128)
    L = Layers(dims, 2, 1, F32)
    bad = L.layer(1)
    bad.norm_w = bad.norm_w + 4                       # misaligned
    L.ldev = torch.frombuffer(bytearray(dfssm.ssm_layers_bytes([L.layers[0], bad])), dtype=torch.uint8).cuda()
    st, bits = L.step()
    assert st == dfssm.DFSSM_ERR_DEVICE_CHECK and bits & dfssm.DFSSM_DEVERR_ENTRY_PTR
    assert torch.isnan(L.out[1]).all()                # layer 1 skipped
    cs, ss = L.state(1)
    np.testing.assert_array_equal(cs, L.inp[1]["conv_state"])
    np.testing.assert_array_equal(ss, L.inp[1]["ssm_state"])
    ref = oracle.ssm_step(dims, L.inp[0])             # layer 0 computed as usual
    e_S, e_out = bounds(dims, L.inp[0], ref)
    check_layer(L, 0, ref, e_S, e_out)
    st, bits = dfssm.dfssm_ssm_read_error(L.ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == dfssm.DFSSM_OK and bits == 0         # cleared by the read

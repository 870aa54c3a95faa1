"""Pins of the oracle's decode step of the Mamba-2 state operations (oracle/ssm_oracle.cpp).

"Density Field State Space Models" (gist.science technical summary), §2.C, state
operations: the state shift register (causal convolution) and the SSM recurrence. Each
part of the step is checked against something other than the oracle's own formula: the
shift register against the inputs fed in, the convolution through one-tap and bias-only
filters against scipy's logistic function, the step size against numpy's log-add-exp and
a closed form of the decay, the recurrence against the closed form of a constant-input
linear recurrence over several steps, the readout through C = 0 and zero-state cases, the
gate and norm through unit-RMS, zero-gate and scaling properties, and the head indexing
through a permutation of the heads.
"""
import numpy as np
import pytest
from scipy.special import expit

import dfssm_synth as synth
import oracle

DIMS = dict(d_inner=128, headdim=64, d_state=16, d_conv=4, eps=1e-5)


def case(seed=3, m=2, dims=DIMS):
    return synth.ssm_layer_inputs(seed, 7, 0, m, dims)


def silu(v):
    return v * expit(v)


def bf16(vals):
    f = np.asarray(vals, np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def bf16_to_f64(b):
    return (np.asarray(b, np.uint32) << 16).view(np.float32).astype(np.float64)


def layout(dims):
    d_inner, d_state = dims["d_inner"], dims["d_state"]
    nheads = d_inner // dims["headdim"]
    conv_dim = d_inner + 2 * d_state
    return d_inner, d_state, nheads, conv_dim


def step(dims, inp):
    """One oracle step; returns its outputs and the next step's inputs (state fed back)."""
    r = oracle.ssm_step(dims, inp)
    nxt = dict(inp)
    nxt["conv_state"] = r["conv_state"]
    nxt["ssm_state"] = r["ssm_state"].astype(np.float32)
    return r, nxt


def test_shift_register_holds_the_last_inputs():
    dims = DIMS
    d_inner, _, _, conv_dim = layout(dims)
    inp = case()
    inp["conv_state"][:] = 0
    fed = []
    for k in range(5):
        v = bf16(np.arange(conv_dim) * 0.25 + k + 1)          # exact in bf16
        inp["zxbcdt"][:, d_inner:d_inner + conv_dim] = v
        fed.append(v)
        _, inp = step(dims, inp)
        want = [np.zeros(conv_dim, np.uint16)] * max(0, 3 - k) + fed[max(0, k - 3):]
        np.testing.assert_array_equal(inp["conv_state"][0], np.stack(want, axis=1))


@pytest.mark.parametrize("tap", [0, 1, 2, 3])
def test_one_tap_convolution_is_silu_of_that_window_entry(tap):
    dims = DIMS
    d_inner, _, _, conv_dim = layout(dims)
    inp = case()
    inp["conv_w"][:] = 0
    inp["conv_w"][:, tap] = 1
    inp["conv_b"][:] = 0
    r = oracle.ssm_step(dims, inp)
    window = np.concatenate([inp["conv_state"][:, :, 1:], inp["zxbcdt"][:, None, d_inner:d_inner + conv_dim]
                             .transpose(0, 2, 1)], axis=2)
    np.testing.assert_allclose(r["xc"], silu(bf16_to_f64(window[:, :, tap])), rtol=1e-14, atol=0)


def test_bias_only_convolution():
    dims = DIMS
    inp = case()
    inp["conv_w"][:] = 0
    r = oracle.ssm_step(dims, inp)
    np.testing.assert_allclose(r["xc"], np.broadcast_to(silu(inp["conv_b"].astype(np.float64)), r["xc"].shape),
                               rtol=1e-14, atol=0)


def test_step_size_and_decay():
    dims = DIMS
    d_inner, _, nheads, conv_dim = layout(dims)
    inp = case()
    # dt = softplus(dt_raw + dt_bias): below 20 numpy's log(e^0 + e^v); above 20 v itself
    raw = np.linspace(-8, 30, nheads)
    inp["zxbcdt"][:, d_inner + conv_dim:] = bf16(raw)
    inp["dt_bias"][:] = 0.5
    inp["a_log"][:] = 0.0                                 # A = -1, so dA = exp(-dt) = 1 / (1 + e^v)
    r = oracle.ssm_step(dims, inp)
    v = bf16_to_f64(bf16(raw)) + 0.5
    want_dt = np.where(v > 20, v, np.logaddexp(0.0, v))
    np.testing.assert_allclose(r["dt"][0], want_dt, rtol=1e-14)
    small = v <= 20
    np.testing.assert_allclose(r["dA"][0][small], expit(-v[small]), rtol=1e-12)


def test_recurrence_matches_the_closed_form_over_steps():
    # a constant input (one-tap filter on the newest entry, the same xBC and dt_raw every step):
    # S_K = dA^K S_0 + dt x B (1 - dA^K) / (1 - dA)
    dims = DIMS
    d_inner, d_state, nheads, conv_dim = layout(dims)
    P = dims["headdim"]
    inp = case(m=1)
    inp["conv_w"][:] = 0
    inp["conv_w"][:, 3] = 1
    s0 = inp["ssm_state"].astype(np.float64).copy()
    K = 6
    for _ in range(K):
        r, inp = step(dims, inp)                           # the state is fp32 between steps
    dt, dA, xc = r["dt"][0], r["dA"][0], r["xc"][0]
    x, B = xc[:d_inner].reshape(nheads, P), xc[d_inner:d_inner + d_state]
    decay = dA[:, None, None] ** K
    want = decay * s0[0] + (dt[:, None, None] * x[:, :, None] * B[None, None, :]) * \
        ((1 - decay) / (1 - dA[:, None, None]))
    # each of the K states fed back is rounded to fp32 (half an ulp, 2^-24 relative)
    bound = K * 2.0 ** -24 * np.abs(want).max()
    assert np.abs(r["ssm_state"][0] - want).max() <= bound


def test_readout_special_cases():
    dims = DIMS
    d_inner, d_state, nheads, conv_dim = layout(dims)
    P = dims["headdim"]
    # C = 0 (its filter and bias zero, silu(0) = 0): y = D x
    inp = case()
    inp["conv_w"][d_inner + d_state:] = 0
    inp["conv_b"][d_inner + d_state:] = 0
    r = oracle.ssm_step(dims, inp)
    x = r["xc"][:, :d_inner]
    np.testing.assert_allclose(r["y"], np.repeat(inp["d_skip"].astype(np.float64), P)[None, :] * x,
                               rtol=1e-14, atol=0)
    # zero state and D = 0: y[h P + p] = dt_h x[h P + p] sum_n B[n] C[n]
    inp = case()
    inp["ssm_state"][:] = 0
    inp["d_skip"][:] = 0
    r = oracle.ssm_step(dims, inp)
    B, C = r["xc"][:, d_inner:d_inner + d_state], r["xc"][:, d_inner + d_state:]
    bc = (B * C).sum(axis=1)
    want = np.repeat(r["dt"], P, axis=1) * r["xc"][:, :d_inner] * bc[:, None]
    np.testing.assert_allclose(r["y"], want, rtol=1e-12)


def test_gate_and_norm_properties():
    dims = dict(DIMS, eps=0.0)
    d_inner = dims["d_inner"]
    inp = case()
    inp["norm_w"][:] = 1
    r = oracle.ssm_step(dims, inp)
    np.testing.assert_allclose((r["out"] ** 2).mean(axis=1), 1.0, rtol=1e-13)    # unit RMS
    inp2 = dict(inp)
    inp2["norm_w"] = np.full(d_inner, 2.0, np.float32)
    r2 = oracle.ssm_step(dims, inp2)
    np.testing.assert_array_equal(r2["out"], 2 * r["out"])
    # a zero gate (z = 0) gives a zero output (eps > 0)
    inp3 = case()
    inp3["zxbcdt"][:, :d_inner] = 0
    r3 = oracle.ssm_step(DIMS, inp3)
    assert np.all(r3["out"] == 0)
    # the gate multiplies y by silu(z): y itself does not depend on z
    np.testing.assert_array_equal(r3["y"], oracle.ssm_step(DIMS, case())["y"])


def test_heads_permute_consistently():
    dims = dict(d_inner=256, headdim=64, d_state=16, d_conv=4, eps=1e-5)
    d_inner, d_state, nheads, conv_dim = layout(dims)
    P = dims["headdim"]
    inp = case(seed=9, dims=dims)
    perm = np.array([2, 0, 3, 1])
    ch = (perm[:, None] * P + np.arange(P)[None, :]).ravel()         # channel order of the permuted heads
    q = {k: np.array(v, copy=True) for k, v in inp.items()}
    z = q["zxbcdt"]
    z[:, :d_inner] = inp["zxbcdt"][:, ch]
    z[:, d_inner:2 * d_inner] = inp["zxbcdt"][:, d_inner + ch]
    z[:, d_inner + conv_dim:] = inp["zxbcdt"][:, d_inner + conv_dim + perm]
    q["conv_state"][:, :d_inner] = inp["conv_state"][:, ch]
    q["conv_w"][:d_inner] = inp["conv_w"][ch]
    q["conv_b"][:d_inner] = inp["conv_b"][ch]
    q["ssm_state"] = inp["ssm_state"][:, perm]
    for k in ("dt_bias", "a_log", "d_skip"):
        q[k] = inp[k][perm]
    q["norm_w"] = inp["norm_w"][ch]
    a, b = oracle.ssm_step(dims, inp), oracle.ssm_step(dims, q)
    np.testing.assert_allclose(b["out"], a["out"][:, ch], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(b["ssm_state"], a["ssm_state"][:, perm], rtol=1e-15, atol=0)
    np.testing.assert_array_equal(b["conv_state"][:, :d_inner], a["conv_state"][:, ch])

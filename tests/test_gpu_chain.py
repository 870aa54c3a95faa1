"""The model's whole decode step through the C ABI, checked stage by stage against the oracle.

The chained step (bench.py ChainRunner) runs as one CUDA graph of the library's calls: the
int8 embedding; per block the residual add + RMS norm, in_proj, the state step and out_proj;
the last residual add + RMS norm; the int8 LM head. Each stage is then checked against the
oracle computed from that stage's own inputs as the GPU left them, so differences do not
compound across blocks:
  * embedding (fp32): bit for bit;
  * residual: bit for bit (one fp32 addition per element); normed output (bf16): the nearest
    bf16 of the oracle's value, or either neighbour where that value lies within 2^-18 |ref|
    of a rounding midpoint (the kernel's relative error is below 1e-6: an fp32 sum of squares
    in a fixed order, correctly rounded square root and division, two products);
  * in_proj and out_proj: the layer's tolerance (tests/gpu_util.py);
  * state step: the bounds of tests/test_gpu_ssm_step.py (shift register bit for bit);
  * LM head: as in tests/test_gpu_int8_table.py.
"""
import numpy as np
import pytest
import torch

import bench
import bit_gemv_gemm_dfssm_b200 as dfssm
import dfssm_synth as synth
import oracle
from gpu_util import check_y, term_bound
from test_gpu_ssm_step import bounds

pytestmark = pytest.mark.gpu
BF16, F32 = dfssm.DFSSM_BF16, dfssm.DFSSM_F32

SMALL = dict(n_layers=3, d_model=256, dims=dict(synth.SSM_DIMS, d_inner=512), vocab=1000)


def bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def check_norm(r_in, delta, w, eps, r_out_gpu, out_gpu):
    ref = oracle.add_rmsnorm(r_in, delta, w, eps)
    np.testing.assert_array_equal(r_out_gpu, ref["resid"])
    check_y(out_gpu, ref["out"], 2.0 ** -18 * np.abs(ref["out"]), BF16)


def check_ssm(dims, inp, conv_gpu, state_gpu, out_gpu):
    ref = oracle.ssm_step(dims, inp)
    e_S, e_out = bounds(dims, inp, ref)
    np.testing.assert_array_equal(conv_gpu, ref["conv_state"])
    err = np.abs(state_gpu.astype(np.float64) - ref["ssm_state"])
    assert not (err > 4 * e_S + 1e-30).any(), f"worst state error {err.max():.3e}"
    check_y(out_gpu, ref["out"], 4 * e_out, BF16)


def check_step(r, states):
    """Every stage of the step just run; states: the (conv, ssm) states each block started from."""
    m, d, eps = r.m, r.d, r.dims["eps"]
    emb, bad = oracle.embed(r.table_host["table"], r.table_host["scale"], r.ids_host)
    assert bad == 0
    np.testing.assert_array_equal(r.emb.cpu().numpy(), emb)
    for i in range(r.n):
        r_in = r.emb.cpu().numpy() if i == 0 else r.resid[i - 1].cpu().numpy()
        delta = None if i == 0 else bits(r.yo[i - 1])
        check_norm(r_in, delta, r.nw_host[i], eps, r.resid[i].cpu().numpy(), bits(r.xn[i]))
        d_in, d_out = r.shapes[0]
        ref = oracle.linear(bits(r.xn[i]), r.w_host[2 * i], m, d_in, d_out)
        check_y(bits(r.zx[i]), ref["y"], term_bound(ref, r.w_host[2 * i]), BF16)
        inp = dict(r.ssm_host[i], zxbcdt=bits(r.zx[i]), conv_state=states[i][0], ssm_state=states[i][1])
        check_ssm(r.dims, inp, bits(r.ssm[i]["conv_state"]), r.ssm[i]["ssm_state"].cpu().numpy(), bits(r.so[i]))
        d_in, d_out = r.shapes[1]
        ref = oracle.linear(bits(r.so[i]), r.w_host[2 * i + 1], m, d_in, d_out)
        check_y(bits(r.yo[i]), ref["y"], term_bound(ref, r.w_host[2 * i + 1]), BF16)
    n = r.n
    check_norm(r.resid[n - 1].cpu().numpy(), bits(r.yo[n - 1]), r.nw_host[n], eps, r.resid[n].cpu().numpy(),
               bits(r.xn[n]))
    ref = oracle.lm_head(r.table_host["table"], r.table_host["scale"], bits(r.xn[n]), m)
    check_y(r.logits.cpu().numpy(), ref["logits"], 2.0 ** -16 * np.abs(ref["logits"]), F32)


def gpu_states(r):
    return [(bits(s["conv_state"]).copy(), s["ssm_state"].cpu().numpy().copy()) for s in r.ssm]


@pytest.mark.parametrize("m", [1, 3])
def test_small_chain_two_steps(m):
    # two replays of the graph: the second step starts from the states the first one left
    r = bench.ChainRunner(m, 17, **SMALL)
    try:
        g = r.graph()
        start = [(x["conv_state"], x["ssm_state"]) for x in r.ssm_host]
        g.replay()
        torch.cuda.synchronize()
        r.check()
        check_step(r, start)
        after = gpu_states(r)
        g.replay()
        torch.cuda.synchronize()
        r.check()
        check_step(r, after)
        del g
    finally:
        r.close()


def test_full_size_decode_step():
    # the bench's configuration: the 48 blocks of Mamba-2 1.3B at one token, every stage checked
    r = bench.ChainRunner(1, synth.MASTER_SEED)
    try:
        g = r.graph()
        start = [(x["conv_state"], x["ssm_state"]) for x in r.ssm_host]
        g.replay()
        torch.cuda.synchronize()
        r.check()
        check_step(r, start)
        assert r.launches() == 1 + 7 * 48 + 2
        del g
    finally:
        r.close()

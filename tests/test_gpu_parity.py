"""CUDA path vs the CPU oracle, through the C ABI (needs a B200).

Small shapes compare every output; full-size workloads (the Mamba-2-1.3B
in_proj / out_proj stack, launched exactly as bench.py launches it) compare
sampled outputs computed one by one by the oracle, plus the per-token
quantities. Integer results are bit-exact; y follows the tolerance stated in
tests/gpu_util.py.
"""
import numpy as np
import pytest
import torch

import bit_gemv_gemm_dfssm_b200 as dfssm
import dfssm_synth as synth
import oracle
from gpu_util import (Linear, check_linear_full, check_linear_sampled, check_y, dev, entries_device, mapped_address,
                      term_bound)

pytestmark = pytest.mark.gpu

SEED = synth.MASTER_SEED
BF16, F32 = dfssm.DFSSM_BF16, dfssm.DFSSM_F32


def run_one(lin: Linear, max_m=None):
    plan = dfssm.dfssm_linear_plan([lin.desc(max_m)])
    try:
        stream = torch.cuda.current_stream().cuda_stream
        dfssm.dfssm_linear_fwd(plan, 0, lin.weights(), lin.dx.data_ptr(), lin.m, lin.dy.data_ptr(), lin.dbg, stream)
        st, bits = dfssm.dfssm_plan_check(plan)
        assert st == dfssm.DFSSM_OK, hex(bits)
    finally:
        dfssm.dfssm_plan_destroy(plan)


# ------------------------------------------------------------------ packing

@pytest.mark.parametrize("d_out,d_in", [(1, 128), (3, 256), (17, 384), (64, 4096)])
@pytest.mark.parametrize("kind", ["i8", "f32"])
def test_pack_sign_matches_oracle(d_out, d_in, kind):
    rng = np.random.default_rng(d_out * 7 + d_in)
    if kind == "i8":
        src = rng.integers(-128, 128, size=(d_out, d_in), dtype=np.int16).astype(np.int8)
        src.ravel()[:5] = [0, -1, 1, 127, -128][: min(5, src.size)]
        code = dfssm.DFSSM_I8
    else:
        src = rng.standard_normal((d_out, d_in)).astype(np.float32)
        src.ravel()[:4] = [0.0, -0.0, 1e-38, -1e-38]
        code = dfssm.DFSSM_F32
    dsrc = dev(src)
    dpk = torch.zeros((d_out, d_in // 8), dtype=torch.uint8, device="cuda")
    dfssm.dfssm_pack_sign(dsrc.data_ptr(), code, d_out, d_in, dpk.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(dpk.cpu().numpy(), oracle.pack_sign(src, d_out, d_in))


# ------------------------------------------------------------------ one linear, every output

DECODE_CASES = [  # (d_in, d_out, m, y_dtype)
    (128, 1, 1, F32), (128, 17, 3, BF16), (384, 200, 1, F32), (384, 64, 8, BF16),
    (256, 130, 9, F32), (2048, 8512, 1, BF16), (4096, 2048, 1, F32), (4096, 100, 16, BF16),
    (8192, 70, 2, F32), (2048, 333, 16, F32),
    # one token: four 2048-column LoRA slices; a ragged second slice of 1152 columns
    (8192, 70, 1, BF16), (3200, 96, 1, F32),
]
PREFILL_CASES = [
    (128, 1, 17, F32), (256, 129, 33, BF16), (384, 300, 300, F32), (2048, 200, 257, BF16),
    (4096, 256, 512, F32), (1024, 128, 100, BF16), (8192, 64, 40, F32),
    # items of 10 and of 5 tokens in the quantiser (32768 / d_in not a power of two), a final
    # half segment, a last row tile of 8 rows, ragged 192-token tiles
    (3200, 520, 300, BF16), (6144, 136, 70, BF16),
    # 241 and 480 tokens: a second tile of 49 tokens; two whole tiles and half a third
    (1024, 200, 241, F32), (512, 130, 480, BF16),
]


@pytest.mark.parametrize("d_in,d_out,m,y_dtype", DECODE_CASES + PREFILL_CASES)
def test_linear_parity(d_in, d_out, m, y_dtype):
    lin = Linear(SEED, 9, d_in * 1000 + d_out, d_in, d_out, m, y_dtype)
    run_one(lin)
    check_linear_full(lin)


def test_max_m_larger_than_m():
    # the plan sized for 600 tokens, called with fewer (decode and prefill paths)
    for m in (5, 40):
        lin = Linear(SEED, 9, 77 + m, 512, 96, m, F32)
        run_one(lin, max_m=600)
        check_linear_full(lin)


def test_decode_and_prefill_agree():
    # the first 16 tokens: m = 16 runs the decode kernel, m = 17 the tcgen05 kernel. The
    # integer sums agree bit for bit; y is computed in different fp32 orders (the prefill runs
    # the LoRA up-projection on bf16 hi/lo warp MMAs), so each is held to the oracle's bound.
    d_in, d_out = 2048, 640
    x = synth.activations(SEED, 9, 5, 17, d_in)
    a = Linear(SEED, 9, 5, d_in, d_out, 16, F32, x=np.ascontiguousarray(x[:16]))
    b = Linear(SEED, 9, 5, d_in, d_out, 17, F32, x=x)
    run_one(a)
    run_one(b)
    np.testing.assert_array_equal(a.dacc.cpu().numpy(), b.dacc.cpu().numpy()[:16])
    ref = oracle.linear(b.x, b.w, 17, d_in, d_out)
    check_y(b.y_host(), ref["y"], term_bound(ref, b.w), F32)
    ref16 = oracle.linear(a.x, a.w, 16, d_in, d_out)
    check_y(a.y_host(), ref16["y"], term_bound(ref16, a.w), F32)


def test_zero_and_single_channel_inputs():
    d_in, d_out, m = 256, 64, 3
    x = np.zeros((m, d_in), np.uint16)
    x[1, 7] = 0x4040            # 3.0
    x[2, :] = 0x3F80            # all 1.0 -> q = 127 everywhere
    for mm in (m, 20):          # decode and prefill
        xx = np.zeros((mm, d_in), np.uint16)
        xx[:m] = x
        lin = Linear(SEED, 9, 3, d_in, d_out, mm, F32, x=xx)
        run_one(lin)
        ref = oracle.linear(xx, lin.w, mm, d_in, d_out)
        assert np.all(ref["y"][0] == 0) and np.all(lin.dy.cpu().numpy()[0] == 0)
        check_linear_full(lin, ref)


def test_all_ones_rows_closed_form():
    # all-ones sign rows: acc = sum_j q (spec invariant), checked on the GPU
    d_in, d_out, m = 512, 32, 4
    w = synth.linear_weights(SEED, 9, 11, d_in, d_out)
    w["sign"][:] = 0xFF
    lin = Linear(SEED, 9, 11, d_in, d_out, m, F32, w=w)
    run_one(lin)
    q = lin.dq.cpu().numpy().astype(np.int64)
    acc = lin.dacc.cpu().numpy()
    np.testing.assert_array_equal(acc, np.repeat(q.sum(axis=1, keepdims=True), d_out, axis=1))
    check_linear_full(lin)


# ------------------------------------------------------------------ stacks

def build_stack(shapes, m, y_dtype=BF16, cfg=9, dbg=True):
    lins = [Linear(SEED, cfg, i, d_in, d_out, m, y_dtype, dbg=dbg) for i, (d_in, d_out) in enumerate(shapes)]
    plan = dfssm.dfssm_linear_plan([l.desc() for l in lins])
    ent = entries_device([l.entry(i) for i, l in enumerate(lins)])
    return lins, plan, ent


@pytest.mark.parametrize("m", [1, 5, 16, 40])
def test_small_stack_parity(m):
    shapes = [(256, 100), (512, 64), (128, 300), (384, 17), (1024, 129), (256, 8)]
    lins, plan, ent = build_stack(shapes, m, F32 if m % 2 else BF16)
    try:
        dfssm.dfssm_linear_stack_fwd(plan, ent.data_ptr(), len(lins), m, torch.cuda.current_stream().cuda_stream)
        st, bits = dfssm.dfssm_plan_check(plan)
        assert st == dfssm.DFSSM_OK, hex(bits)
        for lin in lins:
            check_linear_full(lin)
    finally:
        dfssm.dfssm_plan_destroy(plan)


def test_stack_entry_desc_mismatch_sets_error_word():
    shapes = [(256, 64), (256, 64)]
    lins = [Linear(SEED, 9, i, 256, 64, 1) for i in range(2)]
    plan = dfssm.dfssm_linear_plan([l.desc() for l in lins])
    try:
        ent = entries_device([lins[0].entry(0), lins[1].entry(0)])     # entry 1 claims desc 0
        dfssm.dfssm_linear_stack_fwd(plan, ent.data_ptr(), 2, 1, 0)
        st, bits = dfssm.dfssm_plan_check(plan)
        assert st == dfssm.DFSSM_ERR_DEVICE_CHECK and bits & dfssm.DFSSM_DEVERR_ENTRY_DESC
        st, bits = dfssm.dfssm_plan_check(plan)     # cleared by the read
        assert st == dfssm.DFSSM_OK and bits == 0
    finally:
        dfssm.dfssm_plan_destroy(plan)


@pytest.mark.parametrize("m", [3, 40])
def test_nonfinite_activation_row_sets_error_word(m):
    # an Inf in token 1: the error word reports it (that token's outputs are undefined), while
    # the other tokens, quantised independently, still match the oracle (decode and prefill)
    d_in, d_out = 512, 96
    x = synth.activations(SEED, 9, 11, m, d_in).copy()
    x[1, 5] = 0x7F80                                  # +Inf
    lin = Linear(SEED, 9, 11, d_in, d_out, m, F32, x=x, dbg=False)
    plan = dfssm.dfssm_linear_plan([lin.desc()])
    try:
        stream = torch.cuda.current_stream().cuda_stream
        dfssm.dfssm_linear_fwd(plan, 0, lin.weights(), lin.dx.data_ptr(), m, lin.dy.data_ptr(), None, stream)
        st, bits = dfssm.dfssm_plan_check(plan)
        assert st == dfssm.DFSSM_ERR_DEVICE_CHECK and bits & dfssm.DFSSM_DEVERR_NONFINITE
    finally:
        dfssm.dfssm_plan_destroy(plan)
    keep = [t for t in range(m) if t != 1]
    ref = oracle.linear(np.ascontiguousarray(x[keep]), lin.w, len(keep), d_in, d_out)
    check_y(lin.y_host()[keep], ref["y"], term_bound(ref, lin.w), F32)


def test_bounded_wait_gives_up_with_timeout_status():
    # the decode kernel's first CTA waits on a barrier nothing arrives on: the bounded wait gives
    # up after 2 ms, the call reports DFSSM_DEVERR_TIMEOUT instead of hanging, and the same plan
    # computes correctly afterwards
    shapes = [(2048, 640), (4096, 256)]
    lins, plan, ent = build_stack(shapes, 1, F32)
    stream = torch.cuda.current_stream().cuda_stream
    try:
        dfssm.dfssm_plan_set_test_hooks(plan, 2_000_000, dfssm.DFSSM_TEST_STALL)
        dfssm.dfssm_linear_stack_fwd(plan, ent.data_ptr(), len(lins), 1, stream)
        st, bits = dfssm.dfssm_plan_check(plan)
        assert st == dfssm.DFSSM_ERR_DEVICE_CHECK and bits & dfssm.DFSSM_DEVERR_TIMEOUT, hex(bits)
        dfssm.dfssm_plan_set_test_hooks(plan, 0, 0)
        dfssm.dfssm_linear_stack_fwd(plan, ent.data_ptr(), len(lins), 1, stream)
        st, bits = dfssm.dfssm_plan_check(plan)
        assert st == dfssm.DFSSM_OK, hex(bits)
        for lin in lins:
            check_linear_full(lin)
        with pytest.raises(dfssm.DfssmError):
            dfssm.dfssm_plan_set_test_hooks(plan, 0, 0x80)
    finally:
        dfssm.dfssm_plan_destroy(plan)


@pytest.mark.parametrize("m", [1, 3])
def test_nonfinite_one_token_paths(m):
    # a NaN in one token's row: the slice kernel (one token) and the split quantiser both report
    # it; for m = 3 the other tokens still match the oracle
    d_in, d_out = 4096, 200
    x = synth.activations(SEED, 9, 21, m, d_in).copy()
    x[0, 100] = 0x7FC0                                # NaN
    lin = Linear(SEED, 9, 21, d_in, d_out, m, F32, x=x, dbg=False)
    plan = dfssm.dfssm_linear_plan([lin.desc()])
    try:
        stream = torch.cuda.current_stream().cuda_stream
        dfssm.dfssm_linear_fwd(plan, 0, lin.weights(), lin.dx.data_ptr(), m, lin.dy.data_ptr(), None, stream)
        st, bits = dfssm.dfssm_plan_check(plan)
        assert st == dfssm.DFSSM_ERR_DEVICE_CHECK and bits & dfssm.DFSSM_DEVERR_NONFINITE, hex(bits)
    finally:
        dfssm.dfssm_plan_destroy(plan)
    if m > 1:
        ref = oracle.linear(np.ascontiguousarray(x[1:]), lin.w, m - 1, d_in, d_out)
        check_y(lin.y_host()[1:], ref["y"], term_bound(ref, lin.w), F32)


def test_argument_errors_launch_nothing():
    lin = Linear(SEED, 9, 1, 256, 64, 4, F32)
    plan = dfssm.dfssm_linear_plan([lin.desc()])
    try:
        w = lin.weights()
        call = lambda *a: dfssm.lib().dfssm_linear_fwd(*a)
        x, y = lin.dx.data_ptr(), lin.dy.data_ptr()
        import ctypes
        assert call(plan, 0, ctypes.byref(w), x, 0, y, None, None) == dfssm.DFSSM_ERR_INVALID_ARG
        assert call(plan, 0, ctypes.byref(w), x, 5, y, None, None) == dfssm.DFSSM_ERR_INVALID_ARG
        assert call(plan, 1, ctypes.byref(w), x, 1, y, None, None) == dfssm.DFSSM_ERR_INVALID_ARG
        assert call(plan, 0, ctypes.byref(w), x + 2, 1, y, None, None) == dfssm.DFSSM_ERR_INVALID_ARG
        bad = dfssm.LinearWeights(w.sign + 8, w.alpha, w.wa, w.sa, w.wb, w.sb)
        assert call(plan, 0, ctypes.byref(bad), x, 1, y, None, None) == dfssm.DFSSM_ERR_INVALID_ARG
        bad = dfssm.LinearWeights(None, w.alpha, w.wa, w.sa, w.wb, w.sb)
        assert call(plan, 0, ctypes.byref(bad), x, 1, y, None, None) == dfssm.DFSSM_ERR_INVALID_ARG
        torch.cuda.synchronize()
        assert torch.isnan(lin.dy).all()          # nothing ran
    finally:
        dfssm.dfssm_plan_destroy(plan)


def test_repeated_calls_are_deterministic():
    shapes = [(2048, 1000), (4096, 512)]
    for m in (1, 300):
        lins, plan, ent = build_stack(shapes, m, F32, dbg=False)
        try:
            outs = []
            for _ in range(3):
                dfssm.dfssm_linear_stack_fwd(plan, ent.data_ptr(), 2, m, 0)
                torch.cuda.synchronize()
                outs.append([l.dy.clone() for l in lins])
            for o in outs[1:]:
                for a, b in zip(outs[0], o):
                    assert torch.equal(a, b)
        finally:
            dfssm.dfssm_plan_destroy(plan)


@pytest.mark.parametrize("m", [1, 5, 40])
def test_stack_output_in_pinned_host_memory(m):
    # y may be any memory the GPU can write: outputs in pinned host buffers (written by the kernels
    # over the bus) are byte-identical to outputs in device memory, on the slice, quant and prefill paths
    shapes = [(2048, 1000), (4096, 512), (256, 100)]
    lins, plan, ent = build_stack(shapes, m, F32 if m % 2 else BF16, dbg=False)
    try:
        stream = torch.cuda.current_stream().cuda_stream
        dfssm.dfssm_linear_stack_fwd(plan, ent.data_ptr(), len(lins), m, stream)
        torch.cuda.synchronize()
        hosts = [torch.full_like(l.dy, float("nan"), device="cpu").pin_memory() for l in lins]
        hent = entries_device([dfssm.StackEntry(l.weights(), l.dx.data_ptr(), mapped_address(h.data_ptr()),
                                                dfssm.Debug(0, 0, 0, 0), i, 0) for i, (l, h) in enumerate(zip(lins, hosts))])
        dfssm.dfssm_linear_stack_fwd(plan, hent.data_ptr(), len(lins), m, stream)
        st, bits = dfssm.dfssm_plan_check(plan)
        assert st == dfssm.DFSSM_OK, hex(bits)
        for l, h in zip(lins, hosts):
            assert torch.equal(h.view(torch.uint8), l.dy.cpu().view(torch.uint8))
            check_linear_full(l)
    finally:
        dfssm.dfssm_plan_destroy(plan)


# ------------------------------------------------------------------ full-size workloads

@pytest.mark.parametrize("workload", ["out_proj_m1", "in_proj_m1"])
def test_single_projection_full(workload):
    wl = synth.WORKLOADS[workload]
    (d_in, d_out), m = wl["shapes"][0], wl["m"]
    lin = Linear(SEED, wl["cfg"], 0, d_in, d_out, m, BF16)
    run_one(lin)
    check_linear_full(lin)


@pytest.mark.parametrize("workload,samples", [("stack48_m1", 0), ("stack48_m4", 400), ("stack48_m16", 400),
                                              ("stack48_m64", 300), ("stack48_m512", 200),
                                              ("stack48_m2048", 200)])
def test_stack_full_size(workload, samples):
    # First the call exactly as bench.py makes it (bf16 y, no debug exports: for M = 2048 this
    # is the 16-byte row-piece store path of the tcgen05 epilogue), y checked against the
    # oracle; then the same call with the debug exports, integers checked bit for bit.
    wl = synth.WORKLOADS[workload]
    m = wl["m"]
    lins, plan, ent_dbg = build_stack(wl["shapes"], m, BF16, cfg=wl["cfg"])
    ent_bench = entries_device([l.entry(i, with_dbg=False) for i, l in enumerate(lins)])
    stream = torch.cuda.current_stream().cuda_stream
    try:
        for ent, ints in ((ent_bench, False), (ent_dbg, True)):
            for lin in lins:
                lin.dy.fill_(float("nan"))
            dfssm.dfssm_linear_stack_fwd(plan, ent.data_ptr(), len(lins), m, stream)
            st, bits = dfssm.dfssm_plan_check(plan)
            assert st == dfssm.DFSSM_OK, hex(bits)
            rng = np.random.default_rng(m)
            for i, lin in enumerate(lins):
                if samples == 0:
                    check_linear_full(lin, ints=ints)
                else:
                    check_linear_sampled(lin, samples, rng, ints=ints)
    finally:
        dfssm.dfssm_plan_destroy(plan)


# bf16 output without debug exports and d_out % 8 == 0: the tcgen05 epilogue stores 16-byte row
# pieces for whole 32-row groups and single elements for a last partial group; ragged token tiles
# (192 tokens per tile, 96 per epilogue half; 241 and 480 reach a second and a third tile)
BENCH_STORE_CASES = [(2048, 136, 200), (4096, 520, 400), (1024, 256, 385), (384, 40, 17), (8192, 64, 193),
                     (2048, 256, 241), (1024, 128, 480)]


@pytest.mark.parametrize("d_in,d_out,m", BENCH_STORE_CASES)
def test_prefill_bf16_store_path(d_in, d_out, m):
    lin = Linear(SEED, 9, d_in + 7 * d_out + m, d_in, d_out, m, BF16, dbg=False)
    run_one(lin)
    check_linear_full(lin)

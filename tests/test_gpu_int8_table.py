"""The int8 embedding table and LM head on the GPU against the oracle, through the C ABI.

Embedding rows are bit-exact (one fp32 product, then bf16 rounding if asked); the LM
head's int32 sums are bit-exact and its logits follow the tolerance of tests/gpu_util.py
(eb = 2^-16 |logit| per element; bf16: the nearest bf16 or, near a midpoint, either
neighbour). Full-size: the tied table of Mamba-2 1.3B (50,288 x 2048 int8, technical
summary §3: 37 % of the 278 MB model), sampled outputs computed one by one by the oracle.
"""
import numpy as np
import pytest
import torch

import bit_gemv_gemm_dfssm_b200 as dfssm
import dfssm_synth as synth
import oracle
from gpu_util import check_y, dev

pytestmark = pytest.mark.gpu
BF16, F32 = dfssm.DFSSM_BF16, dfssm.DFSSM_F32


class Table:
    def __init__(self, vocab, d, seed=31):
        self.vocab, self.d = vocab, d
        self.w = synth.int8_table(seed, 5, vocab, d)
        self.dt = dev(self.w["table"])
        self.ds = dev(self.w["scale"])
        self.c = dfssm.Int8Table(self.dt.data_ptr(), self.ds.data_ptr(), vocab, d)


def out_host(t, dtype):
    if dtype == BF16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


@pytest.mark.parametrize("vocab,d,m,dtype", [(100, 16, 1, F32), (257, 48, 5, BF16), (1000, 2048, 16, F32),
                                             (50, 8192, 3, BF16)])
def test_embed_parity(vocab, d, m, dtype):
    tb = Table(vocab, d)
    ids = synth.token_ids(7, 5, m, vocab)
    ids[0] = vocab - 1
    dids = dev(ids)
    out = torch.full((m, d), float("nan"), dtype=torch.bfloat16 if dtype == BF16 else torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dfssm.dfssm_embed_fwd(tb.c, dids.data_ptr(), m, out.data_ptr(), dtype, err.data_ptr(),
                          torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    ref, bad = oracle.embed(tb.w["table"], tb.w["scale"], ids)
    assert bad == 0 and int(err.item()) == 0
    got = out_host(out, dtype)
    if dtype == F32:
        np.testing.assert_array_equal(got, ref)
    else:
        np.testing.assert_array_equal(got, oracle.f64_to_bf16(ref.astype(np.float64)))


def test_embed_bad_ids_give_zero_rows_and_error_bit():
    tb = Table(64, 32)
    ids = np.array([3, -1, 64, 63], np.int32)
    out = torch.full((4, 32), float("nan"), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dfssm.dfssm_embed_fwd(tb.c, dev(ids).data_ptr(), 4, out.data_ptr(), F32, err.data_ptr(), 0)
    torch.cuda.synchronize()
    ref, bad = oracle.embed(tb.w["table"], tb.w["scale"], ids)
    assert bad == 2 and int(err.item()) & dfssm.DFSSM_DEVERR_TOKEN_ID
    np.testing.assert_array_equal(out.cpu().numpy(), ref)


def run_head(tb, h, m, dtype, acc=True):
    dh = dev(h)
    lo = torch.full((m, tb.vocab), float("nan"), dtype=torch.bfloat16 if dtype == BF16 else torch.float32,
                    device="cuda")
    da = torch.zeros((m, tb.vocab), dtype=torch.int32, device="cuda") if acc else None
    dfssm.dfssm_lm_head_fwd(tb.c, dh.data_ptr(), m, lo.data_ptr(), dtype, da.data_ptr() if acc else 0,
                            torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return out_host(lo, dtype), (da.cpu().numpy() if acc else None)


@pytest.mark.parametrize("vocab,d,m,dtype", [(37, 16, 1, F32), (100, 128, 2, BF16), (513, 2048, 4, F32),
                                             (250, 4096, 16, BF16), (77, 8192, 9, F32)])
def test_lm_head_parity(vocab, d, m, dtype):
    tb = Table(vocab, d, seed=vocab + d)
    h = synth.activations(13, 5, vocab, m, d)
    logits, acc = run_head(tb, h, m, dtype)
    ref = oracle.lm_head(tb.w["table"], tb.w["scale"], h, m)
    np.testing.assert_array_equal(acc, ref["acc"])
    check_y(logits, ref["logits"], 2.0 ** -16 * np.abs(ref["logits"]), dtype)


@pytest.mark.parametrize("m", [1, 4])
def test_lm_head_full_size_sampled(m):
    # the bench's configuration: bf16 logits, no sums exported
    tb = Table(synth.VOCAB, synth.D_MODEL, seed=2)
    h = synth.activations(17, 5, 1, m, synth.D_MODEL)
    logits, _ = run_head(tb, h, m, BF16, acc=False)
    rng = np.random.default_rng(m)
    t = np.sort(rng.integers(0, m, 500)).astype(np.int32)
    v = rng.integers(0, synth.VOCAB, 500).astype(np.int32)
    v[:2] = [0, synth.VOCAB - 1]
    s = oracle.lm_head_sampled(tb.w["table"], tb.w["scale"], h, m, t, v)
    check_y(logits[t, v], s["logits"], 2.0 ** -16 * np.abs(s["logits"]), BF16)
    # and the int32 sums, in a second call with the export
    _, acc = run_head(tb, h, m, F32, acc=True)
    np.testing.assert_array_equal(acc[t, v], s["acc"])


def test_table_argument_errors():
    tb = Table(16, 32)
    import ctypes
    L = dfssm.lib()
    bad = dfssm.Int8Table(tb.dt.data_ptr(), tb.ds.data_ptr(), 16, 24)       # d % 16 != 0
    x = torch.zeros((1, 32), dtype=torch.int16, device="cuda")
    y = torch.zeros((1, 16), dtype=torch.float32, device="cuda")
    assert L.dfssm_lm_head_fwd(ctypes.byref(bad), x.data_ptr(), 1, y.data_ptr(), F32, None, None) == \
        dfssm.DFSSM_ERR_UNSUPPORTED_SHAPE
    assert L.dfssm_lm_head_fwd(ctypes.byref(tb.c), x.data_ptr(), 17, y.data_ptr(), F32, None, None) == \
        dfssm.DFSSM_ERR_INVALID_ARG
    assert L.dfssm_embed_fwd(ctypes.byref(tb.c), None, 1, y.data_ptr(), F32, None, None) == dfssm.DFSSM_ERR_INVALID_ARG

"""Pins of the CPU oracle against things other than itself.

Each oracle function is checked against at least one of: hand-worked golden
fixtures (tests/golden/), brute force with an independent library routine
(numpy unpackbits / dense float64 matmul), closed forms, and invariants of the
layer ("Density Field State Space Models", gist.science technical summary,
§2.B frozen 1-bit scaffold + rank-16 int8 LoRA; §2.C int8 scaffold matmul).
The cases are chosen so that a dropped term, a wrong sign, a swapped index or a
transposed operand in the oracle fails at least one of them.
"""
import numpy as np
import pytest

import dfssm_synth as synth
import oracle
from conftest import golden_lines

pytestmark = pytest.mark.filterwarnings("ignore")


def bf16_bits(vals):
    """Exact float -> bf16 bits for values known to be bf16-representable."""
    f = np.asarray(vals, dtype=np.float32)
    b = f.view(np.uint32)
    assert np.all((b & 0xFFFF) == 0), "value not exact in bf16"
    return (b >> 16).astype(np.uint16)


def numpy_unpack(packed, d_out, d_in):
    """Independent unpack: numpy's little-endian bit order, 1 -> +1, 0 -> -1."""
    bits = np.unpackbits(np.asarray(packed, np.uint8).reshape(d_out, d_in // 8), axis=1,
                         bitorder="little")
    return bits.astype(np.int64) * 2 - 1


def rand_case(seed, m, d_in, d_out, rank=16):
    w = synth.linear_weights(seed, 7, 0, d_in, d_out, rank)
    x = synth.activations(seed, 7, 0, m, d_in)
    return x, w


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_rounding_golden():
    for ln in golden_lines("bf16_rounding.txt"):
        v, bits = ln.split()[:2]
        got = int(oracle.f64_to_bf16([float(v)])[0])
        assert got == int(bits, 16), (v, hex(got), bits)


def test_bf16_rounding_matches_library_on_fp32_values():
    # For values exact in fp32 a single rounding equals torch's fp32 -> bf16 (RNE).
    import torch
    rng = np.random.default_rng(1)
    f = (rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))).astype(np.float32)
    f = np.concatenate([f, np.float32([0.0, -0.0, 1.0, 65504.0, 1e-38, -3e38])])
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f64_to_bf16(f.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_bf16_rounding_is_nearest():
    # |v - round(v)| <= half an ulp, and the result is one of the two neighbours.
    rng = np.random.default_rng(2)
    v = rng.standard_normal(5000) * 1000.0
    r = oracle.bf16_bits_to_f64(oracle.f64_to_bf16(v))
    e = np.floor(np.log2(np.abs(v)))
    ulp = 2.0 ** (e - 7)
    assert np.all(np.abs(v - r) <= ulp / 2 * (1 + 1e-15))


# ---------------------------------------------------------------- packing

def test_pack_sign_golden():
    for ln in golden_lines("pack_sign.txt"):
        vals, bytes_ = ln.split("|")
        vals = vals.split()[1:]
        src = np.array([float(v) for v in vals], dtype=np.float32)[None, :]
        expect = np.array([int(b, 16) for b in bytes_.split()], dtype=np.uint8)
        got = oracle.pack_sign(src, 1, 16)[0]
        np.testing.assert_array_equal(got, expect)
        # int8 source agrees where the values fit
        if np.all(np.abs(src) < 127) and np.all(src == np.round(src)):
            got8 = oracle.pack_sign(src.astype(np.int8), 1, 16)[0]
            np.testing.assert_array_equal(got8, expect)


def test_pack_sign_nan_rejected():
    src = np.zeros((1, 8), np.float32)
    src[0, 3] = np.nan
    with pytest.raises(ValueError):
        oracle.pack_sign(src, 1, 8)


@pytest.mark.parametrize("d_out,d_in", [(1, 8), (3, 16), (17, 128), (5, 2048)])
def test_unpack_matches_numpy_and_roundtrips(d_out, d_in):
    rng = np.random.default_rng(d_out * 1000 + d_in)
    packed = rng.integers(0, 256, size=(d_out, d_in // 8), dtype=np.uint8)
    w = oracle.unpack_sign(packed, d_out, d_in)
    np.testing.assert_array_equal(w, numpy_unpack(packed, d_out, d_in))
    np.testing.assert_array_equal(oracle.pack_sign(w, d_out, d_in), packed)
    np.testing.assert_array_equal(oracle.pack_sign(w.astype(np.float32), d_out, d_in), packed)


def test_single_bit_positions():
    # bit i of byte b <-> column 8b + i, LSB first
    d_in = 64
    for col in range(d_in):
        packed = np.zeros((1, d_in // 8), np.uint8)
        packed[0, col // 8] = 1 << (col % 8)
        w = oracle.unpack_sign(packed, 1, d_in)[0]
        assert w[col] == 1 and np.sum(w == 1) == 1


# ---------------------------------------------------------------- quantiser

def test_quantizer_golden():
    rows = [ln.split("|") for ln in golden_lines("quantizer_ties.txt")]
    x = np.stack([bf16_bits([float(v) for v in a.split()]) for a, _ in rows])
    expect = np.array([[int(v) for v in b.split()] for _, b in rows], dtype=np.int8)
    q, sx = oracle.quantize(x, len(rows), 8)
    np.testing.assert_array_equal(q, expect)
    amax = np.abs(oracle.bf16_bits_to_f64(x)).max(axis=1).astype(np.float32)
    # s_x = amax / 127 as one IEEE fp32 division (numpy's float32 divide)
    np.testing.assert_array_equal(sx, np.where(amax == 0, np.float32(0), amax / np.float32(127)))
    assert sx[0] == 1.0 and sx[1] == 0.0


def test_quantizer_properties_random():
    x = synth.activations(11, 7, 0, 6, 4096)
    q, sx = oracle.quantize(x, 6, 4096)
    xf = oracle.bf16_bits_to_f64(x)
    amax = np.abs(xf).max(axis=1)
    assert np.all(np.abs(q.astype(int)) <= 127)
    # the channel holding amax maps to +-127
    for t in range(6):
        j = np.argmax(np.abs(xf[t]))
        assert abs(int(q[t, j])) == 127 and np.sign(q[t, j]) == np.sign(xf[t, j])
    # rounding bound: |q - x*127/amax| <= 1/2 plus the fp32 rounding of inv and the product
    err = np.abs(q - xf * 127.0 / amax[:, None])
    assert np.all(err <= 0.5 + 127 * 2.0 ** -22)
    # odd symmetry (RNE is symmetric about zero)
    qn, sxn = oracle.quantize(x ^ np.uint16(0x8000), 6, 4096)
    np.testing.assert_array_equal(qn, -q)
    np.testing.assert_array_equal(sxn, sx)
    # power-of-two scaling leaves q unchanged and scales s_x exactly
    xs = bf16_bits((xf * 4.0).astype(np.float32))
    qs, sxs = oracle.quantize(xs, 6, 4096)
    np.testing.assert_array_equal(qs, q)
    np.testing.assert_array_equal(sxs, sx * np.float32(4))


def test_quantizer_one_nonzero_channel():
    for v in [1e-3, 0.75, -3.0, 200.0, -1e5]:
        x = np.zeros((1, 32), np.float32)
        x[0, 5] = v
        xb = (x.view(np.uint32) >> 16).astype(np.uint16)
        q, sx = oracle.quantize(xb, 1, 32)
        vv = oracle.bf16_bits_to_f64(xb)[0, 5]
        assert q[0, 5] == (127 if vv > 0 else -127)
        assert np.count_nonzero(q) == 1
        assert sx[0] == np.float32(abs(vv)) / np.float32(127)


def test_quantizer_tiny_amax_saturates():
    # amax below 127 / FLT_MAX (about 3.7e-37): inv = 127 / amax overflows to +inf in fp32, so
    # every nonzero entry maps to +-127 and a zero entry (0 * inf) to 0; s_x stays amax / 127
    for amax_bits in (0x0080, 0x0100, 0x01F0):          # bf16 2^-126, 2^-125, about 1.8e-37
        x = np.zeros((1, 16), np.uint16)
        x[0, 0] = amax_bits
        x[0, 3] = amax_bits ^ 0x8000                     # -amax
        x[0, 7] = 0x0001                                 # the smallest bf16 subnormal
        q, sx = oracle.quantize(x, 1, 16)
        a = oracle.bf16_bits_to_f64(x)[0, 0]
        assert np.float32(127) / np.float32(a) == np.inf
        expect = np.zeros(16, np.int8)
        expect[[0, 7]], expect[3] = 127, -127
        np.testing.assert_array_equal(q[0], expect)
        assert sx[0] == np.float32(a) / np.float32(127)


# ---------------------------------------------------------------- the linear

def test_linear_golden_hand_worked():
    g = {ln.split()[0]: ln.split()[1:] for ln in golden_lines("linear_tiny.txt")}
    d_in, d_out, r = 16, 2, 16
    x0 = np.array([127] + list(range(1, 16)), dtype=np.float32)
    x = bf16_bits(np.stack([x0, 2 * x0, -x0]))
    sign = np.array([[int(b, 16) for b in g["sign_row0"]], [int(b, 16) for b in g["sign_row1"]]], np.uint8)
    wa = np.zeros((d_out, r), np.int8)
    wa[:, 0] = [int(v) for v in g["W_A_col0"]]
    wb = np.zeros((r, d_in), np.int8)
    wb[0] = [int(v) for v in g["W_B_row0"]]
    sb = np.ones(r, np.float32)
    sb[0] = float(g["s_B0"][0])
    w = dict(sign=sign, alpha=np.array(g["alpha"], np.float32), wa=wa,
             sa=np.array(g["s_A"], np.float32), wb=wb, sb=sb)
    out = oracle.linear(x, w, 3, d_in, d_out, r)
    np.testing.assert_array_equal(out["acc"][0], [int(v) for v in g["acc_t0"]])
    np.testing.assert_array_equal(out["acc"][2], [-int(v) for v in g["acc_t0"]])
    assert out["h"][0, 0] == int(g["h0_t0"][0]) and np.all(out["h"][0, 1:] == 0)
    for t, key in enumerate(["y_t0", "y_t1", "y_t2"]):
        np.testing.assert_array_equal(out["y"][t], [float(v) for v in g[key]])
    # sampled path gives the same numbers
    s = oracle.linear_sampled(x, w, 3, d_in, d_out, [0, 0, 1, 2], [0, 1, 1, 0], r)
    np.testing.assert_array_equal(s["y"], [154.375, -91.75, -183.5, -154.375])


@pytest.mark.parametrize("m,d_in,d_out", [(1, 8, 1), (2, 16, 3), (5, 128, 17), (3, 256, 40)])
def test_linear_brute_force(m, d_in, d_out):
    rank = 16
    x, w = rand_case(100 + m + d_in + d_out, m, d_in, d_out, rank)
    out = oracle.linear(x, w, m, d_in, d_out, rank)
    q = out["q"].astype(np.float64)
    W = numpy_unpack(w["sign"], d_out, d_in).astype(np.float64)
    acc_bf = q @ W.T                                     # exact: all values < 2^53
    h_bf = q @ w["wb"].astype(np.float64).T
    np.testing.assert_array_equal(out["acc"], acc_bf.astype(np.int64))
    np.testing.assert_array_equal(out["h"], h_bf.astype(np.int64))
    # y via dense float64 matrices (a different association than the oracle's loop)
    lora = (h_bf * w["sb"].astype(np.float64)[None, :]) @ w["wa"].astype(np.float64).T
    y_bf = out["sx"].astype(np.float64)[:, None] * (
        w["alpha"].astype(np.float64)[None, :] * acc_bf + w["sa"].astype(np.float64)[None, :] * lora)
    np.testing.assert_allclose(out["y"], y_bf, rtol=1e-12, atol=1e-12 * np.abs(y_bf).max())


def test_invariant_all_ones_row_and_zero_lora():
    m, d_in, d_out = 3, 256, 8
    x, w = rand_case(5, m, d_in, d_out)
    w["sign"][2, :] = 0xFF                    # row 2: all +1
    w["sign"][5, :] = 0x00                    # row 5: all -1
    w["wa"][:] = 0                            # zero LoRA
    out = oracle.linear(x, w, m, d_in, d_out)
    sq = out["q"].astype(np.int64).sum(axis=1)
    np.testing.assert_array_equal(out["acc"][:, 2], sq)
    np.testing.assert_array_equal(out["acc"][:, 5], -sq)
    # zero LoRA: y equals the scaffold term alone, s_x * alpha * acc
    y_s = out["sx"].astype(np.float64)[:, None] * w["alpha"].astype(np.float64)[None, :] * out["acc"]
    np.testing.assert_array_equal(out["y"], y_s)
    # zero W_B gives the same
    x2, w2 = rand_case(5, m, d_in, d_out)
    w2["sign"][2, :] = 0xFF
    w2["sign"][5, :] = 0x00
    w2["wb"][:] = 0
    out2 = oracle.linear(x2, w2, m, d_in, d_out)
    assert np.all(out2["h"] == 0)
    np.testing.assert_array_equal(out2["y"], y_s)


def test_invariant_bit_flip():
    m, d_in, d_out = 2, 128, 4
    x, w = rand_case(9, m, d_in, d_out)
    base = oracle.linear(x, w, m, d_in, d_out)
    rng = np.random.default_rng(0)
    for _ in range(20):
        o, j = int(rng.integers(d_out)), int(rng.integers(d_in))
        w2 = {k: v.copy() for k, v in w.items()}
        was_one = (w2["sign"][o, j // 8] >> (j % 8)) & 1
        w2["sign"][o, j // 8] ^= np.uint8(1 << (j % 8))
        out = oracle.linear(x, w2, m, d_in, d_out)
        d = out["acc"].astype(np.int64) - base["acc"]
        qj = base["q"][:, j].astype(np.int64)
        np.testing.assert_array_equal(d[:, o], -2 * qj if was_one else 2 * qj)
        d[:, o] = 0
        assert np.all(d == 0)


def test_invariant_alpha_zero_gives_lora_only():
    m, d_in, d_out = 2, 128, 5
    x, w = rand_case(21, m, d_in, d_out)
    w["alpha"][:] = 0
    out = oracle.linear(x, w, m, d_in, d_out)
    h = out["h"].astype(np.float64)
    lora = (h * w["sb"].astype(np.float64)) @ w["wa"].astype(np.float64).T
    expect = out["sx"].astype(np.float64)[:, None] * w["sa"].astype(np.float64)[None, :] * lora
    np.testing.assert_allclose(out["y"], expect, rtol=1e-12)


def test_invariant_channel_permutation_and_batch():
    m, d_in, d_out = 4, 256, 6
    x, w = rand_case(33, m, d_in, d_out)
    base = oracle.linear(x, w, m, d_in, d_out)
    perm = np.random.default_rng(3).permutation(d_in)
    W = oracle.unpack_sign(w["sign"], d_out, d_in)
    w2 = dict(w)
    w2["sign"] = oracle.pack_sign(W[:, perm], d_out, d_in)
    w2["wb"] = np.ascontiguousarray(w["wb"][:, perm])
    out = oracle.linear(np.ascontiguousarray(x[:, perm]), w2, m, d_in, d_out)
    np.testing.assert_array_equal(out["acc"], base["acc"])
    np.testing.assert_array_equal(out["h"], base["h"])
    np.testing.assert_array_equal(out["y"], base["y"])
    # batch invariance: row t of an m-batch equals an m = 1 run of token t
    for t in range(m):
        one = oracle.linear(np.ascontiguousarray(x[t:t + 1]), w, 1, d_in, d_out)
        np.testing.assert_array_equal(one["y"][0], base["y"][t])


def test_invariant_power_of_two_scaling_of_x():
    m, d_in, d_out = 2, 128, 5
    x, w = rand_case(44, m, d_in, d_out)
    base = oracle.linear(x, w, m, d_in, d_out)
    xs = (oracle.bf16_bits_to_f64(x) * 8.0).astype(np.float32)
    xsb = (xs.view(np.uint32) >> 16).astype(np.uint16)
    out = oracle.linear(xsb, w, m, d_in, d_out)
    np.testing.assert_array_equal(out["acc"], base["acc"])
    np.testing.assert_array_equal(out["y"], base["y"] * 8.0)


def test_sampled_matches_full():
    m, d_in, d_out = 3, 256, 33
    x, w = rand_case(55, m, d_in, d_out)
    full = oracle.linear(x, w, m, d_in, d_out)
    rng = np.random.default_rng(4)
    t = np.sort(rng.integers(0, m, 50)).astype(np.int32)
    o = rng.integers(0, d_out, 50).astype(np.int32)
    s = oracle.linear_sampled(x, w, m, d_in, d_out, t, o)
    np.testing.assert_array_equal(s["acc"], full["acc"][t, o])
    np.testing.assert_array_equal(s["y"], full["y"][t, o])


def test_unpacked_entry_matches_the_layer():
    # the forward pass from the unpacked +-1 matrix (the CPU baseline times the unpack apart)
    x, w = rand_case(21, 3, 384, 50)
    full = oracle.linear(x, w, 3, 384, 50)
    wpm = oracle.unpack_sign(w["sign"], 50, 384)
    np.testing.assert_array_equal(oracle.linear_unpacked(x, wpm, w, 3, 384, 50), full["y"])
    np.testing.assert_array_equal(oracle.linear_unpacked(x, wpm, w, 3, 384, 50, threads=1), full["y"])


def test_threads_do_not_change_results():
    m, d_in, d_out = 3, 512, 64
    x, w = rand_case(66, m, d_in, d_out)
    a = oracle.linear(x, w, m, d_in, d_out, threads=1)
    b = oracle.linear(x, w, m, d_in, d_out, threads=4)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])


def test_accumulator_bounds_fit_int32():
    # |acc| <= 127 * d_in and |h| <= 127 * 127 * d_in stay inside int32 for d_in <= 4096
    d_in = 4096
    x = bf16_bits(np.full((1, d_in), 3.0, np.float32))
    w = dict(sign=np.full((2, d_in // 8), 0xFF, np.uint8), alpha=np.ones(2, np.float32),
             wa=np.full((2, 16), 127, np.int8), sa=np.ones(2, np.float32),
             wb=np.full((16, d_in), 127, np.int8), sb=np.ones(16, np.float32))
    out = oracle.linear(x, w, 1, d_in, 2)
    assert out["acc"][0, 0] == 127 * d_in
    assert np.all(out["h"][0] == 127 * 127 * d_in)


# ---------------------------------------------------------------- layout vs the pages' sizes

def test_scaffold_share_matches_pages():
    g = {ln.split()[0]: ln.split()[1:] for ln in golden_lines("model_composition.txt")}
    total = int(g["total_bytes"][0])
    n_layers = int(g["n_layers"][0])
    shapes = [tuple(int(v) for v in g["in_proj"]), tuple(int(v) for v in g["out_proj"])]
    sign = lora = 0
    for d_in, d_out in shapes:
        s, l, _ = oracle.weight_bytes(d_in, d_out, 16)
        sign += n_layers * s
        lora += n_layers * l
    assert sign == 154_927_104
    assert round(100 * sign / total) == int(g["scaffold_percent"][0])
    # LoRA: 4.6 % of 278 MB against a printed "4 %"; consistent to the page's one digit
    assert abs(100 * lora / total - int(g["lora_percent"][0])) < 1.0


# ---------------------------------------------------------------- int8 embedding table / LM head

def tiny_table():
    g = {ln.split()[0]: ln.split()[1:] for ln in golden_lines("int8_table_tiny.txt")}
    table = np.array([[int(v) for v in g[f"E{i}"]] for i in range(3)], np.int8)
    scale = np.array([float(v) for v in g["scale"]], np.float32)
    return g, table, scale


def test_embed_golden_hand_worked():
    g, table, scale = tiny_table()
    ids = np.array([int(v) for v in g["embed_ids"]], np.int32)
    out, bad = oracle.embed(table, scale, ids)
    assert bad == 0
    np.testing.assert_array_equal(out[0], np.array([float(v) for v in g["embed_row0"]], np.float32))
    np.testing.assert_array_equal(out[1], np.array([float(v) for v in g["embed_row1"]], np.float32))


def test_embed_matches_float64_product_rounded_once_and_flags_bad_ids():
    rng = np.random.default_rng(3)
    table = rng.integers(-127, 128, size=(50, 96)).astype(np.int8)
    scale = rng.uniform(1e-4, 1e-2, 50).astype(np.float32)
    ids = np.array([0, 49, 7, -1, 50, 7], np.int32)
    out, bad = oracle.embed(table, scale, ids)
    assert bad == 2
    ref = (table.astype(np.float64) * scale.astype(np.float64)[:, None]).astype(np.float32)
    for t, i in enumerate(ids):
        if 0 <= i < 50:
            np.testing.assert_array_equal(out[t], ref[i])
        else:
            assert np.all(out[t] == 0)


def test_lm_head_golden_hand_worked():
    g, table, scale = tiny_table()
    h0 = bf16_bits([float(v) for v in g["h_t0"]])
    h = np.stack([h0, bf16_bits(2 * np.array([float(v) for v in g["h_t0"]], np.float32))])
    q, sx = oracle.quantize(h, 2, 4)
    np.testing.assert_array_equal(q[0], np.array([int(v) for v in g["q_t0"]], np.int8))
    out = oracle.lm_head(table, scale, h, 2)
    acc0 = np.array([int(v) for v in g["acc_t0"]], np.int32)
    np.testing.assert_array_equal(out["acc"][0], acc0)
    np.testing.assert_array_equal(out["acc"][1], acc0)
    sx0 = np.float32(2.0) / np.float32(127.0)
    expect = float(sx0) * scale.astype(np.float64) * acc0
    np.testing.assert_array_equal(out["logits"][0], expect)
    np.testing.assert_array_equal(out["logits"][1], 2 * expect)


@pytest.mark.parametrize("m,vocab,d", [(1, 37, 128), (3, 64, 256), (5, 11, 2048)])
def test_lm_head_brute_force(m, vocab, d):
    rng = np.random.default_rng(vocab * d + m)
    table = rng.integers(-127, 128, size=(vocab, d)).astype(np.int8)
    scale = rng.uniform(1e-4, 1e-2, vocab).astype(np.float32)
    h = synth.activations(11, 7, vocab, m, d)
    out = oracle.lm_head(table, scale, h, m)
    q, sx = oracle.quantize(h, m, d)
    acc = q.astype(np.float64) @ table.astype(np.float64).T          # exact below 2^53
    np.testing.assert_array_equal(out["acc"], acc.astype(np.int64))
    ref = sx.astype(np.float64)[:, None] * scale.astype(np.float64)[None, :] * acc
    np.testing.assert_allclose(out["logits"], ref, rtol=1e-15, atol=0)
    # sampled pairs agree with the full head
    t = np.array([0, m - 1, m - 1], np.int32)
    v = np.array([vocab - 1, 0, vocab // 2], np.int32)
    s = oracle.lm_head_sampled(table, scale, h, m, t, v)
    np.testing.assert_array_equal(s["acc"], out["acc"][t, v])
    np.testing.assert_array_equal(s["logits"], out["logits"][t, v])


def test_lm_head_invariants():
    rng = np.random.default_rng(5)
    vocab, d, m = 20, 256, 2
    table = rng.integers(-127, 128, size=(vocab, d)).astype(np.int8)
    scale = rng.uniform(1e-4, 1e-2, vocab).astype(np.float32)
    h = synth.activations(5, 7, 3, m, d)
    base = oracle.lm_head(table, scale, h, m)
    # a row scale times 4 gives that row's logits times 4 (exact), the others unchanged
    s2 = scale.copy()
    s2[3] *= 4
    out = oracle.lm_head(table, s2, h, m)
    np.testing.assert_array_equal(out["logits"][:, 3], 4 * base["logits"][:, 3])
    np.testing.assert_array_equal(np.delete(out["logits"], 3, 1), np.delete(base["logits"], 3, 1))
    # permuting the rows of the table permutes the logits
    perm = rng.permutation(vocab)
    out = oracle.lm_head(table[perm], scale[perm], h, m)
    np.testing.assert_array_equal(out["logits"], base["logits"][:, perm])
    # negating a row negates its sums
    t2 = table.copy()
    t2[5] = -t2[5]
    out = oracle.lm_head(t2, scale, h, m)
    np.testing.assert_array_equal(out["acc"][:, 5], -base["acc"][:, 5])
    # h = 0: every logit is 0
    out = oracle.lm_head(table, scale, np.zeros((m, d), np.uint16), m)
    assert np.all(out["logits"] == 0) and np.all(out["acc"] == 0)


def test_embedding_share_matches_pages():
    g = {ln.split()[0]: ln.split()[1:] for ln in golden_lines("model_composition.txt")}
    total = int(g["total_bytes"][0])
    table_bytes = int(g["vocab"][0]) * int(g["d_model"][0])
    assert table_bytes == 102_989_824
    assert round(100 * table_bytes / total) == int(g["emb_percent"][0])

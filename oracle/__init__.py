"""CPU oracle for the DF-SSM 1-bit scaffold + int8 LoRA linear (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The library (``bit_gemv_gemm_dfssm_b200``)
never imports it, and the two share no code. ``dfssm_oracle.cpp`` (the layer,
the int8 table), ``ssm_oracle.cpp`` (the state operations) and
``block_oracle.cpp`` (the block frame: residual add and RMS norm) and
``density_oracle.cpp`` (the state density field) hold the arithmetic, written as plain loops; this file only loads them and marshals
numpy arrays.

Every function is pinned (``tests/test_oracle_pins.py``,
``tests/test_ssm_oracle_pins.py``, ``tests/test_block_oracle_pins.py``,
``tests/test_density_oracle_pins.py``) against brute force,
closed forms, invariants and hand-computed fixtures; no function here is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dfssm_oracle.cpp")
_SRCS = [_SRC, os.path.join(_HERE, "ssm_oracle.cpp"), os.path.join(_HERE, "block_oracle.cpp"),
         os.path.join(_HERE, "density_oracle.cpp")]
_LIB_PATH = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (no fast-math, no FMA contraction, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or any(os.path.getmtime(_LIB_PATH) < os.path.getmtime(f)
                                                     for f in _SRCS):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c++17",
                               "-ffp-contract=off", "-fno-fast-math", "-o", tmp, *_SRCS])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        vp, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.dfssm_oracle_f64_to_bf16.restype = ctypes.c_uint16
        lib.dfssm_oracle_f64_to_bf16.argtypes = [dbl]
        lib.dfssm_oracle_f64_to_bf16_array.argtypes = [vp, i64, vp]
        lib.dfssm_oracle_unpack_sign.argtypes = [vp, i32, i32, vp]
        lib.dfssm_oracle_pack_sign_f32.argtypes = [vp, i32, i32, vp]
        lib.dfssm_oracle_pack_sign_i8.argtypes = [vp, i32, i32, vp]
        lib.dfssm_oracle_quantize.argtypes = [vp, i32, i32, vp, vp]
        lib.dfssm_oracle_linear.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp,
                                            vp, vp, vp, vp, vp, i32]
        lib.dfssm_oracle_linear_unpacked.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp,
                                                     vp, vp, vp, vp, vp, i32]
        lib.dfssm_oracle_linear_sampled.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp,
                                                    vp, vp, i64, vp, vp]
        lib.dfssm_oracle_weight_bytes.argtypes = [i32, i32, i32, vp, vp, vp]
        lib.dfssm_oracle_embed.restype = i32
        lib.dfssm_oracle_embed.argtypes = [vp, vp, i32, i32, vp, i32, vp]
        lib.dfssm_oracle_lm_head.argtypes = [vp, vp, i32, i32, vp, i32, vp, vp, i32]
        lib.dfssm_oracle_ssm_step.argtypes = [i32, i32, i32, i32, dbl, i32, vp, vp, vp, vp, vp, vp, vp, vp,
                                              vp, vp, vp, vp, vp, vp, vp, vp]
        lib.dfssm_oracle_lm_head_sampled.argtypes = [vp, vp, i32, i32, vp, i32, vp, vp, i64, vp, vp]
        lib.dfssm_oracle_add_rmsnorm.argtypes = [i32, dbl, i32, vp, vp, i32, vp, vp, vp, vp]
        lib.dfssm_oracle_density_encode.argtypes = [i32, i32, i32, vp, vp, vp]
        lib.dfssm_oracle_density_decode.argtypes = [i32, i32, i32, vp, vp, vp]
        _lib = lib
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


def f64_to_bf16(v) -> np.ndarray:
    """Round float64 values to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    v, pv = _c(v, np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    _L().dfssm_oracle_f64_to_bf16_array(pv, v.size, out.ctypes.data)
    return out


def bf16_bits_to_f64(b) -> np.ndarray:
    """Exact widening of bf16 bit patterns (numpy only)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def unpack_sign(packed, d_out: int, d_in: int) -> np.ndarray:
    p, pp = _c(packed, np.uint8)
    assert p.size == d_out * d_in // 8
    w = np.empty((d_out, d_in), dtype=np.int8)
    _L().dfssm_oracle_unpack_sign(pp, d_out, d_in, w.ctypes.data)
    return w


def pack_sign(src, d_out: int, d_in: int) -> np.ndarray:
    """Pack a frozen scaffold (fp32 or int8): value >= 0 -> bit 1 (+1), value < 0 -> bit 0."""
    src = np.asarray(src)
    out = np.empty((d_out, d_in // 8), dtype=np.uint8)
    if src.dtype == np.float32:
        s, ps = _c(src, np.float32)
        rc = _L().dfssm_oracle_pack_sign_f32(ps, d_out, d_in, out.ctypes.data)
    elif src.dtype == np.int8:
        s, ps = _c(src, np.int8)
        rc = _L().dfssm_oracle_pack_sign_i8(ps, d_out, d_in, out.ctypes.data)
    else:
        raise TypeError(src.dtype)
    if rc:
        raise ValueError("NaN in the scaffold source")
    return out


def quantize(x_bf16_bits, m: int, d_in: int):
    """Per-token symmetric absmax int8 quantiser. Returns (q int8 m x d_in, s_x fp32 m)."""
    x, px = _c(x_bf16_bits, np.uint16)
    q = np.empty((m, d_in), dtype=np.int8)
    sx = np.empty(m, dtype=np.float32)
    _L().dfssm_oracle_quantize(px, m, d_in, q.ctypes.data, sx.ctypes.data)
    return q, sx


def linear(x_bf16_bits, w: dict, m: int, d_in: int, d_out: int, rank: int = 16, threads: int = 0):
    """The whole layer. Returns dict(q, sx, acc, h, y) with y in float64."""
    x, px = _c(x_bf16_bits, np.uint16)
    keep = [_c(w["sign"], np.uint8), _c(w["alpha"], np.float32), _c(w["wa"], np.int8),
            _c(w["sa"], np.float32), _c(w["wb"], np.int8), _c(w["sb"], np.float32)]
    out = dict(q=np.empty((m, d_in), np.int8), sx=np.empty(m, np.float32),
               acc=np.empty((m, d_out), np.int32), h=np.empty((m, rank), np.int32),
               y=np.empty((m, d_out), np.float64))
    _L().dfssm_oracle_linear(px, m, d_in, d_out, rank, *[p for _, p in keep],
                             out["q"].ctypes.data, out["sx"].ctypes.data, out["acc"].ctypes.data,
                             out["h"].ctypes.data, out["y"].ctypes.data, threads)
    return out


def linear_unpacked(x_bf16_bits, w_pm1, w: dict, m: int, d_in: int, d_out: int, rank: int = 16, threads: int = 0):
    """The layer from the unpacked +-1 matrix (d_out x d_in int8, see unpack_sign): y (float64) only."""
    x, px = _c(x_bf16_bits, np.uint16)
    keep = [_c(w_pm1, np.int8), _c(w["alpha"], np.float32), _c(w["wa"], np.int8),
            _c(w["sa"], np.float32), _c(w["wb"], np.int8), _c(w["sb"], np.float32)]
    y = np.empty((m, d_out), np.float64)
    _L().dfssm_oracle_linear_unpacked(px, m, d_in, d_out, rank, *[p for _, p in keep], None, None, None, None,
                                      y.ctypes.data, threads)
    return y


def linear_sampled(x_bf16_bits, w: dict, m: int, d_in: int, d_out: int, t_idx, o_idx, rank: int = 16):
    """y (float64) and acc (int32) at the pairs (t_idx[i], o_idx[i]) only."""
    x, px = _c(x_bf16_bits, np.uint16)
    keep = [_c(w["sign"], np.uint8), _c(w["alpha"], np.float32), _c(w["wa"], np.int8),
            _c(w["sa"], np.float32), _c(w["wb"], np.int8), _c(w["sb"], np.float32)]
    t, pt = _c(t_idx, np.int32)
    o, po = _c(o_idx, np.int32)
    n = t.size
    acc = np.empty(n, np.int32)
    y = np.empty(n, np.float64)
    _L().dfssm_oracle_linear_sampled(px, m, d_in, d_out, rank, *[p for _, p in keep], pt, po, n,
                                     acc.ctypes.data, y.ctypes.data)
    return dict(acc=acc, y=y)


def weight_bytes(d_in: int, d_out: int, rank: int = 16):
    """(sign, lora, scale) bytes of one linear as stored."""
    a, b, c = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    _L().dfssm_oracle_weight_bytes(d_in, d_out, rank, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c))
    return a.value, b.value, c.value


def embed(table, scale, ids):
    """Rows of the int8 table times their scales (fp32). Returns (out m x d float32, #bad ids)."""
    tb, ptb = _c(table, np.int8)
    sc, psc = _c(scale, np.float32)
    i, pi = _c(ids, np.int32)
    vocab, d = tb.shape
    out = np.empty((i.size, d), np.float32)
    bad = _L().dfssm_oracle_embed(ptb, psc, vocab, d, pi, i.size, out.ctypes.data)
    return out, bad


def lm_head(table, scale, h_bf16_bits, m: int, threads: int = 0):
    """Logits (float64, m x vocab) and int32 sums of the int8 head over the quantised h."""
    tb, ptb = _c(table, np.int8)
    sc, psc = _c(scale, np.float32)
    h, ph = _c(h_bf16_bits, np.uint16)
    vocab, d = tb.shape
    acc = np.empty((m, vocab), np.int32)
    logits = np.empty((m, vocab), np.float64)
    _L().dfssm_oracle_lm_head(ptb, psc, vocab, d, ph, m, acc.ctypes.data, logits.ctypes.data, threads)
    return dict(acc=acc, logits=logits)


def lm_head_sampled(table, scale, h_bf16_bits, m: int, t_idx, v_idx):
    """Logits and int32 sums at the pairs (t_idx[i], v_idx[i]) only."""
    tb, ptb = _c(table, np.int8)
    sc, psc = _c(scale, np.float32)
    h, ph = _c(h_bf16_bits, np.uint16)
    t, pt = _c(t_idx, np.int32)
    v, pv = _c(v_idx, np.int32)
    vocab, d = tb.shape
    acc = np.empty(t.size, np.int32)
    logits = np.empty(t.size, np.float64)
    _L().dfssm_oracle_lm_head_sampled(ptb, psc, vocab, d, ph, m, pt, pv, t.size, acc.ctypes.data,
                                      logits.ctypes.data)
    return dict(acc=acc, logits=logits)


def ssm_step(dims, inp):
    """One decode step of the Mamba-2 state operations for one layer (ssm_oracle.cpp).

    dims: dict(d_inner, headdim, d_state, d_conv, eps). inp: dict with zxbcdt (m x row, bf16
    bits), conv_state (m x conv_dim x d_conv, bf16 bits), ssm_state (m x nheads x headdim x
    d_state, float32), conv_w (conv_dim x d_conv), conv_b, dt_bias, a_log, d_skip, norm_w
    (float32). The inputs are not modified. Returns float64 ssm_state and out, the new
    conv_state (bf16 bits) and the intermediates xc, dt, dA, y (before the gate) and r."""
    d_inner, headdim, d_state, d_conv = dims["d_inner"], dims["headdim"], dims["d_state"], dims["d_conv"]
    nheads = d_inner // headdim
    conv_dim = d_inner + 2 * d_state
    z, pz = _c(inp["zxbcdt"], np.uint16)
    m = z.shape[0]
    assert z.shape == (m, 2 * d_inner + 2 * d_state + nheads)
    cs = np.array(inp["conv_state"], dtype=np.uint16, copy=True, order="C")
    assert cs.shape == (m, conv_dim, d_conv)
    s_in, ps = _c(inp["ssm_state"], np.float32)
    assert s_in.shape == (m, nheads, headdim, d_state)
    par = [_c(inp[k], np.float32) for k in ("conv_w", "conv_b", "dt_bias", "a_log", "d_skip", "norm_w")]
    s_out = np.empty(s_in.shape, np.float64)
    out = np.empty((m, d_inner), np.float64)
    xc = np.empty((m, conv_dim), np.float64)
    dt = np.empty((m, nheads), np.float64)
    dA = np.empty((m, nheads), np.float64)
    y = np.empty((m, d_inner), np.float64)
    r = np.empty(m, np.float64)
    _L().dfssm_oracle_ssm_step(d_inner, headdim, d_state, d_conv, float(dims["eps"]), m, pz, cs.ctypes.data, ps,
                               s_out.ctypes.data, *[p for _, p in par], out.ctypes.data, xc.ctypes.data,
                               dt.ctypes.data, dA.ctypes.data, y.ctypes.data, r.ctypes.data)
    return dict(ssm_state=s_out, out=out, conv_state=cs, xc=xc, dt=dt, dA=dA, y=y, r=r)


def add_rmsnorm(resid, delta, w, eps):
    """The residual add and RMS norm of the Mamba-2 block frame (block_oracle.cpp).

    resid: m x d float32; delta: m x d bf16 bits (uint16) or float32, or None; w: d float32.
    Returns the new residual (float32: the fp32 sum), the normed output (float64) and the
    per-token factor 1/sqrt(mean(r^2) + eps) (float64)."""
    r_in, pr = _c(resid, np.float32)
    m, d = r_in.shape
    wv, pw = _c(w, np.float32)
    assert wv.shape == (d,)
    pd, bf = None, 0
    if delta is not None:
        dl = np.ascontiguousarray(delta)
        assert dl.shape == (m, d) and dl.dtype in (np.uint16, np.float32)
        bf = 1 if dl.dtype == np.uint16 else 0
        pd = dl.ctypes.data
    r_out = np.empty((m, d), np.float32)
    out = np.empty((m, d), np.float64)
    r = np.empty(m, np.float64)
    _L().dfssm_oracle_add_rmsnorm(d, float(eps), m, pr, pd, bf, pw, r_out.ctypes.data, out.ctypes.data,
                                  r.ctypes.data)
    return dict(resid=r_out, out=out, r=r)


def density_encode(state, K: int):
    """The state density field of each row (density_oracle.cpp): state rows x d_state float32.
    Returns (scale: rows float32, bits: rows x ceil(K*K/8) uint8, LSB-first cells)."""
    st, ps = _c(state, np.float32)
    rows, d = st.shape
    assert K * K >= d, "every value needs at least one cell"
    scale = np.empty(rows, np.float32)
    bits = np.empty((rows, (K * K + 7) // 8), np.uint8)
    _L().dfssm_oracle_density_encode(rows, d, K, ps, scale.ctypes.data, bits.ctypes.data)
    return scale, bits


def density_decode(scale, bits, d_state: int, K: int):
    """The popcount readout: rows x d_state float64 values from the scales and fields."""
    sc, psc = _c(scale, np.float32)
    b, pb = _c(bits, np.uint8)
    rows = sc.size
    assert K * K >= d_state and b.shape == (rows, (K * K + 7) // 8)
    out = np.empty((rows, d_state), np.float64)
    _L().dfssm_oracle_density_decode(rows, d_state, K, psc, pb, out.ctypes.data)
    return out

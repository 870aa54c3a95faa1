"""Seeded synthetic inputs for the DF-SSM scaffold linear (inputs only).

This module draws the tensors the layer consumes; it contains none of the
layer's arithmetic. Both the CPU oracle and the CUDA path read the bytes it
writes. The C side (``synth.c``) defines the generator: SplitMix64 in counter
mode, keyed by ``(seed, stream_id)``.

Shapes follow Mamba-2 1.3B (d_model 2048, 48 layers): in_proj 2048 -> 8512
(2*4096 z/x + 2*128 B/C + 64 dt heads), out_proj 4096 -> 2048, LoRA rank 16
("Density Field State Space Models", gist.science technical summary, §2.B:
rank-16 int8 LoRA on every in_proj and out_proj of all 48 layers).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libdfssm_synth.so")

MASTER_SEED = 0x20260610
RANK = 16
D_MODEL = 2048
IN_PROJ = (2048, 8512)    # (d_in, d_out)
OUT_PROJ = (4096, 2048)
N_LAYERS = 48

# tensor ids inside a stream
T_X, T_COLS, T_SIGN, T_ALPHA, T_WA, T_SA, T_WB, T_SB, T_TABLE, T_TSCALE, T_IDS = range(11)
(T_ZXBCDT, T_CONV_STATE, T_SSM_STATE, T_CONV_W, T_CONV_B, T_DT_BIAS, T_A_LOG, T_D_SKIP,
 T_NORM_W) = range(11, 20)
T_BLOCK_NORM = 20
KIND_WEIGHTS, KIND_ACT = 1, 2
# the tied int8 embedding / LM-head table of Mamba-2 1.3B: its 50,277-token vocabulary padded to
# a multiple of 16, d_model columns
VOCAB = 50288


def build(force: bool = False) -> str:
    """Compile synth.c into libdfssm_synth.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, i64, i32, vp, dbl = (ctypes.c_uint64, ctypes.c_int64, ctypes.c_int,
                                  ctypes.c_void_p, ctypes.c_double)
        lib.dfssm_synth_key.restype = u64
        lib.dfssm_synth_key.argtypes = [u64, u64]
        lib.dfssm_synth_raw.argtypes = [u64, u64, i64, vp]
        lib.dfssm_synth_outlier_cols.argtypes = [u64, i32, i32, vp]
        lib.dfssm_synth_x.argtypes = [u64, u64, i32, i32, vp]
        lib.dfssm_synth_bits.argtypes = [u64, i64, vp]
        lib.dfssm_synth_uniform_f32.argtypes = [u64, i64, dbl, dbl, vp]
        lib.dfssm_synth_int8_sym127.argtypes = [u64, i64, vp]
        lib.dfssm_synth_normal.argtypes = [u64, i64, dbl, ctypes.c_int, vp]
        lib.dfssm_synth_f64_to_bf16.restype = ctypes.c_uint16
        lib.dfssm_synth_f64_to_bf16.argtypes = [dbl]
        _lib = lib
    return _lib


def stream_id(kind: int, cfg: int, m: int, index: int, tensor: int) -> int:
    assert 0 <= m < (1 << 20) and 0 <= index < (1 << 24) and 0 <= tensor < 256
    return (kind << 60) | (cfg << 52) | (m << 32) | (index << 8) | tensor


def key(seed: int, sid: int) -> int:
    return int(_L().dfssm_synth_key(seed & (2**64 - 1), sid))


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def raw(seed: int, sid: int, start: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _L().dfssm_synth_raw(key(seed, sid), start, n, _ptr(out))
    return out


def outlier_cols(seed: int, cfg: int, m: int, index: int, d_in: int) -> np.ndarray:
    n_out = int(np.floor(0.01 * d_in + 0.5))
    out = np.empty(n_out, dtype=np.int32)
    if n_out:
        _L().dfssm_synth_outlier_cols(key(seed, stream_id(KIND_ACT, cfg, m, index, T_COLS)),
                                      d_in, n_out, _ptr(out))
    return out


def activations(seed: int, cfg: int, index: int, m: int, d_in: int, out: np.ndarray | None = None):
    """x for one linear: m x d_in bf16, returned as its uint16 bit patterns."""
    if out is None:
        out = np.empty((m, d_in), dtype=np.uint16)
    assert out.dtype == np.uint16 and out.shape == (m, d_in)
    kx = key(seed, stream_id(KIND_ACT, cfg, m, index, T_X))
    kc = key(seed, stream_id(KIND_ACT, cfg, m, index, T_COLS))
    _L().dfssm_synth_x(kx, kc, m, d_in, _ptr(out))
    return out


def linear_weights(seed: int, cfg: int, index: int, d_in: int, d_out: int, rank: int = RANK,
                   out: dict | None = None) -> dict:
    """Weights of one linear. ``sign`` is packed (d_out x d_in/8 bytes)."""
    assert d_in % 8 == 0
    shapes = {
        "sign": ((d_out, d_in // 8), np.uint8), "alpha": ((d_out,), np.float32),
        "wa": ((d_out, rank), np.int8), "sa": ((d_out,), np.float32),
        "wb": ((rank, d_in), np.int8), "sb": ((rank,), np.float32),
    }
    if out is None:
        out = {k: np.empty(s, dtype=t) for k, (s, t) in shapes.items()}
    for k, (s, t) in shapes.items():
        assert out[k].shape == s and out[k].dtype == t, (k, out[k].shape, s)
    L = _L()

    def k_(t):
        return key(seed, stream_id(KIND_WEIGHTS, cfg, 0, index, t))

    L.dfssm_synth_bits(k_(T_SIGN), out["sign"].size, _ptr(out["sign"]))
    L.dfssm_synth_uniform_f32(k_(T_ALPHA), d_out, 0.005, 0.05, _ptr(out["alpha"]))
    L.dfssm_synth_int8_sym127(k_(T_WA), out["wa"].size, _ptr(out["wa"]))
    L.dfssm_synth_uniform_f32(k_(T_SA), d_out, 1e-4, 1e-3, _ptr(out["sa"]))
    L.dfssm_synth_int8_sym127(k_(T_WB), out["wb"].size, _ptr(out["wb"]))
    L.dfssm_synth_uniform_f32(k_(T_SB), rank, 1e-4, 1e-3, _ptr(out["sb"]))
    return out


def int8_table(seed: int, cfg: int, vocab: int, d: int) -> dict:
    """An int8 table (vocab x d, uniform on -127..127) with one fp32 scale per row (U(1e-4, 1e-3))."""
    out = dict(table=np.empty((vocab, d), np.int8), scale=np.empty(vocab, np.float32))
    L = _L()
    L.dfssm_synth_int8_sym127(key(seed, stream_id(KIND_WEIGHTS, cfg, 0, 0, T_TABLE)), out["table"].size,
                              _ptr(out["table"]))
    L.dfssm_synth_uniform_f32(key(seed, stream_id(KIND_WEIGHTS, cfg, 0, 0, T_TSCALE)), vocab, 1e-4, 1e-3,
                              _ptr(out["scale"]))
    return out


def token_ids(seed: int, cfg: int, m: int, vocab: int) -> np.ndarray:
    """m token ids drawn uniformly from [0, vocab)."""
    r = raw(seed, stream_id(KIND_ACT, cfg, m, 0, T_IDS), 0, m)
    return (r % np.uint64(vocab)).astype(np.int32)


# The Mamba-2 1.3B state operations between in_proj and out_proj: d_inner = 2 d_model, 64 heads of
# 64 channels, d_state 128 (one group of B and C), a 4-tap causal convolution, RMS-norm eps 1e-5.
SSM_DIMS = dict(d_inner=4096, headdim=64, d_state=128, d_conv=4, eps=1e-5)


def ssm_layer_inputs(seed: int, cfg: int, index: int, m: int, dims=None) -> dict:
    """One layer's decode-step inputs for m tokens (inputs only; the state operations themselves
    are in the oracle and the library). zxbcdt ~ N(0,1) and conv_state ~ N(0,1) as bf16 bits,
    ssm_state ~ N(0, 0.5^2) fp32; conv_w ~ U(-0.5, 0.5), conv_b ~ U(-0.1, 0.1); the step size at
    initialisation dt0 ~ U(0.001, 0.1) gives dt_bias = log(expm1(dt0)) (so softplus(dt_bias) = dt0);
    a_log = log(U(1, 16)); d_skip, norm_w ~ U(0.5, 1.5) (all fp32)."""
    d = dims or SSM_DIMS
    d_inner, headdim, d_state, d_conv = d["d_inner"], d["headdim"], d["d_state"], d["d_conv"]
    nheads = d_inner // headdim
    conv_dim = d_inner + 2 * d_state
    row = 2 * d_inner + 2 * d_state + nheads
    L = _L()

    def k_(kind, t):
        return key(seed, stream_id(kind, cfg, m if kind == KIND_ACT else 0, index, t))

    out = dict(zxbcdt=np.empty((m, row), np.uint16), conv_state=np.empty((m, conv_dim, d_conv), np.uint16),
               ssm_state=np.empty((m, nheads, headdim, d_state), np.float32),
               conv_w=np.empty((conv_dim, d_conv), np.float32), conv_b=np.empty(conv_dim, np.float32),
               dt_bias=np.empty(nheads, np.float32), a_log=np.empty(nheads, np.float32),
               d_skip=np.empty(nheads, np.float32), norm_w=np.empty(d_inner, np.float32))
    L.dfssm_synth_normal(k_(KIND_ACT, T_ZXBCDT), out["zxbcdt"].size, 1.0, 1, _ptr(out["zxbcdt"]))
    L.dfssm_synth_normal(k_(KIND_ACT, T_CONV_STATE), out["conv_state"].size, 1.0, 1, _ptr(out["conv_state"]))
    L.dfssm_synth_normal(k_(KIND_ACT, T_SSM_STATE), out["ssm_state"].size, 0.5, 0, _ptr(out["ssm_state"]))
    L.dfssm_synth_uniform_f32(k_(KIND_WEIGHTS, T_CONV_W), out["conv_w"].size, -0.5, 0.5, _ptr(out["conv_w"]))
    L.dfssm_synth_uniform_f32(k_(KIND_WEIGHTS, T_CONV_B), conv_dim, -0.1, 0.1, _ptr(out["conv_b"]))
    dt0 = np.empty(nheads, np.float32)
    L.dfssm_synth_uniform_f32(k_(KIND_WEIGHTS, T_DT_BIAS), nheads, 0.001, 0.1, _ptr(dt0))
    out["dt_bias"][:] = np.log(np.expm1(dt0.astype(np.float64))).astype(np.float32)
    a = np.empty(nheads, np.float32)
    L.dfssm_synth_uniform_f32(k_(KIND_WEIGHTS, T_A_LOG), nheads, 1.0, 16.0, _ptr(a))
    out["a_log"][:] = np.log(a.astype(np.float64)).astype(np.float32)
    L.dfssm_synth_uniform_f32(k_(KIND_WEIGHTS, T_D_SKIP), nheads, 0.5, 1.5, _ptr(out["d_skip"]))
    L.dfssm_synth_uniform_f32(k_(KIND_WEIGHTS, T_NORM_W), d_inner, 0.5, 1.5, _ptr(out["norm_w"]))
    return out


def block_norm_weights(seed: int, cfg: int, index: int, d: int) -> np.ndarray:
    """The RMS-norm weight in front of block `index` (index = the number of blocks: the final
    norm before the LM head), U(0.5, 1.5) fp32."""
    w = np.empty(d, np.float32)
    _L().dfssm_synth_uniform_f32(key(seed, stream_id(KIND_WEIGHTS, cfg, 0, index, T_BLOCK_NORM)), d, 0.5, 1.5,
                                 _ptr(w))
    return w


def stack_shapes(n_layers: int = N_LAYERS):
    """(d_in, d_out) of the 2*n_layers linears in stack order: in_proj, out_proj per layer."""
    return [IN_PROJ if i % 2 == 0 else OUT_PROJ for i in range(2 * n_layers)]


# Named workloads (sizes of the Mamba-2-1.3B scaffold-linear stack).
WORKLOADS = {
    "out_proj_m1": dict(cfg=0, shapes=[OUT_PROJ], m=1),
    "in_proj_m1": dict(cfg=1, shapes=[IN_PROJ], m=1),
    "stack48_m1": dict(cfg=2, shapes=stack_shapes(), m=1),
    "stack48_m4": dict(cfg=3, shapes=stack_shapes(), m=4),
    "stack48_m16": dict(cfg=3, shapes=stack_shapes(), m=16),
    "stack48_m64": dict(cfg=3, shapes=stack_shapes(), m=64),
    "stack48_m512": dict(cfg=4, shapes=stack_shapes(), m=512),
    "stack48_m2048": dict(cfg=4, shapes=stack_shapes(), m=2048),
}

# Stack workloads draw their weights from one stream family (the M=1 stack's),
# so every stack workload runs on identical weights.
def weight_cfg(cfg: int) -> int:
    return 2 if cfg in (2, 3, 4) else cfg

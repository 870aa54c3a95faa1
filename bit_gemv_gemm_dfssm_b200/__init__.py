"""Python binding of libdfssm (argument marshalling only).

Every step of the layer runs in the CUDA kernels of ``libdfssm.so``; this
module only loads the library, declares the C structs of ``include/dfssm.h``
and forwards raw device pointers and stream handles. There is no fallback: if
the library is missing, the first call raises ImportError.

The entry points keep the C names: ``dfssm_linear_plan``, ``dfssm_plan_destroy``,
``dfssm_pack_sign``, ``dfssm_linear_fwd``, ``dfssm_linear_stack_fwd``,
``dfssm_plan_check``, ``dfssm_plan_workspace_bytes``, ``dfssm_status_string``,
``dfssm_linear_fwd_noalloc``, ``dfssm_plan_set_test_hooks``, ``dfssm_embed_fwd``,
``dfssm_lm_head_fwd``, ``dfssm_ssm_workspace_bytes``, ``dfssm_ssm_step``,
``dfssm_ssm_read_error``, ``dfssm_add_rmsnorm``.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# DFSSM_LIBRARY may name another build of the same library (for example a copy built
# with different tile sizes); by default the in-tree build is used.
LIB_PATH = os.environ.get("DFSSM_LIBRARY") or os.path.join(_HERE, "libdfssm.so")

DFSSM_OK = 0
DFSSM_ERR_INVALID_ARG = 1
DFSSM_ERR_UNSUPPORTED_SHAPE = 2
DFSSM_ERR_CUDA = 3
DFSSM_ERR_NO_MEMORY = 4
DFSSM_ERR_DEVICE_CHECK = 5

DFSSM_BF16, DFSSM_F32, DFSSM_I8 = 0, 1, 2

DFSSM_DEVERR_ENTRY_DESC = 0x1
DFSSM_DEVERR_NONFINITE = 0x2
DFSSM_DEVERR_TIMEOUT = 0x4
DFSSM_DEVERR_ENTRY_PTR = 0x8

RANK = 16

# every function the header declares
EXPORTS = (
    "dfssm_linear_plan", "dfssm_plan_destroy", "dfssm_pack_sign", "dfssm_linear_fwd",
    "dfssm_linear_stack_fwd", "dfssm_plan_check", "dfssm_plan_workspace_bytes", "dfssm_status_string",
    "dfssm_linear_fwd_noalloc", "dfssm_plan_set_test_hooks", "dfssm_embed_fwd", "dfssm_lm_head_fwd",
    "dfssm_ssm_workspace_bytes", "dfssm_ssm_step", "dfssm_ssm_read_error", "dfssm_add_rmsnorm",
)
DFSSM_DEVERR_TOKEN_ID = 0x10
DFSSM_TEST_STALL = 0x1
DFSSM_NOALLOC_MAX_M = 16


class DfssmError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {dfssm_status_string(status)} ({status})" if what else dfssm_status_string(status))


class LinearDesc(ctypes.Structure):
    _fields_ = [("d_in", ctypes.c_int32), ("d_out", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("max_m", ctypes.c_int32), ("y_dtype", ctypes.c_int32), ("flags", ctypes.c_uint32)]


class LinearWeights(ctypes.Structure):
    _fields_ = [("sign", ctypes.c_void_p), ("alpha", ctypes.c_void_p), ("wa", ctypes.c_void_p),
                ("sa", ctypes.c_void_p), ("wb", ctypes.c_void_p), ("sb", ctypes.c_void_p)]


class Debug(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("sx", ctypes.c_void_p), ("acc", ctypes.c_void_p),
                ("h", ctypes.c_void_p)]


class StackEntry(ctypes.Structure):
    _fields_ = [("w", LinearWeights), ("x", ctypes.c_void_p), ("y", ctypes.c_void_p), ("dbg", Debug),
                ("desc_index", ctypes.c_int32), ("reserved", ctypes.c_int32)]


assert ctypes.sizeof(StackEntry) == 104


class Int8Table(ctypes.Structure):
    _fields_ = [("table", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("vocab", ctypes.c_int32),
                ("d", ctypes.c_int32)]


class SsmDims(ctypes.Structure):
    _fields_ = [("d_inner", ctypes.c_int32), ("headdim", ctypes.c_int32), ("d_state", ctypes.c_int32),
                ("d_conv", ctypes.c_int32), ("eps", ctypes.c_float), ("out_dtype", ctypes.c_int32)]


class SsmLayer(ctypes.Structure):
    _fields_ = [("zxbcdt", ctypes.c_void_p), ("conv_state", ctypes.c_void_p), ("ssm_state", ctypes.c_void_p),
                ("conv_w", ctypes.c_void_p), ("conv_b", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
                ("a_log", ctypes.c_void_p), ("d_skip", ctypes.c_void_p), ("norm_w", ctypes.c_void_p),
                ("out", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libdfssm.so is not built ({LIB_PATH}); run "
                          "`python -m bit_gemv_gemm_dfssm_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, u32p = ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(ctypes.c_uint32)
    lib.dfssm_linear_plan.argtypes = [ctypes.POINTER(LinearDesc), ctypes.c_int, ctypes.POINTER(vp)]
    lib.dfssm_plan_destroy.argtypes = [vp]
    lib.dfssm_pack_sign.argtypes = [vp, i32, i32, i32, vp, vp]
    lib.dfssm_linear_fwd.argtypes = [vp, i32, ctypes.POINTER(LinearWeights), vp, i32, vp,
                                     ctypes.POINTER(Debug), vp]
    lib.dfssm_linear_stack_fwd.argtypes = [vp, vp, i32, i32, vp]
    lib.dfssm_linear_fwd_noalloc.argtypes = [ctypes.POINTER(LinearDesc), ctypes.POINTER(LinearWeights), vp, i32,
                                             vp, vp]
    lib.dfssm_plan_check.argtypes = [vp, u32p]
    lib.dfssm_plan_workspace_bytes.argtypes = [vp, ctypes.POINTER(ctypes.c_size_t)]
    lib.dfssm_plan_set_test_hooks.argtypes = [vp, ctypes.c_uint64, ctypes.c_uint32]
    lib.dfssm_embed_fwd.argtypes = [ctypes.POINTER(Int8Table), vp, i32, vp, i32, vp, vp]
    lib.dfssm_lm_head_fwd.argtypes = [ctypes.POINTER(Int8Table), vp, i32, vp, i32, vp, vp]
    lib.dfssm_ssm_workspace_bytes.argtypes = [ctypes.POINTER(SsmDims), i32, i32, ctypes.POINTER(ctypes.c_size_t)]
    lib.dfssm_ssm_step.argtypes = [ctypes.POINTER(SsmDims), vp, i32, i32, vp, ctypes.c_size_t, vp]
    lib.dfssm_ssm_read_error.argtypes = [vp, u32p, vp]
    lib.dfssm_add_rmsnorm.argtypes = [vp, i32, ctypes.c_float, vp, vp, i32, i32, vp, vp, i32, vp]
    lib.dfssm_status_string.restype = ctypes.c_char_p
    lib.dfssm_status_string.argtypes = [ctypes.c_int]
    for name in EXPORTS:
        if name != "dfssm_status_string":
            getattr(lib, name).restype = ctypes.c_int
    return lib


_lib = None


def lib():
    """The loaded libdfssm (loaded on first use; raises ImportError if not built)."""
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def dfssm_status_string(status: int) -> str:
    return lib().dfssm_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != DFSSM_OK:
        raise DfssmError(status, what)


def dfssm_linear_plan(descs) -> int:
    """descs: list of LinearDesc (or (d_in, d_out, max_m, y_dtype) tuples). Returns the plan handle."""
    arr = (LinearDesc * len(descs))()
    for i, d in enumerate(descs):
        if not isinstance(d, LinearDesc):
            d_in, d_out, max_m, y_dtype = d
            d = LinearDesc(d_in, d_out, RANK, max_m, y_dtype, 0)
        arr[i] = d
    out = ctypes.c_void_p()
    _check(lib().dfssm_linear_plan(arr, len(descs), ctypes.byref(out)), "dfssm_linear_plan")
    return out.value


def dfssm_plan_destroy(plan: int) -> None:
    _check(lib().dfssm_plan_destroy(plan), "dfssm_plan_destroy")


def dfssm_pack_sign(src_ptr: int, src_dtype: int, d_out: int, d_in: int, packed_ptr: int, stream: int = 0) -> None:
    _check(lib().dfssm_pack_sign(src_ptr, src_dtype, d_out, d_in, packed_ptr, stream), "dfssm_pack_sign")


def dfssm_linear_fwd(plan: int, desc_index: int, w: LinearWeights, x_ptr: int, m: int, y_ptr: int,
                     dbg: Debug | None = None, stream: int = 0) -> None:
    _check(lib().dfssm_linear_fwd(plan, desc_index, ctypes.byref(w), x_ptr, m, y_ptr,
                                 ctypes.byref(dbg) if dbg is not None else None, stream), "dfssm_linear_fwd")


def dfssm_linear_stack_fwd(plan: int, entries_dev_ptr: int, n_entries: int, m: int, stream: int = 0) -> None:
    _check(lib().dfssm_linear_stack_fwd(plan, entries_dev_ptr, n_entries, m, stream), "dfssm_linear_stack_fwd")


def dfssm_linear_fwd_noalloc(desc, w: LinearWeights, x_ptr: int, m: int, y_ptr: int, stream: int = 0) -> None:
    """One linear, m <= 16 tokens, without any device allocation (fixed device scratch)."""
    if not isinstance(desc, LinearDesc):
        d_in, d_out, y_dtype = desc
        desc = LinearDesc(d_in, d_out, RANK, m, y_dtype, 0)
    _check(lib().dfssm_linear_fwd_noalloc(ctypes.byref(desc), ctypes.byref(w), x_ptr, m, y_ptr, stream),
           "dfssm_linear_fwd_noalloc")


def dfssm_plan_check(plan: int):
    """Returns (status, error bits); synchronises the device."""
    bits = ctypes.c_uint32(0)
    st = lib().dfssm_plan_check(plan, ctypes.byref(bits))
    if st not in (DFSSM_OK, DFSSM_ERR_DEVICE_CHECK):
        raise DfssmError(st, "dfssm_plan_check")
    return st, bits.value


def dfssm_embed_fwd(table: Int8Table, ids_ptr: int, m: int, out_ptr: int, out_dtype: int, err_ptr: int = 0,
                    stream: int = 0) -> None:
    """Embedding rows of the int8 table (see include/dfssm.h)."""
    _check(lib().dfssm_embed_fwd(ctypes.byref(table), ids_ptr, m, out_ptr, out_dtype, err_ptr or None, stream),
           "dfssm_embed_fwd")


def dfssm_lm_head_fwd(table: Int8Table, h_ptr: int, m: int, logits_ptr: int, out_dtype: int, acc_ptr: int = 0,
                      stream: int = 0) -> None:
    """Logits of the int8 LM head over the quantised hidden state (see include/dfssm.h)."""
    _check(lib().dfssm_lm_head_fwd(ctypes.byref(table), h_ptr, m, logits_ptr, out_dtype, acc_ptr or None, stream),
           "dfssm_lm_head_fwd")


def dfssm_plan_set_test_hooks(plan: int, wait_limit_ns: int = 0, flags: int = 0) -> None:
    """Error-path test hooks of the decode kernel (see include/dfssm.h)."""
    _check(lib().dfssm_plan_set_test_hooks(plan, wait_limit_ns, flags), "dfssm_plan_set_test_hooks")


def dfssm_plan_workspace_bytes(plan: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().dfssm_plan_workspace_bytes(plan, ctypes.byref(n)), "dfssm_plan_workspace_bytes")
    return n.value


def weights_struct(sign, alpha, wa, sa, wb, sb) -> LinearWeights:
    """Build the C struct from objects exposing data_ptr() (e.g. torch CUDA tensors)."""
    return LinearWeights(sign.data_ptr(), alpha.data_ptr(), wa.data_ptr(), sa.data_ptr(), wb.data_ptr(),
                         sb.data_ptr())


def stack_entries_bytes(entries) -> bytes:
    """Pack a list of StackEntry into the byte image the device array must hold."""
    arr = (StackEntry * len(entries))(*entries)
    return ctypes.string_at(ctypes.addressof(arr), ctypes.sizeof(arr))


def dfssm_ssm_workspace_bytes(dims: SsmDims, n_layers: int, m: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().dfssm_ssm_workspace_bytes(ctypes.byref(dims), n_layers, m, ctypes.byref(n)),
           "dfssm_ssm_workspace_bytes")
    return n.value


def dfssm_ssm_step(dims: SsmDims, layers_dev_ptr: int, n_layers: int, m: int, workspace_ptr: int,
                   workspace_bytes: int, stream: int = 0) -> None:
    """One decode step of the state operations for n_layers layers (see include/dfssm.h)."""
    _check(lib().dfssm_ssm_step(ctypes.byref(dims), layers_dev_ptr, n_layers, m, workspace_ptr, workspace_bytes,
                                stream), "dfssm_ssm_step")


def dfssm_ssm_read_error(workspace_ptr: int, stream: int = 0):
    """(status, bits) of the workspace's device error word, which is cleared."""
    bits = ctypes.c_uint32(0)
    st = lib().dfssm_ssm_read_error(workspace_ptr, ctypes.byref(bits), stream)
    if st not in (DFSSM_OK, DFSSM_ERR_DEVICE_CHECK):
        raise DfssmError(st, "dfssm_ssm_read_error")
    return st, bits.value


def ssm_layers_bytes(layers) -> bytes:
    """Pack a list of SsmLayer into the byte image the device array must hold."""
    arr = (SsmLayer * len(layers))(*layers)
    return ctypes.string_at(ctypes.addressof(arr), ctypes.sizeof(arr))


def dfssm_add_rmsnorm(norm_w_ptr: int, d: int, eps: float, resid_in_ptr: int, delta_ptr: int, delta_dtype: int,
                      m: int, resid_out_ptr: int, out_ptr: int, out_dtype: int, stream: int = 0) -> None:
    """Residual add and RMS norm of the Mamba-2 block frame (see include/dfssm.h)."""
    _check(lib().dfssm_add_rmsnorm(norm_w_ptr, d, eps, resid_in_ptr, delta_ptr or None, delta_dtype, m,
                                   resid_out_ptr, out_ptr, out_dtype, stream), "dfssm_add_rmsnorm")

"""The C-ABI library loads and exports every function include/dfssm.h declares.

No compute call is made here: only argument checks that return before any
CUDA call, and the struct layout against the C compiler's view of the header.
"""
import ctypes
import os
import re
import subprocess

import pytest

import bit_gemv_gemm_dfssm_b200 as dfssm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dfssm.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dfssm_[a-z_]+)\s*\(", src)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(dfssm.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = dfssm.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", dfssm.LIB_PATH], capture_output=True, text=True).stdout
    for name in declared_functions():
        assert re.search(rf"\bT {name}\b", out), name


def test_struct_layout_matches_c(tmp_path):
    prog = tmp_path / "layout.c"
    prog.write_text(f'''
#include <stdio.h>
#include <stddef.h>
#include "{HEADER}"
int main(void) {{
  printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\\n", sizeof(dfssm_linear_desc), sizeof(dfssm_linear_weights),
         sizeof(dfssm_debug), sizeof(dfssm_stack_entry), offsetof(dfssm_stack_entry, x),
         offsetof(dfssm_stack_entry, dbg), offsetof(dfssm_stack_entry, desc_index), sizeof(dfssm_ssm_dims),
         sizeof(dfssm_ssm_layer), offsetof(dfssm_ssm_layer, out));
  return 0;
}}''')
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c99", "-o", str(exe), str(prog)])
    got = [int(v) for v in subprocess.check_output([str(exe)]).split()]
    S = dfssm.StackEntry
    assert got == [ctypes.sizeof(dfssm.LinearDesc), ctypes.sizeof(dfssm.LinearWeights), ctypes.sizeof(dfssm.Debug),
                   ctypes.sizeof(S), S.x.offset, S.dbg.offset, S.desc_index.offset, ctypes.sizeof(dfssm.SsmDims),
                   ctypes.sizeof(dfssm.SsmLayer), dfssm.SsmLayer.out.offset]


def test_argument_errors_without_gpu():
    lib = dfssm.lib()
    out = ctypes.c_void_p(123)
    bad_rank = (dfssm.LinearDesc * 1)(dfssm.LinearDesc(2048, 8512, 8, 1, 0, 0))
    assert lib.dfssm_linear_plan(bad_rank, 1, ctypes.byref(out)) == dfssm.DFSSM_ERR_UNSUPPORTED_SHAPE
    assert out.value is None
    bad_din = (dfssm.LinearDesc * 1)(dfssm.LinearDesc(2000, 8512, 16, 1, 0, 0))
    assert lib.dfssm_linear_plan(bad_din, 1, ctypes.byref(out)) == dfssm.DFSSM_ERR_UNSUPPORTED_SHAPE
    bad_dt = (dfssm.LinearDesc * 1)(dfssm.LinearDesc(2048, 8512, 16, 1, 7, 0))
    assert lib.dfssm_linear_plan(bad_dt, 1, ctypes.byref(out)) == dfssm.DFSSM_ERR_INVALID_ARG
    assert lib.dfssm_linear_plan(None, 1, ctypes.byref(out)) == dfssm.DFSSM_ERR_INVALID_ARG
    assert lib.dfssm_linear_fwd(None, 0, None, None, 1, None, None, None) == dfssm.DFSSM_ERR_INVALID_ARG
    assert lib.dfssm_linear_stack_fwd(None, None, 1, 1, None) == dfssm.DFSSM_ERR_INVALID_ARG
    assert lib.dfssm_pack_sign(None, dfssm.DFSSM_I8, 1, 128, None, None) == dfssm.DFSSM_ERR_INVALID_ARG
    assert lib.dfssm_plan_destroy(None) == dfssm.DFSSM_OK
    # the state step: unsupported shapes and missing buffers return before any CUDA call
    dims = dfssm.SsmDims(4096, 64, 128, 4, 1e-5, dfssm.DFSSM_BF16)
    assert dfssm.dfssm_ssm_workspace_bytes(dims, 48, 1) >= 48 * 4096 * 4       # g of every layer
    for bad in (dfssm.SsmDims(4096, 32, 128, 4, 1e-5, 0), dfssm.SsmDims(4096, 64, 64, 4, 1e-5, 0),
                dfssm.SsmDims(4096, 64, 128, 3, 1e-5, 0), dfssm.SsmDims(4100, 64, 128, 4, 1e-5, 0)):
        n = ctypes.c_size_t(0)
        assert lib.dfssm_ssm_workspace_bytes(ctypes.byref(bad), 1, 1, ctypes.byref(n)) == \
            dfssm.DFSSM_ERR_UNSUPPORTED_SHAPE
    nan_eps = dfssm.SsmDims(4096, 64, 128, 4, float("nan"), 0)
    n = ctypes.c_size_t(0)
    assert lib.dfssm_ssm_workspace_bytes(ctypes.byref(nan_eps), 1, 1, ctypes.byref(n)) == dfssm.DFSSM_ERR_INVALID_ARG
    assert lib.dfssm_ssm_step(ctypes.byref(dims), None, 1, 1, None, 0, None) == dfssm.DFSSM_ERR_INVALID_ARG
    assert lib.dfssm_ssm_step(ctypes.byref(dims), 256, 1, 1, 4096, 16, None) == dfssm.DFSSM_ERR_INVALID_ARG
    # the block frame: shapes, alignment, eps and dtypes are checked before any launch
    A = 1 << 12                                              # 16-byte aligned dummy addresses
    args = dict(w=A, d=2048, eps=1e-5, rin=A, delta=A, ddt=dfssm.DFSSM_BF16, m=1, rout=A, out=A,
                odt=dfssm.DFSSM_BF16)

    def norm(**kw):
        a = dict(args, **kw)
        return lib.dfssm_add_rmsnorm(a["w"], a["d"], a["eps"], a["rin"], a["delta"], a["ddt"], a["m"], a["rout"],
                                     a["out"], a["odt"], None)

    for bad in (dict(d=2044), dict(d=0), dict(d=8200), dict(m=0), dict(m=65537)):
        assert norm(**bad) == dfssm.DFSSM_ERR_UNSUPPORTED_SHAPE, bad
    for bad in (dict(w=None), dict(rin=A + 4), dict(delta=A + 8), dict(out=None), dict(eps=-1.0),
                dict(eps=float("inf")), dict(ddt=dfssm.DFSSM_I8), dict(odt=7)):
        assert norm(**bad) == dfssm.DFSSM_ERR_INVALID_ARG, bad
    assert dfssm.dfssm_status_string(dfssm.DFSSM_ERR_CUDA) == "CUDA error"
    with pytest.raises(dfssm.DfssmError):
        dfssm.dfssm_linear_plan([(100, 10, 1, 0)])


def test_no_cpu_fallback_in_package():
    # the product package never imports the oracle
    pkg = os.path.join(ROOT, "bit_gemv_gemm_dfssm_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "dfssm_oracle" not in text, f

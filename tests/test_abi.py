"""The C-ABI library loads and exports exactly what include/splitkv.h declares (CPU only, no CUDA calls)."""

import ctypes
import os
import re

from context_block_sparse_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "splitkv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(splitkv_\w+)\s*\(", src)))


def test_header_declarations_are_exported(splitkv):
    names = _declared()
    assert len(names) >= 12
    lib = ctypes.CDLL(_abi.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(_abi.SIGNATURES) == names


def test_only_splitkv_symbols_exported(splitkv):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True, text=True).stdout
    syms = [l.split()[-1] for l in out.splitlines() if l.strip()]
    funcs = [s for s in syms if not s.startswith("splitkv_")]
    assert funcs == [] or all(s.startswith(("_init", "_fini")) for s in funcs), funcs


def test_error_strings(splitkv):
    lib = splitkv._lib
    for code in range(0, -8, -1):
        s = lib.splitkv_error_string(code).decode()
        assert s and s != "unknown status"
    assert lib.splitkv_error_string(-99).decode() == "unknown status"


def _c_layout(struct, fields, tmp_path):
    """sizeof and field offsets of a header struct, as gcc lays it out."""
    import subprocess
    body = "".join(f'  printf("%zu\\n", offsetof({struct}, {f}));\n' for f in fields)
    src = (f'#include <stddef.h>\n#include <stdio.h>\n#include "splitkv.h"\n'
           f'int main(void) {{\n  printf("%zu\\n", sizeof({struct}));\n{body}  return 0;\n}}\n')
    c = tmp_path / "layout.c"
    c.write_text(src)
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)], check=True)
    vals = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    return vals[0], vals[1:]


def test_struct_layouts_match_header(tmp_path):
    for struct, cls in (("splitkv_problem", _abi.Problem), ("splitkv_stats", _abi.Stats)):
        fields = [f for f, _ in cls._fields_]
        size, offs = _c_layout(struct, fields, tmp_path)
        assert ctypes.sizeof(cls) == size, struct
        assert [getattr(cls, f).offset for f in fields] == offs, struct


def test_bindings_check_tensor_sizes_against_the_plan(splitkv):
    """The C entry points take bare pointers; the binding refuses a tensor whose element count
    differs from the plan's layout before any pointer is taken (checked here on CPU tensors,
    which then fail the CUDA check)."""
    import pytest
    import torch
    plan = splitkv.splitkv_plan([300, 200], [10, 250, 400], 16, 4, 2, 64, 128, 8)
    Nq, N = 3 * 16, 500
    bf = dict(dtype=torch.bfloat16)
    q, k, v = torch.zeros(Nq, 4, 64, **bf), torch.zeros(N, 2, 64, **bf), torch.zeros(N, 2, 64, **bf)
    ws = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="k has"):
        splitkv.splitkv_attn_fwd(plan, q, k[:-1], v, 0.1, ws)
    with pytest.raises(ValueError, match="q has"):
        splitkv.splitkv_attn_fwd(plan, q[:, :3], k, v, 0.1, ws)
    with pytest.raises(ValueError, match="CUDA"):            # sizes right: the device check speaks
        splitkv.splitkv_attn_fwd(plan, q, k, v, 0.1, ws)
    o, lse = torch.zeros(Nq, 4, 64), torch.zeros(Nq, 4)
    kb = torch.zeros(Nq, 2, 64, **bf)
    with pytest.raises(ValueError, match="lse has"):
        splitkv.splitkv_merge(plan, q, kb, kb, 0.1, ws, o, lse[:-1])
    with pytest.raises(ValueError, match="dvb has"):
        splitkv.splitkv_attn_bwd(plan, q, k, v, kb, kb, o, lse, q, o, o.new_zeros(N, 2, 64), o.new_zeros(N, 2, 64),
                                 o.new_zeros(Nq, 2, 64), o.new_zeros(Nq, 2, 65), 0.1, ws)
    # the sizes follow the plan through an update
    splitkv.splitkv_plan_update(plan, [300, 300], [10, 250, 400])
    with pytest.raises(ValueError, match="k has"):
        splitkv.splitkv_attn_fwd(plan, q, k, v, 0.1, ws)


def test_cast_bf16_rejects_bad_arguments_on_the_host(splitkv):
    """splitkv_cast_bf16 checks its size and pointers before any CUDA call."""
    lib = splitkv._lib
    assert lib.splitkv_cast_bf16(-1, None, None, None) == splitkv._abi.ERR_INVALID_ARG
    assert lib.splitkv_cast_bf16(4, None, None, None) == splitkv._abi.ERR_INVALID_ARG
    assert lib.splitkv_cast_bf16(1 << 43, 16, 16, None) == splitkv._abi.ERR_INVALID_ARG
    assert lib.splitkv_cast_bf16(0, None, None, None) == splitkv._abi.OK   # nothing to do

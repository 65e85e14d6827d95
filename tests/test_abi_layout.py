"""The binding's ctypes mirrors of the C-ABI structs have the header's layout (CPU): a C program built
with gcc against include/vsa.h prints each struct's size and every field's offset, and the ctypes
classes must give the same numbers field by field (a field added on one side only, or out of order,
fails here)."""
import ctypes
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

STRUCTS = {
    "vsa_geometry": "Geometry",
    "vsa_plan_dims": "PlanDims",
    "vsa_seq_parts": "SeqParts",
    "vsa_workspace_layout": "WorkspaceLayout",
}


@pytest.fixture(scope="module")
def c_layout(tmp_path_factory):
    import block_sparse_tiled_b200 as vsa

    d = tmp_path_factory.mktemp("abi")
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "vsa.h"', "int main(void) {"]
    for cname, pyname in STRUCTS.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for field, _ in getattr(vsa, pyname)._fields_:
            lines.append(f'  printf("{cname} {field} %zu\\n", offsetof({cname}, {field}));')
    lines += ["  return 0;", "}"]
    src = d / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = d / "layout"
    subprocess.check_call(["gcc", "-std=c11", f"-I{ROOT}/include", str(src), "-o", str(exe)])
    out = {}
    for ln in subprocess.check_output([str(exe)], text=True).splitlines():
        s, f, v = ln.split()
        out[(s, f)] = int(v)
    return out


@pytest.mark.parametrize("cname", list(STRUCTS))
def test_ctypes_mirror_matches_header(c_layout, cname):
    import block_sparse_tiled_b200 as vsa

    cls = getattr(vsa, STRUCTS[cname])
    assert ctypes.sizeof(cls) == c_layout[(cname, "size")]
    for field, _ in cls._fields_:
        assert getattr(cls, field).offset == c_layout[(cname, field)], field

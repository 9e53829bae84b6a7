"""The ctypes mirrors of the C-ABI argument structs (binding.py) must have the C layout exactly:
a field at a wrong offset would hand the kernels a misread pointer or size.  A small C program,
compiled here with the host compiler against include/kda.h, prints every field's offset and size
and each struct's size; they are compared with the ctypes structures field by field."""
import ctypes
import os
import shutil
import subprocess

import pytest

from linear_attention_serving_rule_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
STRUCTS = {"kda_chunk_args": B.KdaChunkArgs, "kda_decode_args": B.KdaDecodeArgs}


@pytest.fixture(scope="module")
def c_layout(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "kda.h"', "int main(void) {"]
    for cname, cls in STRUCTS.items():
        lines.append(f'  printf("{cname} sizeof %zu %zu\\n", sizeof({cname}), sizeof({cname}));')
        for fname, _ in cls._fields_:
            lines.append(f'  printf("{cname} {fname} %zu %zu\\n", offsetof({cname}, {fname}), '
                         f"sizeof((({cname}*)0)->{fname}));")
    lines += ["  return 0;", "}"]
    d = tmp_path_factory.mktemp("abi")
    src, exe = d / "layout.c", d / "layout"
    src.write_text("\n".join(lines) + "\n")
    subprocess.run([cc, "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    lay = {}
    for line in out.splitlines():
        s, f, a, b = line.split()
        lay[(s, f)] = (int(a), int(b))
    return lay


@pytest.mark.parametrize("cname", list(STRUCTS))
def test_ctypes_mirror_matches_the_c_layout(c_layout, cname):
    cls = STRUCTS[cname]
    assert ctypes.sizeof(cls) == c_layout[(cname, "sizeof")][0]
    for fname, _ in cls._fields_:
        f = getattr(cls, fname)
        assert (f.offset, f.size) == c_layout[(cname, fname)], fname

"""The ctypes mirror of tsa_params in the Python binding matches the C
struct declared in include/tsa.h field by field (offsets and total size), as
the C compiler lays it out.  CPU only: a tiny C program compiled with the
system compiler prints the layout."""
import ctypes
import os
import subprocess
import tempfile

import pytest

import token_sparse_attention_tsa_b200 as T

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def c_layout():
    fields = [f for f, _ in T.tsa_params._fields_]
    body = "\n".join(f'  printf("{f} %zu\\n", offsetof(tsa_params, {f}));' for f in fields)
    src = ("#include <stddef.h>\n#include <stdio.h>\n#include \"tsa.h\"\n"
           "int main(void) {\n" + body + '\n  printf("sizeof %zu\\n", sizeof(tsa_params));\n'
           '  printf("noalloc_bytes %llu\\n", (unsigned long long)TSA_NOALLOC_SCRATCH_BYTES);\n  return 0;\n}\n')
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "layout.c")
        exe = os.path.join(d, "layout")
        with open(c, "w") as f:
            f.write(src)
        try:
            subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True,
                           capture_output=True)
        except (FileNotFoundError, subprocess.CalledProcessError) as e:
            pytest.skip(f"no C compiler: {e}")
        out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    return {k: int(v) for k, v in (line.split() for line in out.splitlines())}


def test_params_struct_layout_matches_the_header():
    lay = c_layout()
    assert lay.pop("sizeof") == ctypes.sizeof(T.tsa_params)
    lay.pop("noalloc_bytes")
    for name, _ in T.tsa_params._fields_:
        assert lay[name] == getattr(T.tsa_params, name).offset, name


def test_params_struct_covers_every_header_field():
    """Every member the header declares in tsa_params has a ctypes field."""
    import re
    text = open(os.path.join(ROOT, "include", "tsa.h")).read()
    body = re.search(r"typedef struct tsa_params \{(.*?)\} tsa_params;", text, re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    declared = []
    for decl in body.split(";"):
        decl = decl.strip()
        if not decl:
            continue
        names = decl.split(None, 1)[1] if not decl.startswith("const") else decl.split(None, 2)[2]
        declared += [n.strip().lstrip("*") for n in names.split(",")]
    assert declared == [f for f, _ in T.tsa_params._fields_]


def test_noalloc_scratch_size_matches_the_header():
    """The binding's copy of TSA_NOALLOC_SCRATCH_BYTES is the header's value."""
    assert c_layout()["noalloc_bytes"] == T.NOALLOC_SCRATCH_BYTES

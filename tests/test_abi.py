"""The C-ABI library loads and exports every entry point include/*.h declares (CPU only).

No compute call is made here: only symbol lookup, struct layout checks against
a C compiler, and argument checks that return before any CUDA call.
"""
import ctypes as C
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        for m in re.finditer(r"\b(vqlin_\w+)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from sparse_compensated_vq_b200 import build
    path = build.build()
    return C.CDLL(path)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 11
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    r = subprocess.run(["nm", "-D", "--defined-only", os.path.join(ROOT, "sparse_compensated_vq_b200", "libvqlin.so")],
                       capture_output=True, text=True, check=True)
    exported = set(l.split()[-1] for l in r.stdout.splitlines() if l.strip())
    assert set(names) <= exported


def test_binding_covers_every_symbol():
    from sparse_compensated_vq_b200 import vqlin
    assert sorted(vqlin.EXPORTS) == declared_functions()


def test_struct_layouts_match_the_header(tmp_path):
    from sparse_compensated_vq_b200 import vqlin
    prog = tmp_path / "layout.c"
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "vqlin.h"', "int main(void) {"]
    for st, cls in (("vqlin_desc", vqlin.vqlin_desc), ("vqlin_info", vqlin.vqlin_info)):
        lines.append('printf("%s sizeof %%zu\\n", sizeof(%s));' % (st, st))
        for f, _ in cls._fields_:
            lines.append('printf("%s %s %%zu\\n", offsetof(%s, %s));' % (st, f, st, f))
    lines.append("return 0; }")
    prog.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), str(prog), "-o", str(exe)])
    out = subprocess.check_output([str(exe)], text=True).split("\n")
    got = {}
    for l in out:
        if l:
            st, f, v = l.split()
            got[(st, f)] = int(v)
    for st, cls in (("vqlin_desc", vqlin.vqlin_desc), ("vqlin_info", vqlin.vqlin_info)):
        assert got[(st, "sizeof")] == C.sizeof(cls)
        for f, _ in cls._fields_:
            assert got[(st, f)] == getattr(cls, f).offset, (st, f)


def test_status_strings_and_version():
    from sparse_compensated_vq_b200 import vqlin
    assert vqlin.vqlin_abi_version() == 1
    for s in range(7):
        assert vqlin.vqlin_status_string(s)


def test_argument_errors_need_no_device():
    from sparse_compensated_vq_b200 import vqlin
    D = vqlin.vqlin_desc()
    D.n_out, D.n_in, D.d = 0, 16, 8
    h = C.c_void_p()
    assert vqlin.vqlin_create(C.byref(D), None, C.byref(h)) == vqlin.VQLIN_ERR_INVALID_ARG
    D.n_out, D.d = 4, 5
    assert vqlin.vqlin_create(C.byref(D), None, C.byref(h)) == vqlin.VQLIN_ERR_UNSUPPORTED
    D.d, D.k1, D.bits1 = 8, 300, 8
    assert vqlin.vqlin_create(C.byref(D), None, C.byref(h)) == vqlin.VQLIN_ERR_INVALID_ARG
    assert b"k1" in vqlin.vqlin_last_error()
    assert vqlin.vqlin_create(None, None, C.byref(h)) == vqlin.VQLIN_ERR_INVALID_ARG
    assert vqlin.vqlin_gemv(None, None, 0, 1, None, 0, None) == vqlin.VQLIN_ERR_INVALID_ARG
    assert vqlin.vqlin_destroy(None) == vqlin.VQLIN_OK

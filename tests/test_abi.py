"""The C-ABI library loads and exports every symbol include/*.h declares (no GPU needed)."""
import glob
import os
import re
import subprocess

import numpy as np

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib():
    from virtual_imaging_b200 import build

    build.build()
    import virtual_imaging_b200 as V

    return V


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b(qem_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return names


def test_every_declared_symbol_is_exported():
    V = _lib()
    declared = _declared()
    assert {"qem_encode", "qem_masked_sum", "qem_masked_sum_delta", "qem_decode_blocks", "qem_free"} <= declared
    out = subprocess.run(["nm", "-D", "--defined-only", V.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = declared - exported
    assert not missing, missing
    assert declared == set(V.EXPORTS), declared ^ set(V.EXPORTS)
    L = V.lib()
    for name in declared:
        getattr(L, name)


def test_abi_string_and_status_names():
    V = _lib()
    assert V.abi() == "qem-pair-v1"
    assert V.status_string(V.QEM_ERR_MALFORMED) == "malformed stream"
    assert V.status_string(99) == "unknown status"


def test_library_model_tables_equal_oracle():
    """Host-side tables of the library, computed independently, equal the oracle's."""
    V = _lib()
    f, a, c = V.model_tables()
    f2, a2, c2 = O.models()
    assert (f == f2).all() and (a == a2).all() and (c == c2).all()
    assert (f.sum(axis=1) == 1024).all()


def test_library_is_sm100a():
    V = _lib()
    log = open(os.path.join(os.path.dirname(V.LIB_PATH), "build.log")).read()
    assert "arch=compute_100a,code=sm_100a" in log
    assert "-lineinfo" in log
    np.zeros(1)


def test_plain_c_consumer(tmp_path):
    """include/qem.h compiles as pedantic C99 and the host-only entry points answer
    through it from a C program linked against libqem.so (no GPU, no Python between)."""
    V = _lib()
    import shutil

    import pytest

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path / "c_abi_host")
    libdir = os.path.dirname(V.LIB_PATH)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_host.c"),
                        "-L", libdir, "-lqem", f"-Wl,-rpath,{libdir}", "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.stdout, r.stderr)

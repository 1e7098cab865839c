"""The C-ABI library loads and exports every symbol include/*.h declares (no GPU needed)."""
import glob
import os
import re
import subprocess

import numpy as np

import oracle as O
from golden_io import frozen_tables as _frozen_tables, tables_sha as _sha

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
    assert V.abi() == "qem-pair-v2"
    assert V.status_string(V.QEM_ERR_MALFORMED) == "malformed stream"
    assert V.status_string(99) == "unknown status"


def test_frozen_tables_file_is_whole():
    """The golden file's tables hash to the digest it states, and have the shapes and
    sums spec S4 fixes (32 models, 256 pair symbols summing to 1024 states)."""
    digest, f, a, c = _frozen_tables()
    assert f.shape == (32, 256) and a.shape == (32,) and c.shape == (32, 16)
    assert (f.astype(np.int64).sum(axis=1) == 1024).all()
    assert _sha(f, a, c) == digest


def test_oracle_rebuild_hashes_to_frozen_tables():
    """The oracle rebuilds the models from spec S4 in double precision on this host;
    its result must hash to the frozen digest (a libm that moved one floor() fails here)."""
    digest, *_ = _frozen_tables()
    assert _sha(*O.models()) == digest


def test_library_tables_equal_frozen_tables():
    """The library's tables (compiled from its own frozen data) equal the golden file."""
    V = _lib()
    digest, f0, a0, c0 = _frozen_tables()
    f, a, c = V.model_tables()
    assert (f == f0).all() and (a == a0).all() and (c == c0).all()
    assert _sha(f, a, c) == digest


def test_library_frozen_data_is_its_generator_output(tmp_path):
    """model_tables.inc is what the library's generator writes on this host."""
    import shutil

    import pytest

    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no C++ compiler")
    csrc = os.path.join(ROOT, "virtual_imaging_b200", "csrc")
    exe = str(tmp_path / "gen")
    r = subprocess.run([cxx, "-O2", "-std=c++17", "-o", exe, os.path.join(csrc, "gen_model_tables.cpp")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([exe], capture_output=True, text=True, timeout=60).stdout
    assert out == open(os.path.join(csrc, "model_tables.inc")).read()


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

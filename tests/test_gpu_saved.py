"""The saved form (QGPUPAIR file): a resident written and reopened holds the
same bytes and answers queries exactly; a foreign ABI, a damaged header or a
truncated file is refused."""
import numpy as np
import pytest

import oracle as O
import virtual_imaging_b200 as V
import workloads as W
from qem_testlib import export_all, gpu_encode, image

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["c1", "c2", "s19"])
def test_save_load_roundtrip(tmp_path, name):
    w = W.workload(name)
    x = w.host_counts()
    valid = W.invalid_mask(w, 5) if name == "s19" else None
    res = gpu_encode(w, x, valid)
    path = str(tmp_path / f"{name}.qgpupair")
    res.save(path)
    back = V.Resident.load(path)
    a, b = res.info(), back.info()
    for k in ("scan_rows", "scan_cols", "det_rows", "det_cols", "dtype_bits", "n_valid", "n_blocks",
              "payload_bytes", "form_count", "out_bits_auto"):
        assert a[k] == b[k], k
    assert (back.valid() == (np.ones(w.n_pixels, np.uint8) if valid is None else valid)).all()
    for (g0, p0), (g1, p1) in zip(export_all(res, w.n_blocks), export_all(back, w.n_blocks)):
        assert (g0 == g1).all() and p0.size == p1.size and (p0 == p1).all()
    for mname, m in w.masks.items():
        assert (image(back, m, 1) == O.dense_masked_sum(x, m, valid)).all(), mname
    with open(path, "rb") as f:
        head = f.read(12 + 1024)
    assert head[:8] == b"QGPUPAIR"
    res.free()
    back.free()


def test_load_refuses_foreign_and_damaged_files(tmp_path):
    w = W.workload("c1")
    x = w.host_counts()
    res = gpu_encode(w, x)
    path = str(tmp_path / "c1.qgpupair")
    res.save(path)
    data = open(path, "rb").read()
    abi = V.abi().encode()
    assert abi in data[:4096]
    other = abi[:-1] + (b"9" if abi[-1:] != b"9" else b"8")       # same length, another ABI
    cases = {
        "abi": data.replace(abi, other, 1),
        "magic": b"QGPUPAIX" + data[8:],
        "truncated": data[: len(data) // 2],
        "geometry": data.replace(b'"det_rows":32', b'"det_rows":33', 1),
    }
    for label, blob in cases.items():
        p = str(tmp_path / f"bad_{label}.qgpupair")
        open(p, "wb").write(blob)
        with pytest.raises(V.QemError):
            V.Resident.load(p)
    with pytest.raises(V.QemError):
        V.Resident.load(str(tmp_path / "missing.qgpupair"))
    part = V.Resident.create((w.scan_rows, w.scan_cols), (w.det_rows, w.det_cols), 8)
    with pytest.raises(V.QemError):                     # not complete
        part.save(str(tmp_path / "part.qgpupair"))
    part.free()
    res.free()


def test_saved_form_then_index(tmp_path):
    w = W.workload("c2")
    x = w.host_counts()
    res = gpu_encode(w, x)
    path = str(tmp_path / "c2.qgpupair")
    res.save(path)
    res.free()
    back = V.Resident.load(path)
    back.build_index((w.det_rows // 2, w.det_cols // 2))
    for mname, m in w.masks.items():
        assert (image(back, m, 2) == O.dense_masked_sum(x, m, None, 2)).all(), mname
    back.free()

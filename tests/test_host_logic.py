"""Host-side logic of the library that needs no GPU: the interaction index's
polar layout (page "Operation pipeline" step 3) and the saved form's header
checks (page "Contract": reopen refuses another ABI)."""
import json
import math
import struct

import numpy as np
import pytest

import virtual_imaging_b200 as V


def _spread(a):
    a = np.sort(np.mod(a, 2 * math.pi))
    gaps = np.diff(np.concatenate([a, a[:1] + 2 * math.pi]))
    return 2 * math.pi - gaps.max()


@pytest.mark.parametrize("rows,cols,centre,invalid", [
    (192, 192, (96, 96), 0),
    (192, 192, (95.5, 95.5), 0),
    (96, 96, (48, 48), 37),
    (17, 17, (8, 8), 0),
    (257, 257, (100.5, 130.25), 11),
    (1, 70, (0, 35), 0),
])
def test_polar_layout_properties(rows, cols, centre, invalid):
    P = rows * cols
    valid = np.ones(P, np.uint8)
    if invalid:
        valid[np.random.default_rng(invalid).choice(P, invalid, replace=False)] = 0
    slots, roots = V.polar_layout(rows, cols, centre, valid)
    real = slots[slots < P]
    # every valid pixel exactly once, padding only at the end of a leaf
    assert np.array_equal(np.sort(real), np.nonzero(valid)[0])
    for leaf in slots:
        pad = leaf >= P
        assert not pad[: (~pad).sum()].any()
        assert (~pad).sum() >= 1
    assert roots[0] == 0 and roots[-1] == slots.shape[0]
    assert (np.diff(roots) >= 1).all() and (np.diff(roots) <= 16).all()
    cr, cc = centre
    sector = 2 * math.pi / 16 + 1e-9
    for i in range(len(roots) - 1):
        grp = slots[roots[i]:roots[i + 1]]
        px = grp[grp < P]
        dr, dc = px // cols - cr, px % cols - cc
        keep = (dr != 0) | (dc != 0)
        assert keep.sum() == 0 or _spread(np.arctan2(dr[keep], dc[keep])) <= sector
        # outward inside a root (leaves in order, pixels in order)
        d2 = dr * dr + dc * dc
        assert (np.diff(d2) >= 0).all()
    # at most 16 partial leaves (one per sector)
    assert ((slots >= P).any(axis=1)).sum() <= 16
    # a disk about the centre covers whole leaves except near its edge
    if rows == 192 and centre == (96, 96):
        rr, cc_ = np.divmod(np.arange(P), cols)
        disk = (rr - 96) ** 2 + (cc_ - 96) ** 2 <= 30 * 30
        full = [l for l in range(slots.shape[0]) if disk[slots[l][slots[l] < P]].all()]
        covered = sum(int((slots[l] < P).sum()) for l in full)
        assert covered >= 0.7 * disk.sum()


def test_polar_layout_rejects_bad_arguments():
    for args in ((0, 5, (0, 0)), (5, 0, (0, 0)), (5, 5, (float("nan"), 0)), (4097, 4097, (0, 0))):
        with pytest.raises(V.QemError):
            V.polar_layout(*args)


def _saved_file(path, header, body=b""):
    js = json.dumps(header, separators=(",", ":")).encode()
    with open(path, "wb") as f:
        f.write(b"QGPUPAIR" + struct.pack("<I", len(js)) + js)
        f.write(b"\0" * (4096 - 12 - len(js)))
        f.write(body)


def test_saved_form_header_checks(tmp_path):
    good = {"format": "qem-pair-resident-v1", "abi": V.abi(), "scan_rows": 16, "scan_cols": 32, "det_rows": 4,
            "det_cols": 4, "dtype_bits": 8, "n_blocks": 1, "valid_off": 4096, "valid_bytes": 16,
            "groups_off": 8192, "groups_bytes": 68, "block_off_off": 12288, "payload_off": 16384,
            "payload_bytes": 0}
    cases = {
        "abi": dict(good, abi=V.abi() + "x"),
        "format": dict(good, format="other"),
        "geometry": dict(good, valid_bytes=15),
        "blocks": dict(good, scan_rows=32),
        "groups": dict(good, groups_bytes=64),
    }
    for name, hdr in cases.items():
        p = str(tmp_path / f"{name}.qgpupair")
        _saved_file(p, hdr, b"\0" * 20000)
        with pytest.raises(V.QemError) as e:
            V.Resident.load(p)
        assert e.value.code == V.QEM_ERR_ARG, name
    # right header, arrays missing (truncated after the header)
    p = str(tmp_path / "short.qgpupair")
    _saved_file(p, good)
    with pytest.raises(V.QemError) as e:
        V.Resident.load(p)
    assert e.value.code == V.QEM_ERR_ARG
    p = str(tmp_path / "magic.qgpupair")
    with open(p, "wb") as f:
        f.write(b"NOTQGPU!" + b"\0" * 100)
    with pytest.raises(V.QemError):
        V.Resident.load(p)

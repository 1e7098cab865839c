"""Scan-range decode and single frames (page "Paired-count resident layout":
"Source map" decode_range / frame kernels; "Contract" queued queries,
session.frame(..., wait=False); "Verification": every frame compared with
direct sums) against the oracle's plain definition, on GPU-encoded and
oracle-encoded residents, with invalid pixels, ranges crossing block
boundaries, queued calls and malformed streams."""
import numpy as np
import pytest
import torch

import oracle as O
import virtual_imaging_b200 as V
import workloads as W
from qem_testlib import device, gpu_encode, oracle_resident, to_dev

pytestmark = pytest.mark.gpu


def _ranges(n_scans, rng):
    out = [(0, 1), (1, 1), (31, 1), (32, 1), (255, 1), (510, 1), (511, 1), (n_scans - 1, 1), (0, 32),
           (5, 27), (480, 32), (0, 512), (n_scans - 7, 7), (0, n_scans)]
    if n_scans > 512:
        out += [(512, 1), (500, 30), (511, 2), (300, 700), (n_scans - 600, 600)]
    for _ in range(6):
        a = int(rng.integers(0, n_scans))
        out.append((a, int(rng.integers(1, n_scans - a + 1))))
    return out


@pytest.mark.parametrize("name", ["c1", "c2", "s17", "u19"])
@pytest.mark.parametrize("source", ["gpu", "oracle"])
def test_decode_range_equals_counts(name, source):
    device()
    w = W.workload(name)
    x = w.host_counts()
    valid = W.invalid_mask(w, 3) if name.startswith("s") else None
    res = gpu_encode(w, x, valid) if source == "gpu" else oracle_resident(w, O.encode(x, w.dtype_bits), valid)
    rng = np.random.default_rng(7)
    for first, n in _ranges(w.n_scans, rng):
        got = res.decode_range(first, n).cpu().numpy()
        want = O.dense_decode_range(x, first, n, valid)
        assert got.dtype == want.dtype and (got == want).all(), (name, source, first, n)
    # a frame is one scan in detector shape
    f = res.frame(w.n_scans // 2).cpu().numpy()
    assert f.shape == (w.det_rows, w.det_cols)
    assert (f.reshape(-1) == O.dense_decode_range(x, w.n_scans // 2, 1, valid)[0]).all()
    res.free()


def test_decode_range_queued_and_args():
    dev = device()
    w = W.workload("c2")
    x = w.host_counts()
    res = gpu_encode(w, x)
    outs = []
    for s in (0, 700, 4095):
        o = torch.empty((3, w.n_pixels), dtype=torch.uint16, device=dev)
        res.decode_range(s if s + 3 <= w.n_scans else s - 2, 3, out=o, wait=False)
        outs.append((s if s + 3 <= w.n_scans else s - 2, o))
    res.finish()
    for s, o in outs:
        assert (o.cpu().numpy() == x[s:s + 3]).all()
    # zero scans is a no-op; ranges past the end are refused
    assert res.decode_range(10, 0).shape == (0, w.n_pixels)
    for first, n in [(-1, 1), (w.n_scans, 1), (w.n_scans - 1, 2)]:
        with pytest.raises(V.QemError) as e:
            res.decode_range(first, n)
        assert e.value.code == V.QEM_ERR_ARG
    res.free()


def test_decode_range_malformed_stream():
    """A reserved header bit in a block the range touches raises; a range elsewhere is exact."""
    device()
    w = W.workload("c2")
    x = w.host_counts()
    enc = O.encode(x, 16)
    p = int(np.nonzero(w.masks["bf"])[0][3])
    g = enc.groups[2]
    gi, j = divmod(p, 32)
    ends = [0] + [(int(g[gi, 1 + t // 2]) >> (16 * (t & 1))) & 0xFFFF for t in range(32)]
    start = int(g[gi, 0]) + ends[j]
    bad = [pl.copy() for pl in enc.payloads]
    bad[2][start + 1] |= 0x40                                # reserved header bit 14 in block 2
    res = oracle_resident(w, enc, payloads=bad)
    with pytest.raises(V.QemError) as e:
        res.decode_range(2 * 512 + 17, 1)
    assert e.value.code == V.QEM_ERR_MALFORMED
    with pytest.raises(V.QemError):
        res.decode_range(1000, 100)                          # crosses into block 2
    assert (res.decode_range(0, 1000).cpu().numpy() == x[:1000]).all()
    assert (res.decode_range(3 * 512, 512).cpu().numpy() == x[1536:2048]).all()
    res.free()

"""Masked moments (fused CoM / DPC numerators and denominator) through the C ABI,
against the oracle's plain definition, exactly."""
import numpy as np
import pytest
import torch

import oracle as O
import virtual_imaging_b200 as V
import workloads as W
from qem_testlib import gpu_encode, oracle_resident, to_dev

pytestmark = pytest.mark.gpu


def com_weights(w):
    rr, cc = np.divmod(np.arange(w.n_pixels), w.det_cols)
    return np.stack([rr - w.det_rows // 2, cc - w.det_cols // 2]).astype(np.int32)


def dpc_weights(w):
    rr, cc = np.divmod(np.arange(w.n_pixels), w.det_cols)
    return np.stack([np.where(rr < w.det_rows // 2, -1, 1), np.where(cc < w.det_cols // 2, -1, 1)]).astype(np.int32)


def moments(res, mask, weights, k=1):
    out = res.masked_moments(to_dev(mask.astype(np.uint8)), to_dev(weights), block_stride=k)
    return out.cpu().numpy()


@pytest.mark.parametrize("name", ["c1", "c2", "s19", "s257"])
@pytest.mark.parametrize("source", ["gpu", "oracle"])
def test_moments_match_oracle(name, source):
    w = W.workload(name)
    x = w.host_counts()
    valid = W.invalid_mask(w, 5) if name == "s19" else None
    if source == "gpu":
        res = gpu_encode(w, x, valid)
    else:
        res = oracle_resident(w, O.encode(x, w.dtype_bits), valid)
    masks = dict(w.masks)
    masks["full"] = np.ones(w.n_pixels, np.uint8)
    for wname, wt in (("com", com_weights(w)), ("dpc", dpc_weights(w))):
        for mname, m in masks.items():
            for k in (1, 3):
                got = moments(res, m, wt, k)
                want = O.dense_masked_moments(x, m, wt, valid, k)
                assert got.shape == want.shape
                assert (got == want).all(), (name, wname, mname, k)
    res.free()


def test_moments_extreme_weights_and_errors():
    w = W.workload("c2")                      # uint16 with full-scale (65535) hot pixels
    x = w.host_counts()
    res = gpu_encode(w, x)
    big = np.full((2, w.n_pixels), 262143, np.int32)
    big[1] = -262143
    full = np.ones(w.n_pixels, np.uint8)
    assert (moments(res, full, big) == O.dense_masked_moments(x, full, big)).all()
    empty = np.zeros(w.n_pixels, np.uint8)
    assert not moments(res, empty, big).any()
    m = to_dev(full)
    wt = to_dev(big)
    with pytest.raises(V.QemError):
        res.masked_moments(m, wt, block_stride=0)
    bad = torch.empty((3 * w.n_blocks * 512 + 1,), dtype=torch.int32, device="cuda")[1:]
    with pytest.raises(V.QemError):           # 4 bytes off an 8-byte boundary
        res.masked_moments(m, wt, out=bad)
    res.free()
    # a malformed stream surfaces as MalformedStream
    enc = O.encode(x, 16)
    bad_groups = [g.copy() for g in enc.groups]
    bad_groups[0][3, 0] = np.uint32(enc.payloads[0].size)
    res = oracle_resident(w, enc, groups=bad_groups)
    with pytest.raises(V.MalformedStream):
        res.masked_moments(m, wt)
    res.free()


def test_moments_leave_delta_baselines_alone():
    w = W.workload("c2")
    x = w.host_counts()
    res = gpu_encode(w, x)
    m0 = to_dev(w.drag[0])
    res.masked_sum(m0)
    moments(res, w.masks["adf"], com_weights(w))
    got = res.masked_sum_delta(to_dev(w.drag[1]))
    assert (V.as_unsigned(got).astype(np.uint64) == O.dense_masked_sum(x, w.drag[1])).all()
    res.free()

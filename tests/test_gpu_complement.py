"""Masked sums by complement (page "Backend Optimization Matrix", CUDA checkpoint
rows: dense dark field as a cached total minus the complement): the image equals
the plain masked sum for dense and sparse masks, strides, invalid pixels and both
output widths; only the complement's streams are decoded once the total is cached;
the result is a delta baseline like any full query; a malformed stream raises."""
import math

import numpy as np
import pytest

import oracle as O
import virtual_imaging_b200 as V
import workloads as W
from qem_testlib import gpu_encode, image, oracle_resident, to_dev

pytestmark = pytest.mark.gpu


def _complement(res, m, k=1, out_bits=0):
    return V.as_unsigned(res.masked_sum_complement(to_dev(m.astype(np.uint8)), block_stride=k,
                                                   out_bits=out_bits)).astype(np.uint64)


@pytest.mark.parametrize("name", ["c1", "c2", "s17", "u19"])
def test_complement_equals_masked_sum(name):
    w = W.workload(name)
    x = w.host_counts()
    valid = W.invalid_mask(w, 5) if name.startswith("s") else None
    res = gpu_encode(w, x, valid)
    P = w.n_pixels
    rng = np.random.default_rng(9)
    masks = [(1 - w.masks["bf"]).astype(np.uint8), np.ones(P, np.uint8), np.zeros(P, np.uint8),
             (rng.random(P) < 0.9).astype(np.uint8), w.masks["bf"]]
    for m in masks:
        for k in (1, 2, 3):
            got = _complement(res, m, k)
            assert got.shape == (math.ceil(w.n_blocks / k), 512)
            assert (got == O.dense_masked_sum(x, m, valid, k)).all(), (name, k)
        assert (_complement(res, m, 1, 64) == O.dense_masked_sum(x, m, valid, 1)).all()
    res.free()


def test_complement_decodes_only_the_complement_and_sets_the_baseline():
    w = W.workload("c2")
    x = w.host_counts()
    res = gpu_encode(w, x)
    df = (1 - w.masks["bf"]).astype(np.uint8)
    _complement(res, df)                                    # builds the cached total
    res.counters()
    got = _complement(res, df, 2)
    rows, streams = res.counters()
    assert streams == int(w.masks["bf"].sum()) * math.ceil(w.n_blocks / 2)
    assert (got == O.dense_masked_sum(x, df, None, 2)).all()
    # the complement result is the stride's baseline: a delta continues from it
    m2 = df.copy()
    m2[np.nonzero(df)[0][:40]] = 0
    d = image(res, m2, 2, delta=True)
    assert (d == O.dense_masked_sum(x, m2, None, 2)).all()
    # an index does not change the complement route's result
    res.build_index((48, 48))
    assert (_complement(res, df) == O.dense_masked_sum(x, df)).all()
    res.free()


def _extent(g, p):
    gi, j = divmod(p, 32)
    e = lambda t: (int(g[gi, 1 + t // 2]) >> (16 * (t & 1))) & 0xFFFF
    return int(g[gi, 0]) + (e(j - 1) if j else 0), int(g[gi, 0]) + e(j)


def test_complement_malformed_stream():
    """A reserved header bit in a stream of the complement raises (the total is not kept);
    the same query on the intact resident is exact."""
    w = W.workload("c1")
    x = w.host_counts()
    enc = O.encode(x, 8)
    g = enc.groups[0]
    df = (1 - w.masks["bf"]).astype(np.uint8)
    p = next(int(q) for q in np.nonzero(df)[0] if _extent(g, int(q))[1] - _extent(g, int(q))[0] >= 2)
    start, _ = _extent(g, p)
    bad = enc.payloads[0].copy()
    bad[start + 1] |= 0x20                                   # reserved header bit 13
    res = oracle_resident(w, enc, payloads=[bad])
    with pytest.raises(V.MalformedStream):
        _complement(res, df)
    res.free()
    res = oracle_resident(w, enc)
    assert (_complement(res, df) == O.dense_masked_sum(x, df)).all()
    res.free()

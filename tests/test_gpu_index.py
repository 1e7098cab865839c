"""The interaction index (page "Operation pipeline" steps 3-4): queries that
take whole radial-angular pixel groups from the index and decode only the
remaining pixels give exactly the oracle's direct sums; the polar layout
covers every valid pixel once; masks made of whole groups decode nothing."""
import math

import numpy as np
import pytest
import torch

import oracle as O
import virtual_imaging_b200 as V
import workloads as W
from qem_testlib import gpu_encode, image, oracle_resident, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def data():
    cache = {}

    def get(name):
        if name not in cache:
            w = W.workload(name)
            x = w.host_counts()
            cache[name] = (w, x, O.encode(x, w.dtype_bits))
        return cache[name]

    return get


def centre(w):
    # the masks of these workloads are centred on (n // 2, n // 2)
    return (w.det_rows // 2, w.det_cols // 2)


def _spread(a):
    """Smallest arc (radians) holding all the angles a."""
    a = np.sort(np.mod(a, 2 * math.pi))
    gaps = np.diff(np.concatenate([a, a[:1] + 2 * math.pi]))
    return 2 * math.pi - gaps.max()


def check_layout(res, w, valid=None):
    """The layout holds every valid pixel once; a leaf (and a root) lies in one
    22.5-degree sector about the centre; a leaf's pixels go outwards."""
    slots, roots = res.index_layout()
    P = w.n_pixels
    real = slots[slots < P]
    want = np.nonzero(np.ones(P, bool) if valid is None else valid)[0]
    assert np.array_equal(np.sort(real), want)
    assert roots[0] == 0 and roots[-1] == slots.shape[0]
    assert (np.diff(roots) >= 1).all() and (np.diff(roots) <= 16).all()
    cr, cc = centre(w)
    sector = 2 * math.pi / 16 + 1e-9

    def angles(px):
        dr, dc = px // w.det_cols - cr, px % w.det_cols - cc
        keep = (dr != 0) | (dc != 0)               # the centre pixel has no direction
        return np.arctan2(dr[keep], dc[keep]), dr * dr + dc * dc

    for l in range(slots.shape[0]):
        px = slots[l][slots[l] < P]
        assert px.size >= 1
        a, d2 = angles(px)
        assert a.size == 0 or _spread(a) <= sector, l
        assert (np.diff(d2) >= 0).all(), l
    for i in range(len(roots) - 1):
        blk = slots[roots[i]:roots[i + 1]]
        a, _ = angles(blk[blk < P])
        assert a.size == 0 or _spread(a) <= sector, i
    return slots, roots


@pytest.mark.parametrize("name", ["c1", "c2", "s17", "s257"])
@pytest.mark.parametrize("source", ["gpu", "oracle"])
def test_index_queries_match_oracle(data, name, source):
    w, x, enc = data(name)
    res = oracle_resident(w, enc) if source == "oracle" else gpu_encode(w, x)
    res.build_index(centre(w))
    info = res.info()
    assert info["index_leaves"] >= -(-w.n_pixels // 64)
    assert info["index_bytes"] > 0
    check_layout(res, w)
    for k in (1, 2, 3):
        for mname, m in w.masks.items():
            got = image(res, m, k)
            assert got.shape == (math.ceil(w.n_blocks / k), 512)
            assert (got == O.dense_masked_sum(x, m, None, k)).all(), (name, mname, k)
    full = np.ones(w.n_pixels, np.uint8)
    assert (image(res, full) == O.dense_masked_sum(x, full)).all()
    res.free()


def test_index_delta_chain_and_leaving_groups(data):
    w, x, enc = data("c2")
    res = gpu_encode(w, x)
    res.build_index(centre(w))
    img = image(res, w.drag[0], 1)
    for t in range(1, len(w.drag)):
        img = image(res, w.drag[t], 1, delta=True)
        assert (img == O.dense_masked_sum(x, w.drag[t])).all(), t
    # whole groups entering and leaving: full detector -> bright field -> annulus -> full
    seq = [np.ones(w.n_pixels, np.uint8), w.masks["bf"], w.masks["adf"], np.ones(w.n_pixels, np.uint8)]
    image(res, seq[0], 2)
    for m in seq[1:]:
        got = image(res, m, 2, delta=True)
        assert (got == O.dense_masked_sum(x, m, None, 2)).all()
    res.free()


def test_whole_groups_decode_nothing(data):
    w, x, enc = data("c2")
    res = gpu_encode(w, x)
    res.build_index(centre(w))
    slots, roots = check_layout(res, w)
    P = w.n_pixels
    # one leaf, one root, and a disk about the centre
    leaf = np.zeros(P, np.uint8)
    leaf[slots[5][slots[5] < P]] = 1
    root = np.zeros(P, np.uint8)
    for l in range(roots[1], roots[2]):
        root[slots[l][slots[l] < P]] = 1
    for m in (leaf, root):
        res.counters()
        got = image(res, m, 1)
        rows, streams = res.counters()
        assert streams == 0
        assert (got == O.dense_masked_sum(x, m)).all()
    res.counters()
    got = image(res, w.masks["bf"], 1)
    rows, streams = res.counters()
    assert (got == O.dense_masked_sum(x, w.masks["bf"])).all()
    assert streams < 0.75 * int(w.masks["bf"].sum()) * w.n_blocks
    res.free()


def test_index_with_invalid_pixels_uint64_and_rebuild(data):
    w, x, enc = data("s257")
    valid = W.invalid_mask(w, 7)
    res = gpu_encode(w, x, valid)
    res.build_index((100.5, 130.25))                 # off-centre: every query still exact
    check_layout_ok = res.index_layout()
    assert (np.sort(check_layout_ok[0][check_layout_ok[0] < w.n_pixels]) == np.nonzero(valid)[0]).all()
    for mname, m in w.masks.items():
        assert (image(res, m, 1) == O.dense_masked_sum(x, m, valid)).all(), mname
    full = np.ones(w.n_pixels, np.uint8)
    assert (image(res, full, 1, out_bits=64) == O.dense_masked_sum(x, full, valid)).all()
    res.build_index(centre(w))
    for mname, m in w.masks.items():
        assert (image(res, m, 2) == O.dense_masked_sum(x, m, valid, 2)).all(), mname
    res.drop_index()
    assert res.info()["index_leaves"] == 0
    assert (image(res, w.masks["bf"], 1) == O.dense_masked_sum(x, w.masks["bf"], valid)).all()
    res.free()


def _ends(g, gi):
    return [int((g[gi, 1 + j // 2] >> (16 * (j & 1))) & 0xFFFF) for j in range(32)]


def test_index_build_rejects_malformed(data):
    w, x, enc = data("c2")
    bad = [g.copy() for g in enc.groups]
    bad[0][3, 0] = np.uint32(enc.payloads[0].size)           # a group whose streams end past the payload
    res = oracle_resident(w, enc, groups=bad)
    with pytest.raises(V.MalformedStream):
        res.build_index(centre(w))
    assert res.info()["index_leaves"] == 0
    res.free()
    part = V.Resident.create((w.scan_rows, w.scan_cols), (w.det_rows, w.det_cols), 16)
    with pytest.raises(V.QemError):                          # not complete
        part.build_index()
    with pytest.raises(V.QemError):                          # no index to show
        part.index_layout()
    part.free()


def test_c4_index_full_size():
    """C4 (512 blocks, uint8) with the index about the bright-field centre:
    strides 1/4/16 and a drag agree with the non-indexed resident exactly,
    and sampled rows with the oracle."""
    from test_gpu_full import build, host_blocks

    w = W.workload("c4")
    res, buf = build(w)
    del buf
    torch.cuda.empty_cache()
    check = [0, 77, 300, 511]
    counts = host_blocks(w, check)
    plain = {}
    for name in ("bf", "adf"):
        for k in (1, 4, 16):
            plain[name, k] = image(res, w.masks[name], k)
    res.build_index((96, 96))
    for name in ("bf", "adf"):
        for k in (1, 4, 16):
            got = image(res, w.masks[name], k)
            assert (got == plain[name, k]).all(), (name, k)
        for b, xb in counts.items():
            assert (plain[name, 1][b] == O.dense_masked_sum(xb, w.masks[name])[0]).all()
    img = image(res, w.drag[0], 1)
    for t in range(1, 9):
        img = image(res, w.drag[t], 1, delta=True)
    for b, xb in counts.items():
        assert (img[b] == O.dense_masked_sum(xb, w.drag[8])[0]).all()
    res.free()


@pytest.mark.parametrize("name", ["c2", "c1"])
def test_planner_follows_its_weights(data, name):
    """The index plan's split follows the planner weights (a pair-by-pair stream 16,
    a light one 1, an item 2): the streams each query decodes are those the host
    rule gives (bench.decompose with the library's pixel classes), a leaf mostly in
    the mask is taken whole minus its other pixels, and the images stay exact."""
    import bench

    w, x, enc = data(name)
    res = gpu_encode(w, x)
    res.build_index(centre(w))
    slots, roots = res.index_layout()
    pclass = res.pixel_classes()
    P = w.n_pixels
    full = np.ones(P, np.uint8)
    rng = np.random.default_rng(3)
    masks = [w.masks["bf"], w.masks["adf"], full, (rng.random(P) < 0.8).astype(np.uint8)]
    took_complement = False
    for m in masks:
        res.counters()
        got = image(res, m, 1)
        rows, streams = res.counters()
        items, resid = bench.decompose(slots, roots, P, m.astype(bool), np.zeros(P, bool), pclass)
        assert (got == O.dense_masked_sum(x, m)).all()
        assert streams == int(resid.sum()) * w.n_blocks
        took_complement |= bool((resid & ~m.astype(bool)).any())
    assert took_complement
    res.free()

"""Edge cases of the CUDA path through the C ABI, against the oracle's direct sums."""
import numpy as np
import pytest
import torch

import oracle as O
import virtual_imaging_b200 as V
import workloads as W
from qem_testlib import gpu_encode, image, oracle_resident, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def c2():
    w = W.workload("c2")
    x = w.host_counts()
    return w, x, O.encode(x, 16)


def test_empty_mask_gives_zero_image(c2):
    w, x, enc = c2
    res = gpu_encode(w, x)
    res.counters()                                   # read and reset
    for k in (1, 3):
        img = image(res, np.zeros(w.n_pixels, np.uint8), k)
        assert img.shape == (-(-w.n_blocks // k), 512) and not img.any()
    rows, streams = res.counters()
    assert streams == 0
    res.free()


def test_stride_at_and_beyond_block_count(c2):
    w, x, enc = c2
    res = gpu_encode(w, x)
    for k in (w.n_blocks, w.n_blocks + 1, 1000):
        img = image(res, w.masks["bf"], k)
        assert img.shape == (1, 512)
        assert (img == O.dense_masked_sum(x, w.masks["bf"], None, k)).all()
    res.free()


def test_delta_with_unchanged_mask_and_toggles(c2):
    w, x, enc = c2
    res = gpu_encode(w, x)
    m = w.masks["bf"]
    full = image(res, m, 2)
    again = image(res, m, 2, delta=True)            # nothing listed: the baseline comes back
    assert (again == full).all()
    m2 = m.copy()
    m2[np.nonzero(m)[0][:5]] = 0                     # five pixels leave
    m2[np.nonzero(m == 0)[0][:7]] = 1                # seven enter
    d = image(res, m2, 2, delta=True)
    assert (d == O.dense_masked_sum(x, m2, None, 2)).all()
    back = image(res, m, 2, delta=True)              # and back
    assert (back == full).all()
    res.free()


def test_delta_with_forced_uint64(c2):
    w, x, enc = c2
    res = gpu_encode(w, x)
    a = image(res, w.drag[0], 1, out_bits=64)
    for t in range(1, 4):
        a = image(res, w.drag[t], 1, delta=True, out_bits=64)
        assert (a == O.dense_masked_sum(x, w.drag[t])).all()
    # switching width on a delta runs a full query of the new mask
    b = image(res, w.drag[4], 1, delta=True)
    assert (b == O.dense_masked_sum(x, w.drag[4])).all()
    res.free()


def test_strides_keep_separate_baselines(c2):
    w, x, enc = c2
    res = gpu_encode(w, x)
    image(res, w.drag[0], 1)
    image(res, w.drag[5], 3)
    d1 = image(res, w.drag[1], 1, delta=True)       # baseline of stride 1 is drag[0]
    d3 = image(res, w.drag[6], 3, delta=True)       # baseline of stride 3 is drag[5]
    assert (d1 == O.dense_masked_sum(x, w.drag[1], None, 1)).all()
    assert (d3 == O.dense_masked_sum(x, w.drag[6], None, 3)).all()
    res.free()


def test_invalid_only_mask_is_zero():
    w = W.workload("s19")
    x = w.host_counts()
    valid = W.invalid_mask(w, 5)
    res = gpu_encode(w, x, valid)
    img = image(res, (valid == 0).astype(np.uint8), 1)
    assert not img.any()
    res.free()


def test_zero_block_decode_and_argument_errors(c2):
    w, x, enc = c2
    res = gpu_encode(w, x)
    out = torch.empty((512, w.n_pixels), dtype=torch.uint16, device="cuda")
    res.decode_blocks(0, 0, out=out)                 # nothing to do
    with pytest.raises(V.QemError):
        res.decode_blocks(w.n_blocks - 1, 2, out=out)
    m = to_dev(w.masks["bf"])
    with pytest.raises(V.QemError):
        res.masked_sum(m, block_stride=0)
    good = torch.empty((w.n_blocks, 512), dtype=torch.int64, device="cuda")
    with pytest.raises(V.QemError):                  # the library itself rejects k = 0
        res.masked_sum(m, block_stride=0, out_bits=64, out=good)
    n = w.n_blocks * 512
    bad = torch.empty((n + 2,), dtype=torch.int64, device="cuda")[1:n + 1]   # 8 bytes off a 16-byte boundary
    with pytest.raises(V.QemError):
        res.masked_sum(m, out_bits=64, out=bad.view(w.n_blocks, 512))
    with pytest.raises(V.QemError):                  # 16 is not a width
        res.masked_sum(m, out_bits=16)
    # an output buffer narrower or shorter than ceil(B/k) x 512 values of the chosen
    # width is refused before the library could write past it
    narrow = torch.empty((w.n_blocks, 512), dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        res.masked_sum(m, out_bits=64, out=narrow)
    short = torch.empty((w.n_blocks - 1, 512), dtype=V.out_dtype(res.info()["out_bits_auto"]), device="cuda")
    with pytest.raises(ValueError):
        res.masked_sum_delta(m, out=short)
    with pytest.raises(ValueError):
        res.masked_sum_noalloc(m, short)
    res.free()
    part = V.Resident.create((w.scan_rows, w.scan_cols), (w.det_rows, w.det_cols), 16)
    part.append(to_dev(x[:512]), 1)
    with pytest.raises(V.QemError):                  # resident not complete
        part.masked_sum(m)
    part.free()


def _starts_ends(g):
    """Per-pixel [start, end) of one block's streams, from its group records."""
    G = g.shape[0]
    ends = np.ascontiguousarray(g[:, 1:]).view(np.uint16).reshape(G, 32).astype(np.int64)
    prev = np.concatenate([np.zeros((G, 1), np.int64), ends[:, :-1]], axis=1)
    base = g[:, :1].astype(np.int64)
    return (base + prev).reshape(-1), (base + ends).reshape(-1)


def test_decreasing_offsets_and_overlong_extent_rejected(c2):
    w, x, enc = c2
    g0 = enc.groups[0]
    a, z = _starts_ends(g0)
    base = np.repeat(g0[:, 0].astype(np.int64), 32)
    cand = [q for q in np.nonzero(w.masks["bf"])[0] if q % 32 and a[q] > base[q]]
    q = int(cand[len(cand) // 2])
    gi, j = divmod(q, 32)
    m = np.zeros(w.n_pixels, np.uint8)
    m[q] = 1
    # rel_end[j] one below rel_end[j-1]
    bad = [g.copy() for g in enc.groups]
    lower = int(a[q] - base[q] - 1)
    word = int(bad[0][gi, 1 + j // 2])
    sh = 16 * (j & 1)
    bad[0][gi, 1 + j // 2] = np.uint32((word & ~(0xFFFF << sh)) | (lower << sh))
    res = oracle_resident(w, enc, groups=bad)
    with pytest.raises(V.MalformedStream):
        image(res, m, 1)
    res.free()
    # a stream that ends beyond its block's payload
    bad = [g.copy() for g in enc.groups]
    bad[0][gi, 0] = np.uint32(enc.payloads[0].size)
    res = oracle_resident(w, enc, groups=bad)
    with pytest.raises(V.MalformedStream):
        image(res, m, 1)
    res.free()


def test_info_counts_match_oracle_forms(c2):
    w, x, enc = c2
    res = gpu_encode(w, x)
    info = res.info()
    forms = np.zeros(len(V.FORMS), np.int64)
    for b in range(w.n_blocks):
        p = enc.payloads[b]
        a, z = _starts_ends(enc.groups[b])
        a, z = a[:w.n_pixels], z[:w.n_pixels]
        code = np.where(z == a, 0, p[np.minimum(a, p.size - 1)] & 7)
        forms += np.bincount(code, minlength=len(V.FORMS))
    assert info["form_count"] == dict(zip(V.FORMS, forms.tolist()))
    assert info["payload_bytes"] == enc.payload_bytes()
    res.free()

"""GPU parity on the small workloads: the CUDA path (through the C ABI) against
the CPU oracle, element by element and byte by byte.

Covers: encoder bitstream identity (payload bytes and grouped offsets),
decode+reduce on oracle-encoded and GPU-encoded residents, block_stride k,
delta chains, uint64 promotion, invalid pixels, block decode, malformed
streams and delta invalidation, deferred (wait=False) status.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import virtual_imaging_b200 as V
import workloads as W
from qem_testlib import export_all, gpu_encode, image, oracle_resident, to_dev

pytestmark = pytest.mark.gpu

SMALL = ["c1", "c2", "s17", "s19", "s257", "u19"]


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


@pytest.mark.parametrize("name", SMALL)
def test_encoder_bitstream_identical(data, name):
    w, x, enc = data(name)
    res = gpu_encode(w, x)
    for b, (g, p) in enumerate(export_all(res, w.n_blocks)):
        assert (g == enc.groups[b]).all(), (name, b)
        assert p.size == enc.payloads[b].size and (p == enc.payloads[b]).all(), (name, b)
    info = res.info()
    assert info["payload_bytes"] == enc.payload_bytes()
    assert sum(info["form_count"].values()) == w.n_blocks * w.n_pixels
    res.free()


@pytest.mark.parametrize("name", SMALL)
@pytest.mark.parametrize("source", ["oracle", "gpu"])
def test_masked_sum_matches(data, name, source):
    w, x, enc = data(name)
    res = oracle_resident(w, enc) if source == "oracle" else gpu_encode(w, x)
    for k in (1, 2, 3):
        for mname, m in w.masks.items():
            want = O.dense_masked_sum(x, m, None, k)
            got = image(res, m, k)
            assert got.shape == (math.ceil(w.n_blocks / k), 512)
            assert (got == want).all(), (name, mname, k)
    # the full-detector image is all pixels
    full = np.ones(w.n_pixels, np.uint8)
    assert (image(res, full) == O.dense_masked_sum(x, full)).all()
    res.free()


@pytest.mark.parametrize("name", SMALL)
def test_decode_blocks_roundtrip(data, name):
    w, x, enc = data(name)
    res = gpu_encode(w, x)
    out = res.decode_blocks(0, w.n_blocks)
    assert (out.cpu().numpy() == x).all()
    if w.n_blocks > 1:
        part = res.decode_blocks(w.n_blocks - 1, 1)
        assert (part.cpu().numpy() == x[-512:]).all()
    res.free()


@pytest.mark.parametrize("name", ["c2", "u19"])
def test_delta_chain(data, name):
    w, x, enc = data(name)
    res = gpu_encode(w, x)
    for k in (1, 3):
        img = image(res, w.drag[0], k)
        assert (img == O.dense_masked_sum(x, w.drag[0], None, k)).all()
        for t in range(1, len(w.drag)):
            img = image(res, w.drag[t], k, delta=True)
            assert (img == O.dense_masked_sum(x, w.drag[t], None, k)).all(), (k, t)
    res.free()


def test_invalid_pixels(data):
    w, x, enc = data("s19")
    valid = W.invalid_mask(w, 3)
    res = gpu_encode(w, x, valid)
    for mname, m in w.masks.items():
        assert (image(res, m, 1) == O.dense_masked_sum(x, m, valid, 1)).all(), mname
    frames = res.decode_blocks(0, w.n_blocks).cpu().numpy()
    assert (frames == O.dense_decode_blocks(x, 0, w.n_blocks, valid)).all()
    assert res.info()["n_valid"] == w.n_pixels - 3
    res.free()


def test_uint64_promotion_257():
    """Page "Contract": uint64 when a full-detector sum could exceed 2**32."""
    w = W.workload("s257")
    P = w.n_pixels
    x = np.full((512, P), 65535, np.uint16)
    x[::7, ::3] = 65534
    res = gpu_encode(w, x)
    assert res.info()["out_bits_auto"] == 64
    img = res.masked_sum(to_dev(np.ones(P, np.uint8)))
    assert img.dtype == torch.int64
    got = V.as_unsigned(img)[0]
    closed = P * 65535 - np.array([len(range(0, P, 3)) if i % 7 == 0 else 0 for i in range(512)])
    assert (got == closed.astype(np.uint64)).all()
    assert int(got.max()) > 2 ** 32
    with pytest.raises(V.QemError):
        res.masked_sum(to_dev(np.ones(P, np.uint8)), out_bits=32)
    res.free()


def test_forced_uint64_and_auto_uint32(data):
    w, x, enc = data("c2")
    res = gpu_encode(w, x)
    assert res.info()["out_bits_auto"] == 32
    full = np.ones(w.n_pixels, np.uint8)
    a = image(res, full, 1, out_bits=64)
    b = image(res, full, 1)
    assert (a == b).all() and (a == O.dense_masked_sum(x, full)).all()
    res.free()


def test_stride_counters(data):
    w, x, enc = data("c2")
    res = gpu_encode(w, x)
    res.counters()
    for k in (1, 2, 3, 5, 8, 9):
        image(res, w.masks["bf"], k)
        rows, streams = res.counters()
        assert rows == math.ceil(w.n_blocks / k)
        assert streams == rows * int(w.masks["bf"].sum())
    res.free()


def _corrupt_reserved(enc, b, p_idx):
    g = enc.groups[b]
    gi, j = divmod(p_idx, 32)
    e = lambda j: int((g[gi, 1 + j // 2] >> (16 * (j & 1))) & 0xFFFF)
    a = int(g[gi, 0]) + (e(j - 1) if j else 0)
    pay = [p.copy() for p in enc.payloads]
    pay[b][a + 1] |= 0x80
    return pay


def test_malformed_reserved_bit_and_taint(data):
    w, x, enc = data("c2")
    q = int(np.nonzero(w.masks["bf"])[0][5])
    pay = _corrupt_reserved(enc, 1, q)
    res = oracle_resident(w, enc, payloads=pay)
    # the oracle agrees it is malformed
    with pytest.raises(O.MalformedStream):
        O.block_masked_sum(enc.groups[1], pay[1], 16, w.n_pixels, np.array([q]), np.array([1]))
    # stride 2 touches blocks 0,2,4,6 only: no error
    assert (image(res, w.masks["bf"], 2) == O.dense_masked_sum(x, w.masks["bf"], None, 2)).all()
    # stride 1 touches block 1: the query raises and taints the stride-1 baseline
    with pytest.raises(V.MalformedStream):
        image(res, w.masks["bf"], 1)
    with pytest.raises(V.TaintedBaseline):
        image(res, w.masks["adf"], 1, delta=True)
    # a full query with a mask that avoids the stream clears the taint
    m = w.masks["adf"]
    assert (image(res, m, 1) == O.dense_masked_sum(x, m, None, 1)).all()
    d = image(res, w.masks["adf"] | (np.arange(w.n_pixels) == 0).astype(np.uint8), 1, delta=True)
    assert (d == O.dense_masked_sum(x, w.masks["adf"] | (np.arange(w.n_pixels) == 0), None, 1)).all()
    # block decode of the bad block raises too
    with pytest.raises(V.MalformedStream):
        res.decode_blocks(1, 1)
    res.free()


def test_malformed_shortened_extent(data):
    """Page "Verification": a shortened stream extent is rejected."""
    w, x, enc = data("s17")
    for form in (1, 2, 3, 4):
        for b in range(w.n_blocks):
            g, pay = enc.groups[b], enc.payloads[b]
            found = None
            for q in range(w.n_pixels):
                gi, j = divmod(q, 32)
                e = lambda jj: int((g[gi, 1 + jj // 2] >> (16 * (jj & 1))) & 0xFFFF)
                a = int(g[gi, 0]) + (e(j - 1) if j else 0)
                if e(j) > (e(j - 1) if j else 0) and (pay[a] & 7) == form:
                    found = (q, gi, j)
                    break
            if found:
                break
        if not found:
            continue
        q, gi, j = found
        bad = [gg.copy() for gg in enc.groups]
        bad[b][gi, 1 + j // 2] = np.uint32(int(bad[b][gi, 1 + j // 2]) - (1 << (16 * (j & 1))))
        res = oracle_resident(w, enc, groups=bad)
        m = np.zeros(w.n_pixels, np.uint8)
        m[q] = 1
        with pytest.raises(V.MalformedStream):
            image(res, m, 1)
        res.free()


def test_malformed_flipped_bits_match_oracle(data):
    """Every single-bit flip in a paired stream: GPU and oracle agree on error/no-error and value."""
    w, x, enc = data("c1")
    g, pay = enc.groups[0], enc.payloads[0]
    bf = np.nonzero(w.masks["bf"])[0]
    q = int(bf[3])
    gi, j = divmod(q, 32)
    e = lambda jj: int((g[gi, 1 + jj // 2] >> (16 * (jj & 1))) & 0xFFFF)
    a, z = int(g[gi, 0]) + (e(j - 1) if j else 0), int(g[gi, 0]) + e(j)
    assert pay[a] & 7 == 3
    m = np.zeros(w.n_pixels, np.uint8)
    m[q] = 1
    for pos in range(a, z, max(1, (z - a) // 12)):
        for bit in (0, 3, 7):
            bad = pay.copy()
            bad[pos] ^= 1 << bit
            try:
                want = O.block_masked_sum(g, bad, 8, w.n_pixels, np.array([q]), np.array([1]))
            except O.MalformedStream:
                want = None
            res = oracle_resident(w, enc, payloads=[bad])
            if want is None:
                with pytest.raises(V.MalformedStream):
                    image(res, m, 1)
            else:
                assert (image(res, m, 1)[0] == want.astype(np.uint64)).all()
            res.free()


def test_async_queries_and_finish(data):
    w, x, enc = data("c2")
    res = gpu_encode(w, x)
    outs = []
    for mname in ("bf", "adf"):
        for k in (1, 2):
            outs.append((mname, k, res.masked_sum(to_dev(w.masks[mname]), block_stride=k, wait=False)))
    res.finish()
    for mname, k, o in outs:
        assert (V.as_unsigned(o).astype(np.uint64) == O.dense_masked_sum(x, w.masks[mname], None, k)).all()
    res.free()


def test_append_in_pieces(data):
    w, x, enc = data("c2")
    res = V.Resident.create((w.scan_rows, w.scan_cols), (w.det_rows, w.det_cols), w.dtype_bits)
    xd = to_dev(x)
    res.append(xd[: 3 * 512], 3)
    res.append(xd[3 * 512: 4 * 512], 1)
    res.append(xd[4 * 512:], 4)
    for b, (g, p) in enumerate(export_all(res, w.n_blocks)):
        assert (g == enc.groups[b]).all() and (p == enc.payloads[b]).all()
    with pytest.raises(V.QemError):
        res.append(xd[:512], 1)
    res.free()


def test_library_tables_equal_oracle():
    f, a, c = V.model_tables()
    f2, a2, c2 = O.models()
    assert (f == f2).all() and (a == a2).all() and (c == c2).all()


def test_uint8_warps_with_base_and_raw_bits():
    """uint8 pixels of the two-state models with a base (every count at least 4) or raw
    low bits (one count of 16 or more) sit in the same 32-pixel groups as plain ones and
    run-decoded ones; full queries, strides and delta chains (whose decode adds the base
    and the raw bits after the table steps) match the plain sums, and the bitstreams the
    oracle's byte for byte."""
    rng = np.random.default_rng(77)
    det, scans = 17, 1024
    P = det * det
    lam = rng.uniform(0.5, 4.0, size=P)
    kind = rng.integers(0, 4, size=P)                     # 0 plain, 1 base, 2 raw bits, 3 low dose
    lam[kind == 3] = 0.01
    x = rng.poisson(np.broadcast_to(lam, (scans, P))).astype(np.int64)
    x[:, kind == 1] += 4
    rows = rng.integers(0, scans, size=(kind == 2).sum())
    x[rows, np.nonzero(kind == 2)[0]] = rng.integers(16, 120, size=rows.size)
    x = np.minimum(x, 255).astype(np.uint8)
    w = W.Workload("mix8", scans // 32, 32, det, det, 8, 0, "host")
    hdrs = [O.stream_header(O.encode_stream(x[:512, p], 1)) for p in range(P)]
    paired = [h for h in hdrs if h is not None and h[0] == 3]
    assert any(h[3] for h in paired) and any(h[2] for h in paired) and any(h[1] >= 8 and not h[2] and not h[3] for h in paired)
    res = gpu_encode(w, x)
    g, pay = res.export_block(1)
    og, op = O.encode_block(x[512:], 8)
    assert (g == og).all() and (pay == op).all()
    drag = [W.disk(det, det, 8, 3 + t, 4) for t in range(11)]
    for k in (1, 2):
        for m in (np.ones(P, np.uint8), W.disk(det, det, 8, 8, 5)):
            assert (image(res, m, k) == O.dense_masked_sum(x, m, None, k)).all()
        img = image(res, drag[0], k)
        for t in range(1, len(drag)):
            img = image(res, drag[t], k, delta=True)
            assert (img == O.dense_masked_sum(x, drag[t], None, k)).all(), (k, t)
    res.free()


def _raw_pixel(rng, scans, shift, base):
    """Counts of one uint8 pixel whose streams carry `shift` raw low bits (spec S3): a
    lambda = 3 pixel plus `base`, with spikes that set the span of every block."""
    v = rng.poisson(3.0, size=scans) + base
    span_lo, span_hi = 1 << (shift + 3), (1 << (shift + 4)) - 1
    for b0 in range(0, scans, 512):
        at = rng.choice(np.arange(b0, b0 + 512), size=3, replace=False)
        v[at] = base + rng.integers(span_lo, min(span_hi, 255 - base) + 1, size=3)
    return np.minimum(v, 255)


def test_uint8_delta_single_raw_lane():
    """Deltas whose 32-lane tiles hold exactly one stream with raw low bits (the whole
    warp reads that lane's low bits) or two (each lane reads its own), entering and
    leaving, with shifts 1-3 and with bases: every image equals the oracle's dense sum."""
    rng = np.random.default_rng(91)
    det, scans = 32, 1024
    P = det * det
    x = rng.poisson(3.0, size=(scans, P)).astype(np.int64)
    raw = [40, 77, 131, 250, 301, 402]
    spec = [(1, 0), (2, 0), (3, 5), (3, 0), (1, 9), (2, 3)]      # (shift, base)
    for p, (sh, base) in zip(raw, spec):
        x[:, p] = _raw_pixel(rng, scans, sh, base)
    x = np.minimum(x, 255).astype(np.uint8)
    for p, (sh, base) in zip(raw, spec):
        for b0 in (0, 512):
            h = O.stream_header(O.encode_stream(x[b0:b0 + 512, p], 1))
            assert h[0] == 3 and h[2] == sh and h[1] >= 8, (p, h)
    w = W.Workload("raw1", scans // 32, 32, det, det, 8, 0, "host")
    res = gpu_encode(w, x)
    plain = [p for p in range(500, 1024) if p not in raw]
    m = np.zeros(P, np.uint8)
    m[plain[:200]] = 1
    steps = []
    m1 = m.copy(); m1[[raw[0]] + plain[200:210]] = 1; steps.append(m1)            # one raw lane enters
    m2 = m1.copy(); m2[[raw[1], raw[2]] + plain[210:215]] = 1; steps.append(m2)   # two raw lanes enter
    m3 = m2.copy(); m3[[raw[0]] + plain[:3]] = 0; steps.append(m3)                # one raw lane leaves
    m4 = m3.copy(); m4[raw[1]] = 0; m4[raw[3]] = 1; steps.append(m4)               # one leaves, one enters
    m5 = m4.copy(); m5[raw[2]] = 0; steps.append(m5)                               # a raw lane alone
    m6 = m5.copy(); m6[[raw[4], raw[5]]] = 1; m6[plain[100:140]] = 0; steps.append(m6)
    m7 = m6.copy(); m7[raw[5]] = 0; m7[plain[140:141]] = 0; steps.append(m7)
    for k in (1, 2):
        img = image(res, m, k)
        assert (img == O.dense_masked_sum(x, m, None, k)).all()
        for t, mt in enumerate(steps):
            img = image(res, mt, k, delta=True)
            assert (img == O.dense_masked_sum(x, mt, None, k)).all(), (k, t)
    res.free()


def test_uint8_delta_raw_value_out_of_range():
    """A raw low bit that lifts a count past 255 (base 225, shift 1, a 255 whose low bit is
    0, flipped) is malformed for the oracle and for a delta that decodes that stream alone;
    the same delta on the intact resident is exact."""
    rng = np.random.default_rng(5)
    det, scans = 8, 512
    P = det * det
    x = rng.poisson(3.0, size=(scans, P)).astype(np.uint8)
    bad_p, bad_scan = 19, 7
    v = rng.integers(225, 255, size=scans)
    v[0], v[bad_scan] = 225, 255
    x[:, bad_p] = v.astype(np.uint8)
    enc = O.encode(x, 8)
    g = enc.groups[0]
    gi, j = divmod(bad_p, 32)
    e = lambda t: (int(g[gi, 1 + t // 2]) >> (16 * (t & 1))) & 0xFFFF
    start = int(g[gi, 0]) + (e(j - 1) if j else 0)
    end = int(g[gi, 0]) + e(j)
    h = O.stream_header(bytes(enc.payloads[0][start:start + 2]))
    assert h[0] == 3 and h[2] == 1 and h[3] == 1 and h[1] >= 8, h
    bad = enc.payloads[0].copy()
    bad[start + 3] ^= 0x80                      # raw section after header + base: scan 7, shift 1
    assert O.decode_stream(bytes(bad[start:end]), 1)[0] != 0
    assert O.decode_stream(bytes(enc.payloads[0][start:end]), 1)[0] == 0
    w = W.Workload("rawbad", 1, scans, det, det, 8, 0, "host")
    m0 = np.zeros(P, np.uint8)
    m0[:10] = 1
    m1 = m0.copy()
    m1[bad_p] = 1
    for payloads, ok in (([bad], False), (None, True)):
        res = oracle_resident(w, enc, payloads=payloads)
        assert (image(res, m0) == O.dense_masked_sum(x, m0)).all()
        if ok:
            assert (image(res, m1, delta=True) == O.dense_masked_sum(x, m1)).all()
        else:
            with pytest.raises(V.MalformedStream):
                image(res, m1, delta=True)
        res.free()


def test_uint16_raw_value_out_of_range():
    """uint16: a raw low bit that lifts a count past 65535 (base 65505, shift 1, a 65535 whose
    low bit is 0, flipped) is malformed for the oracle, for a full query and for a delta
    that decode that stream; on the intact resident both are exact.  The pixel's other
    counts are high, so its warp's segments are reduced scan by scan."""
    rng = np.random.default_rng(6)
    det, scans = 8, 512
    P = det * det
    x = rng.poisson(3.0, size=(scans, P)).astype(np.uint16)
    bad_p, bad_scan = 37, 9
    v = rng.integers(65505, 65535, size=scans)
    v[0], v[bad_scan] = 65505, 65535
    x[:, bad_p] = v.astype(np.uint16)
    enc = O.encode(x, 16)
    g = enc.groups[0]
    gi, j = divmod(bad_p, 32)
    e = lambda t: (int(g[gi, 1 + t // 2]) >> (16 * (t & 1))) & 0xFFFF
    start = int(g[gi, 0]) + (e(j - 1) if j else 0)
    end = int(g[gi, 0]) + e(j)
    h = O.stream_header(bytes(enc.payloads[0][start:start + 2]))
    assert h[0] == 3 and h[2] == 1 and h[3] == 1 and h[1] >= 8, h
    bad = enc.payloads[0].copy()
    bad[start + 4 + 1] ^= 0x02                  # raw section after header + 2-byte base: scan 9 = byte 1, bit 1
    assert O.decode_stream(bytes(bad[start:end]), 2)[0] != 0
    assert O.decode_stream(bytes(enc.payloads[0][start:end]), 2)[0] == 0
    w = W.Workload("rawbad16", 1, scans, det, det, 16, 0, "host")
    m0 = np.zeros(P, np.uint8)
    m0[:10] = 1
    m1 = m0.copy()
    m1[bad_p] = 1
    for payloads, ok in (([bad], False), (None, True)):
        res = oracle_resident(w, enc, payloads=payloads)
        assert (image(res, m0) == O.dense_masked_sum(x, m0)).all()
        if ok:
            assert (image(res, m1, delta=True) == O.dense_masked_sum(x, m1)).all()
            assert (image(res, m1) == O.dense_masked_sum(x, m1)).all()
        else:
            with pytest.raises(V.MalformedStream):
                image(res, m1, delta=True)
        res.free()
    res = oracle_resident(w, enc, payloads=[bad])
    with pytest.raises(V.MalformedStream):
        image(res, m1)
    res.free()

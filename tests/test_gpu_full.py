"""GPU parity at full size (the 192x192-detector workloads), in the launch
configuration the bench uses: counts generated on the device by the
counter-based generator, encoded by the GPU, queried through the C ABI.

The oracle cannot hold these acquisitions, so it checks sampled blocks: it
regenerates their counts on the host (its own generator implementation),
encodes them, and compares bitstreams byte for byte and virtual-image rows
value for value.  Whole-array properties that hold at any size are checked
on the GPU results directly (stride rows are a subset of the stride-1 rows,
DPC quadrants sum to the bright-field image, a delta chain ends at the full
query of its last mask, the uint64 image equals the uint32 one).
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle as O
import virtual_imaging_b200 as V
import workloads as W
from qem_testlib import device, image, to_dev

pytestmark = pytest.mark.gpu


def generate(w, b0, nb, out=None):
    spec = w.counter
    dev = device()
    if out is None:
        out = torch.empty((nb * 512, w.n_pixels), dtype=torch.uint8 if w.dtype_bits == 8 else torch.uint16,
                          device=dev)
    V.generate_counts(out, w.dtype_bits, spec.seed, b0 * 512, nb * 512, w.n_pixels,
                      to_dev(spec.pixel_class.astype(np.int32)), to_dev(spec.class_desc.astype(np.int32)),
                      to_dev(spec.thresholds.view(np.int64)))
    return out


def host_blocks(w, blocks):
    with ThreadPoolExecutor(8) as ex:
        return dict(zip(blocks, ex.map(w.block_counts, blocks)))


def build(w, chunk_blocks=None):
    chunk_blocks = chunk_blocks or w.n_blocks
    res = V.Resident.create((w.scan_rows, w.scan_cols), (w.det_rows, w.det_cols), w.dtype_bits)
    buf = None
    for b0 in range(0, w.n_blocks, chunk_blocks):
        nb = min(chunk_blocks, w.n_blocks - b0)
        buf = generate(w, b0, nb, None if buf is None or buf.shape[0] != nb * 512 else buf)
        res.append(buf, nb)
    torch.cuda.synchronize()
    return res, buf


def check_bitstreams(res, w, counts):
    for b, x in counts.items():
        g, p = res.export_block(b)
        og, op = O.encode_block(x, w.dtype_bits)
        assert (g == og).all(), b
        assert p.size == op.size and (p == op).all(), b


@pytest.mark.parametrize("name", ["c3", "c4", "c5"])
def test_generator_matches_host(name):
    w = W.workload(name)
    for b in (0, w.n_blocks - 1):
        dev = generate(w, b, 1).cpu().numpy()
        assert (dev == w.block_counts(b)).all(), (name, b)


def test_c3_full():
    w = W.workload("c3")
    res, buf = build(w)
    check = sorted(set(w.decode_blocks[:3]) | {0})
    counts = host_blocks(w, check)
    check_bitstreams(res, w, counts)
    imgs = {}
    for name, m in w.masks.items():
        imgs[name] = image(res, m, 1)
        for b, x in counts.items():
            assert (imgs[name][b] == O.dense_masked_sum(x, m)[0]).all(), (name, b)
    dpc = sum(imgs[f"dpc{q}"] for q in range(4))
    assert (dpc == imgs["bf"]).all()
    # block decode of the 16 listed blocks, one call each (n=1), against the device counts
    for b in w.decode_blocks:
        out = res.decode_blocks(b, 1)
        assert torch.equal(out, buf[b * 512:(b + 1) * 512]), b
        if b in counts:
            assert (out.cpu().numpy() == counts[b]).all()
    res.free()


def test_c4_full():
    w = W.workload("c4")
    res, buf = build(w)
    del buf
    torch.cuda.empty_cache()
    check = sorted(set(w.sample_blocks[:4]) | {0, 16, 256})
    counts = host_blocks(w, check)
    check_bitstreams(res, w, counts)
    for name in ("bf", "adf"):
        m = w.masks[name]
        full = image(res, m, 1)
        for b, x in counts.items():
            assert (full[b] == O.dense_masked_sum(x, m)[0]).all(), (name, b)
        for k in (4, 16):
            img = image(res, m, k)
            assert img.shape[0] == -(-w.n_blocks // k)
            assert (img == full[::k]).all(), (name, k)
    # drag: 64 deltas end at the full query of the last mask, rows match the oracle
    img = image(res, w.drag[0], 1)
    for t in range(1, len(w.drag)):
        img = image(res, w.drag[t], 1, delta=True)
        if t % 16 == 0:
            for b, x in counts.items():
                assert (img[b] == O.dense_masked_sum(x, w.drag[t])[0]).all(), (t, b)
    assert (img == image(res, w.drag[-1], 1)).all()
    rows, streams = res.counters()
    res.free()


def test_c5_chunks():
    w = W.workload("c5")
    res, buf = build(w, chunk_blocks=1)
    del buf
    torch.cuda.empty_cache()
    info = res.info()
    assert info["n_blocks_encoded"] == 2048 and info["out_bits_auto"] == 32
    check = sorted(w.sample_blocks)
    counts = host_blocks(w, check)
    check_bitstreams(res, w, counts)
    full = w.masks["full"]
    a64 = image(res, full, 1, out_bits=64)
    a32 = image(res, full, 1)
    assert (a64 == a32).all()
    for b, x in counts.items():
        assert (a64[b] == O.dense_masked_sum(x, full)[0]).all(), b
    for name in ("bf", "adf"):
        img = image(res, w.masks[name], 1)
        for b, x in counts.items():
            assert (img[b] == O.dense_masked_sum(x, w.masks[name])[0]).all(), (name, b)
    res.free()

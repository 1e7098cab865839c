"""The allocation-free masked sum (qem_masked_sum_noalloc).

Some callers must not allocate device memory while they query: a render or
acquisition thread that must never block on the CUDA allocator (cudaMalloc
can synchronise the device), or code under a memory budget fixed at set-up.
qem_masked_sum_noalloc serves them with a fixed working array in the
library's device globals.  These tests call it through the C ABI and check,
on two calls in a row, that its images equal both the allocating entry
point's and the plain masked sums of the counts; that a malformed stream is
reported; that an indexed resident gives the same images; and that the
device's free memory does not change across its first calls.  The file is
collected last and passes alone in a fresh process as well as after the
other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import virtual_imaging_b200 as V
import workloads as W
from qem_testlib import device, gpu_encode, oracle_resident, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(res, mask, k, out_bits, out):
    """Direct C-ABI call: int qem_masked_sum_noalloc(res, d_mask, k, out_bits, d_out, stream)."""
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return V.lib().qem_masked_sum_noalloc(res._h, ctypes.c_void_p(mask.data_ptr()), k, out_bits,
                                          ctypes.c_void_p(out.data_ptr()), stream)


@pytest.mark.parametrize("name", ["c1", "c2", "u19"])
def test_noalloc_equals_masked_sum_and_oracle(name):
    device()
    w = W.workload(name)
    x = w.host_counts()
    res = gpu_encode(w, x)
    bits = res.info()["out_bits_auto"]
    masks = list(w.masks.values()) + [np.ones(w.n_pixels, np.uint8)]
    for k in (1, 2, 3):
        rows = -(-w.n_blocks // k)
        for m in masks:
            md = to_dev(m.astype(np.uint8))
            want = O.dense_masked_sum(x, m, None, k)
            lib_img = V.as_unsigned(res.masked_sum(md, block_stride=k)).astype(np.uint64)
            assert (lib_img == want).all()
            for out_bits in (0, 64):
                width = bits if out_bits == 0 else 64
                for call in range(2):                       # two calls in a row share the array
                    out = torch.full((rows, 512), -1, dtype=V.out_dtype(width), device=md.device)
                    assert _noalloc(res, md, k, out_bits, out) == V.QEM_OK
                    got = V.as_unsigned(out).astype(np.uint64)
                    assert (got == want).all(), (name, k, out_bits, call)
    res.free()


def test_noalloc_allocates_nothing():
    """The device's free memory is the same before the first call on a new resident
    and after two calls (outputs allocated beforehand)."""
    dev = device()
    w = W.workload("c2")
    x = w.host_counts()
    res = gpu_encode(w, x)
    md = to_dev(w.masks["bf"])
    outs = [torch.zeros((w.n_blocks, 512), dtype=torch.int32, device=dev) for _ in range(2)]
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for out in outs:
        assert _noalloc(res, md, 1, 0, out) == V.QEM_OK
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    assert free1 == free0, (free0, free1)
    want = O.dense_masked_sum(x, w.masks["bf"])
    for out in outs:
        assert (V.as_unsigned(out).astype(np.uint64) == want).all()
    res.free()


def test_noalloc_indexed_resident():
    """With an interaction index built, the call still decodes every masked pixel and
    gives the plain masked sums."""
    device()
    w = W.workload("c2")
    x = w.host_counts()
    res = gpu_encode(w, x)
    res.build_index((48, 48))
    for m in list(w.masks.values()) + [w.drag[3]]:
        md = to_dev(m)
        for call in range(2):
            out = torch.zeros((w.n_blocks, 512), dtype=torch.int32, device=md.device)
            assert _noalloc(res, md, 1, 0, out) == V.QEM_OK
            assert (V.as_unsigned(out).astype(np.uint64) == O.dense_masked_sum(x, m)).all()
    res.free()


def test_noalloc_malformed_stream():
    """A stream with a reserved header bit set inside the mask gives
    QEM_ERR_MALFORMED; the next call on an intact resident is exact again (the
    status lives in the shared array and every call clears it)."""
    device()
    w = W.workload("c1")
    x = w.host_counts()
    enc = O.encode(x, 8)
    p = int(np.nonzero(w.masks["bf"])[0][5])
    g = enc.groups[0]
    gi, j = divmod(p, 32)
    ends = [0] + [(int(g[gi, 1 + t // 2]) >> (16 * (t & 1))) & 0xFFFF for t in range(32)]
    start, end = int(g[gi, 0]) + ends[j], int(g[gi, 0]) + ends[j + 1]
    assert end - start >= 2
    bad = enc.payloads[0].copy()
    bad[start + 1] |= 0x80                                  # reserved header bit 15
    res_bad = oracle_resident(w, enc, payloads=[bad])
    res_ok = oracle_resident(w, enc)
    md = to_dev(w.masks["bf"])
    out = torch.zeros((1, 512), dtype=torch.int32, device=md.device)
    assert _noalloc(res_bad, md, 1, 0, out) == V.QEM_ERR_MALFORMED
    assert _noalloc(res_ok, md, 1, 0, out) == V.QEM_OK
    assert (V.as_unsigned(out).astype(np.uint64) == O.dense_masked_sum(x, w.masks["bf"])).all()
    # a mask that leaves the damaged pixel out is exact on the damaged resident
    m2 = w.masks["bf"].copy()
    m2[p] = 0
    assert _noalloc(res_bad, to_dev(m2), 1, 0, out) == V.QEM_OK
    assert (V.as_unsigned(out).astype(np.uint64) == O.dense_masked_sum(x, m2)).all()
    res_bad.free()
    res_ok.free()


def test_noalloc_rejects_oversize_and_bad_args():
    device()
    side = 363                                               # 131769 pixels > QEM_NOALLOC_MAX_PIXELS
    res = V.Resident.create((16, 32), (side, side), 8)
    mask = torch.ones(side * side, dtype=torch.uint8, device="cuda")
    out = torch.zeros((1, 512), dtype=torch.int32, device="cuda")
    assert _noalloc(res, mask, 1, 0, out) == V.QEM_ERR_ARG
    res.free()
    w = W.workload("c1")
    res = gpu_encode(w, w.host_counts())
    mask = to_dev(w.masks["bf"])
    assert _noalloc(res, mask, 0, 0, out) == V.QEM_ERR_ARG      # stride 0
    assert _noalloc(res, mask, 1, 16, out) == V.QEM_ERR_ARG     # width 16
    res.free()

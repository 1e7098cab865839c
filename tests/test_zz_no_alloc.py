"""The allocation-free masked sum (qem_masked_sum_noalloc) against qem_masked_sum.

Some callers must not allocate device memory while they query (a thread that
must never block on the CUDA allocator, or code under an allocation budget
fixed at set-up).  qem_masked_sum_noalloc serves them with a fixed working
array in the library's device globals.  This test calls it through the C ABI
and checks that two calls in a row give exactly the images the allocating
entry point gives.  It lives in its own file that pytest collects last, and
passes alone in a fresh process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import virtual_imaging_b200 as V
import workloads as W
from qem_testlib import device, gpu_encode, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(res, mask, k, out_bits, out):
    """Direct C-ABI call: int qem_masked_sum_noalloc(res, d_mask, k, out_bits, d_out, stream)."""
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return V.lib().qem_masked_sum_noalloc(res._h, ctypes.c_void_p(mask.data_ptr()), k, out_bits,
                                          ctypes.c_void_p(out.data_ptr()), stream)


@pytest.mark.parametrize("name", ["c1", "c2"])
def test_noalloc_equals_masked_sum(name):
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
            want = V.as_unsigned(res.masked_sum(md, block_stride=k))
            for out_bits in (0, 64):
                width = bits if out_bits == 0 else 64
                for call in range(2):                       # two calls in a row share the array
                    out = torch.full((rows, 512), -1, dtype=V.out_dtype(width), device=md.device)
                    assert _noalloc(res, md, k, out_bits, out) == V.QEM_OK
                    got = V.as_unsigned(out)
                    assert (got.astype(np.uint64) == want.astype(np.uint64)).all(), (name, k, out_bits, call)
    res.free()


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

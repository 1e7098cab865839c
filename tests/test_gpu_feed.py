"""Block decode with float32 square-root amplitude, and the prefetching feed
over a series of residents: every block in order, counts equal to the
acquisition, amplitude equal to numpy's correctly rounded float32 sqrt."""
import numpy as np
import pytest
import torch

import workloads as W
from qem_testlib import gpu_encode
from virtual_imaging_b200.feed import Feed

pytestmark = pytest.mark.gpu


def amp_of(x, valid=None):
    a = np.sqrt(x.astype(np.float32))
    if valid is not None:
        a[:, valid == 0] = 0.0
    return a


@pytest.mark.parametrize("name", ["c1", "c2", "s19"])
def test_decode_blocks_amplitude(name):
    w = W.workload(name)
    x = w.host_counts()
    valid = W.invalid_mask(w, 5) if name == "s19" else None
    res = gpu_encode(w, x, valid)
    counts, amp = res.decode_blocks_amplitude(0, w.n_blocks)
    want = x.copy()
    if valid is not None:
        want[:, valid == 0] = 0
    assert (counts.cpu().numpy() == want).all()
    got = amp.cpu().numpy()
    assert got.dtype == np.float32
    assert np.array_equal(got.view(np.uint32), amp_of(want).view(np.uint32))
    if w.n_blocks > 2:
        c2, a2 = res.decode_blocks_amplitude(1, 2)
        assert (c2.cpu().numpy() == want[512:1536]).all()
        assert np.array_equal(a2.cpu().numpy(), amp_of(want[512:1536]))
    res.free()


@pytest.mark.parametrize("amplitude", [False, True])
def test_feed_over_a_series(amplitude):
    ws = [W.workload("c2"), W.workload("c1"), W.workload("s17")]
    xs = [w.host_counts() for w in ws]
    series = [gpu_encode(w, x) for w, x in zip(ws, xs)]
    seen = []
    consumer = torch.cuda.current_stream()
    for item in Feed(series, blocks=3, amplitude=amplitude, depth=2, stream=consumer):
        x = xs[item.source][item.first_block * 512:(item.first_block + item.n_blocks) * 512]
        assert (item.counts.cpu().numpy() == x).all(), (item.source, item.first_block)
        if amplitude:
            assert np.array_equal(item.amplitude.cpu().numpy(), amp_of(x))
        else:
            assert item.amplitude is None
        seen.append((item.source, item.first_block, item.n_blocks))
    want = []
    for si, w in enumerate(ws):
        for b0 in range(0, w.n_blocks, 3):
            want.append((si, b0, min(3, w.n_blocks - b0)))
    assert seen == want
    for r in series:
        r.free()

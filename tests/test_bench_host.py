"""Host-side helpers of bench.py that need no GPU: the query schedule, the split of
a query over the interaction index (which must mirror the plan kernel's rule),
the algorithmic byte count behind the roofline, and the source hash that ties a
committed DRAM-traffic capture to the code it measured."""
import os
import shutil

import numpy as np
import pytest

import bench
import virtual_imaging_b200 as V
import workloads as W


def test_schedule_c4():
    w = W.workload("c4")
    s = bench.schedule(w)
    assert len(s) == 71
    assert [x[0] for x in s[:7]] == ["bf_k1", "adf_k1", "bf_k4", "adf_k4", "bf_k16", "adf_k16", "drag_full"]
    assert all(x[0] == "drag_delta" and x[3] and x[2] == 1 for x in s[7:])
    assert not any(x[3] for x in s[:7])


def _layout(w):
    return V.polar_layout(w.det_rows, w.det_cols, (w.det_rows // 2, w.det_cols // 2))


@pytest.mark.parametrize("case", ["bf", "adf", "delta"])
@pytest.mark.parametrize("classes", [False, True])
def test_decompose_partitions_the_query(case, classes):
    """Items plus signed residual pixels add up to exactly the query, items are
    disjoint, no whole leaf is left residual, and with pixel classes (the c4 light /
    heavy split: heavy inside the bright-field disk) a leaf becomes item-minus-rest
    only when that is cheaper by the planner weights."""
    w = W.workload("c4")
    slots, roots = _layout(w)
    P = w.n_pixels
    if case == "delta":
        old, new = w.drag[0].astype(bool), w.drag[1].astype(bool)
        add, rem = new & ~old, old & ~new
    else:
        add, rem = w.masks[case].astype(bool), np.zeros(P, bool)
    pclass = (~W.disk(192, 192, 96, 96, 30).astype(bool)).astype(np.uint8) if classes else None
    items, resid = bench.decompose(slots, roots, P, add, rem, pclass)
    covered = np.zeros(P, np.int64)
    sign = np.zeros(P, np.int64)
    for lvl, g in items:
        leaves = range(roots[g], roots[g + 1]) if lvl == 1 else [g]
        px = np.concatenate([slots[l][slots[l] < P] for l in leaves])
        covered[px] += 1
        sign[px] += -1 if (rem.any() and rem[px].all()) else 1
    assert covered.max(initial=0) <= 1                       # items are disjoint
    # residual pixels inside an item leaf are subtracted (not in the query), others added
    contrib = sign + np.where(resid & (covered > 0), -1, 0) + np.where(resid & (covered == 0), np.where(rem, -1, 1), 0)
    want = add.astype(np.int64) - rem.astype(np.int64)
    assert np.array_equal(contrib, want)
    for l in range(slots.shape[0]):
        px = slots[l][slots[l] < P]
        assert not (add[px].all() and resid[px].all())
        assert not (rem.any() and rem[px].all() and resid[px].all())
        if classes and case != "delta" and covered[px].any() and not add[px].all():
            wgt = np.where(pclass[px] != 0, bench.PLAN_LIGHT, bench.PLAN_HEAVY)
            assert bench.PLAN_ITEM + wgt[~add[px]].sum() < wgt[add[px]].sum()
    if case == "adf":
        assert len(items) > 0 and resid.sum() < add.sum() // 3
    if case == "bf" and classes:
        # edge leaves of the disk are taken whole: few heavy pixels stay residual
        assert (resid & (pclass == 0)).sum() < (add & (pclass == 0)).sum() // 10


def test_algorithmic_bytes_hand_count():
    w = W.Workload("t", 32, 32, 8, 8, 8, 0, "host")           # 2 blocks, 64 pixels
    lens = np.full((2, 64), 10, np.uint32)
    lens[1, 40] = 50
    m = np.zeros(64, np.uint8)
    m[[3, 5, 40]] = 1
    (a,) = bench.algorithmic_bytes(lens, w, [("q", m, 1, False)], 32)
    enc = 10 * 3 + 10 * 2 + 50
    assert a["enc"] == enc
    assert a["streams"] == 6
    # encoded bytes + 2 B offset per stream + 4 B base per touched group (2 groups x 2 rows)
    # + the image (2 rows x 512 x 4 B) + 4 B list entry per listed pixel
    assert a["bytes"] == enc + 2 * 6 + 4 * 4 + 2 * 512 * 4 + 4 * 3
    assert a["raw"] == 3 * 512 * 2
    # stride 2 touches one block; a delta from that mask lists only the changed pixel
    m2 = m.copy()
    m2[5] = 0
    q = bench.algorithmic_bytes(lens, w, [("a", m, 2, False), ("d", m2, 2, True)], 32)
    assert q[0]["enc"] == 30 and q[1]["enc"] == 10 and q[1]["streams"] == 1


def test_kernel_source_hash_ignores_comments(tmp_path, monkeypatch):
    src = os.path.join(bench.ROOT, "virtual_imaging_b200", "csrc")
    dst = tmp_path / "virtual_imaging_b200" / "csrc"
    dst.mkdir(parents=True)
    for name in ("kernels.cu", "qem_internal.h"):
        shutil.copy(os.path.join(src, name), dst / name)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    k = dst / "kernels.cu"
    text = k.read_text()
    k.write_text("// a new comment\n/* and a block\n   comment */\n\n" + text.replace("\n", "  \n", 3))
    assert bench.kernel_source_hash() == h0
    k.write_text(text.replace("kFull = 0xFFFFFFFFu", "kFull = 0xFFFFFFFEu", 1))
    assert "kFull = 0xFFFFFFFEu" in k.read_text()
    assert bench.kernel_source_hash() != h0


def _fake_nvml(fail=False):
    import types

    fake = types.ModuleType("pynvml")
    st = {"init": 0, "shutdown": 0, "i": 0}

    def init():
        if fail:
            raise RuntimeError("no driver")
        st["init"] += 1

    def by_uuid(u):
        assert u.startswith("GPU-")
        return "h"

    def clock(h, c):
        st["i"] += 1
        return (1965, 1965, 1800)[st["i"] % 3]

    fake.NVML_CLOCK_SM = 1
    fake.nvmlInit = init
    fake.nvmlShutdown = lambda: st.__setitem__("shutdown", st["shutdown"] + 1)
    fake.nvmlDeviceGetHandleByUUID = by_uuid
    fake.nvmlDeviceGetHandleByIndex = lambda i: "h"
    fake.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    fake.nvmlDeviceGetClockInfo = clock
    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x4 if st["i"] % 2 else 0x1
    return fake, st


def test_clock_sampler_reads_nvml(monkeypatch):
    import sys
    import time

    fake, st = _fake_nvml()
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    with bench.Clocks(0, "0000-1111", period=0.001) as c:
        time.sleep(0.05)
    s = c.summary()
    assert s["source"] == "nvml" and s["samples"] >= 5
    assert s["sm_max_mhz"] == 1965 and s["sm_mhz"] in (1800, 1965)
    assert s["reasons"] == ["sw_power_cap"]            # idle (0x1) is not a reason that matters
    assert st["init"] == 1 and st["shutdown"] == 1


def test_clock_sampler_without_nvml(monkeypatch):
    import sys

    fake, _ = _fake_nvml(fail=True)
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    with bench.Clocks(0) as c:
        pass
    s = c.summary()
    assert s["sm_mhz"] is None and s["reasons"]

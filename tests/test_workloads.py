"""Pins for the seeded input generators (no codec arithmetic lives here)."""
import math

import numpy as np
from scipy import stats

import workloads as W


def test_splitmix64_published_vector():
    """SplitMix64 seeded with 1234567: first five outputs of Vigna's splitmix64.c."""
    z = W.counter_draw(1234567, np.zeros(5, np.int64), np.arange(5), 10 ** 9)
    assert [int(x) for x in z] == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                                   4593380528125082431, 16408922859458223821]


def _gauss_circle(r: int, r2: int | None = None) -> int:
    """Lattice points with x^2 + y^2 <= n (n = r^2 by default):
    1 + 4 floor(sqrt n) + 4 sum_{i=1..floor(sqrt n)} floor(sqrt(n - i^2))."""
    n = r * r if r2 is None else r2
    s = math.isqrt(n)
    return 1 + 4 * s + 4 * sum(math.isqrt(n - i * i) for i in range(1, s + 1))


def test_mask_pixel_counts_closed_form():
    for det, R in [(32, 8), (96, 24), (192, 30), (192, 48), (192, 10)]:
        assert int(W.disk(det, det, det // 2, det // 2, R).sum()) == _gauss_circle(R)
    assert _gauss_circle(8) == 197
    a = W.annulus(192, 192, 96, 96, 40, 90)
    assert int(a.sum()) == _gauss_circle(90) - _gauss_circle(0, 40 * 40 - 1)
    q = W.quadrants(192, 192, 96, 96, 30)
    tot = np.sum(q, axis=0)
    assert (tot == W.disk(192, 192, 96, 96, 30)).all()          # disjoint cover of the disk


def test_poisson_thresholds_match_scipy():
    for lam in [0.01, 0.3, 3.0, 20.0, 400.0, 1000.0]:
        t = W.poisson_thresholds(lam, 65535).astype(np.float64)
        assert (np.diff(t) >= 0).all() and t[-1] == 2.0 ** 53
        pmf = np.diff(np.concatenate([[0.0], t])) / 2.0 ** 53
        ref = stats.poisson.pmf(np.arange(t.size), lam)
        assert np.abs(pmf[:-1] - ref[:-1]).max() < 1e-9


def test_counter_counts_are_poisson():
    w = W.workload("c4")
    x = w.block_counts(5).astype(np.float64)
    bf = W.disk(192, 192, 96, 96, 30).astype(bool)
    v = x[:, bf].ravel()
    n = v.size
    assert abs(v.mean() - 3.0) < 5 * math.sqrt(3.0 / n)
    assert abs(v.var() - 3.0) < 0.05
    hist = np.bincount(v.astype(int), minlength=12)[:12]
    exp = stats.poisson.pmf(np.arange(12), 3.0) * n
    chi2 = float((((hist - exp) ** 2) / exp).sum())
    assert chi2 < stats.chi2.ppf(0.9999, 11)
    df = x[:, ~bf].ravel()
    assert abs(df.mean() - 0.01) < 5 * math.sqrt(0.01 / df.size)


def test_counter_regeneration_is_positional():
    """Any scan range regenerates identically (the generator is counter-based)."""
    w = W.workload("c3")
    a = W.counter_counts(w.counter, 512 * 3, 512)
    b = W.counter_counts(w.counter, 512 * 3 + 100, 50)
    assert (a[100:150] == b).all()
    uni = w.counter.class_desc[w.counter.pixel_class][:, 0] == W.KIND_UNIFORM
    assert int(uni.sum()) == 184


def test_c_generator_equals_numpy_generator():
    """The C host generator (used to regenerate whole full-size acquisitions for the
    parity tests) gives the NumPy generator's counts bit for bit, on scans from the
    start, the middle and the end of every counter workload."""
    assert W._cgen_lib() is not None, "counter_gen.c did not build"
    for name in ("c3", "c4", "c5"):
        w = W.workload(name)
        for s0 in (0, 511, w.n_scans // 2 + 3, w.n_scans - 6):
            a = W.counter_counts(w.counter, s0, 6)
            b = W.counter_counts_fast(w.counter, s0, 6)
            assert a.dtype == b.dtype and (a == b).all(), (name, s0)

"""Seeded synthetic 4D-STEM count workloads.

This module only *generates inputs*: count acquisitions, detector masks and the
query schedules that exercise the paired-count resident.  It holds none of the
codec's arithmetic (no models, no tANS, no stream forms, no sums), so both the
CUDA library and the CPU oracle can take their inputs from here without sharing
any of the method.

Two kinds of generator exist:

* ``host`` workloads (the 32x32 and 96x96 detectors) are drawn with NumPy's
  ``default_rng`` and uploaded as-is.
* ``counter`` workloads (the 192x192 detectors) are defined by a counter-based
  hash so that any block can be regenerated independently:
  ``z = splitmix64_mix(seed + (s*P + p + 1) * 0x9E3779B97F4A7C15)`` (the n-th
  output of Steele, Lea & Flood's SplitMix64 seeded with ``seed``, Vigna's
  ``splitmix64.c``), ``u = z >> 11`` (53 bits), and the count is the Poisson
  inverse CDF read from an integer threshold table per pixel class
  (``count = min{k : u < T[k]}``).  Uniform ("incompressible") pixels take
  ``z & dtype_max``; constant pixels take a fixed value.  The CUDA library has
  its own device implementation of this generator; :func:`counter_counts` is
  the host one.

Scan index ``s = scan_row * scan_cols + scan_col`` (row-major), pixel index
``p = det_row * det_cols + det_col``; count arrays are ``[scans][pixels]``.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading
from dataclasses import dataclass, field

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

KIND_POISSON = 0
KIND_UNIFORM = 1
KIND_CONSTANT = 2

SCANS_PER_BLOCK = 512


# ----------------------------------------------------------------------------
# counter-based generator (host implementation)
# ----------------------------------------------------------------------------
def splitmix64_mix(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output mix (Steele, Lea & Flood 2014) on a uint64 array."""
    z = np.asarray(z, dtype=np.uint64).copy()
    z ^= z >> np.uint64(30)
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def counter_draw(seed: int, scan: np.ndarray, pixel: np.ndarray, n_pixels: int) -> np.ndarray:
    """64-bit draw for (scan, pixel): SplitMix64 output number s*P + p + 1."""
    idx = scan.astype(np.uint64) * np.uint64(n_pixels) + pixel.astype(np.uint64) + np.uint64(1)
    with np.errstate(over="ignore"):
        state = np.uint64(seed) + idx * GAMMA
    return splitmix64_mix(state)


def poisson_thresholds(lam: float, dtype_max: int) -> np.ndarray:
    """Integer inverse-CDF table for Poisson(lam): T[k] = floor(F(k) * 2**53).

    The table stops at the first k whose threshold reaches 2**53 (or at
    dtype_max, where the last entry is forced to 2**53), so that
    ``min{k : u < T[k]}`` always exists for u < 2**53.  The pmf is evaluated in
    float64 through log-space (``-lam + k ln lam - lgamma(k+1)``) so that large
    means do not underflow.
    """
    full = 1 << 53
    out = []
    cdf = 0.0
    k = 0
    while True:
        term = math.exp(-lam + k * math.log(lam) - math.lgamma(k + 1)) if lam > 0 else float(k == 0)
        cdf += term
        t = min(full, int(math.floor(min(cdf, 1.0) * full)))
        # past the mean, once the next terms cannot move a threshold, close the table
        if k >= dtype_max or (k > lam and term * full < 0.25):
            t = full
        out.append(t)
        if t >= full:
            break
        k += 1
    return np.asarray(out, dtype=np.uint64)


@dataclass
class CounterSpec:
    """Everything the counter-based generator needs, as plain arrays."""

    seed: int
    n_pixels: int
    dtype_bits: int
    pixel_class: np.ndarray          # uint32 [P]
    class_desc: np.ndarray           # uint32 [C][4]: kind, offset, length, value
    thresholds: np.ndarray           # uint64 [sum of lengths]


def counter_counts(spec: CounterSpec, scan0: int, n_scans: int) -> np.ndarray:
    """Host regeneration of scans [scan0, scan0+n_scans) of a counter workload.

    Poisson pixels take ``min{k : u < T[k]}`` over their class's threshold
    table, found by a vectorised binary search over the whole [scans][pixels]
    array at once.
    """
    P = spec.n_pixels
    dmax = (1 << spec.dtype_bits) - 1
    dt = np.uint8 if spec.dtype_bits == 8 else np.uint16
    pix = np.arange(P, dtype=np.int64)[None, :]
    scan = np.arange(scan0, scan0 + n_scans, dtype=np.int64)[:, None]
    z = counter_draw(spec.seed, np.broadcast_to(scan, (n_scans, P)), np.broadcast_to(pix, (n_scans, P)), P)
    u = z >> np.uint64(11)
    desc = spec.class_desc.astype(np.int64)
    cls = spec.pixel_class.astype(np.int64)
    kind = desc[cls, 0][None, :]
    off = desc[cls, 1][None, :]
    ln = desc[cls, 2][None, :]
    val = desc[cls, 3][None, :]
    lo = np.broadcast_to(off, (n_scans, P)).copy()
    hi = np.broadcast_to(off + np.maximum(ln, 1) - 1, (n_scans, P)).copy()
    T = spec.thresholds
    if T.size == 0:
        T = np.zeros(1, dtype=np.uint64)
    for _ in range(int(max(1, desc[:, 2].max())).bit_length() + 1):
        active = lo < hi
        mid = (lo + hi) // 2
        right = u >= T[np.minimum(mid, T.size - 1)]
        lo = np.where(active & right, mid + 1, lo)
        hi = np.where(active & ~right, mid, hi)
    poisson = lo - off
    row = np.where(kind == KIND_POISSON, poisson,
                   np.where(kind == KIND_UNIFORM, (z & np.uint64(dmax)).astype(np.int64),
                            np.broadcast_to(val, (n_scans, P))))
    return np.minimum(row, dmax).astype(dt)


_HERE = os.path.dirname(os.path.abspath(__file__))
_CGEN_SRC = os.path.join(_HERE, "counter_gen.c")
_CGEN_SO = os.path.join(_HERE, "libcountergen.so")
_cgen_lock = threading.Lock()
_cgen = None


def _cgen_lib():
    """The C implementation of the counter generator (counter_gen.c), built with gcc on
    first use; None when no C compiler is available."""
    global _cgen
    with _cgen_lock:
        if _cgen is None:
            try:
                if not os.path.exists(_CGEN_SO) or os.path.getmtime(_CGEN_SO) < os.path.getmtime(_CGEN_SRC):
                    tmp = _CGEN_SO + f".tmp{os.getpid()}"
                    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _CGEN_SRC])
                    os.replace(tmp, _CGEN_SO)
                L = ctypes.CDLL(_CGEN_SO)
                P = ctypes.c_void_p
                L.wl_counter_counts.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                                                P, P, P, ctypes.c_int32, P]
                _cgen = L
            except (OSError, subprocess.CalledProcessError):
                _cgen = False
    return _cgen or None


def counter_counts_fast(spec: CounterSpec, scan0: int, n_scans: int) -> np.ndarray:
    """Same counts as :func:`counter_counts`, from the C implementation (falls back to
    the NumPy one without a C compiler).  Releases the GIL, so threads run in parallel."""
    L = _cgen_lib()
    if L is None:
        return counter_counts(spec, scan0, n_scans)
    dt = np.uint8 if spec.dtype_bits == 8 else np.uint16
    out = np.empty((n_scans, spec.n_pixels), dtype=dt)
    cls = np.ascontiguousarray(spec.pixel_class, dtype=np.uint32)
    desc = np.ascontiguousarray(spec.class_desc, dtype=np.uint32)
    thr = np.ascontiguousarray(spec.thresholds if spec.thresholds.size else np.zeros(1, np.uint64), dtype=np.uint64)
    L.wl_counter_counts(ctypes.c_uint64(spec.seed), scan0, n_scans, spec.n_pixels, cls.ctypes.data,
                        desc.ctypes.data, thr.ctypes.data, spec.dtype_bits, out.ctypes.data)
    return out


# ----------------------------------------------------------------------------
# detector geometry and masks
# ----------------------------------------------------------------------------
def radius2(det_rows: int, det_cols: int, cr: float, cc: float) -> np.ndarray:
    r = np.arange(det_rows)[:, None] - cr
    c = np.arange(det_cols)[None, :] - cc
    return (r * r + c * c).reshape(-1)


def disk(det_rows, det_cols, cr, cc, R) -> np.ndarray:
    """BF disk: integer pixel centres with d^2 <= R^2."""
    return (radius2(det_rows, det_cols, cr, cc) <= R * R).astype(np.uint8)


def annulus(det_rows, det_cols, cr, cc, r_in, r_out) -> np.ndarray:
    """ADF annulus: r_in^2 <= d^2 <= r_out^2 (inclusive)."""
    d2 = radius2(det_rows, det_cols, cr, cc)
    return ((d2 >= r_in * r_in) & (d2 <= r_out * r_out)).astype(np.uint8)


def quadrants(det_rows, det_cols, cr, cc, R) -> list[np.ndarray]:
    """DPC quadrant masks q = 2*[r>=cr] + [c>=cc] within the BF disk."""
    bf = disk(det_rows, det_cols, cr, cc, R).astype(bool)
    rr = np.repeat(np.arange(det_rows), det_cols)
    cc_ = np.tile(np.arange(det_cols), det_rows)
    q = 2 * (rr >= cr) + (cc_ >= cc)
    return [(bf & (q == k)).astype(np.uint8) for k in range(4)]


# ----------------------------------------------------------------------------
# workload definitions
# ----------------------------------------------------------------------------
@dataclass
class Workload:
    name: str
    scan_rows: int
    scan_cols: int
    det_rows: int
    det_cols: int
    dtype_bits: int
    seed: int
    kind: str                                     # "host" | "counter"
    masks: dict = field(default_factory=dict)     # name -> uint8 [P]
    strides: tuple = (1,)
    drag: list = field(default_factory=list)      # list of uint8 [P] masks (first is full, rest deltas)
    counter: CounterSpec | None = None
    decode_blocks: list = field(default_factory=list)
    sample_blocks: list = field(default_factory=list)

    @property
    def n_scans(self) -> int:
        return self.scan_rows * self.scan_cols

    @property
    def n_blocks(self) -> int:
        return self.n_scans // SCANS_PER_BLOCK

    @property
    def n_pixels(self) -> int:
        return self.det_rows * self.det_cols

    @property
    def np_dtype(self):
        return np.uint8 if self.dtype_bits == 8 else np.uint16

    @property
    def raw_bytes(self) -> int:
        return self.n_scans * self.n_pixels * (self.dtype_bits // 8)

    def host_counts(self) -> np.ndarray:
        """Full count array [scans][pixels] (host workloads, or small counter ones)."""
        if self.kind == "host":
            return _HOST_GEN[self.name](self)
        return counter_counts_fast(self.counter, 0, self.n_scans)

    def block_counts(self, b: int) -> np.ndarray:
        """Counts of one 512-scan block [512][P]."""
        if self.kind == "host":
            return self.host_counts()[b * 512:(b + 1) * 512]
        return counter_counts_fast(self.counter, b * 512, 512)


def _c1_counts(w: Workload) -> np.ndarray:
    rng = np.random.default_rng(w.seed)
    u = rng.integers(0, 3, size=4)
    v = rng.integers(0, 4, size=4)
    a = rng.uniform(0.5, 1.0, size=4)
    phi = rng.uniform(0.0, 2 * np.pi, size=4)
    rr = np.arange(w.scan_rows)[:, None, None]
    cc = np.arange(w.scan_cols)[None, :, None]
    s = (a[None, None, :] * np.cos(2 * np.pi * (u * rr / 16.0 + v * cc / 32.0) + phi)).sum(-1) / a.sum()
    s = s.reshape(-1)                                   # [scans]
    inside = disk(w.det_rows, w.det_cols, 16, 16, 8).astype(bool)
    lam = np.where(inside[None, :], 20.0 * (1.0 + 0.3 * s[:, None]), 0.05)
    counts = rng.poisson(lam)
    perm = rng.permutation(w.n_pixels)
    dead = perm[:20]
    hot = perm[20:30]
    counts[:, dead] = 0
    counts[:, hot] = 255
    return np.minimum(counts, 255).astype(np.uint8)


def _c2_counts(w: Workload) -> np.ndarray:
    rng = np.random.default_rng(w.seed)
    fr, fc = rng.integers(1, 4, size=2)
    phi = rng.uniform(0.0, 2 * np.pi)
    rr = np.repeat(np.arange(w.scan_rows), w.scan_cols)
    cc = np.tile(np.arange(w.scan_cols), w.scan_rows)
    mod = 1.0 + 0.2 * np.sin(2 * np.pi * (fr * rr + fc * cc) / 64.0 + phi)
    d = np.sqrt(radius2(w.det_rows, w.det_cols, 48, 48))
    inside = d <= 24
    lam = np.where(inside[None, :], 200.0 * mod[:, None], 0.2 * np.exp(-(d[None, :] - 24.0) / 20.0))
    counts = rng.poisson(lam)
    perm = rng.permutation(w.n_pixels)
    unif = perm[:92]
    sent = perm[92:184]
    counts[:, unif] = rng.integers(0, 65536, size=(w.n_scans, 92))
    counts[:, sent] = 65535
    return np.minimum(counts, 65535).astype(np.uint16)


def _small_counts(w: Workload) -> np.ndarray:
    """Contract fixtures: wide literal row, saturated row, invalid pixel (17/19/257 detectors)."""
    rng = np.random.default_rng(w.seed)
    dmax = (1 << w.dtype_bits) - 1
    lam = rng.uniform(0.0, 4.0, size=w.n_pixels)
    counts = rng.poisson(np.broadcast_to(lam, (w.n_scans, w.n_pixels)))
    counts = np.minimum(counts, dmax)
    counts[:, : w.det_cols] = rng.integers(0, dmax + 1, size=(w.n_scans, w.det_cols))   # wide literal row
    counts[:, w.det_cols: 2 * w.det_cols] = dmax                                       # saturated row
    return counts.astype(w.np_dtype)


def _u8_mixed_counts(w: Workload) -> np.ndarray:
    """uint8 fixture for warps mixing stream kinds: per-pixel Poisson means
    in [0.3, 3.5] (streams of plain pair steps) and a fifth of the pixels at
    0.01 (run events or sparse), and 48 planted counts in [16, 200] that give
    their streams raw low bits (shift > 0) beside plain neighbours."""
    rng = np.random.default_rng(w.seed)
    lam = rng.uniform(0.3, 3.5, size=w.n_pixels)
    lam[rng.random(w.n_pixels) < 0.2] = 0.01
    counts = rng.poisson(np.broadcast_to(lam, (w.n_scans, w.n_pixels)))
    s = rng.integers(0, w.n_scans, size=48)
    p = rng.integers(0, w.n_pixels, size=48)
    counts[s, p] = rng.integers(16, 201, size=48)
    return np.minimum(counts, 255).astype(np.uint8)


_HOST_GEN = {"c1": _c1_counts, "c2": _c2_counts}


def _counter_spec(seed, det, dtype_bits, lam_of_d2, n_uniform) -> CounterSpec:
    P = det * det
    dmax = (1 << dtype_bits) - 1
    d2 = radius2(det, det, det // 2, det // 2)
    classes: dict = {}
    desc = []
    thr = []
    off = 0
    pixel_class = np.zeros(P, dtype=np.uint32)
    for p in range(P):
        key = int(d2[p])
        if key not in classes:
            t = poisson_thresholds(lam_of_d2(key), dmax)
            classes[key] = len(desc)
            desc.append((KIND_POISSON, off, len(t), 0))
            thr.append(t)
            off += len(t)
        pixel_class[p] = classes[key]
    if n_uniform:
        rng = np.random.default_rng(seed)
        uni = rng.choice(P, n_uniform, replace=False)
        desc.append((KIND_UNIFORM, 0, 0, 0))
        pixel_class[uni] = len(desc) - 1
    return CounterSpec(seed=seed, n_pixels=P, dtype_bits=dtype_bits, pixel_class=pixel_class,
                       class_desc=np.asarray(desc, dtype=np.uint32).reshape(-1, 4),
                       thresholds=np.concatenate(thr).astype(np.uint64))


def workload(name: str) -> Workload:
    """The named synthetic workload: c1..c5, or small fixtures s17/s19/s257."""
    if name == "c1":
        w = Workload("c1", 16, 32, 32, 32, 8, 0, "host")
        w.masks = {"bf": disk(32, 32, 16, 16, 8), "adf": annulus(32, 32, 16, 16, 10, 15)}
        return w
    if name == "c2":
        w = Workload("c2", 64, 64, 96, 96, 16, 1, "host")
        w.masks = {"bf": disk(96, 96, 48, 48, 24), "adf": annulus(96, 96, 48, 48, 30, 45)}
        w.drag = [disk(96, 96, 48, 32 + 2 * t, 10) for t in range(17)]
        return w
    if name == "c3":
        lam = lambda d2: 1000.0 if d2 <= 900 else 0.5 * math.exp(-(math.sqrt(d2) - 30.0) / 40.0)
        w = Workload("c3", 256, 256, 192, 192, 16, 2, "counter")
        w.counter = _counter_spec(2, 192, 16, lam, 184)
        w.masks = {"bf": disk(192, 192, 96, 96, 30), "adf": annulus(192, 192, 96, 96, 40, 90)}
        for k, q in enumerate(quadrants(192, 192, 96, 96, 30)):
            w.masks[f"dpc{k}"] = q
        w.decode_blocks = sorted(int(x) for x in np.random.default_rng(2).choice(128, 16, replace=False))
        return w
    if name == "c4":
        lam = lambda d2: 3.0 if d2 <= 900 else 0.01
        w = Workload("c4", 512, 512, 192, 192, 8, 3, "counter")
        w.counter = _counter_spec(3, 192, 8, lam, 0)
        w.masks = {"bf": disk(192, 192, 96, 96, 30), "adf": annulus(192, 192, 96, 96, 40, 90)}
        w.strides = (1, 4, 16)
        w.drag = [disk(192, 192, 96, 64 + t, 30) for t in range(65)]
        w.sample_blocks = sorted(int(x) for x in np.random.default_rng(3).choice(512, 8, replace=False))
        return w
    if name == "c5":
        lam = lambda d2: 400.0 if d2 <= 48 * 48 else 0.3 * math.exp(-(math.sqrt(d2) - 48.0) / 30.0)
        w = Workload("c5", 1024, 1024, 192, 192, 16, 4, "counter")
        w.counter = _counter_spec(4, 192, 16, lam, 0)
        w.masks = {"full": np.ones(192 * 192, dtype=np.uint8), "bf": disk(192, 192, 96, 96, 48),
                   "adf": annulus(192, 192, 96, 96, 60, 90)}
        w.sample_blocks = sorted(int(x) for x in np.random.default_rng(4).choice(2048, 16, replace=False))
        return w
    if name in ("s17", "s19", "s257"):
        det = int(name[1:])
        bits = 16
        scans = 1024 if det < 100 else 512
        w = Workload(name, scans // 32, 32, det, det, bits, det, "host")
        c = det // 2
        w.masks = {"full": np.ones(det * det, dtype=np.uint8), "bf": disk(det, det, c, c, det // 4),
                   "adf": annulus(det, det, c, c, det // 4 + 1, det // 2)}
        _HOST_GEN[name] = _small_counts
        return w
    if name == "u19":
        det, c = 19, 9
        w = Workload(name, 32, 32, det, det, 8, 19, "host")
        w.masks = {"full": np.ones(det * det, dtype=np.uint8), "bf": disk(det, det, c, c, 4),
                   "adf": annulus(det, det, c, c, 5, 9)}
        w.drag = [disk(det, det, c, 4 + t, 4) for t in range(11)]
        _HOST_GEN[name] = _u8_mixed_counts
        return w
    raise KeyError(name)


def invalid_mask(w: Workload, n_invalid: int = 1) -> np.ndarray:
    """A detector-validity mask with ``n_invalid`` pixels switched off (seeded)."""
    v = np.ones(w.n_pixels, dtype=np.uint8)
    rng = np.random.default_rng(w.seed + 1000)
    v[rng.choice(w.n_pixels, n_invalid, replace=False)] = 0
    return v


ALL = ("c1", "c2", "c3", "c4", "c5")

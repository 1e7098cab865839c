"""CPU oracle for the paired-count resident (qem-pair-v2).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
bench's ``cpu_baseline`` / ``--impl reference`` leg may import this package.
It shares no code with the CUDA library (``virtual_imaging_b200``) and never
imports it.

Two layers:

* plain definitions in NumPy (exact integer arithmetic, uint64 / int64):
  :func:`dense_masked_sum`, :func:`dense_delta`, :func:`dense_decode_blocks`,
  :func:`dense_masked_moments` --
  these are the results the method must reach, written out directly from the
  source page "Paired-count resident layout" (section "Operation pipeline"
  step 4: exact integer virtual images, ``block_stride=k`` touches every k-th
  512-scan block; section "Contract": uint32 sums, uint64 when a full-detector
  sum could exceed 2**32, invalid pixels reported as zero);
* the codec in plain C (``oracle.c``): model tables, stream encoder/decoder,
  block layout with grouped offsets, and the decode-based masked sum, wrapped
  here with ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_SRC = [os.path.join(_HERE, "oracle.c"), os.path.join(_HERE, "oracle.h")]
_lock = threading.Lock()
_lib = None

ORC_ERRORS = {
    0: "ok", 1: "reserved header bit set", 2: "invalid form code", 3: "fields invalid for form",
    4: "length does not match form", 5: "sparse stream invalid", 6: "constant value zero",
    7: "final tANS state is not 1024", 8: "nonzero pad bits", 9: "offsets invalid", 10: "model",
}


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain gcc, -O2)."""
    newest = max(os.path.getmtime(p) for p in _SRC)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < newest:
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-fPIC", "-shared",
                               "-o", tmp, _SRC[0], "-lm"])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_SO)
            P = ctypes.c_void_p
            L.orc_models.argtypes = [P, P, P]
            L.orc_decode_table.argtypes = [ctypes.c_int, P, P, P]
            L.orc_encode_stream.argtypes = [P, ctypes.c_int, P, P]
            L.orc_decode_stream.argtypes = [P, ctypes.c_int, ctypes.c_int, P]
            L.orc_decode_stream.restype = ctypes.c_int
            L.orc_encode_block.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P]
            L.orc_encode_block.restype = ctypes.c_uint64
            L.orc_block_masked_sum.argtypes = [P, P, ctypes.c_uint64, ctypes.c_int, ctypes.c_int,
                                               P, P, ctypes.c_int, P]
            L.orc_block_masked_sum.restype = ctypes.c_int
            L.orc_decode_block.argtypes = [P, P, ctypes.c_uint64, ctypes.c_int, ctypes.c_int, P]
            L.orc_decode_block.restype = ctypes.c_int
            L.orc_paired_size.argtypes = [P, ctypes.c_int, ctypes.c_int]
            L.orc_paired_size.restype = ctypes.c_int
            L.orc_stream_sizes.argtypes = [P, ctypes.c_int, P]
            # build the model tables once, before any threads use them
            f = np.zeros((32, 256), np.uint16)
            a = np.zeros(32, np.uint8)
            c = np.zeros((32, 16), np.uint32)
            L.orc_models(f.ctypes.data, a.ctypes.data, c.ctypes.data)
            _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


class MalformedStream(ValueError):
    """A stream failed a qem-pair-v2 check (the query returns no result)."""


# ----------------------------------------------------------------------------
# tables
# ----------------------------------------------------------------------------
def models():
    """(freq [32][256] uint16, amax [32] uint8, cost [32][16] uint32)."""
    f = np.zeros((32, 256), np.uint16)
    a = np.zeros(32, np.uint8)
    c = np.zeros((32, 16), np.uint32)
    lib().orc_models(_ptr(f), _ptr(a), _ptr(c))
    return f, a, c


def decode_table(m: int):
    sym = np.zeros(1024, np.uint8)
    nb = np.zeros(1024, np.uint8)
    nbase = np.zeros(1024, np.uint16)
    lib().orc_decode_table(m, _ptr(sym), _ptr(nb), _ptr(nbase))
    return sym, nb, nbase


# ----------------------------------------------------------------------------
# streams
# ----------------------------------------------------------------------------
def encode_stream(values: np.ndarray, w: int) -> bytes:
    v = np.ascontiguousarray(values, dtype=np.uint16)
    assert v.shape == (512,)
    out = np.zeros(2 + 1024, np.uint8)
    n = ctypes.c_int(0)
    lib().orc_encode_stream(_ptr(v), w, _ptr(out), ctypes.byref(n))
    return out[: n.value].tobytes()


def decode_stream(data: bytes, w: int):
    """(status, values uint16[512])."""
    buf = np.frombuffer(bytes(data) + b"\0" * 8, np.uint8).copy()
    v = np.zeros(512, np.uint16)
    rc = lib().orc_decode_stream(_ptr(buf), len(data), w, _ptr(v))
    return rc, v


def paired_size(values: np.ndarray, w: int, model: int) -> int:
    """Exact paired-form length with a forced model (-1 if its box is too small)."""
    v = np.ascontiguousarray(values, dtype=np.uint16)
    return int(lib().orc_paired_size(_ptr(v), w, model))


def stream_sizes(values: np.ndarray, w: int):
    """(S_sparse, S_paired, S_literal, selected model) for one stream."""
    v = np.ascontiguousarray(values, dtype=np.uint16)
    info = np.zeros(4, np.int32)
    lib().orc_stream_sizes(_ptr(v), w, _ptr(info))
    return tuple(int(x) for x in info)


def stream_header(data: bytes):
    """(form, model, shift, has_base, reserved) of an encoded stream (None if empty)."""
    if len(data) == 0:
        return None
    h = data[0] | (data[1] << 8)
    return h & 7, (h >> 3) & 31, (h >> 8) & 15, (h >> 12) & 1, h >> 13


# ----------------------------------------------------------------------------
# blocks and whole acquisitions
# ----------------------------------------------------------------------------
@dataclass
class Encoded:
    """Oracle-encoded resident: per block, the group table and the payload."""

    n_pixels: int
    dtype_bits: int
    groups: list = field(default_factory=list)     # list of uint32 [G][17]
    payloads: list = field(default_factory=list)   # list of uint8 [len]

    @property
    def w(self) -> int:
        return self.dtype_bits // 8

    @property
    def n_blocks(self) -> int:
        return len(self.groups)

    def payload_bytes(self) -> int:
        return int(sum(p.size for p in self.payloads))


def encode_block(counts_block: np.ndarray, dtype_bits: int):
    """One 512-scan block [512][P] -> (groups uint32 [G][17], payload uint8)."""
    w = dtype_bits // 8
    c = np.ascontiguousarray(counts_block, dtype=np.uint8 if w == 1 else np.uint16)
    P = c.shape[1]
    G = (P + 31) // 32
    groups = np.zeros((G, 17), np.uint32)
    payload = np.zeros((2 + 512 * w) * P + 16, np.uint8)
    n = lib().orc_encode_block(_ptr(c), w, P, _ptr(groups), _ptr(payload))
    return groups, payload[:n].copy()


def _workers(n_tasks: int, threads: int | None) -> int:
    if threads is None:
        threads = os.cpu_count() or 1
    return max(1, min(threads, n_tasks))


def encode(counts: np.ndarray, dtype_bits: int, threads: int | None = None) -> Encoded:
    """Encode a whole acquisition [scans][P] (scans a multiple of 512)."""
    S, P = counts.shape
    assert S % 512 == 0
    B = S // 512
    enc = Encoded(P, dtype_bits, [None] * B, [None] * B)

    def job(b):
        g, p = encode_block(counts[b * 512:(b + 1) * 512], dtype_bits)
        enc.groups[b] = g
        enc.payloads[b] = p

    with ThreadPoolExecutor(_workers(B, threads)) as ex:
        list(ex.map(job, range(B)))
    return enc


def block_masked_sum(groups, payload, dtype_bits, P, pix, sign):
    """Decode-based signed masked sum of one block: int64[512] (raises on malformed)."""
    w = dtype_bits // 8
    pix = np.ascontiguousarray(pix, np.int32)
    sign = np.ascontiguousarray(sign, np.int8)
    out = np.zeros(512, np.int64)
    buf = np.concatenate([payload, np.zeros(16, np.uint8)])
    rc = lib().orc_block_masked_sum(_ptr(np.ascontiguousarray(groups, np.uint32)), _ptr(buf),
                                    payload.size, w, P, _ptr(pix), _ptr(sign), pix.size, _ptr(out))
    if rc:
        raise MalformedStream(ORC_ERRORS.get(rc, str(rc)))
    return out


def decode_block(groups, payload, dtype_bits, P) -> np.ndarray:
    w = dtype_bits // 8
    out = np.zeros((512, P), np.uint8 if w == 1 else np.uint16)
    buf = np.concatenate([payload, np.zeros(16, np.uint8)])
    rc = lib().orc_decode_block(_ptr(np.ascontiguousarray(groups, np.uint32)), _ptr(buf),
                                payload.size, w, P, _ptr(out))
    if rc:
        raise MalformedStream(ORC_ERRORS.get(rc, str(rc)))
    return out


# ----------------------------------------------------------------------------
# queries
# ----------------------------------------------------------------------------
def out_bits_auto(n_valid: int, dtype_bits: int) -> int:
    """uint64 when a full-detector sum could exceed 2**32 - 1 (page "Contract")."""
    return 64 if n_valid * ((1 << dtype_bits) - 1) > 0xFFFFFFFF else 32


def touched_blocks(n_blocks: int, k: int) -> list:
    """block_stride=k touches blocks 0, k, 2k, ...: ceil(n_blocks / k) of them."""
    return list(range(0, n_blocks, k))


def dense_masked_sum(counts: np.ndarray, mask: np.ndarray, valid: np.ndarray | None = None,
                     k: int = 1) -> np.ndarray:
    """Plain definition: V[r][i] = sum over p with mask&valid of x[512*(r*k) + i][p] (uint64)."""
    sel = mask.astype(bool)
    if valid is not None:
        sel &= valid.astype(bool)
    B = counts.shape[0] // 512
    rows = touched_blocks(B, k)
    out = np.zeros((len(rows), 512), np.uint64)
    for r, b in enumerate(rows):
        out[r] = counts[b * 512:(b + 1) * 512][:, sel].astype(np.uint64).sum(axis=1)
    return out


def dense_block_sums(counts_block: np.ndarray, masks, valid: np.ndarray | None = None) -> np.ndarray:
    """Plain definition for one 512-scan block and several masks at once:
    V[m][i] = sum over p with masks[m][p] & valid[p] of x[i][p] (uint64 [n_masks][512]).

    Written as one matrix product x[512][P] @ S[P][n_masks] in float64 (a library
    primitive standing for the sums): every partial sum is an integer below
    P * 65535 < 2^53, so each float64 addition is exact and the order of the
    additions cannot change the result."""
    sel = np.asarray(masks, dtype=bool).reshape(-1, counts_block.shape[1])
    if valid is not None:
        sel = sel & valid.astype(bool)[None, :]
    assert counts_block.shape[1] * 65535 < 2 ** 53
    out = counts_block.astype(np.float64) @ sel.T.astype(np.float64)
    return np.rint(out.T).astype(np.uint64)


def dense_masked_moments(counts: np.ndarray, mask: np.ndarray, weights: np.ndarray,
                         valid: np.ndarray | None = None, k: int = 1) -> np.ndarray:
    """Plain definition of the fused moment reduction (page "Backend Optimization Matrix",
    CoM/DPC rows: a fused moment reducer whose centre of mass is exact before the divide):
    for each touched block row r and scan i, over the pixels p with mask & valid,
    M[0][r][i] = sum x*w[0][p], M[1][r][i] = sum x*w[1][p], M[2][r][i] = sum x (int64)."""
    sel = mask.astype(bool)
    if valid is not None:
        sel &= valid.astype(bool)
    B = counts.shape[0] // 512
    rows = touched_blocks(B, k)
    w0 = weights[0][sel].astype(np.int64)
    w1 = weights[1][sel].astype(np.int64)
    out = np.zeros((3, len(rows), 512), np.int64)
    for r, b in enumerate(rows):
        x = counts[b * 512:(b + 1) * 512][:, sel].astype(np.int64)
        out[0, r] = x @ w0
        out[1, r] = x @ w1
        out[2, r] = x.sum(axis=1)
    return out


def dense_decode_blocks(counts: np.ndarray, first: int, n: int, valid: np.ndarray | None = None):
    out = counts[first * 512:(first + n) * 512].copy()
    if valid is not None:
        out[:, ~valid.astype(bool)] = 0
    return out


def dense_decode_range(counts: np.ndarray, first_scan: int, n_scans: int, valid: np.ndarray | None = None):
    """Plain definition of a scan-range decode: out[i][p] = valid[p] ? x[first_scan + i][p] : 0."""
    out = counts[first_scan:first_scan + n_scans].copy()
    if valid is not None:
        out[:, ~valid.astype(bool)] = 0
    return out


def masked_pixels(mask: np.ndarray, valid: np.ndarray | None = None) -> np.ndarray:
    sel = mask.astype(bool)
    if valid is not None:
        sel &= valid.astype(bool)
    return np.nonzero(sel)[0].astype(np.int32)


def delta_lists(old: np.ndarray, new: np.ndarray, valid: np.ndarray | None = None):
    """(pixels, signs): +1 for pixels entering the mask, -1 for pixels leaving it."""
    o = old.astype(bool)
    n = new.astype(bool)
    if valid is not None:
        o &= valid.astype(bool)
        n &= valid.astype(bool)
    add = np.nonzero(n & ~o)[0]
    rem = np.nonzero(o & ~n)[0]
    pix = np.concatenate([add, rem]).astype(np.int32)
    sign = np.concatenate([np.ones(add.size, np.int8), -np.ones(rem.size, np.int8)])
    order = np.argsort(pix, kind="stable")
    return pix[order], sign[order]


def resident_masked_sum(enc: Encoded, mask: np.ndarray, valid: np.ndarray | None = None,
                        k: int = 1, blocks=None, threads: int | None = None) -> np.ndarray:
    """Decode-based masked sum over the oracle-encoded resident (uint64 rows)."""
    pix = masked_pixels(mask, valid)
    sign = np.ones(pix.size, np.int8)
    rows = touched_blocks(enc.n_blocks, k) if blocks is None else list(blocks)
    out = np.zeros((len(rows), 512), np.uint64)

    def job(r):
        b = rows[r]
        out[r] = block_masked_sum(enc.groups[b], enc.payloads[b], enc.dtype_bits, enc.n_pixels,
                                  pix, sign).astype(np.uint64)

    with ThreadPoolExecutor(_workers(len(rows), threads)) as ex:
        list(ex.map(job, range(len(rows))))
    return out


def resident_delta(enc: Encoded, prev: np.ndarray, old: np.ndarray, new: np.ndarray,
                   valid: np.ndarray | None = None, k: int = 1, threads: int | None = None):
    """V_new = V_prev + sum(entering) - sum(leaving), in wide integers, then uint64."""
    pix, sign = delta_lists(old, new, valid)
    rows = touched_blocks(enc.n_blocks, k)
    out = prev.astype(np.int64).copy()

    def job(r):
        b = rows[r]
        out[r] += block_masked_sum(enc.groups[b], enc.payloads[b], enc.dtype_bits, enc.n_pixels,
                                   pix, sign)

    with ThreadPoolExecutor(_workers(len(rows), threads)) as ex:
        list(ex.map(job, range(len(rows))))
    assert (out >= 0).all()
    return out.astype(np.uint64)


def resident_decode_blocks(enc: Encoded, first: int, n: int, valid: np.ndarray | None = None):
    parts = [decode_block(enc.groups[b], enc.payloads[b], enc.dtype_bits, enc.n_pixels)
             for b in range(first, first + n)]
    out = np.concatenate(parts, axis=0)
    if valid is not None:
        out[:, ~valid.astype(bool)] = 0
    return out

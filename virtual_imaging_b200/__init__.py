"""B200-native paired-count resident for 4D-STEM counts (bitstream ``qem-pair-v2``).

Thin ctypes binding over ``libqem.so`` (declared in ``include/qem.h``): it only
marshals arguments -- torch tensors become device pointers, the current CUDA
stream becomes ``cudaStream_t`` -- and turns status codes into exceptions.
Every step of encoding, querying and decoding runs in the library's kernels.
There is no CPU fallback: without the built library (or a CUDA device) every
call raises.

Source: page "Paired-count resident layout" (quantem.gpu developer docs),
"Operation pipeline" steps 1-6 and "Contract".
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqem.so")

QEM_OK, QEM_ERR_ARG, QEM_ERR_MALFORMED, QEM_ERR_CUDA, QEM_ERR_OOM, QEM_ERR_TIMEOUT, QEM_ERR_TAINTED, QEM_ERR_STATE = range(8)
KERNELS = ("plan", "decode_reduce", "finalize", "decode_blocks", "enc_streams", "enc_layout", "enc_compact",
           "generate")
FORMS = ("empty", "constant", "sparse", "paired", "literal")

# every symbol include/qem.h declares
EXPORTS = ("qem_abi", "qem_status_string", "qem_create", "qem_encode", "qem_encode_append", "qem_masked_sum",
           "qem_masked_sum_delta", "qem_decode_blocks", "qem_finish", "qem_info", "qem_query_counters",
           "qem_profile", "qem_profile_read", "qem_free", "qem_block_bytes", "qem_export_block", "qem_import",
           "qem_model_tables", "qem_generate_counts", "qem_masked_sum_noalloc", "qem_build_index",
           "qem_drop_index", "qem_index_layout", "qem_index_desc", "qem_export_valid", "qem_save", "qem_load",
           "qem_decode_blocks_amplitude", "qem_masked_moments", "qem_polar_layout", "qem_decode_range",
           "qem_pixel_classes", "qem_masked_sum_complement")


class QemError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


class MalformedStream(QemError, ValueError):
    """A decoded stream failed a qem-pair-v2 check; the query has no result."""


class TaintedBaseline(QemError):
    """Delta refused: the stride's baseline was invalidated by a failed decode."""


class Info(ctypes.Structure):
    _fields_ = [("scan_rows", ctypes.c_int64), ("scan_cols", ctypes.c_int64), ("det_rows", ctypes.c_int32),
                ("det_cols", ctypes.c_int32), ("dtype_bits", ctypes.c_int32), ("n_pixels", ctypes.c_int32),
                ("n_valid", ctypes.c_int32), ("out_bits_auto", ctypes.c_int32), ("n_blocks", ctypes.c_int64),
                ("n_blocks_encoded", ctypes.c_int64), ("payload_bytes", ctypes.c_uint64),
                ("group_bytes", ctypes.c_uint64), ("device_bytes", ctypes.c_uint64),
                ("form_count", ctypes.c_uint64 * 5), ("model_count", ctypes.c_uint64 * 32),
                ("n_arenas", ctypes.c_int32), ("index_leaves", ctypes.c_int32), ("index_roots", ctypes.c_int32),
                ("index_bytes", ctypes.c_uint64)]


class Profile(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_int64 * 8), ("ms", ctypes.c_double * 8)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libqem.so; raises if it has not been built (no fallback exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m virtual_imaging_b200.build` "
                           "(the paired-count resident has no CPU path)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64
    pp = ctypes.POINTER(ctypes.c_void_p)
    sig = {
        "qem_abi": ([], ctypes.c_char_p),
        "qem_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "qem_create": ([i64, i64, i32, i32, i32, vp, vp, pp], ctypes.c_int),
        "qem_encode": ([vp, i32, i64, i64, i32, i32, vp, vp, pp], ctypes.c_int),
        "qem_encode_append": ([vp, vp, i64, vp], ctypes.c_int),
        "qem_masked_sum": ([vp, vp, i32, i32, vp, ctypes.POINTER(i32), i32, vp], ctypes.c_int),
        "qem_masked_sum_delta": ([vp, vp, i32, i32, vp, ctypes.POINTER(i32), i32, vp], ctypes.c_int),
        "qem_masked_sum_complement": ([vp, vp, i32, i32, vp, ctypes.POINTER(i32), i32, vp], ctypes.c_int),
        "qem_decode_blocks": ([vp, i64, i64, vp, i32, vp], ctypes.c_int),
        "qem_decode_range": ([vp, i64, i64, vp, i32, vp], ctypes.c_int),
        "qem_pixel_classes": ([vp, vp], ctypes.c_int),
        "qem_finish": ([vp, vp], ctypes.c_int),
        "qem_info": ([vp, ctypes.POINTER(Info)], ctypes.c_int),
        "qem_query_counters": ([vp, ctypes.POINTER(u64), ctypes.POINTER(u64), vp], ctypes.c_int),
        "qem_profile": ([vp, i32], ctypes.c_int),
        "qem_profile_read": ([vp, ctypes.POINTER(Profile)], ctypes.c_int),
        "qem_free": ([vp], None),
        "qem_block_bytes": ([vp, i64, ctypes.POINTER(u64)], ctypes.c_int),
        "qem_export_block": ([vp, i64, vp, vp, vp], ctypes.c_int),
        "qem_import": ([i64, i64, i32, i32, i32, vp, vp, vp, vp, vp, pp], ctypes.c_int),
        "qem_model_tables": ([vp, vp, vp], ctypes.c_int),
        "qem_generate_counts": ([vp, i32, u64, i64, i64, i32, vp, vp, vp, vp], ctypes.c_int),
        "qem_masked_sum_noalloc": ([vp, vp, i32, i32, vp, vp], ctypes.c_int),
        "qem_build_index": ([vp, ctypes.c_double, ctypes.c_double, vp], ctypes.c_int),
        "qem_drop_index": ([vp, vp], ctypes.c_int),
        "qem_index_layout": ([vp, vp, vp, ctypes.POINTER(i32), ctypes.POINTER(i32)], ctypes.c_int),
        "qem_index_desc": ([vp, vp], ctypes.c_int),
        "qem_export_valid": ([vp, vp], ctypes.c_int),
        "qem_save": ([vp, ctypes.c_char_p, vp], ctypes.c_int),
        "qem_load": ([ctypes.c_char_p, vp, pp], ctypes.c_int),
        "qem_decode_blocks_amplitude": ([vp, i64, i64, vp, vp, i32, vp], ctypes.c_int),
        "qem_masked_moments": ([vp, vp, vp, i32, vp, i32, vp], ctypes.c_int),
        "qem_polar_layout": ([i32, i32, vp, ctypes.c_double, ctypes.c_double, vp, vp, ctypes.POINTER(i32),
                              ctypes.POINTER(i32)], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def status_string(code: int) -> str:
    return lib().qem_status_string(code).decode()


def abi() -> str:
    return lib().qem_abi().decode()


def _check(code: int, where: str):
    if code == QEM_OK:
        return
    if code == QEM_ERR_MALFORMED:
        raise MalformedStream(code, where)
    if code == QEM_ERR_TAINTED:
        raise TaintedBaseline(code, where)
    raise QemError(code, where)


def _stream(stream=None) -> int:
    if stream is None:
        if not torch.cuda.is_available():
            return 0        # the default stream; calls that need a device then fail in the library
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dev_ptr(t: torch.Tensor | None) -> int:
    if t is None:
        return 0
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    return t.data_ptr()


def _count_dtype(bits: int):
    return torch.uint8 if bits == 8 else torch.uint16


def out_dtype(bits: int):
    """Torch storage for uint32/uint64 images (same bits, signed view)."""
    return torch.int32 if bits == 32 else torch.int64


def as_unsigned(img: torch.Tensor) -> np.ndarray:
    """Host copy of an image buffer as uint32/uint64."""
    a = img.detach().cpu().numpy()
    return a.view(np.uint32 if a.dtype == np.int32 else np.uint64)


class Resident:
    """An encoded acquisition resident on one GPU (owns all its device memory)."""

    def __init__(self, handle: ctypes.c_void_p):
        self._h = handle
        self._geom = None

    def _static(self):
        """(n_blocks, n_pixels, dtype_bits, out_bits_auto): fixed once the resident exists."""
        if self._geom is None:
            i = self.info()
            self._geom = (i["n_blocks"], i["n_pixels"], i["dtype_bits"], i["out_bits_auto"])
        return self._geom

    # ---- construction -------------------------------------------------------
    @classmethod
    def create(cls, scan_shape, det_shape, dtype_bits: int, valid: torch.Tensor | None = None, stream=None):
        h = ctypes.c_void_p()
        _check(lib().qem_create(scan_shape[0], scan_shape[1], det_shape[0], det_shape[1], dtype_bits,
                                _dev_ptr(valid), _stream(stream), ctypes.byref(h)), "qem_create")
        return cls(h)

    @classmethod
    def encode(cls, counts: torch.Tensor, scan_shape, det_shape, valid: torch.Tensor | None = None,
               stream=None):
        """Encode device counts [scans][pixels] (or 4-D) of uint8/uint16."""
        bits = 8 if counts.dtype == torch.uint8 else 16
        if counts.dtype not in (torch.uint8, torch.uint16):
            raise ValueError("counts must be uint8 or uint16")
        h = ctypes.c_void_p()
        _check(lib().qem_encode(_dev_ptr(counts), bits, scan_shape[0], scan_shape[1], det_shape[0], det_shape[1],
                                _dev_ptr(valid), _stream(stream), ctypes.byref(h)), "qem_encode")
        return cls(h)

    @classmethod
    def from_encoded(cls, scan_shape, det_shape, dtype_bits: int, groups: np.ndarray, payload: np.ndarray,
                     block_off: np.ndarray, valid: np.ndarray | None = None, stream=None):
        """Build a resident from a host encoded form (groups [B][G][17] u32, payload u8, offsets [B+1])."""
        g = np.ascontiguousarray(groups, np.uint32)
        p = np.ascontiguousarray(payload, np.uint8)
        if p.size == 0:
            p = np.zeros(1, np.uint8)
        o = np.ascontiguousarray(block_off, np.uint64)
        v = None if valid is None else np.ascontiguousarray(valid, np.uint8)
        h = ctypes.c_void_p()
        _check(lib().qem_import(scan_shape[0], scan_shape[1], det_shape[0], det_shape[1], dtype_bits,
                                g.ctypes.data, p.ctypes.data, o.ctypes.data,
                                None if v is None else v.ctypes.data, _stream(stream), ctypes.byref(h)),
               "qem_import")
        return cls(h)

    def append(self, counts: torch.Tensor, n_blocks: int, stream=None):
        _check(lib().qem_encode_append(self._h, _dev_ptr(counts), n_blocks, _stream(stream)),
               "qem_encode_append")

    # ---- queries ---------------------------------------------------------------
    def _query(self, fn, name, mask, block_stride, out_bits, out, wait, stream):
        if out is None:
            if block_stride < 1:
                raise QemError(QEM_ERR_ARG, name)
            n_blocks, _, _, auto = self._static()
            rows = -(-n_blocks // block_stride)
            bits = auto if out_bits == 0 else out_bits
            out = torch.empty((rows, 512), dtype=out_dtype(bits), device=mask.device)
        elif block_stride >= 1 and out_bits in (0, 32, 64):
            # the library writes ceil(B/k) x 512 values of the chosen width through a raw
            # pointer: a smaller or narrower buffer is refused here (other arguments are
            # the library's to refuse)
            n_blocks, _, _, auto = self._static()
            rows = -(-n_blocks // block_stride)
            bits = auto if out_bits == 0 else out_bits
            if out.dtype != out_dtype(bits) or out.numel() < rows * 512:
                raise ValueError(f"{name}: out must hold {rows} x 512 {out_dtype(bits)} values")
        _check(fn(self._h, _dev_ptr(mask), block_stride, out_bits, _dev_ptr(out), None,
                  1 if wait else 0, _stream(stream)), name)
        return out

    def masked_sum(self, mask: torch.Tensor, block_stride: int = 1, out_bits: int = 0,
                   out: torch.Tensor | None = None, wait: bool = True, stream=None) -> torch.Tensor:
        """Exact virtual image [ceil(B/k)][512] (int32/int64 storage of uint32/uint64)."""
        return self._query(lib().qem_masked_sum, "qem_masked_sum", mask, block_stride, out_bits, out, wait,
                           stream)

    def masked_sum_delta(self, mask: torch.Tensor, block_stride: int = 1, out_bits: int = 0,
                         out: torch.Tensor | None = None, wait: bool = True, stream=None) -> torch.Tensor:
        return self._query(lib().qem_masked_sum_delta, "qem_masked_sum_delta", mask, block_stride, out_bits,
                           out, wait, stream)

    def masked_sum_complement(self, mask: torch.Tensor, block_stride: int = 1, out_bits: int = 0,
                              out: torch.Tensor | None = None, wait: bool = True, stream=None) -> torch.Tensor:
        """The same image as masked_sum, as the cached full-detector image minus the valid pixels
        outside the mask (the cheaper route for dense masks such as a dark field)."""
        return self._query(lib().qem_masked_sum_complement, "qem_masked_sum_complement", mask, block_stride,
                           out_bits, out, wait, stream)

    def masked_sum_noalloc(self, mask: torch.Tensor, out: torch.Tensor, block_stride: int = 1,
                           out_bits: int = 0, stream=None) -> torch.Tensor:
        """Masked sum that allocates no device memory (qem_masked_sum_noalloc): for callers that
        must not allocate while querying.  `out` must be preallocated ([ceil(B/k)][512] of the
        chosen width); calls that overlap on the GPU race on the library's fixed working memory."""
        if block_stride >= 1 and out_bits in (0, 32, 64):
            n_blocks, _, _, auto = self._static()
            bits = auto if out_bits == 0 else out_bits
            if out.dtype != out_dtype(bits) or out.numel() < -(-n_blocks // block_stride) * 512:
                raise ValueError("qem_masked_sum_noalloc: out must hold ceil(B/k) x 512 values of the chosen width")
        _check(lib().qem_masked_sum_noalloc(self._h, _dev_ptr(mask), block_stride, out_bits, _dev_ptr(out),
                                            _stream(stream)), "qem_masked_sum_noalloc")
        return out

    def masked_moments(self, mask: torch.Tensor, weights: torch.Tensor, block_stride: int = 1,
                       out: torch.Tensor | None = None, wait: bool = True, stream=None) -> torch.Tensor:
        """int64 [3][ceil(B/k)][512]: (sum x*w0, sum x*w1, sum x) per scan over mask & valid pixels.
        weights: int32 [2][pixels] on the device, |w| <= 262143."""
        if out is None:
            n_blocks = self._static()[0]
            if block_stride < 1:
                raise QemError(QEM_ERR_ARG, "qem_masked_moments")
            out = torch.empty((3, -(-n_blocks // block_stride), 512), dtype=torch.int64, device=mask.device)
        _check(lib().qem_masked_moments(self._h, _dev_ptr(mask), _dev_ptr(weights), block_stride, _dev_ptr(out),
                                        1 if wait else 0, _stream(stream)), "qem_masked_moments")
        return out

    def decode_blocks(self, first: int, n: int, out: torch.Tensor | None = None, wait: bool = True,
                      stream=None) -> torch.Tensor:
        if out is None:
            _, n_pixels, bits, _ = self._static()
            out = torch.empty((n * 512, n_pixels), dtype=_count_dtype(bits),
                              device=torch.device("cuda", torch.cuda.current_device()))
        _check(lib().qem_decode_blocks(self._h, first, n, _dev_ptr(out), 1 if wait else 0, _stream(stream)),
               "qem_decode_blocks")
        return out

    def decode_range(self, first_scan: int, n_scans: int, out: torch.Tensor | None = None, wait: bool = True,
                     stream=None) -> torch.Tensor:
        """Counts of scans [first_scan, first_scan + n_scans) as [n_scans][pixels] (native dtype)."""
        if out is None:
            _, n_pixels, bits, _ = self._static()
            out = torch.empty((n_scans, n_pixels), dtype=_count_dtype(bits),
                              device=torch.device("cuda", torch.cuda.current_device()))
        _check(lib().qem_decode_range(self._h, first_scan, n_scans, _dev_ptr(out), 1 if wait else 0,
                                      _stream(stream)), "qem_decode_range")
        return out

    def frame(self, scan: int, out: torch.Tensor | None = None, wait: bool = True, stream=None) -> torch.Tensor:
        """One diffraction pattern (scan index scan_row * scan_cols + scan_col) as [det_rows][det_cols]."""
        i = self.info()
        return self.decode_range(scan, 1, out, wait, stream).view(i["det_rows"], i["det_cols"])

    # ---- interaction index ----------------------------------------------------
    def build_index(self, center=None, stream=None):
        """Build the interaction index about `center` (detector row, col; default the detector centre)."""
        if center is None:
            i = self.info()
            center = ((i["det_rows"] - 1) / 2.0, (i["det_cols"] - 1) / 2.0)
        _check(lib().qem_build_index(self._h, float(center[0]), float(center[1]), _stream(stream)),
               "qem_build_index")

    def drop_index(self, stream=None):
        _check(lib().qem_drop_index(self._h, _stream(stream)), "qem_drop_index")

    def index_layout(self):
        """(slots int64 [leaves][64] with n_pixels for unused slots, root_leaf0 int64 [roots + 1])."""
        nl, nr = ctypes.c_int32(0), ctypes.c_int32(0)
        _check(lib().qem_index_layout(self._h, None, None, ctypes.byref(nl), ctypes.byref(nr)), "qem_index_layout")
        slots = np.zeros((nl.value, 64), np.uint32)
        roots = np.zeros(nr.value + 1, np.int32)
        _check(lib().qem_index_layout(self._h, slots.ctypes.data, roots.ctypes.data, None, None), "qem_index_layout")
        return slots.astype(np.int64), roots.astype(np.int64)

    # ---- saved form -------------------------------------------------------------
    def save(self, path: str, stream=None):
        """Write the resident's saved form (QGPUPAIR file) to `path`."""
        _check(lib().qem_save(self._h, os.fsencode(path), _stream(stream)), "qem_save")

    @classmethod
    def load(cls, path: str, stream=None):
        """Reopen a saved form written by save()."""
        h = ctypes.c_void_p()
        _check(lib().qem_load(os.fsencode(path), _stream(stream), ctypes.byref(h)), "qem_load")
        return cls(h)

    def valid(self) -> np.ndarray:
        i = self.info()
        v = np.zeros(i["n_pixels"], np.uint8)
        _check(lib().qem_export_valid(self._h, v.ctypes.data), "qem_export_valid")
        return v

    def pixel_classes(self) -> np.ndarray:
        """uint8 [pixels]: 1 for light streams (empty, sparse, run-decoded), 0 for pair-by-pair ones."""
        i = self.info()
        c = np.zeros(i["n_pixels"], np.uint8)
        _check(lib().qem_pixel_classes(self._h, c.ctypes.data), "qem_pixel_classes")
        return c

    def index_desc(self):
        """uint32 [n_blocks][leaves + roots] storage descriptors (width code in bits 30-31)."""
        i = self.info()
        d = np.zeros((i["n_blocks"], i["index_leaves"] + i["index_roots"]), np.uint32)
        _check(lib().qem_index_desc(self._h, d.ctypes.data), "qem_index_desc")
        return d

    def decode_blocks_amplitude(self, first: int, n: int, counts: torch.Tensor | None = None,
                                amp: torch.Tensor | None = None, wait: bool = True, stream=None):
        """(counts [n*512][P] native, amplitude float32 sqrt(counts) of the same shape)."""
        _, n_pixels, bits, _ = self._static()
        dev = torch.device("cuda", torch.cuda.current_device())
        if counts is None:
            counts = torch.empty((n * 512, n_pixels), dtype=_count_dtype(bits), device=dev)
        if amp is None:
            amp = torch.empty((n * 512, n_pixels), dtype=torch.float32, device=dev)
        _check(lib().qem_decode_blocks_amplitude(self._h, first, n, _dev_ptr(counts), _dev_ptr(amp),
                                                 1 if wait else 0, _stream(stream)), "qem_decode_blocks_amplitude")
        return counts, amp

    def finish(self, stream=None):
        _check(lib().qem_finish(self._h, _stream(stream)), "qem_finish")

    # ---- introspection ---------------------------------------------------------
    def info(self) -> dict:
        i = Info()
        _check(lib().qem_info(self._h, ctypes.byref(i)), "qem_info")
        d = {k: getattr(i, k) for k, _ in Info._fields_}
        d["form_count"] = dict(zip(FORMS, list(i.form_count)))
        d["model_count"] = list(i.model_count)
        return d

    def counters(self, stream=None):
        rows, streams = ctypes.c_uint64(0), ctypes.c_uint64(0)
        _check(lib().qem_query_counters(self._h, ctypes.byref(rows), ctypes.byref(streams), _stream(stream)),
               "qem_query_counters")
        return rows.value, streams.value

    def profile(self, enable: bool = True):
        _check(lib().qem_profile(self._h, 1 if enable else 0), "qem_profile")

    def profile_read(self) -> dict:
        p = Profile()
        _check(lib().qem_profile_read(self._h, ctypes.byref(p)), "qem_profile_read")
        return {k: (int(p.launches[i]), float(p.ms[i])) for i, k in enumerate(KERNELS)}

    def export_block(self, b: int, stream=None):
        """(groups uint32 [G][17], payload uint8) of block b."""
        n = ctypes.c_uint64(0)
        _check(lib().qem_block_bytes(self._h, b, ctypes.byref(n)), "qem_block_bytes")
        info = self.info()
        G = (info["n_pixels"] + 31) // 32
        groups = np.zeros((G, 17), np.uint32)
        payload = np.zeros(max(1, n.value), np.uint8)
        _check(lib().qem_export_block(self._h, b, groups.ctypes.data, payload.ctypes.data, _stream(stream)),
               "qem_export_block")
        return groups, payload[: n.value]

    def free(self):
        if self._h:
            lib().qem_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def polar_layout(det_rows: int, det_cols: int, center, valid: np.ndarray | None = None):
    """Host-only: (slots int64 [leaves][64], root_leaf0 int64 [roots + 1]) of the index layout."""
    v = None if valid is None else np.ascontiguousarray(valid, np.uint8)
    nl, nr = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib().qem_polar_layout(det_rows, det_cols, None if v is None else v.ctypes.data, float(center[0]),
                                  float(center[1]), None, None, ctypes.byref(nl), ctypes.byref(nr)),
           "qem_polar_layout")
    slots = np.zeros((nl.value, 64), np.uint32)
    roots = np.zeros(nr.value + 1, np.int32)
    _check(lib().qem_polar_layout(det_rows, det_cols, None if v is None else v.ctypes.data, float(center[0]),
                                  float(center[1]), slots.ctypes.data, roots.ctypes.data, None, None),
           "qem_polar_layout")
    return slots.astype(np.int64), roots.astype(np.int64)


def model_tables():
    f = np.zeros((32, 256), np.uint16)
    a = np.zeros(32, np.uint8)
    c = np.zeros((32, 16), np.uint32)
    _check(lib().qem_model_tables(f.ctypes.data, a.ctypes.data, c.ctypes.data), "qem_model_tables")
    return f, a, c


def generate_counts(out: torch.Tensor, dtype_bits: int, seed: int, scan0: int, n_scans: int, n_pixels: int,
                    pixel_class: torch.Tensor, class_desc: torch.Tensor, thresholds: torch.Tensor, stream=None):
    """Counter-based synthetic counts on the device (see qem_generate_counts)."""
    _check(lib().qem_generate_counts(_dev_ptr(out), dtype_bits, seed, scan0, n_scans, n_pixels,
                                     _dev_ptr(pixel_class), _dev_ptr(class_desc), _dev_ptr(thresholds),
                                     _stream(stream)), "qem_generate_counts")
    return out

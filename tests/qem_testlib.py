"""Helpers shared by the GPU tests: move workloads to the device, build residents
from GPU or oracle encodings, and compare through the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import virtual_imaging_b200 as V
import workloads as W


def device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    V.lib()
    return torch.device("cuda", torch.cuda.current_device())


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device())


def gpu_encode(w: W.Workload, counts: np.ndarray, valid: np.ndarray | None = None) -> V.Resident:
    return V.Resident.encode(to_dev(counts), (w.scan_rows, w.scan_cols), (w.det_rows, w.det_cols),
                             None if valid is None else to_dev(valid))


def oracle_resident(w: W.Workload, enc: O.Encoded, valid: np.ndarray | None = None,
                    payloads=None, groups=None) -> V.Resident:
    """Upload an oracle-encoded form through the library's import entry point."""
    payloads = enc.payloads if payloads is None else payloads
    groups = enc.groups if groups is None else groups
    off = np.zeros(len(payloads) + 1, np.uint64)
    off[1:] = np.cumsum([p.size for p in payloads])
    payload = np.concatenate(payloads) if payloads else np.zeros(0, np.uint8)
    g = np.stack(groups).astype(np.uint32)
    return V.Resident.from_encoded((w.scan_rows, w.scan_cols), (w.det_rows, w.det_cols), w.dtype_bits, g,
                                   payload, off, valid)


def image(res: V.Resident, mask: np.ndarray, k: int = 1, delta: bool = False, out_bits: int = 0) -> np.ndarray:
    m = to_dev(mask.astype(np.uint8))
    fn = res.masked_sum_delta if delta else res.masked_sum
    return V.as_unsigned(fn(m, block_stride=k, out_bits=out_bits)).astype(np.uint64)


def export_all(res: V.Resident, n_blocks: int):
    return [res.export_block(b) for b in range(n_blocks)]

"""Readers for the golden fixtures under tests/golden/ (plain text, cited there)."""
from __future__ import annotations

import hashlib
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def frozen_tables():
    """The frozen pair models of model_tables.txt: (sha256, freq [32][256], box [32], cost [32][16])."""
    digest, freq, box, cost = None, [], [], []
    for line in open(os.path.join(GOLDEN, "model_tables.txt")):
        parts = line.split()
        if not parts or parts[0].startswith("#"):
            continue
        if parts[0] == "sha256":
            digest = parts[1]
        elif parts[0] == "model":
            assert int(parts[1]) == len(box)
            box.append(int(parts[3]))
        elif parts[0] == "cost":
            cost.append([int(v) for v in parts[1:]])
        elif parts[0] == "freq":
            freq.append([int(v) for v in parts[1:]])
    return (digest, np.asarray(freq, np.uint16), np.asarray(box, np.uint8), np.asarray(cost, np.uint32))


def tables_sha(freq, box, cost) -> str:
    """SHA-256 of freq <u2 [32][256] | box u1 [32] | cost <u4 [32][16]."""
    return hashlib.sha256(np.asarray(freq, "<u2").tobytes() + np.asarray(box, "u1").tobytes() +
                          np.asarray(cost, "<u4").tobytes()).hexdigest()

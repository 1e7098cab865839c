"""Write tests/golden/model_tables.txt from the CPU oracle's rebuild of the
32 Poisson pair models (page "Paired-count resident layout", "Operation
pipeline" step 2: a 1024-state tANS table from 32 Poisson pair models;
section "Contract": the coding parameters are fixed by the ABI string).

The file freezes the models of the bitstream qem-pair-v2: per model its box
(largest codable count), its 16 selection costs and its 256 pair frequencies,
plus the SHA-256 of their canonical bytes:

    freq  uint16 little-endian [32][256]   (pair (a, b) at a + 16 b)
    box   uint8 [32]
    cost  uint32 little-endian [32][16]    (0xFFFFFFFF outside the box)

concatenated in that order.  Only the oracle is called here.

Usage: python tests/golden/make_model_tables.py
"""
from __future__ import annotations

import hashlib
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

OUT = os.path.join(HERE, "model_tables.txt")


def canonical_bytes(freq, box, cost) -> bytes:
    import numpy as np

    return (np.asarray(freq, "<u2").tobytes() + np.asarray(box, "u1").tobytes() +
            np.asarray(cost, "<u4").tobytes())


def main() -> None:
    import oracle as O

    freq, box, cost = O.models()
    digest = hashlib.sha256(canonical_bytes(freq, box, cost)).hexdigest()
    lines = [
        "# Frozen pair models of qem-pair-v2 (spec S4), written by make_model_tables.py from the oracle.",
        "# Page \"Paired-count resident layout\", Operation pipeline step 2 (32 Poisson pair models,",
        "# 1024-state tANS) and Contract (coding parameters fixed by the ABI string).",
        "# sha256 covers freq <u2 [32][256] | box u1 [32] | cost <u4 [32][16], in that order.",
        f"sha256 {digest}",
    ]
    for m in range(32):
        lines.append(f"model {m} box {int(box[m])}")
        lines.append("cost " + " ".join(str(int(v)) for v in cost[m]))
        lines.append("freq " + " ".join(str(int(v)) for v in freq[m]))
    with open(OUT, "w") as f:
        f.write("\n".join(lines) + "\n")
    print(OUT, digest)


if __name__ == "__main__":
    main()

"""Feeding a consumer from the resident form (page "Paired-count resident
layout", "Operation pipeline" step 6: the blocks of a series are decoded on
a prefetch stream, `depth` buffers ahead, with events in both directions, so
a reconstruction reads native counts, and optionally their float32 square-
root amplitude, without a dense copy of the acquisition).

Every decode runs in the library's kernels (qem_decode_blocks and
qem_decode_blocks_amplitude); this module only orders them on CUDA streams.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import Resident


@dataclass
class FeedItem:
    source: int              # index of the resident in the series
    first_block: int         # first 512-scan block of the batch
    n_blocks: int
    counts: torch.Tensor     # native [n_blocks * 512][pixels], valid until the next item is requested
    amplitude: torch.Tensor | None


class Feed:
    """Iterate the blocks of one or more residents, `blocks` at a time.

    Decodes run on a side stream, up to `depth` batches ahead of the consumer;
    each yielded item's tensors are ready on the consumer's stream (it waits on
    the decode's event), and a buffer is reused only after the consumer's
    stream has passed the point where the next item was requested (an event
    recorded there), so consumer work queued on that stream may keep reading
    an item until it asks for the next one.
    """

    def __init__(self, sources: list[Resident], blocks: int = 1, amplitude: bool = False, depth: int = 2,
                 stream: torch.cuda.Stream | None = None):
        if blocks < 1 or depth < 1:
            raise ValueError("blocks and depth must be >= 1")
        self.sources = list(sources)
        self.blocks = blocks
        self.amplitude = amplitude
        self.depth = depth
        self.consumer = stream or torch.cuda.current_stream()
        self.side = torch.cuda.Stream(device=self.consumer.device)
        self.plan = []
        for si, r in enumerate(self.sources):
            nb = r.info()["n_blocks"]
            for b0 in range(0, nb, blocks):
                self.plan.append((si, b0, min(blocks, nb - b0)))

    def __len__(self):
        return len(self.plan)

    def __iter__(self):
        dev = self.consumer.device
        bufs = []
        for _ in range(self.depth):
            bufs.append({"free": None, "ready": None, "item": None})
        shapes = {}

        def start(k):
            si, b0, nb = self.plan[k]
            r = self.sources[si]
            slot = bufs[k % self.depth]
            info = r.info()
            shape = (nb * 512, info["n_pixels"])
            dtype = torch.uint8 if info["dtype_bits"] == 8 else torch.uint16
            key = (k % self.depth, shape, dtype)
            if shapes.get(k % self.depth) != key:
                slot["counts"] = torch.empty(shape, dtype=dtype, device=dev)
                slot["amp"] = torch.empty(shape, dtype=torch.float32, device=dev) if self.amplitude else None
                shapes[k % self.depth] = key
            if slot["free"] is not None:
                self.side.wait_event(slot["free"])
            if self.amplitude:
                r.decode_blocks_amplitude(b0, nb, slot["counts"], slot["amp"], wait=False, stream=self.side)
            else:
                r.decode_blocks(b0, nb, out=slot["counts"], wait=False, stream=self.side)
            ev = torch.cuda.Event()
            ev.record(self.side)
            slot["ready"] = ev
            slot["item"] = FeedItem(si, b0, nb, slot["counts"], slot["amp"])

        n = len(self.plan)
        for k in range(min(self.depth, n)):
            start(k)
        for k in range(n):
            slot = bufs[k % self.depth]
            self.consumer.wait_event(slot["ready"])
            yield slot["item"]
            # the consumer has asked for the next item: its stream, from here
            # on, no longer reads this buffer
            free = torch.cuda.Event()
            free.record(self.consumer)
            slot["free"] = free
            if k + self.depth < n:
                start(k + self.depth)
        for r in self.sources:
            r.finish(stream=self.side)

"""Block-by-block decode that overlaps the next block's decode with this block's compute.

The pages keep every weight coded in GPU memory and decode a transformer block's weights into a
buffer just before that block runs, alternating decompression and forward kernels ("Float8@2bits"
summary, "Decodificacion en Tiempo de Inferencia"; DFloat11 page, "Descompresion por bloque
transformer").  BlockPipeline does that with two decode buffers and a side stream: while block i
computes on the caller's stream out of buffer i % 2, block i + 1 decodes into the other buffer;
CUDA events order the two streams, nothing on the host waits.
"""
from __future__ import annotations

import torch

from . import api


class BlockPipeline:
    def __init__(self, blocks, device=None):
        """blocks: list (one per transformer block) of lists of DeviceRans; every block has the
        same tensor shapes, position by position."""
        self.blocks = [list(b) for b in blocks]
        if not self.blocks:
            raise ValueError("no blocks")
        shapes = [(t.rows, t.cols) for t in self.blocks[0]]
        for b in self.blocks:
            if [(t.rows, t.cols) for t in b] != shapes:
                raise ValueError("blocks differ in shape")
        dev = torch.device(device) if device is not None else self.blocks[0][0].words.device
        self.device = dev
        self.bufs = [[torch.empty(r, c, dtype=torch.bfloat16, device=dev) for r, c in shapes]
                     for _ in range(2)]
        self.status = api.new_status(dev)
        self.side = torch.cuda.Stream(dev)

    def run(self, compute, overlap: bool = True) -> None:
        """compute(i, weights) enqueues block i's work on the current stream, reading the decoded
        bf16 weights (a list, same order as the block's tensors).  With overlap=False every
        decode runs on the current stream right before its block."""
        main = torch.cuda.current_stream(self.device)
        n = len(self.blocks)
        if not overlap:
            for i in range(n):
                api.decode(self.blocks[i], self.bufs[i % 2], self.status, main)
                compute(i, self.bufs[i % 2])
            return
        ready = [torch.cuda.Event() for _ in range(2)]
        free = [torch.cuda.Event() for _ in range(2)]
        self.side.wait_stream(main)  # the caller's earlier work (uploads, zeroed status) first

        def decode_into(i):
            b = i % 2
            self.side.wait_event(free[b])  # block i - 2 is done reading this buffer
            api.decode(self.blocks[i], self.bufs[b], self.status, self.side)
            ready[b].record(self.side)

        decode_into(0)
        for i in range(n):
            if i + 1 < n:
                decode_into(i + 1)
            main.wait_event(ready[i % 2])
            compute(i, self.bufs[i % 2])
            free[i % 2].record(main)
        main.wait_stream(self.side)

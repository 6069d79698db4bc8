"""Decompress transformer blocks ahead of their use.

The pages decompress all DF11 matrices of a transformer block as one batch
right before that block's forward pass, and drop the BF16 copy once the matrix
multiplications are done ("DFloat11: compressao sem perda para inferencia em
GPU ...", sections "Descompressao adaptada para inferencia em GPU" and
"Descompressao por bloco de transformer").  `BlockPrefetcher` runs that
pattern with the decode of block i+1 on a side CUDA stream, into the spare one
of a few reused BF16 buffers, while the caller computes with block i on its own
stream; CUDA events order every buffer reuse after the caller's work on it.
"""
from __future__ import annotations

import torch

from .codec import CompressedStream, decode_options, decompress


class BlockPrefetcher:
    """Iterate over compressed blocks with the next block's decode overlapped.

    Iterating yields ``(i, views)``: block i's matrices as BF16 views, ready
    for use on the stream that was current when iteration started.  Work that
    the caller enqueues on that stream before asking for the next block is
    ordered before the buffer holding block i is overwritten; keep no view
    past that point without copying it.

    n_buffers   BF16 buffers cycled through (2 = double buffering)
    max_sms     cap on the SMs each decode occupies (None = all), so that the
                caller's kernels can run beside it
    options     decode options (decode_options), e.g. many small CTAs that
                queue behind the caller's kernels and fill the SMs they leave
                idle; overrides max_sms
    status      optional int32 device word, OR-ed with DF11_ERR_CORRUPT by a
                decode that finds its stream inconsistent
    split       None, or the fraction of block i+1's thread blocks decoded on
                at most side_sms SMs while the caller works on block i; the
                rest is decoded on every SM once the caller's work on block i
                is done.  For consumers that leave SMs idle: cuBLAS's BF16
                GEMMs on B200 run 128 CTAs, one per SM, on 128 of 148 SMs.
    side_sms    SMs for the overlapped part (split mode)
    """

    def __init__(self, streams: list[CompressedStream], n_buffers: int = 2, max_sms: int | None = None,
                 status: torch.Tensor | None = None, decode_stream: torch.cuda.Stream | None = None,
                 options=None, split: float | None = None, side_sms: int = 20):
        if n_buffers < 2:
            raise ValueError("n_buffers must be at least 2")
        if not streams:
            raise ValueError("no blocks")
        self.streams = list(streams)
        if split is not None and not 0.0 <= split <= 1.0:
            raise ValueError("split must lie in [0, 1]")
        self.max_sms = max_sms
        self.options = options
        self.split = split
        self.side_sms = side_sms
        self.status = status
        dev = self.streams[0].exp.device
        n_max = max(max(cs.n_elems for cs in self.streams), 1)
        self.buffers = [torch.empty(n_max, dtype=torch.bfloat16, device=dev) for _ in range(n_buffers)]
        self.decode_stream = decode_stream or torch.cuda.Stream(device=dev)

    def __len__(self) -> int:
        return len(self.streams)

    def _decode(self, i: int, options=None) -> None:
        cs = self.streams[i]
        slot = i % len(self.buffers)
        decompress(cs, out=self.buffers[slot][: cs.n_elems], status=self.status, stream=self.decode_stream,
                   max_sms=None if options is not None else self.max_sms,
                   options=options if options is not None else self.options)

    def _launch(self, i: int, free: list) -> torch.cuda.Event | None:
        """Block i's decode (split mode: its first part only); returns the
        event that marks it ready, or None when a second part follows."""
        slot = i % len(self.buffers)
        if free[slot] is not None:
            self.decode_stream.wait_event(free[slot])
        if self.split is None:
            self._decode(i)
        else:
            cut = int(self.streams[i].header.n_blocks * self.split)
            if cut > 0:
                self._decode(i, decode_options(max_sms=self.side_sms, block_begin=0, block_end=cut))
            return None
        ready = torch.cuda.Event()
        ready.record(self.decode_stream)
        return ready

    def _finish(self, i: int) -> torch.cuda.Event:
        """Split mode: the rest of block i on every SM."""
        nb = int(self.streams[i].header.n_blocks)
        cut = int(nb * self.split)
        if cut < nb:
            self._decode(i, decode_options(block_begin=cut, block_end=nb))
        ready = torch.cuda.Event()
        ready.record(self.decode_stream)
        return ready

    def __iter__(self):
        compute = torch.cuda.current_stream()
        # the compressed arrays may have been written on the caller's stream
        self.decode_stream.wait_stream(compute)
        free = [None] * len(self.buffers)
        ready = self._launch(0, free)
        if ready is None:
            ready = self._finish(0)
        for i, cs in enumerate(self.streams):
            compute.wait_event(ready)
            nxt = i + 1 < len(self.streams)
            if nxt:
                ready = self._launch(i + 1, free)
            slot = i % len(self.buffers)
            yield i, cs.views(self.buffers[slot][: cs.n_elems])
            done = torch.cuda.Event()
            done.record(compute)
            free[slot] = done
            if nxt and ready is None:  # split: the rest after the caller's work on block i
                self.decode_stream.wait_event(done)
                ready = self._finish(i + 1)

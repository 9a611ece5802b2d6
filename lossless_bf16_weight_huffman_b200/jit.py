"""Just-in-time, layer-by-layer decode that runs ahead of the compute using it.

mlx-dfloat (PyPI page), "Status" and "Measured numbers": blocks are decoded
on the GPU just before they are used, with a run-ahead of one or two blocks,
and the cost is reported per step against weights kept as BF16. This module is
that schedule on CUDA streams: while the caller computes with layer l on its
stream, layers l+1 .. l+depth are decoded on a side stream into a ring of
depth+1 buffer sets; CUDA events order each decode after the computation
that last read its buffer set, and each computation after its layer's decode.
Every decode is one grouped launch of the layer's tensors (df_decode_batch_run
for the Huffman format, df_nf12_decode_batch_run for the fixed 12-bit one).

HostLayerStreamer adds the copy of each layer's container from pinned host
memory into device staging buffers on a copy stream, one layer ahead of the
decode, so that the weights need not stay in HBM at all.
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch

from . import api, codec, nf12


def _flat_views(buf: torch.Tensor, sizes: Sequence[int]) -> list[torch.Tensor]:
    views, off = [], 0
    for n in sizes:
        views.append(buf[off: off + n])
        off += n
    return views


def _device_of(c) -> torch.device:
    return c.slots.device if isinstance(c, nf12.Nf12) else c.stream.device


def _batch_decoder(comps, views, max_ctas: int):
    """One prepared grouped launch over a layer's containers: the Huffman
    format's (df_decode_batch_*) or the fixed 12-bit format's
    (df_nf12_decode_batch_*)."""
    if all(isinstance(c, nf12.Nf12) for c in comps):
        return nf12.BatchDecoder(comps, views)
    if any(isinstance(c, nf12.Nf12) for c in comps):
        raise TypeError("a layer mixes the two formats")
    dec = codec.BatchDecoder(comps, views)
    dec.plan.max_ctas = max_ctas
    return dec


class LayerStreamer:
    """Decode `layers` (each a list of device-resident containers, of either
    format) one layer at a time into a ring of depth+1 buffer sets, `depth`
    layers ahead of the consumer. depth=0 decodes each layer on the
    consumer's own stream right before it is used (no overlap). max_ctas caps
    the CUDA blocks of a Huffman-format decode (0: all that fit)."""

    def __init__(self, layers: Sequence[Sequence[codec.Compressed]], depth: int = 1, max_ctas: int = 0,
                 device=None):
        if depth < 0:
            raise ValueError("depth must be >= 0")
        if not layers:
            raise ValueError("no layers")
        self.layers = [list(l) for l in layers]
        self.depth = depth
        dev = torch.device(device) if device is not None else _device_of(self.layers[0][0])
        self.device = dev
        self.nslots = depth + 1
        cap = max(sum(c.n for c in l) for l in self.layers)
        self.bufs = [torch.empty(max(cap, 1), dtype=torch.int16, device=dev) for _ in range(self.nslots)]
        self.side = torch.cuda.Stream(dev) if depth > 0 else None
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        # one prepared grouped launch per (layer, slot): the plans hold the
        # output pointers, so they are built once
        self.decoders = []
        self.views = []
        for l in self.layers:
            per_slot, per_views = [], []
            for s in range(self.nslots):
                views = _flat_views(self.bufs[s], [c.n for c in l])
                per_slot.append(_batch_decoder(l, views, max_ctas))
                per_views.append(views)
            self.decoders.append(per_slot)
            self.views.append(per_views)
        torch.cuda.synchronize(dev)
        self.ready = [torch.cuda.Event() for _ in range(self.nslots)]
        self.free = [torch.cuda.Event() for _ in range(self.nslots)]

    def _issue(self, l: int) -> None:
        s = l % self.nslots
        self.side.wait_event(self.free[s])  # the computation that last read this set is done
        self.decoders[l][s].run(self.err, self.side)
        self.ready[s].record(self.side)

    def run(self, consume: Callable[[int, list[torch.Tensor]], None]) -> None:
        """consume(l, views) is called for every layer in order, on the
        current stream, with the layer's tensors decoded into `views` (flat
        int16 tensors holding the BF16 bit patterns)."""
        main = torch.cuda.current_stream(self.device)
        n = len(self.layers)
        if self.depth == 0:
            for l in range(n):
                self.decoders[l][0].run(self.err, main)
                consume(l, self.views[l][0])
            return
        for s in range(self.nslots):  # every buffer set starts free
            self.free[s].record(main)
        for l in range(min(self.depth, n)):
            self._issue(l)
        for l in range(n):
            if l + self.depth < n:
                self._issue(l + self.depth)
            s = l % self.nslots
            main.wait_event(self.ready[s])
            consume(l, self.views[l][s])
            self.free[s].record(main)

    def errors(self) -> int:
        """The OR of the decode error flags so far (waits for the device)."""
        return api.df_read_error(self.err)


class HostLayerStreamer:
    """Layers whose containers sit in pinned host memory: each layer's parts
    are copied into one of two device staging sets on a copy stream, decoded
    on a decode stream into one of two output sets, and handed to the
    consumer on its stream; copy, decode and consumption of consecutive layers
    overlap."""

    PARTS = ("stream", "gaps", "index", "sm")  # index: uint64 offsets or the compact index

    def __init__(self, layers: Sequence[Sequence[codec.Compressed]], device=None):
        self.layers = [list(l) for l in layers]
        dev = torch.device(device) if device is not None else self.layers[0][0].stream.device
        self.device = dev
        # pinned host copies of every container part
        self.host = [[{k: self._part(c, k).cpu().pin_memory() for k in self.PARTS} for c in l] for l in self.layers]
        # two device staging sets, each sized for the largest layer, and
        # containers that point into them
        self.stage = []
        for s in range(2):
            bufs = {}
            for k in self.PARTS:
                need = max(sum(self.host[i][j][k].numel() * self.host[i][j][k].element_size()
                               for j in range(len(self.layers[i]))) for i in range(len(self.layers)))
                bufs[k] = torch.empty(max(need, 16) + 16 * max(len(l) for l in self.layers), dtype=torch.uint8,
                                      device=dev)
            self.stage.append(bufs)
        self.h2d_bytes = sum(self.host[i][j][k].numel() * self.host[i][j][k].element_size()
                             for i in range(len(self.layers)) for j in range(len(self.layers[i])) for k in self.PARTS)
        self.copy = torch.cuda.Stream(dev)
        self.dec = torch.cuda.Stream(dev)
        cap = max(sum(c.n for c in l) for l in self.layers)
        self.outs = [torch.empty(max(cap, 1), dtype=torch.int16, device=dev) for _ in range(2)]
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.decoders = []
        for i, l in enumerate(self.layers):
            per = []
            for s in range(2):
                comps = [self._staged(c, i, j, s) for j, c in enumerate(l)]
                views = _flat_views(self.outs[s], [c.n for c in l])
                per.append((codec.BatchDecoder(comps, views), views))
            self.decoders.append(per)
        torch.cuda.synchronize(dev)
        self.copied = [torch.cuda.Event() for _ in range(2)]
        self.stage_free = [torch.cuda.Event() for _ in range(2)]
        self.decoded = [torch.cuda.Event() for _ in range(2)]
        self.out_free = [torch.cuda.Event() for _ in range(2)]

    @staticmethod
    def _part(c: codec.Compressed, k: str) -> torch.Tensor:
        t = getattr(c, k)
        return t[: c.n] if k == "sm" else t

    def _staged(self, c: codec.Compressed, i: int, j: int, s: int) -> codec.Compressed:
        """A container whose parts live in staging set s at 16-byte-aligned offsets."""
        parts = {}
        for k in self.PARTS:
            off = 0
            for jj in range(j):
                h = self.host[i][jj][k]
                off += (h.numel() * h.element_size() + 15) // 16 * 16
            h = self.host[i][j][k]
            view = self.stage[s][k][off: off + h.numel() * h.element_size()]
            parts[k] = view.view(h.dtype)
        u64 = c.offsets is not None
        return codec.Compressed(n=c.n, shape=c.shape, code=c.code, lut=c.lut, sizes=c.sizes,
                                chunk_bytes=c.chunk_bytes, threads_per_block=c.threads_per_block,
                                stream=parts["stream"], gaps=parts["gaps"], offsets=parts["index"] if u64 else None,
                                sm=parts["sm"], index8=None if u64 else parts["index"], index8_wide=c.index8_wide)

    def _copy_in(self, i: int) -> None:
        s = i % 2
        self.copy.wait_event(self.stage_free[s])
        with torch.cuda.stream(self.copy):
            for j, c in enumerate(self.layers[i]):
                dc = self.decoders[i][s][0].comps[j]
                for k in self.PARTS:
                    getattr(dc, k).copy_(self.host[i][j][k], non_blocking=True)
        self.copied[s].record(self.copy)

    def run(self, consume: Callable[[int, list[torch.Tensor]], None]) -> None:
        main = torch.cuda.current_stream(self.device)
        n = len(self.layers)
        for s in range(2):
            self.stage_free[s].record(main)
            self.out_free[s].record(main)
        self._copy_in(0)
        for i in range(n):
            s = i % 2
            if i + 1 < n:
                self._copy_in(i + 1)
            self.dec.wait_event(self.copied[s])
            self.dec.wait_event(self.out_free[s])
            dec, views = self.decoders[i][s]
            dec.run(self.err, self.dec)
            self.stage_free[s].record(self.dec)
            self.decoded[s].record(self.dec)
            main.wait_event(self.decoded[s])
            consume(i, views)
            self.out_free[s].record(main)

    def errors(self) -> int:
        return api.df_read_error(self.err)

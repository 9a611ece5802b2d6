"""The fixed 12-bit format (include/nf12.h) at the tensor level: compress a
BF16 CUDA tensor into slots, bitmap and side buffer, and decode one or many
tensors. Every step runs in libdf11.so; CPU tensors are rejected.

Fixed 12-bit format: agihunt.info, "Developer open-sources nf12: lossless
12-bit compression for BF16 models", section "Confirmed".
"""
from __future__ import annotations

import numpy as np
import torch

from . import api
from ._native import DF_NF12_TOP, DfNf12EncodeTensor, DfNf12Tensor
from .codec import _as_u16


class Nf12:
    """One tensor in the fixed 12-bit format, in device memory."""

    def __init__(self, *, n, shape, top, slots, bitmap, side, n_escaped):
        self.n = int(n)
        self.shape = tuple(shape)
        self.top = int(top)
        self.slots = slots
        self.bitmap = bitmap
        self.side = side
        self.n_escaped = int(n_escaped)

    @property
    def groups(self) -> int:
        return (self.n + 7) // 8

    @property
    def container_bytes(self) -> int:
        """Slots + bitmap + side entries (12 B per group, 16 B more per escaped group)."""
        return 12 * self.groups + 4 * ((self.groups + 31) // 32) + 16 * self.n_escaped

    @property
    def ratio(self) -> float:
        return self.container_bytes / (2 * self.n) if self.n else 1.0

    def read_bytes(self) -> int:
        """Bytes a decode reads: slots, bitmap and the side entries."""
        return self.container_bytes

    def descriptor(self) -> DfNf12Tensor:
        t = DfNf12Tensor()
        t.n = self.n
        t.n_escaped = self.n_escaped
        t.slots = self.slots.data_ptr() if self.n else None
        t.bitmap = self.bitmap.data_ptr() if self.n else None
        t.side = self.side.data_ptr() if self.n_escaped else None
        t.top = self.top
        t.reserved = 0
        return t


def compress(w: torch.Tensor, top: int = DF_NF12_TOP, d_err: torch.Tensor | None = None, stream=None) -> Nf12:
    """Encode w: one pass over the groups, a read of the escape count (the
    side buffer is sized from it), then the escaped groups."""
    x = _as_u16(w)
    dev = x.device
    n = x.numel()
    z = api.df_nf12_sizes_for(n)
    slots = torch.empty(max(z.slots_bytes, 16), dtype=torch.uint8, device=dev)
    bitmap = torch.empty(max(z.bitmap_bytes, 16), dtype=torch.uint8, device=dev)
    ws = torch.empty(z.encode_ws_bytes, dtype=torch.uint8, device=dev)
    escaped = torch.empty(1, dtype=torch.int64, device=dev)
    api.df_nf12_encode_groups(x, top, slots, bitmap, ws, escaped, stream)
    e = int(escaped.cpu().numpy().view(np.uint64)[0])  # waits for the stream's work
    side = torch.empty(max(16 * e, 16), dtype=torch.uint8, device=dev)
    if e:
        api.df_nf12_encode_escapes(x, top, slots, bitmap, ws, side, d_err, stream)
    return Nf12(n=n, shape=tuple(w.shape), top=top, slots=slots, bitmap=bitmap, side=side, n_escaped=e)


class BatchEncoder:
    """A grouped encode of many tensors (one launch per step for all of them):
    run() packs every tensor and counts its escapes, reads the counts (one
    wait), sizes the side buffers and writes them."""

    def __init__(self, ws: list[torch.Tensor], top: int = DF_NF12_TOP):
        if not ws:
            raise ValueError("no tensors")
        self.xs = [_as_u16(w) for w in ws]
        self.shapes = [tuple(w.shape) for w in ws]
        self.top = top
        dev = self.xs[0].device
        self.parts = []
        for x in self.xs:
            z = api.df_nf12_sizes_for(x.numel())
            self.parts.append((torch.empty(max(z.slots_bytes, 16), dtype=torch.uint8, device=dev),
                               torch.empty(max(z.bitmap_bytes, 16), dtype=torch.uint8, device=dev)))
        self.escaped = torch.empty(len(self.xs), dtype=torch.int64, device=dev)
        self.sides = [None] * len(self.xs)
        self.ws = torch.empty(max(api.df_nf12_encode_batch_workspace(self.descriptors()), 16), dtype=torch.uint8,
                              device=dev)
        self.plan = api.df_nf12_encode_batch_prepare(self.descriptors(), self.ws)

    def descriptors(self) -> list[DfNf12EncodeTensor]:
        out = []
        for i, (x, (slots, bitmap)) in enumerate(zip(self.xs, self.parts)):
            t = DfNf12EncodeTensor()
            t.input = x.data_ptr() if x.numel() else None
            t.n = x.numel()
            t.slots = slots.data_ptr()
            t.bitmap = bitmap.data_ptr()
            side = self.sides[i]
            t.side = side.data_ptr() if side is not None else None
            t.side_capacity = side.numel() // 16 if side is not None else 0
            t.top = self.top
            out.append(t)
        return out

    def run(self, d_err: torch.Tensor | None = None, stream=None) -> list[Nf12]:
        api.df_nf12_encode_batch_groups(self.plan, self.escaped, stream)
        counts = [int(v) for v in self.escaped.cpu().numpy().view(np.uint64)]  # waits for the stream
        dev = self.xs[0].device
        for i, e in enumerate(counts):
            if self.sides[i] is None or self.sides[i].numel() < 16 * e:
                self.sides[i] = torch.empty(max(16 * e, 16), dtype=torch.uint8, device=dev)
        self.plan = api.df_nf12_encode_batch_prepare(self.descriptors(), self.ws, stream)
        api.df_nf12_encode_batch_escapes(self.plan, d_err, stream)
        return [Nf12(n=x.numel(), shape=shp, top=self.top, slots=sl, bitmap=bm, side=sd, n_escaped=e)
                for x, shp, (sl, bm), sd, e in zip(self.xs, self.shapes, self.parts, self.sides, counts)]


def compress_batch(ws: list[torch.Tensor], top: int = DF_NF12_TOP, d_err: torch.Tensor | None = None,
                   stream=None) -> list[Nf12]:
    """compress() of many tensors with one launch per kernel for all."""
    return BatchEncoder(ws, top).run(d_err, stream)


def decompress(c: Nf12, out: torch.Tensor | None = None, d_err: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(c.shape, dtype=torch.bfloat16, device=c.slots.device)
    if out.numel() != c.n:
        raise ValueError("output size differs from the tensor's")
    if c.n:
        api.df_nf12_decode(c.descriptor(), out.view(torch.int16).reshape(-1), d_err, stream)
    return out


class BatchDecoder:
    """A grouped decode of many tensors in the fixed 12-bit format, prepared
    once and launched many times (one kernel launch per run)."""

    def __init__(self, comps: list[Nf12], outs: list[torch.Tensor] | None = None, stream=None):
        if not comps:
            raise ValueError("no tensors")
        dev = comps[0].slots.device
        self.comps = comps
        self.outs = outs if outs is not None else [
            torch.empty(c.shape, dtype=torch.bfloat16, device=dev) for c in comps]
        self.ws = torch.empty(api.df_nf12_decode_batch_workspace(len(comps)), dtype=torch.uint8, device=dev)
        flat = [o.view(torch.int16).reshape(-1) for o in self.outs]
        self.plan = api.df_nf12_decode_batch_prepare([c.descriptor() for c in comps], flat, self.ws, stream)

    def run(self, d_err: torch.Tensor | None = None, stream=None) -> list[torch.Tensor]:
        api.df_nf12_decode_batch_run(self.plan, d_err, stream)
        return self.outs

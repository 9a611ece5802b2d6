"""Tensor-level helpers over the C ABI: compress a BF16 CUDA tensor into a
container held in torch CUDA buffers, and decode one or many containers.

PyTorch only allocates memory here; every step of the codec runs in
libdf11.so (df_histogram, df_encode, df_encode_batch_*, df_decode,
df_decode_batch_*). Building
the code table is host work done by df_build_code / df_build_lut in the same
library. There is no CPU fallback: CPU tensors are rejected.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import api
from ._native import DfEncodeTensor, DfTensor

DEFAULT_MAX_LEN = 32
DEFAULT_CHUNK_BYTES = 32
DEFAULT_THREADS_PER_BLOCK = 32


def _as_u16(w: torch.Tensor) -> torch.Tensor:
    if not w.is_cuda:
        raise TypeError("compress takes a CUDA tensor (there is no CPU path)")
    if w.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError(f"expected BF16 bit patterns (bfloat16/int16/uint16), got {w.dtype}")
    return w.contiguous().reshape(-1).view(torch.int16)


class Compressed:
    """One tensor's container in device memory."""

    def __init__(self, *, n, shape, code, lut, sizes, chunk_bytes, threads_per_block, stream, gaps, offsets, sm,
                 index8=None, index8_wide=0):
        if (offsets is None) == (index8 is None):
            raise ValueError("a container holds exactly one block index: offsets or index8")
        self.n = int(n)
        self.shape = tuple(shape)
        self.code = code
        self.lut = lut
        self.sizes = sizes
        self.chunk_bytes = chunk_bytes
        self.threads_per_block = threads_per_block
        self.stream = stream
        self.gaps = gaps
        self.offsets = offsets      # uint64 block offsets, or None with the compact index
        self.index8 = index8        # compact block index (df_index8_build), or None
        self.index8_wide = int(index8_wide)
        self.sm = sm
        self._desc = None

    @property
    def total_bits(self) -> int:
        return self.sizes["total_bits"]

    @property
    def index_kind(self) -> str:
        return "u64" if self.offsets is not None else "idx8"

    @property
    def index_bytes(self) -> int:
        """Bytes of the block index this container holds."""
        if self.offsets is not None:
            return self.sizes["offsets_bytes"]
        return api.df_index8_bytes(self.sizes["n_blocks"], self.index8_wide)

    @property
    def index(self) -> torch.Tensor:
        """The block index part: uint64 offsets or the compact index bytes."""
        return self.offsets if self.offsets is not None else self.index8

    @property
    def container_bytes(self) -> int:
        return self.sizes["container_bytes"] - self.sizes["offsets_bytes"] + self.index_bytes

    @property
    def ratio(self) -> float:
        return self.container_bytes / (2 * self.n) if self.n else 1.0

    @property
    def lengths(self) -> np.ndarray:
        return np.frombuffer(bytes(self.code.lengths), np.uint8).copy()

    def read_bytes(self) -> int:
        """Bytes a full decode must read: the stream, gaps, block index and sm bytes."""
        z = self.sizes
        return z["stream_bytes"] + z["gap_bytes"] + self.index_bytes + z["sm_bytes"]

    def block_offsets(self, stream=None) -> torch.Tensor:
        """The uint64 block offsets on the device (expanded from the compact
        index into a new tensor when that is what the container holds)."""
        if self.offsets is not None:
            return self.offsets
        o = torch.empty(self.sizes["n_blocks"] + 1, dtype=torch.int64, device=self.stream.device)
        api.df_index8_expand(self.index8, self.sizes["n_blocks"], self.index8_wide, o, None, stream)
        return o

    def use_index8(self, d_err: torch.Tensor | None = None, stream=None) -> "Compressed":
        """Replace the uint64 block offsets by the compact index (df11pack,
        "What is checked": --index idx8). Waits for the stream once to learn
        the number of wide superblocks."""
        if self.offsets is None:
            return self
        nb = self.sizes["n_blocks"]
        dev = self.offsets.device
        wide = torch.zeros(1, dtype=torch.int64, device=dev)
        ix = torch.empty(max(api.df_index8_bytes(nb, 0), 16), dtype=torch.uint8, device=dev)
        api.df_index8_build(self.offsets, nb, ix, wide, None, stream)
        w = int(wide.cpu().item())
        if w:  # room for the wide superblocks' counts, then again
            ix = torch.empty(api.df_index8_bytes(nb, w), dtype=torch.uint8, device=dev)
            api.df_index8_build(self.offsets, nb, ix, wide, d_err, stream)
        self.index8, self.index8_wide, self.offsets, self._desc = ix, w, None, None
        return self

    def descriptor(self) -> DfTensor:
        if self._desc is None:
            d = DfTensor()
            d.n = self.n
            d.total_bits = self.total_bits
            d.chunk_bytes = self.chunk_bytes
            d.threads_per_block = self.threads_per_block
            d.max_len = self.code.max_len
            d.n_tables = self.code.n_tables
            d.stream = self.stream.data_ptr()
            d.gaps = self.gaps.data_ptr()
            if self.offsets is not None:
                d.block_offsets = self.offsets.data_ptr()
            else:
                d.index8 = self.index8.data_ptr()
                d.index8_wide = self.index8_wide
            d.sm = self.sm.data_ptr() if self.n else self.stream.data_ptr()
            d.lut = self.lut.data_ptr()
            d.lengths[:] = self.code.lengths[:]
            self._desc = d
        return self._desc

    @classmethod
    def from_host(cls, *, lengths, max_len, total_bits, n, stream, gaps, offsets, sm, shape=None,
                  chunk_bytes=DEFAULT_CHUNK_BYTES, threads_per_block=DEFAULT_THREADS_PER_BLOCK,
                  device="cuda", index8=None, index8_wide=0):
        """Upload a container whose parts are host arrays (e.g. read from a
        file); give either offsets or index8 (with index8_wide)."""
        code = api.df_code_from_lengths(lengths, max_len)
        lut = torch.from_numpy(api.df_build_lut(code).view(np.int32)).to(device)
        if offsets is not None:
            n_blocks = int(np.asarray(offsets).size) - 1
        else:
            n_blocks = api.df_container_sizes(int(n), int(total_bits), chunk_bytes, threads_per_block).n_blocks
        hist_free = {
            "total_bits": int(total_bits),
            "stream_bytes": int(np.asarray(stream).size),
            "gap_bytes": int(np.asarray(gaps).size),
            "offsets_bytes": 8 * (n_blocks + 1),
            "sm_bytes": int(n),
            "n_blocks": n_blocks,
        }
        hist_free["container_bytes"] = (hist_free["stream_bytes"] + hist_free["gap_bytes"] +
                                        hist_free["offsets_bytes"] + int(n) + 256 + 64)
        t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(device)  # noqa: E731
        sm_arr = np.asarray(sm, np.uint8)
        return cls(n=n, shape=shape or (n,), code=code, lut=lut, sizes=hist_free, chunk_bytes=chunk_bytes,
                   threads_per_block=threads_per_block, stream=t(np.asarray(stream, np.uint8), np.uint8),
                   gaps=t(np.asarray(gaps, np.uint8), np.uint8),
                   offsets=t(np.asarray(offsets, np.uint64), np.int64) if offsets is not None else None,
                   sm=t(sm_arr if sm_arr.size else np.zeros(16, np.uint8), np.uint8),
                   index8=t(np.asarray(index8, np.uint8), np.uint8) if index8 is not None else None,
                   index8_wide=index8_wide)


def auto_chunk_bytes(code) -> int:
    """32-byte chunks; 16 when the shortest code is 1 bit, so that no chunk
    holds more than 128 codes (the decoder's per-thread region stays small)."""
    return DEFAULT_CHUNK_BYTES if code.min_len >= 2 else 16


class SafeCheckError(RuntimeError):
    pass


def compress(w: torch.Tensor, max_len: int = DEFAULT_MAX_LEN, chunk_bytes: int | None = None,
             threads_per_block: int = DEFAULT_THREADS_PER_BLOCK, d_err: torch.Tensor | None = None,
             stream=None, safe: bool = False, index: str = "u64") -> Compressed:
    """Histogram on the GPU, code build on the host, encode on the GPU.
    chunk_bytes=None picks auto_chunk_bytes(code). safe=True decodes the new
    container and compares it with w on the GPU before returning (df11pack,
    "Use": --safe), raising SafeCheckError on any difference. index="idx8"
    keeps the compact block index in place of the uint64 offsets."""
    if index not in ("u64", "idx8"):
        raise ValueError("index is 'u64' or 'idx8'")
    x = _as_u16(w)
    dev = x.device
    n = x.numel()
    hist_d = torch.empty(256, dtype=torch.int64, device=dev)
    api.df_histogram(x, hist_d, stream)
    hist = hist_d.cpu().numpy().view(np.uint64)
    code = api.df_build_code(hist, max_len)
    if chunk_bytes is None:
        chunk_bytes = auto_chunk_bytes(code)
    lut = torch.from_numpy(api.df_build_lut(code).view(np.int32)).to(dev)
    z = api.df_plan(code, hist, n, chunk_bytes, threads_per_block).as_dict()
    stream_buf = torch.empty(z["stream_bytes"], dtype=torch.uint8, device=dev)
    gaps = torch.empty(z["gap_bytes"], dtype=torch.uint8, device=dev)
    offsets = torch.empty(z["n_blocks"] + 1, dtype=torch.int64, device=dev)
    sm = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
    ws = torch.empty(max(z["encode_ws_bytes"], 16), dtype=torch.uint8, device=dev)
    api.df_encode(code, x, z["total_bits"], chunk_bytes, threads_per_block, stream_buf, gaps, offsets,
                  sm, ws, d_err, stream)
    c = Compressed(n=n, shape=tuple(w.shape), code=code, lut=lut, sizes=z, chunk_bytes=chunk_bytes,
                   threads_per_block=threads_per_block, stream=stream_buf, gaps=gaps, offsets=offsets, sm=sm)
    if index == "idx8":
        c.use_index8(d_err, stream)
    if safe and n:
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        api.df_read_error(err, stream)
        back = torch.empty(n, dtype=torch.int16, device=dev)
        decompress(c, back, err, stream)
        first = torch.empty(1, dtype=torch.int64, device=dev)
        api.df_compare(back, x, first, stream)
        if api.df_read_error(err, stream) or int(first.cpu().numpy().view(np.uint64)[0]) != 2**64 - 1:
            raise SafeCheckError("the container does not decode to its source")
    return c


def _per_tensor(value, count: int, name: str) -> list:
    if isinstance(value, (list, tuple)):
        if len(value) != count:
            raise ValueError(f"{name}: one value per tensor")
        return list(value)
    return [value] * count


class BatchEncoder:
    """A grouped encode of many tensors (df_encode_batch_*): one launch for
    all the exponent histograms, the codes built on the host (one wait for
    the histograms), then one launch that zeroes every output and one that
    encodes every tensor. Each container equals compress()'s for the same
    tensor and format. chunk_bytes (None: auto_chunk_bytes per tensor) and
    threads_per_block may be one value or one per tensor. prepare() reads the
    histograms and allocates the containers; run() encodes into them (again
    on every call, e.g. to time it)."""

    def __init__(self, ws: list[torch.Tensor], max_len: int = DEFAULT_MAX_LEN, chunk_bytes=None,
                 threads_per_block=DEFAULT_THREADS_PER_BLOCK, stream=None):
        if not ws:
            raise ValueError("no tensors")
        self.xs = [_as_u16(w) for w in ws]
        self.shapes = [tuple(w.shape) for w in ws]
        self.dev = self.xs[0].device
        if any(x.device != self.dev for x in self.xs):
            raise ValueError("all tensors must be on one device")
        self.max_len = max_len
        self.chunk_bytes = _per_tensor(chunk_bytes, len(self.xs), "chunk_bytes")
        self.tpb = _per_tensor(threads_per_block, len(self.xs), "threads_per_block")
        self.hist = torch.empty((len(self.xs), 256), dtype=torch.int64, device=self.dev)
        descs = self.descriptors()
        self.ws = torch.empty(max(api.df_encode_batch_workspace(descs), 16), dtype=torch.uint8, device=self.dev)
        self.plan = api.df_encode_batch_prepare(descs, self.ws, stream)
        self.comps: list[Compressed] | None = None

    def descriptors(self, comps: list[Compressed] | None = None) -> list[DfEncodeTensor]:
        """The C descriptors of the inputs, with each container's code,
        format and outputs when `comps` is given (histograms only otherwise)."""
        out = []
        for i, x in enumerate(self.xs):
            t = DfEncodeTensor()
            t.input = x.data_ptr() if x.numel() else None
            t.n = x.numel()
            if comps is not None:
                c = comps[i]
                t.code = ctypes.pointer(c.code)
                t.total_bits = c.total_bits
                t.chunk_bytes = c.chunk_bytes
                t.threads_per_block = c.threads_per_block
                t.stream = c.stream.data_ptr()
                t.gaps = c.gaps.data_ptr()
                t.block_offsets = c.offsets.data_ptr()
                t.sm = c.sm.data_ptr()
            out.append(t)
        return out

    def run_histograms(self, stream=None) -> None:
        """Every tensor's exponent histogram into self.hist (one launch)."""
        api.df_histogram_batch_run(self.plan, self.hist, stream)

    def histograms(self, stream=None) -> np.ndarray:
        self.run_histograms(stream)
        if stream is not None:
            stream.synchronize()
        return self.hist.cpu().numpy().view(np.uint64)

    def prepare(self, stream=None) -> list[Compressed]:
        hist = self.histograms(stream)
        comps = []
        for i, x in enumerate(self.xs):
            n = x.numel()
            code = api.df_build_code(hist[i], self.max_len)
            C = self.chunk_bytes[i] or auto_chunk_bytes(code)
            T = self.tpb[i]
            lut = torch.from_numpy(api.df_build_lut(code).view(np.int32)).to(self.dev)
            z = api.df_plan(code, hist[i], n, C, T).as_dict()
            comps.append(Compressed(
                n=n, shape=self.shapes[i], code=code, lut=lut, sizes=z, chunk_bytes=C, threads_per_block=T,
                stream=torch.empty(z["stream_bytes"], dtype=torch.uint8, device=self.dev),
                gaps=torch.empty(z["gap_bytes"], dtype=torch.uint8, device=self.dev),
                offsets=torch.empty(z["n_blocks"] + 1, dtype=torch.int64, device=self.dev),
                sm=torch.empty(max(n, 16), dtype=torch.uint8, device=self.dev)))
        self.plan = api.df_encode_batch_prepare(self.descriptors(comps), self.ws, stream)
        self.comps = comps
        return comps

    def run(self, d_err: torch.Tensor | None = None, stream=None) -> list[Compressed]:
        if self.comps is None:
            self.prepare(stream)
        api.df_encode_batch_run(self.plan, d_err, stream)
        return self.comps


def compress_batch(ws: list[torch.Tensor], max_len: int = DEFAULT_MAX_LEN, chunk_bytes=None,
                   threads_per_block=DEFAULT_THREADS_PER_BLOCK, d_err: torch.Tensor | None = None,
                   stream=None) -> list[Compressed]:
    """compress() of many tensors with one launch per step for all of them."""
    return BatchEncoder(ws, max_len, chunk_bytes, threads_per_block, stream).run(d_err, stream)


def decompress(c: Compressed, out: torch.Tensor | None = None, d_err: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """Decode into `out` (BF16 or 16-bit integer CUDA tensor of c.n elements)."""
    if out is None:
        out = torch.empty(c.shape, dtype=torch.bfloat16, device=c.stream.device)
    if out.numel() != c.n:
        raise ValueError("output size differs from the container's")
    api.df_decode(c.descriptor(), out.view(torch.int16).reshape(-1) if c.n else out, d_err, stream)
    return out


class BatchDecoder:
    """A grouped decode of many containers, prepared once and launched many
    times (one kernel launch per run)."""

    def __init__(self, comps: list[Compressed], outs: list[torch.Tensor] | None = None, stream=None):
        if not comps:
            raise ValueError("no tensors")
        dev = comps[0].stream.device
        self.comps = comps
        self.outs = outs if outs is not None else [
            torch.empty(c.shape, dtype=torch.bfloat16, device=dev) for c in comps]
        self.ws = torch.empty(api.df_decode_batch_workspace(len(comps)), dtype=torch.uint8, device=dev)
        descs = [c.descriptor() for c in comps]
        flat = [o.view(torch.int16).reshape(-1) for o in self.outs]
        self.plan = api.df_decode_batch_prepare(descs, flat, self.ws, stream)

    def run(self, d_err: torch.Tensor | None = None, stream=None) -> list[torch.Tensor]:
        api.df_decode_batch_run(self.plan, d_err, stream)
        return self.outs


def decompress_batch(comps: list[Compressed], outs: list[torch.Tensor] | None = None,
                     d_err: torch.Tensor | None = None, stream=None) -> list[torch.Tensor]:
    dec = BatchDecoder(comps, outs, stream)
    return dec.run(d_err, stream)

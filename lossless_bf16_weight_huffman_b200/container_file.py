"""A file of compressed tensors: save containers from the GPU, load them back.

df11pack (GitHub page), "What is checked": a per-tensor SHA-256 can sit in the
header (--hashes) so that verify catches corruption without the source. The
file layout is this library's own (little-endian):

    b"DF11B200"  u32 version (1)  u32 count  u64 header bytes
    header: UTF-8 JSON {"tensors": [entry, ...]}
    zero padding to a multiple of 64 bytes
    every tensor's parts (stream, gaps, its block index, sm), each at a
    64-byte-aligned offset from the start of the file

entry: name, shape, n, total_bits, chunk_bytes, threads_per_block, max_len,
lengths (256 code lengths, hex), index ("u64": the part "offsets"; "idx8":
the part "index8", the compact block index of df_index8_build, with
index8_wide), parts {part: [offset, bytes]}, and sha256: the leaf-tree
SHA-256 (df_sha256_device) of the tensor's BF16 bytes, or null. The decode
tables are not stored: loading rebuilds them from the lengths.
"""
from __future__ import annotations

import json
import struct
import warnings

import numpy as np

from . import api, codec

MAGIC = b"DF11B200"
VERSION = 1
ALIGN = 64
_DTYPES = {"stream": np.uint8, "gaps": np.uint8, "offsets": np.uint64, "index8": np.uint8, "sm": np.uint8}


def _parts(index: str) -> tuple[str, ...]:
    if index not in ("u64", "idx8"):
        raise FormatError(f"unknown block index {index!r}")
    return ("stream", "gaps", "offsets" if index == "u64" else "index8", "sm")


class FormatError(ValueError):
    pass


def _part_host(c: codec.Compressed, part: str) -> np.ndarray:
    t = getattr(c, part)
    if part == "sm":
        t = t[: c.n]
    a = t.detach().cpu().numpy()
    return np.ascontiguousarray(a.view(_DTYPES[part]))


def _pad(n: int) -> int:
    return (-n) % ALIGN


def save(path: str, tensors, hashes: dict | None = None) -> None:
    """Write (name, Compressed) pairs; hashes maps a name to its 32-byte digest."""
    hashes = hashes or {}
    entries, blobs = [], []
    for name, c in tensors:
        parts = {p: _part_host(c, p) for p in _parts(c.index_kind)}
        entries.append({"name": name, "shape": list(c.shape), "n": c.n, "total_bits": c.total_bits,
                        "chunk_bytes": c.chunk_bytes, "threads_per_block": c.threads_per_block,
                        "max_len": int(c.code.max_len), "lengths": bytes(c.code.lengths).hex(),
                        "index": c.index_kind, "index8_wide": c.index8_wide,
                        "sha256": hashes[name].hex() if name in hashes else None, "parts": {}})
        blobs.append(parts)
    # offsets depend on the header size, which depends on the offsets: lay
    # out with a fixed-width placeholder first, then fill in
    def header_bytes():
        return json.dumps({"tensors": entries}, separators=(",", ":")).encode()

    for e, parts in zip(entries, blobs):
        e["parts"] = {p: [0, int(parts[p].nbytes)] for p in parts}
    for _ in range(3):  # converges: offsets only grow the header by a few digits
        pos = 24 + len(header_bytes())
        pos += _pad(pos)
        for e, parts in zip(entries, blobs):
            for p in parts:
                e["parts"][p][0] = pos
                pos += parts[p].nbytes + _pad(parts[p].nbytes)
    head = header_bytes()
    with open(path, "wb") as f:
        f.write(MAGIC + struct.pack("<IIQ", VERSION, len(entries), len(head)))
        f.write(head)
        f.write(b"\0" * _pad(24 + len(head)))
        for e, parts in zip(entries, blobs):
            for p in parts:
                if f.tell() != e["parts"][p][0]:
                    raise FormatError("layout mismatch while writing")
                f.write(parts[p].tobytes())
                f.write(b"\0" * _pad(parts[p].nbytes))


def read_header(path: str) -> dict:
    with open(path, "rb") as f:
        fixed = f.read(24)
        if len(fixed) < 24 or fixed[:8] != MAGIC:
            raise FormatError("not a container file")
        version, count, hlen = struct.unpack("<IIQ", fixed[8:])
        if version != VERSION:
            raise FormatError(f"unknown version {version}")
        head = json.loads(f.read(hlen).decode())
    if len(head.get("tensors", [])) != count:
        raise FormatError("header count mismatch")
    return head


def read_host(path: str):
    """(entry, {part: numpy array}) per tensor, the arrays mapped from the file."""
    head = read_header(path)
    mm = np.memmap(path, dtype=np.uint8, mode="r")
    out = []
    for e in head["tensors"]:
        parts = {}
        for p in _parts(e.get("index", "u64")):
            off, nbytes = e["parts"][p]
            if off + nbytes > mm.size:
                raise FormatError(f"{e['name']}: part {p} runs past the end of the file")
            parts[p] = np.asarray(mm[off: off + nbytes]).view(_DTYPES[p])
        out.append((e, parts))
    return out


def load(path: str, device="cuda"):
    """(name, Compressed on `device`, digest or None) per tensor."""
    out = []
    for e, parts in read_host(path):
        # the decoder reads as many bytes as n and total_bits imply: refuse
        # parts of any other size before anything reaches the GPU
        try:
            z = api.df_container_sizes(e["n"], e["total_bits"], e["chunk_bytes"], e["threads_per_block"]).as_dict()
        except Exception as exc:
            raise FormatError(f"{e['name']}: impossible sizes ({exc})") from exc
        wide = int(e.get("index8_wide", 0))
        if not 0 <= wide <= (z["n_blocks"] + 63) // 64:
            raise FormatError(f"{e['name']}: {wide} wide superblocks")
        want = {"stream": z["stream_bytes"], "gaps": z["gap_bytes"], "offsets": z["offsets_bytes"],
                "index8": api.df_index8_bytes(z["n_blocks"], wide), "sm": z["sm_bytes"]}
        for p in parts:
            if parts[p].nbytes != want[p]:
                raise FormatError(f"{e['name']}: part {p} holds {parts[p].nbytes} bytes, the layout needs {want[p]}")
        lengths = np.frombuffer(bytes.fromhex(e["lengths"]), np.uint8)
        if lengths.size != 256:
            raise FormatError(f"{e['name']}: {lengths.size} code lengths")
        with warnings.catch_warnings():  # the parts are read-only views of the file; they are only copied
            warnings.simplefilter("ignore", UserWarning)
            c = codec.Compressed.from_host(
                lengths=lengths, max_len=e["max_len"], total_bits=e["total_bits"], n=e["n"], stream=parts["stream"],
                gaps=parts["gaps"], offsets=parts.get("offsets"), sm=parts["sm"], shape=tuple(e["shape"]),
                chunk_bytes=e["chunk_bytes"], threads_per_block=e["threads_per_block"], device=device,
                index8=parts.get("index8"), index8_wide=wide)
        c.sizes.update({k: z[k] for k in ("n_chunks", "n_blocks", "container_bytes")})
        out.append((e["name"], c, bytes.fromhex(e["sha256"]) if e["sha256"] else None))
    return out

"""Check compressed tensors, with or without their source.

df11pack (GitHub page), "Use": verify checks a container's structure with no
source needed; with the source it also decodes 1000 sampled chunks and compares
them; at level full it decodes and compares everything; it exits 0 on pass, 1
when a check fails, 2 when it could not check. "What is checked" (--hashes): a
per-tensor SHA-256 stored with the container lets verify catch corruption
without the source.

Levels here (a "chunk" is one format block of T chunks of the stream, the unit
one warp decodes on its own):
  structure  sizes and code lengths on the host, block offsets on the GPU
             (df_check_structure); no decode
  sampled    + `samples` format blocks drawn at random (seeded), decoded alone
             by one grouped launch and compared with the source on the GPU
             (df_compare); without a source: could not check (2)
  full       + every tensor decoded and compared with the source, or, with no
             source, its digest (df_sha256_device) compared with the stored one;
             with neither: could not check (2)
Every step runs in libdf11.so; this module builds descriptors and reads flags.

    python -m lossless_bf16_weight_huffman_b200.verify FILE [--source NPZ] [--level structure|sampled|full]
"""
from __future__ import annotations

import argparse
import ctypes
import sys

import numpy as np
import torch

from . import api, codec
from ._native import DfError, DfTensor

PASS, FAIL, CANNOT = 0, 1, 2
LEVELS = ("structure", "sampled", "full")


def _flags(dev) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=dev)


def _first_diff(a: torch.Tensor, b: torch.Tensor) -> int:
    out = torch.empty(1, dtype=torch.int64, device=a.device)
    api.df_compare(a.view(torch.int16).reshape(-1), b.view(torch.int16).reshape(-1), out)
    v = int(out.cpu().numpy().view(np.uint64)[0])
    return -1 if v == 0xFFFFFFFFFFFFFFFF else v


def check_structure(c: codec.Compressed) -> str | None:
    """None when the container's structure is sound, else what is wrong."""
    try:
        z = api.df_container_sizes(c.n, c.total_bits, c.chunk_bytes, c.threads_per_block).as_dict()
    except DfError as e:
        return f"impossible sizes: {e}"
    have = {"stream_bytes": c.stream.numel(), "gap_bytes": c.gaps.numel()}
    if c.offsets is not None:
        have["offsets_bytes"] = 8 * c.offsets.numel()
    for k, v in have.items():
        if v < z[k]:
            return f"{k}: {v} < {z[k]}"
    if c.index8 is not None:
        need = api.df_index8_bytes(z["n_blocks"], c.index8_wide)
        if c.index8.numel() < need or c.index8_wide > (z["n_blocks"] + 63) // 64:
            return f"compact block index: {c.index8.numel()} bytes for {c.index8_wide} wide superblocks"
    if c.sm.numel() < c.n:
        return "sign|fraction bytes shorter than n"
    try:
        api.df_code_from_lengths(c.lengths, c.code.max_len)
    except DfError as e:
        return f"code lengths: {e}"
    if c.n == 0:
        return None
    fl = _flags(c.stream.device)
    d = _with_offsets(c, _offsets_of(c, fl))
    api.df_check_structure(d, fl)
    return "block offsets" if api.df_read_error(fl) else None


def _offsets_of(c: codec.Compressed, fl: torch.Tensor) -> torch.Tensor:
    """The container's uint64 block offsets (expanded on the GPU from a
    compact index; a bad overflow slot there sets DF_EFLAG_INDEX8 in fl)."""
    if c.offsets is not None:
        return c.offsets
    o = torch.empty(c.sizes["n_blocks"] + 1, dtype=torch.int64, device=c.stream.device)
    api.df_index8_expand(c.index8, c.sizes["n_blocks"], c.index8_wide, o, fl)
    return o


def _with_offsets(c: codec.Compressed, offsets: torch.Tensor) -> DfTensor:
    d = DfTensor()
    ctypes.memmove(ctypes.byref(d), ctypes.byref(c.descriptor()), ctypes.sizeof(d))
    d.block_offsets = offsets.data_ptr()
    d.index8 = None
    d.index8_wide = 0
    d._keep = offsets
    return d


def _block_descriptor(c: codec.Compressed, offsets: torch.Tensor, b: int, offs: tuple[int, int]) -> DfTensor:
    """A descriptor of format block b alone: the stream, gaps and offsets from
    the block's start; output indices stay absolute (n = the block's end)."""
    T, C = c.threads_per_block, c.chunk_bytes
    cbits = 8 * C
    d = DfTensor()
    d.n = offs[1]
    d.total_bits = min(c.total_bits - b * T * cbits, T * cbits)
    d.chunk_bytes = C
    d.threads_per_block = T
    d.max_len = c.code.max_len
    d.n_tables = c.code.n_tables
    d.stream = c.stream.data_ptr() + b * T * C
    d.gaps = c.gaps.data_ptr() + (5 * T * b) // 8  # T is a multiple of 32: the block's fields start on a byte
    d.block_offsets = offsets.data_ptr() + 8 * b
    d.sm = c.sm.data_ptr()
    d.lut = c.lut.data_ptr()
    d.lengths[:] = c.code.lengths[:]
    return d


def check_sampled(entries, source: dict, samples: int = 1000, seed: int = 0) -> tuple[int, str]:
    """Decode `samples` random format blocks (all tensors, weighted by block
    count) in one grouped launch and compare each with the source."""
    comps = [(name, c) for name, c, _ in entries if c.n]
    if not comps:
        return PASS, "nothing to sample"
    dev = comps[0][1].stream.device
    nb = np.array([c.sizes["n_blocks"] if "n_blocks" in c.sizes else
                   api.df_container_sizes(c.n, c.total_bits, c.chunk_bytes, c.threads_per_block).n_blocks
                   for _, c in comps], np.int64)
    rng = np.random.default_rng(seed)
    picks = rng.choice(int(nb.sum()), size=min(samples, int(nb.sum())), replace=False)
    starts = np.concatenate([[0], np.cumsum(nb)])
    chosen = []
    for g in np.sort(picks):
        ti = int(np.searchsorted(starts, g, side="right") - 1)
        chosen.append((ti, int(g - starts[ti])))
    # the block offsets of the chosen blocks
    fl0 = _flags(dev)
    full = {ti: _offsets_of(comps[ti][1], fl0) for ti in sorted({ti for ti, _ in chosen})}
    if api.df_read_error(fl0):
        return FAIL, "compact block index"
    offs = []
    for ti, b in chosen:
        o = full[ti][b: b + 2].cpu().numpy().view(np.uint64)
        offs.append((int(o[0]), int(o[1])))
    if any(o[1] < o[0] or o[1] > comps[ti][1].n for (ti, _), o in zip(chosen, offs)):
        return FAIL, "block offsets out of range"
    sizes = [o[1] - o[0] for o in offs]
    buf = torch.empty(sum(sizes) + 8 * len(sizes) + 8, dtype=torch.int16, device=dev)
    descs, outs, views, pos = [], [], [], 0
    for (ti, b), o, n in zip(chosen, offs, sizes):
        # place the block's outputs so that its absolute index o[0] lands at a
        # 16-byte-aligned view (the decoder then takes its vector path)
        pos += (-(pos - o[0])) % 8
        descs.append(_block_descriptor(comps[ti][1], full[ti], b, o))
        outs.append(buf.data_ptr() + 2 * (pos - o[0]))
        views.append(buf[pos: pos + n])
        pos += n
    ws = torch.empty(api.df_decode_batch_workspace(len(descs)), dtype=torch.uint8, device=dev)
    fl = _flags(dev)
    api.df_decode_batch(descs, outs, ws, fl)
    if api.df_read_error(fl):
        return FAIL, "a sampled block does not decode"
    for (ti, b), o, v in zip(chosen, offs, views):
        name = comps[ti][0]
        src = source[name].reshape(-1)[o[0]: o[1]]
        if _first_diff(v, src) >= 0:
            return FAIL, f"{name}: block {b} differs from the source"
    return PASS, f"{len(chosen)} sampled blocks equal the source"


def check_full(entries, source: dict | None) -> tuple[int, str]:
    """Decode everything; compare with the source, else with the stored digest."""
    for name, c, sha in entries:
        if c.n == 0:
            continue
        if (source is None or name not in source) and sha is None:
            return CANNOT, f"{name}: no source and no stored digest"
        out = torch.empty(c.n, dtype=torch.int16, device=c.stream.device)
        fl = _flags(c.stream.device)
        codec.decompress(c, out, fl)
        if api.df_read_error(fl):
            return FAIL, f"{name}: does not decode"
        if source is not None and name in source:
            if _first_diff(out, source[name].reshape(-1)) >= 0:
                return FAIL, f"{name}: differs from the source"
        elif api.df_sha256_device(out) != sha:
            return FAIL, f"{name}: digest differs from the stored one"
    return PASS, "every tensor decodes to its source" if source is not None else "every digest matches"


def verify(entries, level: str = "structure", source: dict | None = None, samples: int = 1000,
           seed: int = 0) -> tuple[int, str]:
    """entries: (name, Compressed, digest or None); source: name -> CUDA tensor
    of the original BF16 bits. Returns (0 pass | 1 fail | 2 could not check, why)."""
    if level not in LEVELS:
        raise ValueError(f"level must be one of {LEVELS}")
    for name, c, _ in entries:
        why = check_structure(c)
        if why:
            return FAIL, f"{name}: {why}"
    if level == "structure":
        return PASS, "structure sound"
    if level == "sampled":
        if source is None:
            return CANNOT, "sampled chunks need the source"
        missing = [n for n, _, _ in entries if n not in source]
        if missing:
            return CANNOT, f"no source for {missing[0]}"
        return check_sampled(entries, source, samples, seed)
    return check_full(entries, source)


def main(argv=None) -> int:
    from . import container_file

    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("file")
    p.add_argument("--source", help=".npz of uint16 arrays (the original BF16 bits) keyed by tensor name")
    p.add_argument("--level", choices=LEVELS, default=None)
    p.add_argument("--samples", type=int, default=1000)
    a = p.parse_args(argv)
    level = a.level or ("sampled" if a.source else "structure")
    try:
        entries = container_file.load(a.file)
    except (container_file.FormatError, DfError, OSError) as e:
        print(f"FAIL: {e}")
        return FAIL
    source = None
    if a.source:
        with np.load(a.source) as z:
            source = {k: torch.from_numpy(np.ascontiguousarray(z[k]).view(np.int16)).cuda() for k in z.files}
    code, why = verify(entries, level, source, a.samples)
    print({PASS: "PASS", FAIL: "FAIL", CANNOT: "COULD NOT CHECK"}[code] + ": " + why)
    return code


if __name__ == "__main__":
    sys.exit(main())

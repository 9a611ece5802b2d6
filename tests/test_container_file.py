"""The container file on the CPU: oracle-made containers saved and loaded back
part for part, the header fields, and files that must be refused (truncated,
wrong magic, parts of the wrong size) before anything could reach a decoder."""
import hashlib
import os

import numpy as np
import pytest

import oracle
from lossless_bf16_weight_huffman_b200 import codec, container_file, synth


def _containers():
    out = []
    w1 = synth.generate(synth.single_1024x4096()[0])[:100_003]
    w2 = synth.generate(synth.heavy_tail_64m()[0])[:50_000]
    for name, w, C, T in (("a.weight", w1, 32, 32), ("b.weight", w2, 16, 64), ("empty", w1[:0], 32, 32)):
        enc = oracle.encode(w, chunk_bytes=C, threads_per_block=T)
        c = codec.Compressed.from_host(lengths=enc.lengths, max_len=32, total_bits=enc.total_bits, n=enc.n,
                                       stream=enc.stream, gaps=enc.gaps, offsets=enc.offsets, sm=enc.sm,
                                       shape=(w.size,), chunk_bytes=C, threads_per_block=T, device="cpu")
        out.append((name, c, enc, w))
    return out


def test_save_load_round_trip(tmp_path):
    items = _containers()
    path = os.path.join(tmp_path, "set.df11")
    digests = {items[0][0]: hashlib.sha256(b"x").digest()}
    container_file.save(path, [(n, c) for n, c, _, _ in items], digests)
    back = container_file.load(path, device="cpu")
    assert [b[0] for b in back] == [n for n, _, _, _ in items]
    for (name, c, enc, w), (bname, bc, sha) in zip(items, back):
        assert bc.n == enc.n and bc.total_bits == enc.total_bits
        assert bc.chunk_bytes == c.chunk_bytes and bc.threads_per_block == c.threads_per_block
        assert (bc.lengths == enc.lengths).all()
        assert (bc.stream.numpy() == enc.stream).all()
        assert (bc.gaps.numpy() == enc.gaps).all()
        assert (bc.offsets.numpy().view(np.uint64) == enc.offsets).all()
        assert (bc.sm.numpy()[: enc.n] == enc.sm).all()
        assert sha == digests.get(name)
        # the oracle decodes what came back
        if enc.n:
            out = oracle.decode(bc.stream.numpy(), bc.total_bits, bc.sm.numpy()[: bc.n], bc.n, bc.lengths,
                                bc.chunk_bytes, bc.threads_per_block)
            assert (out == w).all()
    head = container_file.read_header(path)
    for e in head["tensors"]:
        for p, (off, nbytes) in e["parts"].items():
            assert off % container_file.ALIGN == 0


def test_damaged_files_are_refused(tmp_path):
    items = _containers()
    path = os.path.join(tmp_path, "set.df11")
    container_file.save(path, [(n, c) for n, c, _, _ in items])
    raw = open(path, "rb").read()
    bad = os.path.join(tmp_path, "bad.df11")
    open(bad, "wb").write(b"NOTDF11!" + raw[8:])
    with pytest.raises(container_file.FormatError):
        container_file.load(bad, device="cpu")
    open(bad, "wb").write(raw[: len(raw) - 100])  # the last parts run past the end
    with pytest.raises(container_file.FormatError):
        container_file.load(bad, device="cpu")
    # a header whose total_bits does not match its stream size (the header
    # padded to its old length, so the parts stay where they were)
    import json
    import struct

    head = container_file.read_header(path)
    head["tensors"][0]["total_bits"] += 4096
    old_len = struct.unpack("<Q", raw[16:24])[0]
    hb = json.dumps(head, separators=(",", ":")).encode()
    assert len(hb) <= old_len
    hb = hb + b" " * (old_len - len(hb))
    open(bad, "wb").write(raw[:24] + hb + raw[24 + old_len:])
    with pytest.raises(container_file.FormatError):
        container_file.load(bad, device="cpu")


def _index8_bytes(offsets):
    from oracle import index8

    a, b, d, o = index8.build(offsets)
    return np.concatenate([a.view(np.uint8), b.view(np.uint8), d, o.view(np.uint8)]), o.size // 64


def test_save_load_compact_index(tmp_path):
    """A container that holds the compact block index (oracle-built) in place
    of the uint64 offsets: saved, loaded back byte for byte, with a wide
    superblock among its superblocks."""
    w = np.concatenate([synth.generate(synth.single_1024x4096()[0])[:600_000], np.full(400_000, 0x3F80, np.uint16),
                        synth.generate(synth.heavy_tail_64m()[0])[:300_001]])
    enc = oracle.encode(w, chunk_bytes=32, threads_per_block=32)
    ix, wide = _index8_bytes(enc.offsets)
    assert wide >= 1  # the constant run packs many more codes per block
    c = codec.Compressed.from_host(lengths=enc.lengths, max_len=32, total_bits=enc.total_bits, n=enc.n,
                                   stream=enc.stream, gaps=enc.gaps, offsets=None, sm=enc.sm, shape=(w.size,),
                                   device="cpu", index8=ix, index8_wide=wide)
    assert c.index_kind == "idx8" and c.index_bytes == ix.size < 8 * enc.offsets.size
    path = os.path.join(tmp_path, "ix.df11")
    container_file.save(path, [("t", c)])
    (name, bc, _), = container_file.load(path, device="cpu")
    assert bc.index_kind == "idx8" and bc.index8_wide == wide
    assert (bc.index8.numpy() == ix).all() and (bc.stream.numpy() == enc.stream).all()
    assert bc.container_bytes == c.container_bytes
    head = container_file.read_header(path)
    assert head["tensors"][0]["index"] == "idx8"


def test_compact_index_of_wrong_size_is_refused(tmp_path):
    w = synth.generate(synth.single_1024x4096()[0])[:200_000]
    enc = oracle.encode(w, chunk_bytes=32, threads_per_block=32)
    ix, wide = _index8_bytes(enc.offsets)
    c = codec.Compressed.from_host(lengths=enc.lengths, max_len=32, total_bits=enc.total_bits, n=enc.n,
                                   stream=enc.stream, gaps=enc.gaps, offsets=None, sm=enc.sm, device="cpu",
                                   index8=np.concatenate([ix, np.zeros(4, np.uint8)]), index8_wide=wide)
    path = os.path.join(tmp_path, "bad.df11")
    container_file.save(path, [("t", c)])
    with pytest.raises(container_file.FormatError):
        container_file.load(path, device="cpu")

"""Helpers for the GPU parity tests: move oracle containers to the device and
compare device results with oracle results byte for byte."""
import numpy as np
import torch

import oracle
from lossless_bf16_weight_huffman_b200 import api, codec


def to_dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def dev_u16(w: np.ndarray) -> torch.Tensor:
    return to_dev(np.ascontiguousarray(w, np.uint16).view(np.int16))


def host_u16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).reshape(-1).cpu().numpy().view(np.uint16)


def from_oracle(enc: oracle.Encoded, max_len: int | None = None) -> codec.Compressed:
    return codec.Compressed.from_host(
        lengths=enc.lengths, max_len=max_len or enc.max_len, total_bits=enc.total_bits, n=enc.n,
        stream=enc.stream, gaps=enc.gaps, offsets=enc.offsets, sm=enc.sm, chunk_bytes=enc.chunk_bytes,
        threads_per_block=enc.threads_per_block)


def err_word() -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def gpu_decode(c: codec.Compressed, fill: int = -1) -> tuple[np.ndarray, int]:
    """Decode into a buffer pre-filled with `fill` (so unwritten outputs show)."""
    out = torch.full((max(c.n, 1),), fill, dtype=torch.int16, device="cuda")[: c.n]
    err = err_word()
    codec.decompress(c, out, err)
    flags = api.df_read_error(err)
    return host_u16(out), flags


def assert_container_equal(c: codec.Compressed, enc: oracle.Encoded):
    assert c.total_bits == enc.total_bits
    assert (np.frombuffer(bytes(c.code.lengths), np.uint8) == enc.lengths).all()
    assert (c.stream.cpu().numpy() == enc.stream).all(), "stream bytes differ"
    assert (c.gaps.cpu().numpy() == enc.gaps).all(), "gap bytes differ"
    assert (c.offsets.cpu().numpy().view(np.uint64) == enc.offsets).all(), "block offsets differ"
    assert (c.sm[: enc.n].cpu().numpy() == enc.sm).all(), "sign|fraction bytes differ"

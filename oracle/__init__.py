"""The CPU oracle: a plain, single-threaded restatement of the codec.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline may import this package; the product library never does. The C source
(``df11_oracle.c``) shares no code with the CUDA library.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "df11_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")

OK, EINVAL, ECORRUPT, ENOMEM = 0, -1, -2, -3

_lib = None


class Sizes(ctypes.Structure):
    _fields_ = [
        ("total_bits", ctypes.c_uint64),
        ("n_chunks", ctypes.c_uint64),
        ("stream_bytes", ctypes.c_uint64),
        ("gap_bytes", ctypes.c_uint64),
        ("n_blocks", ctypes.c_uint64),
        ("offsets_bytes", ctypes.c_uint64),
        ("sm_bytes", ctypes.c_uint64),
        ("container_bytes", ctypes.c_uint64),
    ]

    def as_dict(self) -> dict:
        return {name: int(getattr(self, name)) for name, _ in self._fields_}


def build_oracle(force: bool = False) -> str:
    """Compile the oracle with gcc -O2 (plain C11, no threads)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra", "-o", tmp, _SRC])
        os.replace(tmp, _SO)
    return _SO


def _p(a: np.ndarray | None):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def lib():
    global _lib
    if _lib is None:
        build_oracle()
        L = ctypes.CDLL(_SO)
        vp, u64, u32, i32 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int
        L.oracle_split.argtypes = [vp, u64, vp, vp]
        L.oracle_join.argtypes = [vp, vp, u64, vp]
        L.oracle_histogram.argtypes = [vp, u64, vp]
        L.oracle_package_merge.argtypes = [vp, i32, vp]
        L.oracle_package_merge.restype = i32
        L.oracle_canonical_codes.argtypes = [vp, vp]
        L.oracle_sizes.argtypes = [u64, u64, u32, u32, ctypes.POINTER(Sizes)]
        L.oracle_sizes.restype = i32
        L.oracle_total_bits.argtypes = [vp, vp]
        L.oracle_total_bits.restype = u64
        L.oracle_encode.argtypes = [vp, u64, vp, vp, u32, u32, vp, vp, vp, vp]
        L.oracle_encode.restype = i32
        L.oracle_decode.argtypes = [vp, u64, vp, u64, vp, u32, u32, vp, vp, vp]
        L.oracle_decode.restype = i32
        _lib = L
    return _lib


def _u16(w) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(w, dtype=np.uint16).reshape(-1))


def split(w):
    w = _u16(w)
    e = np.empty(w.size, np.uint8)
    sm = np.empty(w.size, np.uint8)
    lib().oracle_split(_p(w), w.size, _p(e), _p(sm))
    return e, sm


def join(e, sm) -> np.ndarray:
    e = np.ascontiguousarray(e, np.uint8)
    sm = np.ascontiguousarray(sm, np.uint8)
    w = np.empty(e.size, np.uint16)
    lib().oracle_join(_p(e), _p(sm), e.size, _p(w))
    return w


def histogram(w) -> np.ndarray:
    w = _u16(w)
    h = np.zeros(256, np.uint64)
    lib().oracle_histogram(_p(w), w.size, _p(h))
    return h


def package_merge(hist, max_len: int = 32) -> np.ndarray:
    h = np.ascontiguousarray(hist, np.uint64)
    assert h.size == 256
    lengths = np.zeros(256, np.uint8)
    rc = lib().oracle_package_merge(_p(h), int(max_len), _p(lengths))
    if rc != OK:
        raise ValueError(f"oracle_package_merge: {rc}")
    return lengths


def canonical_codes(lengths) -> np.ndarray:
    lengths = np.ascontiguousarray(lengths, np.uint8)
    codes = np.zeros(256, np.uint32)
    lib().oracle_canonical_codes(_p(lengths), _p(codes))
    return codes


def sizes(n: int, total_bits: int, chunk_bytes: int = 32, threads_per_block: int = 32) -> dict:
    s = Sizes()
    rc = lib().oracle_sizes(n, total_bits, chunk_bytes, threads_per_block, ctypes.byref(s))
    if rc != OK:
        raise ValueError(f"oracle_sizes: {rc}")
    return s.as_dict()


def total_bits(hist, lengths) -> int:
    h = np.ascontiguousarray(hist, np.uint64)
    lengths = np.ascontiguousarray(lengths, np.uint8)
    return int(lib().oracle_total_bits(_p(h), _p(lengths)))


class Encoded:
    """The oracle's container for one tensor (host arrays)."""

    def __init__(self, n, lengths, codes, chunk_bytes, threads_per_block, max_len, sz, stream, gaps, offsets, sm):
        self.n = n
        self.lengths = lengths
        self.codes = codes
        self.chunk_bytes = chunk_bytes
        self.threads_per_block = threads_per_block
        self.max_len = max_len
        self.sizes = sz
        self.total_bits = sz["total_bits"]
        self.stream = stream
        self.gaps = gaps
        self.offsets = offsets
        self.sm = sm

    @property
    def container_bytes(self) -> int:
        return self.sizes["container_bytes"]


def encode(w, max_len: int = 32, chunk_bytes: int = 32, threads_per_block: int = 32, lengths=None) -> Encoded:
    w = _u16(w)
    h = histogram(w)
    if lengths is None:
        lengths = package_merge(h, max_len)
    lengths = np.ascontiguousarray(lengths, np.uint8)
    codes = canonical_codes(lengths)
    sz = sizes(w.size, total_bits(h, lengths), chunk_bytes, threads_per_block)
    stream = np.zeros(sz["stream_bytes"], np.uint8)
    gaps = np.zeros(sz["gap_bytes"], np.uint8)
    offsets = np.zeros(sz["n_blocks"] + 1, np.uint64)
    sm = np.zeros(w.size, np.uint8)
    rc = lib().oracle_encode(_p(w), w.size, _p(lengths), _p(codes), chunk_bytes, threads_per_block,
                             _p(stream), _p(gaps), _p(offsets), _p(sm))
    if rc != OK:
        raise ValueError(f"oracle_encode: {rc}")
    return Encoded(w.size, lengths, codes, chunk_bytes, threads_per_block, max_len, sz, stream, gaps, offsets, sm)


def decode(stream, total_bits_: int, sm, n: int, lengths, chunk_bytes: int = 32, threads_per_block: int = 32,
           rederive: bool = False):
    """Bit-serial decode. Returns the BF16 bit patterns, or (w, gaps, offsets)
    with ``rederive``; raises ValueError on a corrupt container."""
    stream = np.ascontiguousarray(stream, np.uint8)
    sm = np.ascontiguousarray(sm, np.uint8)
    lengths = np.ascontiguousarray(lengths, np.uint8)
    out = np.zeros(n, np.uint16)
    gaps = offsets = None
    if rederive:
        sz = sizes(n, total_bits_, chunk_bytes, threads_per_block)
        gaps = np.zeros(sz["gap_bytes"], np.uint8)
        offsets = np.zeros(sz["n_blocks"] + 1, np.uint64)
    rc = lib().oracle_decode(_p(stream), total_bits_, _p(sm), n, _p(lengths), chunk_bytes, threads_per_block,
                             _p(out), _p(gaps), _p(offsets))
    if rc != OK:
        raise ValueError(f"oracle_decode: {rc}")
    return (out, gaps, offsets) if rederive else out


def decode_encoded(enc: Encoded, rederive: bool = False):
    return decode(enc.stream, enc.total_bits, enc.sm, enc.n, enc.lengths, enc.chunk_bytes,
                  enc.threads_per_block, rederive)


def unpack_gaps(gaps, n_chunks: int) -> np.ndarray:
    """The 5-bit gap fields as integers (MSB-first bit order)."""
    bits = np.unpackbits(np.asarray(gaps, np.uint8))
    out = np.zeros(n_chunks, np.int64)
    for b in range(5):
        out = (out << 1) | bits[5 * np.arange(n_chunks) + b]
    return out

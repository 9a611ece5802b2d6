"""Lossless BF16 weight compression for B200: the exponent of every weight is
replaced by a canonical, length-limited Huffman code and the sign|fraction
byte is kept raw; encode and decode run in hand-written sm_100a CUDA kernels
behind a C ABI (include/df11.h, libdf11.so).

``api`` mirrors the C entry points one to one; ``codec`` wraps them for torch
CUDA tensors (compress, decompress, BatchDecoder); ``synth`` generates the
seeded synthetic weight sets.
"""

__all__ = ["api", "codec", "synth"]


def __getattr__(name):
    if name in ("api", "codec"):
        import importlib

        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)

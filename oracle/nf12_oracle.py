"""Oracle for the fixed 12-bit format (nf12): plain numpy, TEST INFRASTRUCTURE
ONLY (the tests, the smoke check and the benchmark's CPU baseline use it; the
product library never does). It shares no code with the CUDA library.

What the page fixes (agihunt.info news item "Developer open-sources nf12:
lossless 12-bit compression for BF16 models", section "Confirmed" and the
related posts below it):
  - post-training weights rarely use the full exponent range: the top four
    exponent bits are the same for almost all weights, so they can be left
    out, leaving 1 sign + 4 exponent + 7 fraction bits = 12 bits per weight;
  - weights are handled in groups of 8: a normal group packs from 16 bytes
    to 12; a group that does not fit escapes, and an escaped group takes 28
    bytes in all;
  - decoding gives back the BF16 bits exactly.
Readings taken where the page is silent (this library's layout):
  - the shared top nibble is the page's 0111 unless the caller names another
    (``top``); one value holds for a whole tensor;
  - a group escapes when any of its 8 weights has other top bits; its 12-byte
    slot then holds its index in a side buffer (uint32, little-endian, then 8
    zero bytes) and the side buffer holds its 8 raw weights (16 bytes):
    12 + 16 = 28 bytes;
  - an escape bitmap marks escaped groups, bit g & 7 of byte g >> 3, padded
    with zero bits to a whole number of 32-bit words;
  - in a normal group, weight k's 12-bit field is
    f = sign << 11 | (low 4 exponent bits) << 7 | fraction, and fields 2j and
    2j + 1 fill bytes 3j .. 3j+2 little-endian (f0 | f1 << 12);
  - the last group is padded with weights whose top bits are the shared ones
    and whose other bits are 0; padding is not part of the output.
Sizes: slots 12 G, bitmap 4 ceil(G / 32), side 16 E bytes, G = ceil(n / 8), E = escaped groups.
"""
from __future__ import annotations

import numpy as np


TOP = 0b0111  # the top four exponent bits the page names


def encode(w, top: int = TOP):
    """(slots, bitmap, side) of the weights w (uint16 BF16 bit patterns)."""
    w = np.ascontiguousarray(np.asarray(w, np.uint16).reshape(-1))
    n = w.size
    G = (n + 7) // 8
    pad = np.full(8 * G - n, top << 11, np.uint16)
    g = np.concatenate([w, pad]).reshape(G, 8)
    escaped = (((g >> 11) & 0xF) != top).any(axis=1)
    bitmap = np.zeros(4 * ((G + 31) // 32), np.uint8)
    for gi in np.nonzero(escaped)[0]:
        bitmap[gi >> 3] |= np.uint8(1 << (gi & 7))
    slots = np.zeros((G, 12), np.uint8)
    f = (((g >> 15) & 1) << 11 | (g & 0x7FF)).astype(np.uint32)  # 12-bit fields
    for j in range(4):
        v = f[:, 2 * j] | (f[:, 2 * j + 1] << 12)
        slots[:, 3 * j] = v & 0xFF
        slots[:, 3 * j + 1] = (v >> 8) & 0xFF
        slots[:, 3 * j + 2] = (v >> 16) & 0xFF
    esc = np.nonzero(escaped)[0]
    side = g[esc].reshape(-1).copy()
    slots[esc] = 0
    idx = np.arange(esc.size, dtype=np.uint32)
    for b in range(4):
        slots[esc, b] = (idx >> (8 * b)) & 0xFF
    return slots.reshape(-1), bitmap, side


def decode(slots, bitmap, side, n: int, top: int = TOP) -> np.ndarray:
    """The n weights back from the parts."""
    G = (n + 7) // 8
    slots = np.asarray(slots, np.uint8).reshape(G, 12)
    out = np.zeros((G, 8), np.uint16)
    for j in range(4):
        v = (slots[:, 3 * j].astype(np.uint32) | slots[:, 3 * j + 1].astype(np.uint32) << 8 |
             slots[:, 3 * j + 2].astype(np.uint32) << 16)
        for k, fk in ((2 * j, v & 0xFFF), (2 * j + 1, v >> 12)):
            out[:, k] = ((fk >> 11) << 15 | top << 11 | (fk & 0x7FF)).astype(np.uint16)
    bits = np.unpackbits(np.asarray(bitmap, np.uint8), bitorder="little")[:G].astype(bool)
    side = np.asarray(side, np.uint16).reshape(-1, 8)
    for gi in np.nonzero(bits)[0]:
        i = int(slots[gi, 0]) | int(slots[gi, 1]) << 8 | int(slots[gi, 2]) << 16 | int(slots[gi, 3]) << 24
        out[gi] = side[i]
    return out.reshape(-1)[:n]


def sizes(n: int, escaped: int) -> dict:
    G = (n + 7) // 8
    bitmap = 4 * ((G + 31) // 32)
    return {"groups": G, "slots_bytes": 12 * G, "bitmap_bytes": bitmap, "side_bytes": 16 * escaped,
            "total_bytes": 12 * G + bitmap + 16 * escaped}

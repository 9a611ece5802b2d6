"""Oracle for the compact 8-bit block index ("idx8"): plain numpy, TEST
INFRASTRUCTURE ONLY (tests, smoke check and benchmark CPU baseline); the
product library never imports it and it shares no code with the CUDA library.

What the page fixes (df11pack, GitHub page, "What is checked, and what is
not", the opt-in list: --index idx8, an experimental 8-bit block index that
makes the file smaller). It gives no layout; this library's reading:

The full index is one uint64 output offset per format block, O[0] = 0 ..
O[B] = n, so block b decodes O[b+1] - O[b] codes (its count c_b). The compact
index groups blocks into superblocks of 64 and stores, per superblock s:
  anchor[s]  uint64, O[64 s];
  base[s]    uint32: the smallest count in s when every count of s is within
             255 of it; otherwise 2^31 | k, k = how many such wide
             superblocks come before s;
  delta[b]   uint8 per block (64 per superblock, the last one padded with 0):
             c_b - base[s], or 0 in a wide superblock;
  overflow   uint32 counts, 64 per wide superblock in order (k-th wide
             superblock at 64 k; padding 0).
So O[64 s + j] = anchor[s] + sum of the counts of blocks 64 s .. 64 s + j - 1.
Sizes: 76 bytes per superblock + 256 per wide one, against 8 (B + 1) bytes.
"""
from __future__ import annotations

import numpy as np

SUPER = 64
WIDE = 1 << 31


def build(offsets):
    """(anchor, base, delta, overflow) of the block offsets O[0..B]."""
    O = np.asarray(offsets, np.uint64)
    B = O.size - 1
    S = (B + SUPER - 1) // SUPER
    counts = np.zeros(S * SUPER, np.int64)
    counts[:B] = (O[1:] - O[:-1]).astype(np.int64)
    anchor = np.zeros(S, np.uint64)
    base = np.zeros(S, np.uint32)
    delta = np.zeros(S * SUPER, np.uint8)
    over = []
    for s in range(S):
        anchor[s] = O[SUPER * s]
        blk = counts[SUPER * s: SUPER * s + SUPER]
        real = blk[: min(SUPER, B - SUPER * s)]
        lo, hi = int(real.min()), int(real.max())
        if hi - lo <= 255:
            base[s] = lo
            delta[SUPER * s: SUPER * s + real.size] = real - lo
        else:
            base[s] = WIDE | (len(over) // SUPER)
            over.extend(int(c) for c in blk)  # the padding entries past B are 0
    return anchor, base, delta, np.array(over, np.uint32)


def expand(anchor, base, delta, overflow, n_blocks: int) -> np.ndarray:
    """The block offsets O[0..B] back from the compact index."""
    O = np.zeros(n_blocks + 1, np.uint64)
    for b in range(n_blocks):
        s, j = divmod(b, SUPER)
        if j == 0:
            O[b] = anchor[s]
        w = int(base[s])
        c = int(overflow[SUPER * (w & (WIDE - 1)) + j]) if w & WIDE else w + int(delta[b])
        O[b + 1] = int(O[b]) + c
    return O


def index_bytes(n_blocks: int, n_wide: int) -> int:
    S = (n_blocks + SUPER - 1) // SUPER
    return 76 * S + 4 * SUPER * n_wide

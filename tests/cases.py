"""Hand-made test tensors shared by the CPU and GPU tests."""
import numpy as np


def long_code_tensor(n, seed=5):
    """Weights whose code (given lengths) has many codes longer than the wide
    window: codes of 1..7 bits for exponents 120..126 (Kraft sum 127/128) and
    14-bit codes for 128 others (the last 1/128), drawn so that 30% of the
    weights take a long code."""
    rng = np.random.default_rng(seed)
    lengths = np.zeros(256, np.uint8)
    lengths[120:127] = np.arange(1, 8)
    longs = [s for s in range(256) if not 120 <= s <= 126][:128]
    lengths[longs] = 14
    short = np.array([120, 121, 122, 123, 124, 125, 126])
    e = np.where(rng.random(n) < 0.3, np.array(longs)[rng.integers(0, 128, n)],
                 short[np.minimum(rng.geometric(0.5, n) - 1, 6)])
    sm = rng.integers(0, 256, n)
    w = (((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)).astype(np.uint16)
    return w, lengths

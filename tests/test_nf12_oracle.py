"""The fixed 12-bit format's oracle (oracle/nf12_oracle.py) pinned to what the
page and arithmetic fix, without the GPU:

* a worked example derived by hand (tests/golden/nf12_worked_example.txt);
* the page's sizes: 12 bytes for a normal group of 8, 28 for an escaped one;
* the escape rule restated through float magnitudes: the top exponent bits
  are 0111 exactly when a finite value has magnitude in [2^-15, 2);
* each 12-bit field, read as sign, 4 exponent bits and 7 fraction bits with
  exponent 112 + e4, gives the weight's value by float arithmetic;
* every one of the 65,536 BF16 bit patterns round-trips.
"""
import os

import numpy as np
import pytest

from oracle import nf12_oracle as nf

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "nf12_worked_example.txt")


def _golden():
    d = {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        key, *vals = line.split()
        d[key] = vals
    return d


def _as_float(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32)


def test_worked_example():
    g = _golden()
    n = int(g["n"][0])
    w = np.array([int(v, 16) for v in g["weights"]], np.uint16)
    assert w.size == n
    slots, bitmap, side = nf.encode(w)
    assert slots.tolist() == [int(v, 16) for v in g["slots"]]
    assert bitmap.tolist() == [int(v, 16) for v in g["bitmap"]]
    assert side.tolist() == [int(v, 16) for v in g["side"]]
    assert np.array_equal(nf.decode(slots, bitmap, side, n), w)


def test_page_sizes_normal_12_escaped_28():
    w = np.full(8 * 64, 0x3F80, np.uint16)  # 64 groups, none escapes
    s0, b0, e0 = nf.encode(w)
    w[8 * 5 + 3] = 0x4000  # one weight outside: its group escapes
    s1, b1, e1 = nf.encode(w)
    assert s0.size == s1.size == 12 * 64 and e0.size == 0
    assert (s1.size + 2 * e1.size) - (s0.size + 2 * e0.size) == 16  # 12 + 16 = 28 bytes for that group
    z = nf.sizes(w.size, 1)
    assert z["slots_bytes"] + z["side_bytes"] == 12 * 63 + 28
    # no escapes: 12 of every 16 bytes, plus one bit per group
    assert nf.sizes(8 * 1024, 0)["total_bytes"] == 12 * 1024 + 1024 // 8


def test_escape_rule_is_the_magnitude_range():
    """Top exponent bits 0111 <=> exponent field 112..127 <=> a finite
    nonzero normal value with 2^-15 <= |x| < 2 (checked on all patterns)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):  # NaN payloads
        x = _as_float(bits).astype(np.float64)
    in_range = np.isfinite(x) & (np.abs(x) >= 2.0 ** -15) & (np.abs(x) < 2.0)
    w = np.repeat(bits, 8)  # group i = eight copies of pattern i
    _, bitmap, side = nf.encode(w)
    esc = np.unpackbits(bitmap, bitorder="little")[:65536].astype(bool)
    assert np.array_equal(esc, ~in_range)
    assert side.size == 8 * int((~in_range).sum())


def test_fields_give_the_value_by_float_arithmetic():
    rng = np.random.default_rng(11)
    x = rng.normal(0, 0.05, 8 * 4096).astype(np.float32)
    x = x[(np.abs(x) >= 2.0 ** -15) & (np.abs(x) < 2.0)][: 8 * 2048]
    w = (x.view(np.uint32) >> 16).astype(np.uint16)  # truncate to BF16 bits
    slots, bitmap, side = nf.encode(w)
    assert side.size == 0 and not bitmap.any()
    b = slots.reshape(-1, 12).astype(np.int64)
    got = []
    for j in range(4):
        v = b[:, 3 * j] + 256 * b[:, 3 * j + 1] + 65536 * b[:, 3 * j + 2]
        for f in (v % 4096, v // 4096):
            s, e4, m = f // 2048, (f // 128) % 16, f % 128
            got.append((-1.0) ** s * 2.0 ** (112 + e4 - 127) * (1 + m / 128))
    got = np.stack(got, axis=1).reshape(-1)
    assert np.array_equal(got, _as_float(w).astype(np.float64))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_round_trip_all_patterns(seed):
    rng = np.random.default_rng(seed)
    w = rng.permutation(np.arange(65536, dtype=np.uint32)).astype(np.uint16)
    # mostly in-range weights with the patterns sprinkled in, ragged length
    base = (rng.normal(0, 0.02, 300_000).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    mixed = np.concatenate([base[:150_000], w, base[150_000:]])[: 365_533]
    for arr in (w, mixed, mixed[:1], mixed[:7], mixed[:9], np.zeros(0, np.uint16)):
        slots, bitmap, side = nf.encode(arr)
        assert np.array_equal(nf.decode(slots, bitmap, side, arr.size), arr)
        z = nf.sizes(arr.size, side.size // 8)
        assert (slots.size, bitmap.size, 2 * side.size) == (z["slots_bytes"], z["bitmap_bytes"], z["side_bytes"])


def test_other_top_nibble():
    """A tensor whose weights sit in another exponent band names its own top
    bits (0110: magnitudes in [2^-31, 2^-15))."""
    rng = np.random.default_rng(4)
    x = (rng.uniform(1, 2, 800) * 2.0 ** rng.integers(-31, -15, 800)).astype(np.float32)
    w = (x.view(np.uint32) >> 16).astype(np.uint16)
    s7, b7, e7 = nf.encode(w)
    s6, b6, e6 = nf.encode(w, top=0b0110)
    assert e6.size == 0 and e7.size == w.size
    assert np.array_equal(nf.decode(s6, b6, e6, w.size, top=0b0110), w)

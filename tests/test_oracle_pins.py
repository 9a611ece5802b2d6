"""Pins for the CPU oracle: facts fixed by the pages, by the mathematics of
prefix codes, or by hand-worked examples, so that a plausible mistake anywhere
in the oracle (a wrong tie rule, shift, bit order, index or sentinel) fails at
least one of them. None of these tests uses the oracle to check itself: each
compares it with brute force, a textbook routine written here, a closed form
or a stored hand-traced value.
"""
import heapq
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from lossless_bf16_weight_huffman_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _hist(d):
    h = np.zeros(256, np.uint64)
    for k, v in d.items():
        h[int(k)] = v
    return h


def heap_huffman_lengths(freqs):
    """Textbook Huffman (a binary heap of subtrees); returns depth per input."""
    if len(freqs) == 1:
        return [1]
    heap = [(f, i, [i]) for i, f in enumerate(freqs)]
    heapq.heapify(heap)
    depth = [0] * len(freqs)
    tick = len(freqs)
    while len(heap) > 1:
        fa, _, a = heapq.heappop(heap)
        fb, _, b = heapq.heappop(heap)
        for s in a + b:
            depth[s] += 1
        heapq.heappush(heap, (fa + fb, tick, a + b))
        tick += 1
    return depth


def brute_force_min_cost(freqs, max_len):
    best = None
    for ls in itertools.product(range(1, max_len + 1), repeat=len(freqs)):
        if sum(2.0 ** -l for l in ls) <= 1.0 + 1e-12:
            c = sum(f * l for f, l in zip(freqs, ls))
            best = c if best is None or c < best else best
    return best


def kraft_units(lengths):
    return sum(1 << (32 - int(l)) for l in lengths if l > 0)


# ---------------------------------------------------------------- hand-worked examples


def test_hand_worked_codes():
    g = json.load(open(os.path.join(GOLDEN, "hand_worked.json")))
    for case in g["cases"]:
        lengths = oracle.package_merge(_hist(case["hist"]), case["max_len"])
        codes = oracle.canonical_codes(lengths)
        want_l = {int(k): v for k, v in case["lengths"].items()}
        want_c = {int(k): v for k, v in case["codes"].items()}
        got_l = {s: int(lengths[s]) for s in range(256) if lengths[s]}
        assert got_l == want_l, case["name"]
        assert {s: int(codes[s]) for s in want_c} == want_c, case["name"]


def test_hand_worked_stream():
    g = json.load(open(os.path.join(GOLDEN, "hand_worked.json")))
    cases = {c["name"]: c for c in g["cases"]}
    for st in g["streams"]:
        case = cases[st["lengths_from"]]
        w = np.array(st["weights"], np.uint16)
        lengths = np.zeros(256, np.uint8)
        for k, v in case["lengths"].items():
            lengths[int(k)] = v
        enc = oracle.encode(w, lengths=lengths)
        assert enc.total_bits == st["total_bits"]
        pre = bytes.fromhex(st["stream_prefix_hex"])
        assert bytes(enc.stream[: len(pre)]) == pre
        assert not enc.stream[len(pre):].any()
        assert bytes(enc.sm) == bytes.fromhex(st["sm_hex"])
        assert (oracle.decode_encoded(enc) == w).all()


# ---------------------------------------------------------------- code construction


@pytest.mark.parametrize("seed", range(40))
def test_kraft_equality_and_limit(seed):
    rng = np.random.default_rng(seed)
    k = int(rng.integers(2, 257))
    max_len = int(rng.integers(max(1, math.ceil(math.log2(k))), 33))
    syms = rng.choice(256, size=k, replace=False)
    h = np.zeros(256, np.uint64)
    # heavy-tailed frequencies, so that the limit binds for small max_len
    h[syms] = (rng.pareto(0.7, size=k) * 1000).astype(np.uint64) + 1
    lengths = oracle.package_merge(h, max_len)
    assert set(np.nonzero(lengths)[0]) == set(syms.tolist())
    assert lengths.max() <= max_len
    assert kraft_units(lengths) == 1 << 32


def test_brute_force_optimality_tiny_alphabets():
    rng = np.random.default_rng(7)
    checked = 0
    for k in range(2, 8):
        for max_len in range(max(1, math.ceil(math.log2(k))), k):
            for _ in range(10):
                freqs = [int(x) for x in rng.integers(1, 50, size=k)]
                h = np.zeros(256, np.uint64)
                syms = rng.choice(256, size=k, replace=False)
                for s, f in zip(syms, freqs):
                    h[s] = f
                lengths = oracle.package_merge(h, max_len)
                cost = sum(int(h[s]) * int(lengths[s]) for s in syms)
                assert cost == brute_force_min_cost(freqs, max_len), (freqs, max_len)
                assert lengths.max() <= max_len
                checked += 1
    assert checked > 100


@pytest.mark.parametrize("seed", range(25))
def test_equals_heap_huffman_when_limit_does_not_bind(seed):
    rng = np.random.default_rng(100 + seed)
    k = int(rng.integers(2, 257))
    freqs = [int(x) for x in rng.integers(1, 10**6, size=k)]
    depth = heap_huffman_lengths(freqs)
    h = np.zeros(256, np.uint64)
    syms = rng.choice(256, size=k, replace=False)
    for s, f in zip(syms, freqs):
        h[s] = f
    max_len = 32
    assert max(depth) <= max_len
    lengths = oracle.package_merge(h, max_len)
    cost = sum(int(h[s]) * int(lengths[s]) for s in syms)
    assert cost == sum(f * d for f, d in zip(freqs, depth))


def test_dyadic_frequencies_give_minus_log2_p():
    # p = 2^-1, 2^-2, ..., 2^-8, 2^-8 : lengths 1..8, 8 and cost = entropy
    freqs = [128, 64, 32, 16, 8, 4, 2, 1, 1]
    syms = [200, 3, 77, 120, 121, 5, 255, 0, 9]
    h = np.zeros(256, np.uint64)
    for s, f in zip(syms, freqs):
        h[s] = f
    lengths = oracle.package_merge(h, 32)
    n = sum(freqs)
    for s, f in zip(syms, freqs):
        assert lengths[s] == -math.log2(f / n)
    entropy_bits = -sum(f * math.log2(f / n) for f in freqs)
    assert oracle.total_bits(h, lengths) == entropy_bits


def test_uniform_256_stream_is_the_exponent_bytes():
    # all 256 exponents equally often: every length 8, canonical code = symbol,
    # so the MSB-first stream is the exponent bytes themselves
    rng = np.random.default_rng(3)
    e = np.repeat(np.arange(256, dtype=np.uint16), 37)
    rng.shuffle(e)
    sm = rng.integers(0, 256, size=e.size).astype(np.uint16)
    w = (((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)).astype(np.uint16)
    enc = oracle.encode(w)
    assert (enc.lengths == 8).all()
    assert (enc.codes == np.arange(256)).all()
    assert enc.total_bits == 8 * e.size
    assert bytes(enc.stream[: e.size]) == bytes(e.astype(np.uint8))
    assert bytes(enc.sm) == bytes(sm.astype(np.uint8))


def test_fibonacci_frequencies_limit_binds():
    fib = [1, 1]
    while len(fib) < 40:
        fib.append(fib[-1] + fib[-2])
    assert max(heap_huffman_lengths(fib)) == 39
    h = np.zeros(256, np.uint64)
    h[:40] = fib
    lengths = oracle.package_merge(h, 32)
    assert lengths.max() == 32
    assert kraft_units(lengths) == 1 << 32
    unrestricted = sum(f * d for f, d in zip(fib, heap_huffman_lengths(fib)))
    assert oracle.total_bits(h, lengths) >= unrestricted
    # a length-32 code can never beat the unrestricted optimum; a looser limit
    # never costs more than a tighter one
    prev = None
    for L in range(6, 40):
        if L > 32:
            break
        cost = oracle.total_bits(h, oracle.package_merge(h, L))
        if prev is not None:
            assert cost <= prev
        prev = cost


def test_single_and_empty_alphabets():
    assert not oracle.package_merge(np.zeros(256, np.uint64)).any()
    h = np.zeros(256, np.uint64)
    h[42] = 1000
    l = oracle.package_merge(h)
    assert l[42] == 1 and l.sum() == 1
    with pytest.raises(ValueError):
        oracle.package_merge(np.ones(256, np.uint64), 7)  # 256 symbols need 8 bits


def test_canonical_codes_are_prefix_free_and_ordered():
    rng = np.random.default_rng(11)
    for _ in range(20):
        k = int(rng.integers(2, 257))
        h = np.zeros(256, np.uint64)
        h[rng.choice(256, k, replace=False)] = rng.integers(1, 10**5, size=k)
        lengths = oracle.package_merge(h, int(rng.integers(max(8, math.ceil(math.log2(k))), 33)))
        codes = oracle.canonical_codes(lengths)
        words = sorted(
            (format(int(codes[s]), f"0{int(lengths[s])}b"), s) for s in range(256) if lengths[s]
        )
        for (a, _), (b, _) in zip(words, words[1:]):
            assert not b.startswith(a)
        # canonical: ordering by (length, symbol) is ordering by left-aligned code value
        by_ls = sorted((int(lengths[s]), s) for s in range(256) if lengths[s])
        vals = [int(codes[s]) << (32 - int(lengths[s])) for _, s in by_ls]
        assert vals == sorted(vals) and len(set(vals)) == len(vals)


# ---------------------------------------------------------------- bounds


@pytest.mark.parametrize("name", ["single_1024x4096", "heavy_tail_64m"])
def test_entropy_bound(name):
    spec = synth.weight_set(name)[0]
    w = synth.generate(spec)
    if w.size > 4_000_000:
        w = w[:4_000_000]
    h = oracle.histogram(w).astype(np.float64)
    n = h.sum()
    p = h[h > 0] / n
    H = float(-(p * np.log2(p)).sum())
    enc = oracle.encode(w)
    assert enc.total_bits >= n * H - 1e-6 * n
    assert enc.total_bits < n * (H + 1)
    # container: at least entropy plus the raw byte per weight
    assert 8 * enc.container_bytes >= n * (H + 8)


# ---------------------------------------------------------------- round trips


def test_all_65536_patterns_round_trip():
    w = synth.all_bf16_patterns()
    e, sm = oracle.split(w)
    assert (oracle.join(e, sm) == w).all()
    assert (e == ((w >> 7) & 0xFF)).all()
    enc = oracle.encode(w)
    assert (oracle.decode_encoded(enc) == w).all()
    # +-0, subnormals, Inf and NaN payloads are all among them
    for max_len in (8, 9, 12, 32):
        enc = oracle.encode(w, max_len=max_len)
        assert (oracle.decode_encoded(enc) == w).all()


@pytest.mark.parametrize("name", ["single_1024x4096", "heavy_tail_64m"])
def test_weight_sets_round_trip(name):
    spec = synth.weight_set(name)[0]
    w = synth.generate(spec)
    for max_len in (32, 12):
        enc = oracle.encode(w, max_len=max_len)
        out, gaps, offs = oracle.decode_encoded(enc, rederive=True)
        assert (out == w).all()
        assert (gaps == enc.gaps).all() and (offs == enc.offsets).all()


def test_mixed_set_round_trip_sample():
    specs = synth.mixed_2000()
    assert len(specs) == 2000
    for spec in specs[:60]:
        w = synth.generate(spec)
        enc = oracle.encode(w)
        assert (oracle.decode_encoded(enc) == w).all(), spec.name
    w0 = synth.generate(specs[0])
    assert len(set(((w0 >> 7) & 0xFF).tolist())) == 1
    w1 = synth.generate(specs[1])
    assert (np.bincount((w1 >> 7) & 0xFF, minlength=256) == 256).all()


def test_degenerate_tensors():
    for w in (np.zeros(0, np.uint16), np.array([0x3F80], np.uint16), np.array([0x8000, 0x7FC1], np.uint16)):
        enc = oracle.encode(w)
        assert (oracle.decode_encoded(enc) == w).all()
        assert enc.offsets[-1] == w.size and enc.sizes["n_chunks"] == 1
    enc = oracle.encode(np.zeros(0, np.uint16))
    assert enc.total_bits == 0 and not enc.stream.any()
    # single-symbol tensor: one zero bit per weight
    w = (0x3F80 | np.arange(1000) % 128).astype(np.uint16)
    enc = oracle.encode(w)
    assert enc.total_bits == 1000 and not enc.stream.any()
    assert (oracle.decode_encoded(enc) == w).all()


@pytest.mark.parametrize("chunk_bytes,tpb", [(16, 32), (32, 256), (64, 64)])
def test_stream_ending_on_chunk_boundary(chunk_bytes, tpb):
    # all lengths 8: total_bits = 8n lands exactly on a chunk boundary when n % C == 0
    n = chunk_bytes * 5 * 256
    w = ((np.arange(n) % 256) << 7).astype(np.uint16)
    enc = oracle.encode(w, chunk_bytes=chunk_bytes, threads_per_block=tpb)
    assert enc.total_bits == 8 * n and enc.total_bits % (8 * chunk_bytes) == 0
    assert enc.sizes["n_chunks"] == n // chunk_bytes
    gaps = oracle.unpack_gaps(enc.gaps, enc.sizes["n_chunks"])
    assert not gaps.any()
    out, g2, o2 = oracle.decode_encoded(enc, rederive=True)
    assert (out == w).all() and (g2 == enc.gaps).all() and (o2 == enc.offsets).all()


# ---------------------------------------------------------------- index: gaps and block offsets


@pytest.mark.parametrize("chunk_bytes,tpb,max_len", [(16, 32, 32), (32, 256, 32), (16, 64, 9), (128, 32, 16)])
def test_gaps_and_offsets_from_code_starts(chunk_bytes, tpb, max_len):
    spec = synth.heavy_tail_64m()[0]
    w = synth.generate(spec)[:300_000]
    enc = oracle.encode(w, max_len=max_len, chunk_bytes=chunk_bytes, threads_per_block=tpb)
    # code start positions by a cumulative sum of lengths; the end of the stream closes the list
    l = enc.lengths[(w >> 7) & 0xFF].astype(np.int64)
    starts = np.concatenate([[0], np.cumsum(l)])
    n_chunks = enc.sizes["n_chunks"]
    cb = 8 * chunk_bytes
    bounds = cb * np.arange(n_chunks, dtype=np.int64)
    first = np.searchsorted(starts, bounds, side="left")  # first start >= boundary
    gaps = starts[first] - bounds
    assert (gaps >= 0).all() and (gaps < max_len).all()
    assert (oracle.unpack_gaps(enc.gaps, n_chunks) == gaps).all()
    n_blocks = enc.sizes["n_blocks"]
    offs = np.searchsorted(starts[:-1], cb * tpb * np.arange(n_blocks, dtype=np.int64), side="left")
    assert (enc.offsets[:-1] == offs).all()
    assert enc.offsets[-1] == w.size
    assert enc.total_bits == starts[-1]
    # padding after the last code is zero
    tb = enc.total_bits
    bits = np.unpackbits(enc.stream)
    assert not bits[tb:].any()


def test_sizes_match_layout():
    h = oracle.histogram(synth.generate(synth.single_1024x4096()[0]))
    lengths = oracle.package_merge(h)
    tb = oracle.total_bits(h, lengths)
    assert tb == int((h * lengths.astype(np.uint64)).sum())
    s = oracle.sizes(int(h.sum()), tb, 32, 256)
    assert s["n_chunks"] == -(-tb // 256)
    assert s["stream_bytes"] == 32 * s["n_chunks"] + 16
    assert s["n_blocks"] == -(-s["n_chunks"] // 256)
    assert s["gap_bytes"] % 16 == 0 and s["gap_bytes"] * 8 >= 5 * s["n_chunks"] + 8


# ---------------------------------------------------------------- corruption is detected


def test_corrupt_containers_are_rejected():
    w = synth.generate(synth.single_1024x4096()[0])[:50_000]
    enc = oracle.encode(w)
    with pytest.raises(ValueError):  # truncated stream length
        oracle.decode(enc.stream, enc.total_bits - 1, enc.sm, enc.n, enc.lengths)
    with pytest.raises(ValueError):  # one weight too many
        oracle.decode(enc.stream, enc.total_bits, np.concatenate([enc.sm, [0]]), enc.n + 1, enc.lengths)
    bad = enc.stream.copy()
    bad[100] ^= 0x10
    try:
        out = oracle.decode(bad, enc.total_bits, enc.sm, enc.n, enc.lengths)
        assert not (out == w).all()
    except ValueError:
        pass


@pytest.mark.parametrize("tpb", [1, 2, 32])
def test_last_chunk_without_a_code_start(tpb):
    # lengths A=1, B=2, C=2 (codes 0, 10, 11). 127 A's then one B: B starts at
    # bit 127 and ends at 129, so no code starts in chunk 1 (bits 128..255).
    # Its gap points at the end of the stream (129 - 128 = 1) and a block that
    # begins there counts every code as starting before it.
    A, B = 0x3F80, 0x4000  # exponents 127 and 128
    lengths = np.zeros(256, np.uint8)
    lengths[127], lengths[128], lengths[129] = 1, 2, 2
    w = np.array([A] * 127 + [B], np.uint16)
    enc = oracle.encode(w, chunk_bytes=16, threads_per_block=tpb, lengths=lengths)
    assert enc.total_bits == 129 and enc.sizes["n_chunks"] == 2
    assert list(oracle.unpack_gaps(enc.gaps, 2)) == [0, 1]
    if tpb == 1:
        assert list(enc.offsets) == [0, 128, 128]
    else:
        assert list(enc.offsets) == [0, 128]
    out, g2, o2 = oracle.decode_encoded(enc, rederive=True)
    assert (out == w).all() and (g2 == enc.gaps).all() and (o2 == enc.offsets).all()

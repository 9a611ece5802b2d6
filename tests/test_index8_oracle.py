"""The compact 8-bit block index's oracle (oracle/index8.py) pinned without
the GPU: two worked examples derived by hand (tests/golden/), the round trip
on block offsets that the DF11 oracle encoder produces for synthetic weights
and on random offsets with narrow and wide superblocks, the narrow/wide rule
at its boundary (a range of 255 is narrow, 256 is wide), and the size
formula against the arrays."""
import os

import numpy as np
import pytest

import oracle
from oracle import index8 as ix
from lossless_bf16_weight_huffman_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "index8_worked_example.txt")


def _expand_list(tokens):
    out = []
    for t in tokens:
        if "*" in t:
            v, k = t.split("*")
            out.extend([int(v)] * int(k))
        else:
            out.append(int(t))
    return out


def _cases():
    cases, cur = [], None
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        key, *vals = line.split()
        if key == "case":
            cur = {"name": vals[0]}
            cases.append(cur)
        else:
            cur[key] = _expand_list(vals)
    return cases


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
def test_worked_examples(case):
    counts = np.array(case["counts"], np.uint64)
    O = np.concatenate([[0], np.cumsum(counts)]).astype(np.uint64)
    anchor, base, delta, over = ix.build(O)
    assert anchor.tolist() == case["anchor"]
    assert base.tolist() == case["base"]
    head = case["delta_head"]
    assert delta[: len(head)].tolist() == head and not delta[len(head):].any()
    S = len(case["anchor"])
    want_over = case["overflow"] + [0] * (-len(case["overflow"]) % 64)
    assert over.tolist() == want_over
    size = anchor.nbytes + base.nbytes + delta.nbytes + over.nbytes
    assert size == case["bytes"][0] == ix.index_bytes(counts.size, len(want_over) // 64)
    assert delta.size == 64 * S
    assert np.array_equal(ix.expand(anchor, base, delta, over, counts.size), O)


def test_round_trip_on_encoder_offsets():
    w = synth.generate(synth.single_1024x4096()[0])[:3_000_001]
    for tpb in (32, 4):
        enc = oracle.encode(w, chunk_bytes=32, threads_per_block=tpb)
        O = enc.offsets
        a, b, d, o = ix.build(O)
        assert np.array_equal(ix.expand(a, b, d, o, O.size - 1), O)
        assert O[-1] == w.size
        # per superblock: the counts sum to the next anchor
        for s in range(a.size - 1):
            assert int(a[s + 1]) - int(a[s]) == int(O[64 * s + 64] - O[64 * s])
        assert ix.index_bytes(O.size - 1, o.size // 64) < 8 * O.size


@pytest.mark.parametrize("seed", range(5))
def test_round_trip_random(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 700))
    counts = rng.integers(2000, 2000 + int(rng.choice([10, 255, 256, 5000])), B)
    if seed % 2:
        counts[rng.integers(0, B, 3)] = 0  # empty blocks
    O = np.concatenate([[0], np.cumsum(counts)]).astype(np.uint64)
    a, b, d, o = ix.build(O)
    assert np.array_equal(ix.expand(a, b, d, o, B), O)


def test_narrow_wide_boundary():
    for spread, wide in ((255, False), (256, True)):
        counts = np.full(64, 1000, np.int64)
        counts[17] += spread
        O = np.concatenate([[0], np.cumsum(counts)]).astype(np.uint64)
        a, b, d, o = ix.build(O)
        assert bool(b[0] & ix.WIDE) == wide
        assert o.size == (64 if wide else 0)
        assert np.array_equal(ix.expand(a, b, d, o, 64), O)

"""The compact block index on the GPU against its oracle (oracle/index8.py):

* df_index8_build writes the oracle's bytes (anchors, bases, deltas,
  overflow) for the offsets of GPU-encoded containers and for hand-made
  offsets with wide superblocks; too little room for the overflow is
  reported and nothing is written past it;
* df_index8_expand gives the offsets back;
* decode through the compact index (single and grouped, mixed with uint64
  offsets, wide superblocks included) equals the source, and equals the
  decode through the offsets;
* a bad overflow slot is reported and nothing lands outside the output.
"""
import numpy as np
import pytest
import torch

from lossless_bf16_weight_huffman_b200 import api, codec, synth
from lossless_bf16_weight_huffman_b200._native import DF_EFLAG_INDEX8
from oracle import index8 as ixo
from tests.gpu_util import dev_u16, err_word, host_u16, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda(cuda_device):
    from lossless_bf16_weight_huffman_b200 import build

    build.build_native()


def _oracle_bytes(offsets):
    a, b, d, o = ixo.build(offsets)
    return np.concatenate([a.view(np.uint8), b.view(np.uint8), d, o.view(np.uint8)]), o.size // 64


def _with_wide_blocks(n_rand=900_000):
    """Random weights around a run of one value (1-bit codes): the block counts
    jump at the run's edges, so some superblocks spread over more than 255."""
    a = synth.generate(synth.single_1024x4096()[0])
    return np.concatenate([a[:n_rand], np.full(500_000, 0x3F80, np.uint16), a[n_rand: 2 * n_rand + 17]])


def _build(offs_dev, nb, wide_room):
    ix = torch.full((api.df_index8_bytes(nb, wide_room) + 64,), 0x5A, dtype=torch.uint8, device="cuda")
    wide = torch.zeros(1, dtype=torch.int64, device="cuda")
    err = err_word()
    api.df_index8_build(offs_dev, nb, ix[: api.df_index8_bytes(nb, wide_room)], wide, err)
    return ix, int(wide.item()), api.df_read_error(err)


CASES = ["single", "heavy", "wide", "tiny"]


def _weights(kind):
    if kind == "single":
        return synth.generate(synth.single_1024x4096()[0])
    if kind == "heavy":
        return synth.generate(synth.heavy_tail_64m()[0])[:5_000_003]
    if kind == "wide":
        return _with_wide_blocks()
    return synth.generate(synth.single_1024x4096()[0])[:777]


@pytest.mark.parametrize("kind", CASES)
def test_build_matches_oracle_and_expands(kind):
    w = _weights(kind)
    c = codec.compress(dev_u16(w))
    O = c.offsets.cpu().numpy().view(np.uint64)
    want, wide = _oracle_bytes(O)
    nb = O.size - 1
    ix, got_wide, flags = _build(c.offsets, nb, wide)
    assert flags == 0 and got_wide == wide
    if kind == "wide":
        assert wide >= 1
    assert np.array_equal(ix[: want.size].cpu().numpy(), want)
    assert (ix[want.size:].cpu().numpy() == 0x5A).all()
    back = torch.empty(nb + 1, dtype=torch.int64, device="cuda")
    api.df_index8_expand(ix, nb, wide, back)
    assert np.array_equal(back.cpu().numpy().view(np.uint64), O)


def test_build_hand_made_offsets():
    rng = np.random.default_rng(3)
    for B, spread in ((1, 5), (64, 255), (64, 256), (129, 4000), (10_000, 300)):
        counts = rng.integers(1000, 1000 + spread + 1, B)
        O = np.concatenate([[0], np.cumsum(counts)]).astype(np.uint64)
        want, wide = _oracle_bytes(O)
        ix, got_wide, flags = _build(to_dev(O.view(np.int64)), B, wide)
        assert flags == 0 and got_wide == wide
        assert np.array_equal(ix[: want.size].cpu().numpy(), want)


def test_build_without_room_reports_and_stays_inside():
    w = _with_wide_blocks()
    c = codec.compress(dev_u16(w))
    nb = c.sizes["n_blocks"]
    ix, wide, flags = _build(c.offsets, nb, 0)
    assert wide >= 1 and flags & DF_EFLAG_INDEX8
    assert (ix[api.df_index8_bytes(nb, 0):].cpu().numpy() == 0x5A).all()


@pytest.mark.parametrize("kind", CASES)
def test_decode_through_compact_index(kind):
    w = _weights(kind)
    x = dev_u16(w)
    c = codec.compress(x)
    ref = codec.decompress(c, torch.empty_like(x))
    c.use_index8()
    assert c.index_kind == "idx8" and c.index_bytes < c.sizes["offsets_bytes"] or c.sizes["n_blocks"] < 64
    out = torch.full((w.size + 8,), -1, dtype=torch.int16, device="cuda")
    err = err_word()
    codec.decompress(c, out[: w.size], err)
    assert api.df_read_error(err) == 0
    assert torch.equal(out[: w.size], x) and torch.equal(ref, x)
    assert (host_u16(out[w.size:]) == 0xFFFF).all()


def test_grouped_decode_mixed_indexes():
    rng = np.random.default_rng(7)
    base = _with_wide_blocks(1_500_000)
    ws, comps, off = [], [], 0
    for i, k in enumerate([1, 5000, 2_000_000, 31, 700_000] + [int(v) for v in rng.integers(1, 300_000, 20)]):
        w = base[off: off + k] if off + k <= base.size else base[:k]
        off += k
        ws.append(w)
        comps.append(codec.compress(dev_u16(w), index="idx8" if i % 2 == 0 else "u64"))
    outs = [torch.full((len(w),), -1, dtype=torch.int16, device="cuda") for w in ws]
    dec = codec.BatchDecoder(comps, outs)
    err = err_word()
    dec.run(err)
    assert api.df_read_error(err) == 0
    for o, w in zip(outs, ws):
        assert np.array_equal(host_u16(o), w)


def test_bad_overflow_slot_is_reported():
    w = _with_wide_blocks()
    x = dev_u16(w)
    c = codec.compress(x, index="idx8")
    assert c.index8_wide >= 1
    nb = c.sizes["n_blocks"]
    S = (nb + 63) // 64
    bases = c.index8[8 * S: 12 * S].view(torch.int32)
    k = int(torch.nonzero(bases < 0)[0])  # a wide superblock (bit 31 set)
    bad = c.index8.clone()
    bad[8 * S: 12 * S].view(torch.int32)[k] = torch.tensor(-2**31 + c.index8_wide + 3, dtype=torch.int32)
    c.index8, c._desc = bad, None
    out = torch.full((w.size + 8,), -1, dtype=torch.int16, device="cuda")
    err = err_word()
    codec.decompress(c, out[: w.size], err)
    assert api.df_read_error(err) != 0
    assert (host_u16(out[w.size:]) == 0xFFFF).all()
    fl = err_word()
    back = torch.empty(nb + 1, dtype=torch.int64, device="cuda")
    api.df_index8_expand(bad, nb, c.index8_wide, back, fl)
    assert api.df_read_error(fl) & DF_EFLAG_INDEX8

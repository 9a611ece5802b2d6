"""The fixed 12-bit format on the GPU against its oracle (oracle/nf12_oracle.py):

* encode: slots, bitmap, side buffer and escape count equal the oracle's
  byte for byte, over sizes that span several 2048-group tiles and ragged
  tails, for 16-byte-aligned and 2-byte-aligned inputs, and another top;
* decode of the ORACLE's parts (independent of the GPU encoder) gives the
  source back, for aligned and unaligned outputs;
* the grouped decode over many tensors, empty and tiny ones included, and the
  grouped encode (one launch per kernel for all tensors) against the oracle;
* a side index past the escaped groups and a side buffer too small are
  reported in the error word, and nothing is written outside the outputs;
* at full size (the 8B-shaped set's largest tensor) the round trip is exact
  and sampled groups equal the oracle's encoding of the same groups.
"""
import numpy as np
import pytest
import torch

from lossless_bf16_weight_huffman_b200 import api, nf12, synth
from lossless_bf16_weight_huffman_b200._native import DF_EFLAG_NF12_SIDE
from oracle import nf12_oracle as nfo
from tests.gpu_util import dev_u16, err_word, host_u16, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda(cuda_device):
    from lossless_bf16_weight_huffman_b200 import build

    build.build_native()


def _weights(n, seed=0, heavy=False):
    w = synth.generate((synth.heavy_tail_64m() if heavy else synth.single_1024x4096())[0])
    rng = np.random.default_rng(seed)
    start = int(rng.integers(0, w.size - n)) if n < w.size else 0
    return np.ascontiguousarray(w[start: start + n])


def _host(t, nbytes):
    return t[:nbytes].cpu().numpy()


def _check_encode(c: nf12.Nf12, w: np.ndarray, top=7):
    slots, bitmap, side = nfo.encode(w, top)
    assert c.n_escaped == side.size // 8
    assert np.array_equal(_host(c.slots, slots.size), slots), "slot bytes differ"
    assert np.array_equal(_host(c.bitmap, bitmap.size), bitmap), "bitmap differs"
    assert np.array_equal(_host(c.side, 2 * side.size).view(np.uint16), side), "side entries differ"


SIZES = [1, 7, 8, 9, 255, 256, 257, 16383, 16384, 16385, 3 * 16384 + 77, 1_000_003]


@pytest.mark.parametrize("n", SIZES)
@pytest.mark.parametrize("heavy", [False, True])
def test_encode_matches_oracle(n, heavy):
    w = _weights(n, seed=n, heavy=heavy)
    _check_encode(nf12.compress(dev_u16(w)), w)


@pytest.mark.parametrize("n", [9, 16385, 300_001])
def test_encode_unaligned_input(n):
    w = _weights(n + 1, seed=5, heavy=True)
    x = dev_u16(w)[1:]  # 2-byte aligned, not 16
    assert x.data_ptr() % 16 != 0
    _check_encode(nf12.compress(x), w[1:])


def test_encode_all_patterns_and_all_escaped():
    pats = synth.all_bf16_patterns()
    _check_encode(nf12.compress(dev_u16(pats)), pats)
    big = np.full(50_001, 0x4000, np.uint16)  # 2.0: every group escapes
    c = nf12.compress(dev_u16(big))
    assert c.n_escaped == c.groups
    _check_encode(c, big)
    none = np.full(40_000, 0x3F80, np.uint16)
    c = nf12.compress(dev_u16(none))
    assert c.n_escaped == 0
    _check_encode(c, none)


def test_encode_other_top():
    rng = np.random.default_rng(4)
    x = (rng.uniform(1, 2, 70_001) * 2.0 ** rng.integers(-31, -14, 70_001)).astype(np.float32)
    w = (x.view(np.uint32) >> 16).astype(np.uint16)
    c = nf12.compress(dev_u16(w), top=6)
    _check_encode(c, w, top=6)
    assert np.array_equal(host_u16(nf12.decompress(c)), w)


def _from_oracle(w, top=7):
    slots, bitmap, side = nfo.encode(w, top)
    return nf12.Nf12(n=w.size, shape=(w.size,), top=top, slots=to_dev(np.concatenate([slots, np.zeros(16, np.uint8)])),
                     bitmap=to_dev(np.concatenate([bitmap, np.zeros(16, np.uint8)])),
                     side=to_dev(np.concatenate([side.view(np.uint8), np.zeros(16, np.uint8)])),
                     n_escaped=side.size // 8)


@pytest.mark.parametrize("n", SIZES)
def test_decode_oracle_parts(n):
    w = _weights(n, seed=n + 1, heavy=True)
    c = _from_oracle(w)
    out = torch.full((n + 8,), -1, dtype=torch.int16, device="cuda")
    err = err_word()
    nf12.decompress(c, out[:n], err)
    assert api.df_read_error(err) == 0
    o = host_u16(out)
    assert np.array_equal(o[:n], w)
    assert (o[n:] == 0xFFFF).all()  # nothing past the output


@pytest.mark.parametrize("n", [5, 16385, 200_003])
def test_decode_unaligned_output(n):
    w = _weights(n, seed=2, heavy=True)
    c = _from_oracle(w)
    buf = torch.full((n + 10,), -1, dtype=torch.int16, device="cuda")
    out = buf[1: n + 1]
    assert out.data_ptr() % 16 != 0
    nf12.decompress(c, out)
    o = host_u16(buf)
    assert np.array_equal(o[1: n + 1], w) and o[0] == 0xFFFF and (o[n + 1:] == 0xFFFF).all()


def test_batch_decode_many_tensors():
    rng = np.random.default_rng(9)
    base = _weights(3_000_000, heavy=True)
    lens = [0, 1, 7, 8, 2048 * 8, 2048 * 8 + 1] + [int(k) for k in rng.integers(1, 200_000, 60)]
    ws, comps, off = [], [], 0
    for k in lens:
        w = base[off: off + k]
        off += k
        ws.append(w)
        comps.append(_from_oracle(w) if len(comps) % 2 else nf12.compress(dev_u16(w)))
    outs = [torch.full((len(w),), -1, dtype=torch.int16, device="cuda") for w in ws]
    dec = nf12.BatchDecoder(comps, outs)
    for _ in range(2):
        err = err_word()
        dec.run(err)
        assert api.df_read_error(err) == 0
        for o, w in zip(outs, ws):
            assert np.array_equal(host_u16(o), w)


def test_bad_side_index_is_reported():
    w = _weights(50_000, heavy=True)
    slots, bitmap, side = nfo.encode(w)
    g = int(np.nonzero(np.unpackbits(bitmap, bitorder="little"))[0][3])
    bad = slots.copy()
    bad[12 * g: 12 * g + 4] = np.frombuffer(np.uint32(side.size // 8 + 5).tobytes(), np.uint8)
    c = _from_oracle(w)
    c.slots = to_dev(np.concatenate([bad, np.zeros(16, np.uint8)]))
    out = torch.full((w.size + 8,), -1, dtype=torch.int16, device="cuda")
    err = err_word()
    nf12.decompress(c, out[: w.size], err)
    assert api.df_read_error(err) & DF_EFLAG_NF12_SIDE
    o = host_u16(out)
    keep = np.ones(w.size, bool)
    keep[8 * g: 8 * g + 8] = False
    assert np.array_equal(o[: w.size][keep], w[keep]) and (o[w.size:] == 0xFFFF).all()


def test_side_capacity_too_small_is_reported():
    w = _weights(100_000, heavy=True)
    x = dev_u16(w)
    z = api.df_nf12_sizes_for(w.size)
    slots = torch.empty(z.slots_bytes, dtype=torch.uint8, device="cuda")
    bitmap = torch.empty(z.bitmap_bytes, dtype=torch.uint8, device="cuda")
    ws = torch.empty(z.encode_ws_bytes, dtype=torch.uint8, device="cuda")
    esc = torch.empty(1, dtype=torch.int64, device="cuda")
    api.df_nf12_encode_groups(x, 7, slots, bitmap, ws, esc)
    e = int(esc.item())
    assert e > 4
    side = torch.full((16 * e,), 0x5A, dtype=torch.uint8, device="cuda")
    err = err_word()
    api.df_nf12_encode_escapes(x, 7, slots, bitmap, ws, side[: 16 * (e - 3)], err)
    assert api.df_read_error(err) & DF_EFLAG_NF12_SIDE
    assert (side[16 * (e - 3):].cpu().numpy() == 0x5A).all()  # nothing past the capacity


def test_full_size_round_trip_and_sampled_groups():
    """The 8B-shaped set's largest tensor (128256 x 4096): exact round trip on
    the GPU, and 4096 sampled groups against the oracle's encoding of them."""
    spec = synth.llama8b_shaped()[0]
    w = synth.generate(spec)
    x = dev_u16(w)
    c = nf12.compress(x)
    back = nf12.decompress(c, torch.empty_like(x))
    assert torch.equal(back, x)
    rng = np.random.default_rng(1)
    G = c.groups
    gs = np.sort(rng.choice(G, 4096, replace=False))
    slots = c.slots.view(-1)[: 12 * G].view(G, 12)[torch.from_numpy(gs).cuda()].cpu().numpy()
    bits = np.unpackbits(c.bitmap[: 4 * ((G + 31) // 32)].cpu().numpy(), bitorder="little")[gs]
    for k, g in enumerate(gs):
        grp = w[8 * g: 8 * g + 8]
        s, b, e = nfo.encode(grp)
        assert bits[k] == (e.size > 0)
        if e.size:  # the slot holds a side index whose entry is the raw group
            idx = int(slots[k, :4].view(np.uint32)[0])
            assert idx < c.n_escaped and not slots[k, 4:].any()
            assert np.array_equal(c.side[16 * idx: 16 * idx + 16].cpu().numpy().view(np.uint16), grp)
        else:
            assert np.array_equal(slots[k], s)


def test_grouped_encode_matches_oracle():
    """nf12.compress_batch (one launch per kernel over every tensor) writes the
    oracle's bytes for each tensor: empty, tiny, ragged, tile-spanning, all
    escaped, 2-byte-aligned input; run twice (the side buffers are reused)."""
    rng = np.random.default_rng(12)
    base = _weights(3_000_000, heavy=True)
    ws = [base[:0], base[:1], base[5:12], np.full(40_001, 0x4000, np.uint16)]
    ws += [base[int(a): int(a) + int(k)] for a, k in zip(rng.integers(0, 2_000_000, 40), rng.integers(1, 70_000, 40))]
    xs = [dev_u16(w) for w in ws]
    xs.append(dev_u16(base[:100_001])[1:])  # 2-byte aligned only
    ws.append(base[1:100_001])
    enc = nf12.BatchEncoder(xs)
    for _ in range(2):
        err = err_word()
        comps = enc.run(err)
        assert api.df_read_error(err) == 0
        for c, w in zip(comps, ws):
            _check_encode(c, w)
            if w.size:
                assert np.array_equal(host_u16(nf12.decompress(c, torch.empty(w.size, dtype=torch.int16, device="cuda"))), w)


def test_grouped_encode_short_side_buffer_is_reported():
    w = _weights(200_000, heavy=True)
    enc = nf12.BatchEncoder([dev_u16(w)])
    enc.run()
    enc.sides[0] = enc.sides[0][: 16 * (enc.sides[0].numel() // 16 // 2)]  # half the room
    enc.plan = api.df_nf12_encode_batch_prepare(enc.descriptors(), enc.ws)
    err = err_word()
    api.df_nf12_encode_batch_escapes(enc.plan, err)
    assert api.df_read_error(err) & DF_EFLAG_NF12_SIDE

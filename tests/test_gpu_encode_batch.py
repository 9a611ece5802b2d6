"""The grouped encode (df_histogram_batch_run, df_encode_batch_run through
codec.BatchEncoder) against the oracle, through the C ABI:

* every tensor's histogram equals the oracle's, and every container part
  equals the oracle's byte for byte, over a table mixing empty, tiny, ragged,
  tile-spanning, single-symbol and all-exponent tensors, a 2-byte-aligned
  input, and a different chunk size and block size per tensor;
* the 2000-tensor set: every container equals the per-tensor df_encode's;
* a run repeated on the same plan writes the same bytes (the zeroing launch
  clears what the last run wrote);
* a wrong total_bits on one tensor sets DF_EFLAG_ENC_TOTAL while the others
  still equal the oracle's; a plan without codes is refused by the encode run.
"""
import numpy as np
import pytest
import torch

import oracle
from lossless_bf16_weight_huffman_b200 import api, codec, synth
from lossless_bf16_weight_huffman_b200._native import DF_EFLAG_ENC_TOTAL, DfError
from tests.gpu_util import assert_container_equal, dev_u16, err_word

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda(cuda_device):
    from lossless_bf16_weight_huffman_b200 import build

    build.build_native()
    return cuda_device


FORMATS = [(32, 32), (16, 32), (64, 256), (32, 1024), (48, 64)]


def _table():
    """(weights, chunk_bytes, threads_per_block) per tensor, and the device
    inputs (one of them 2-byte aligned only)."""
    base = synth.generate(synth.heavy_tail_64m()[0])
    rng = np.random.default_rng(21)
    ws = [base[:0], base[:1], base[3:10], np.full(5_000, 0x3F80, np.uint16), synth.all_bf16_patterns(),
          synth.generate(synth.mixed_2000()[1]), base[100: 100 + 4095], base[9_000: 9_000 + 4096],
          base[20_000: 20_000 + 4097], base[50_000: 50_000 + 70_001], base[200_000: 200_000 + 1_000_003]]
    for a, k in zip(rng.integers(0, 60_000_000, 24), rng.integers(1, 300_000, 24)):
        ws.append(base[int(a): int(a) + int(k)])
    fmts = [FORMATS[i % len(FORMATS)] for i in range(len(ws))]
    xs = [dev_u16(w) if w.size else torch.empty(0, dtype=torch.int16, device="cuda") for w in ws]
    odd = base[1_500_000: 1_500_000 + 300_007]
    xs.append(dev_u16(np.concatenate([np.zeros(1, np.uint16), odd]))[1:])
    assert xs[-1].data_ptr() % 16 != 0
    ws.append(odd)
    fmts.append((32, 32))
    return ws, xs, fmts


def test_grouped_histograms_and_containers_match_the_oracle():
    ws, xs, fmts = _table()
    enc = codec.BatchEncoder(xs, chunk_bytes=[f[0] for f in fmts], threads_per_block=[f[1] for f in fmts])
    hist = enc.histograms()
    for i, w in enumerate(ws):
        assert (hist[i] == oracle.histogram(w)).all(), i
    err = err_word()
    comps = enc.run(err)
    assert api.df_read_error(err) == 0
    for c, w, (C, T) in zip(comps, ws, fmts):
        assert_container_equal(c, oracle.encode(w, chunk_bytes=C, threads_per_block=T))
    first = [(c.stream.clone(), c.gaps.clone(), c.offsets.clone(), c.sm.clone()) for c in comps]
    enc.run(err)  # same plan again: the outputs are zeroed and rewritten
    assert api.df_read_error(err) == 0
    for c, (s, g, o, m) in zip(comps, first):
        assert torch.equal(c.stream, s) and torch.equal(c.gaps, g) and torch.equal(c.offsets, o)
        assert torch.equal(c.sm[: c.n], m[: c.n])


def test_grouped_encode_of_the_2000_tensor_set_equals_per_tensor_encode():
    specs = synth.mixed_2000()
    xs = [dev_u16(synth.generate(s)) for s in specs]
    err = err_word()
    comps = codec.compress_batch(xs, d_err=err)
    assert api.df_read_error(err) == 0
    for k, (x, c) in enumerate(zip(xs, comps)):
        ref = codec.compress(x)
        assert c.total_bits == ref.total_bits and c.chunk_bytes == ref.chunk_bytes, k
        assert torch.equal(c.stream, ref.stream) and torch.equal(c.gaps, ref.gaps), k
        assert torch.equal(c.offsets, ref.offsets) and torch.equal(c.sm[: c.n], ref.sm[: ref.n]), k
    for s, c in list(zip(specs, comps))[:: 97]:
        enc = oracle.encode(synth.generate(s), chunk_bytes=c.chunk_bytes, threads_per_block=c.threads_per_block)
        assert_container_equal(c, enc)


def test_grouped_encode_reports_a_wrong_total_and_keeps_the_others_intact():
    base = synth.generate(synth.single_1024x4096()[0])
    ws = [base[:200_000], base[200_000:450_001], base[500_000:530_000]]
    enc = codec.BatchEncoder([dev_u16(w) for w in ws], chunk_bytes=32)
    comps = enc.prepare()
    descs = enc.descriptors(comps)
    descs[1].total_bits = comps[1].total_bits - 1  # the buffers stay large enough: one bit less
    enc.plan = api.df_encode_batch_prepare(descs, enc.ws)
    err = err_word()
    enc.run(err)
    assert api.df_read_error(err) & DF_EFLAG_ENC_TOTAL
    for i in (0, 2):
        assert_container_equal(comps[i], oracle.encode(ws[i], chunk_bytes=32))


def test_encode_run_needs_a_plan_with_codes():
    enc = codec.BatchEncoder([dev_u16(np.arange(1000, dtype=np.uint16))])
    with pytest.raises(DfError):
        api.df_encode_batch_run(enc.plan)

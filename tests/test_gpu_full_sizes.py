"""GPU parity at the full sizes of the decoder-layer and 8B-shaped weight sets,
in the launch configuration the benchmark times (one grouped decode of every
tensor of the set, and layer by layer into reused buffers).

At these sizes the checks are the ones that hold at any size, plus sampled
tensors the oracle encodes whole:
  - every decoded tensor equals its source bit for bit (the round trip the
    method promises: mlx-dfloat, PyPI page, intro);
  - the GPU-encoded containers of sampled tensors equal the oracle's byte for
    byte (stream, gaps, block offsets, sign|fraction bytes);
  - the error word stays 0.
"""
import numpy as np
import pytest
import torch

import oracle
from lossless_bf16_weight_huffman_b200 import api, codec, synth
from tests.gpu_util import assert_container_equal, err_word

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _cuda(cuda_device):
    from lossless_bf16_weight_huffman_b200 import build

    build.build_native()
    return cuda_device


def _compress_set(specs, keep_source=True):
    """Generate each tensor on the host, encode it on the GPU; returns the
    containers and (optionally) the device copies of the sources."""
    staging = torch.empty(max(s.numel for s in specs), dtype=torch.int16, pin_memory=True)
    comps, srcs = [], []
    err = err_word()
    for s in specs:
        n = s.numel
        synth.fill_ptr(s, staging.data_ptr(), n)
        x = staging[:n].to("cuda")
        comps.append(codec.compress(x, d_err=err))
        srcs.append(x if keep_source else None)
    assert api.df_read_error(err) == 0
    return comps, srcs


def _oracle_container_check(spec, c):
    w = synth.generate(spec)
    enc = oracle.encode(w, chunk_bytes=c.chunk_bytes, threads_per_block=c.threads_per_block)
    assert_container_equal(c, enc)


def test_llama_layer_full_size():
    specs = synth.llama_layer()
    comps, srcs = _compress_set(specs)
    # every tensor of the layer against the oracle's container
    for s, c in zip(specs, comps):
        _oracle_container_check(s, c)
    err = err_word()
    dec = codec.BatchDecoder(comps)
    for _ in range(2):  # twice into the same buffers, as the benchmark does
        outs = dec.run(err)
        for o, x in zip(outs, srcs):
            assert torch.equal(o.view(torch.int16).reshape(-1), x)
    assert api.df_read_error(err) == 0


def test_llama8b_shaped_full_size():
    specs = synth.llama8b_shaped()
    assert sum(s.numel for s in specs) == 8_030_257_152
    comps, srcs = _compress_set(specs)
    by_name = {s.name: (s, c) for s, c in zip(specs, comps)}
    # sampled tensors against the oracle: the first and a middle layer's
    # projections, and the largest tensor (the embedding)
    for name in ("layers.0.q_proj", "layers.17.down_proj", "embed_tokens"):
        s, c = by_name[name]
        _oracle_container_check(s, c)

    # the whole set in one grouped launch
    err = err_word()
    outs = codec.BatchDecoder(comps).run(err)
    assert api.df_read_error(err) == 0
    for o, x in zip(outs, srcs):
        assert torch.equal(o.view(torch.int16).reshape(-1), x)
    del outs

    # layer by layer into reused buffers (two layers and the embedding)
    groups = [[c for s, c in zip(specs, comps) if s.name.startswith(p)] for p in ("layers.0.", "layers.31.")]
    groups.append([by_name["embed_tokens"][1]])
    for g in groups:
        dec = codec.BatchDecoder(g)
        outs = dec.run(err)
        idx = [comps.index(c) for c in g]
        for o, i in zip(outs, idx):
            assert torch.equal(o.view(torch.int16).reshape(-1), srcs[i])
    assert api.df_read_error(err) == 0

"""Just-in-time layer decode (jit.py) on the GPU: every layer handed to the
consumer equals its source bit for bit, at run-ahead depth 0, 1 and 2, from
containers in HBM and from pinned host memory; a grouped launch limited to a
few CUDA blocks (df_batch_plan.max_ctas) decodes the same bytes."""
import numpy as np
import pytest
import torch

from lossless_bf16_weight_huffman_b200 import api, codec, jit, synth
from tests.gpu_util import err_word

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layers(cuda_device):
    rng = np.random.default_rng(3)
    base = synth.generate(synth.heavy_tail_64m()[0])
    src, comps = [], []
    off = 0
    for l in range(5):
        sl, cl = [], []
        for n in (int(rng.integers(1, 50_000)), 300_001 + 17 * l, 4096, 1):
            w = base[off: off + n]
            off += n
            x = torch.from_numpy(w.view(np.int16)).cuda()
            sl.append(x)
            cl.append(codec.compress(x))
        src.append(sl)
        comps.append(cl)
    return src, comps


@pytest.mark.parametrize("depth", [0, 1, 2])
def test_layer_streamer_every_layer_equals_its_source(layers, depth):
    src, comps = layers
    st = jit.LayerStreamer(comps, depth=depth)
    seen = {}

    def consume(l, views):
        seen[l] = [v.clone() for v in views]

    for _ in range(2):  # the ring is reused across passes
        seen.clear()
        st.run(consume)
        torch.cuda.synchronize()
        assert st.errors() == 0
        assert sorted(seen) == list(range(len(src)))
        for l in range(len(src)):
            for v, x in zip(seen[l], src[l]):
                assert torch.equal(v, x)


def test_host_layer_streamer_round_trip(layers):
    src, comps = layers
    hls = jit.HostLayerStreamer(comps)
    seen = {}
    hls.run(lambda l, views: seen.__setitem__(l, [v.clone() for v in views]))
    torch.cuda.synchronize()
    assert hls.errors() == 0
    for l in range(len(src)):
        for v, x in zip(seen[l], src[l]):
            assert torch.equal(v, x)
    assert hls.h2d_bytes == sum(c.read_bytes() for l in comps for c in l)


@pytest.mark.parametrize("max_ctas", [1, 3, 1000])
def test_grouped_launch_with_few_blocks(layers, max_ctas):
    src, comps = layers
    flat = [c for l in comps for c in l]
    outs = [torch.full((c.n,), -1, dtype=torch.int16, device="cuda") for c in flat]
    dec = codec.BatchDecoder(flat, outs)
    dec.plan.max_ctas = max_ctas
    err = err_word()
    dec.run(err)
    assert api.df_read_error(err) == 0
    for o, x in zip(outs, [x for l in src for x in l]):
        assert torch.equal(o, x)


@pytest.mark.parametrize("depth", [0, 2])
def test_layer_streamer_fixed_12_bit_format(layers, depth):
    """The same schedule over layers held in the fixed 12-bit format."""
    from lossless_bf16_weight_huffman_b200 import nf12

    src, _ = layers
    n12 = [[nf12.compress(x) for x in l] for l in src]
    st = jit.LayerStreamer(n12, depth=depth)
    seen = {}
    st.run(lambda l, views: seen.__setitem__(l, [v.clone() for v in views]))
    torch.cuda.synchronize()
    assert st.errors() == 0
    for l in range(len(src)):
        for v, x in zip(seen[l], src[l]):
            assert torch.equal(v, x)

"""The seeded input generators: stable bits and the stated shapes/distributions."""
import hashlib
import json
import os

import numpy as np

from lossless_bf16_weight_huffman_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "oracle_digests.json")


def bf16_to_f64(w):
    return (w.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_input_digests_are_stable():
    g = json.load(open(GOLDEN))
    seen = set()
    for t in g["tensors"]:
        key = (t["set"], t["index"])
        if key in seen:
            continue
        seen.add(key)
        w = synth.generate(synth.weight_set(t["set"])[t["index"]])
        assert hashlib.sha256(w.tobytes()).hexdigest() == t["input_sha256"], key


def test_splitmix64_reference_values():
    # SplitMix64 with state 0: the first outputs of the published generator
    assert synth.splitmix64(0, 0) == 0xE220A8397B1DCDAF
    assert synth.splitmix64(0, 1) == 0x6E789E6AA1B965F4
    assert synth.splitmix64(0, 2) == 0x06C45D188009454F


def test_rne_to_bf16():
    lib = synth._load()
    assert lib.synth_f32_to_bf16_rne(1.0) == 0x3F80
    # 1 + 2^-8 is a tie between 1.0 and 1 + 2^-7: even mantissa wins (1.0)
    assert lib.synth_f32_to_bf16_rne(1.0 + 2.0**-8) == 0x3F80
    # 1 + 3*2^-8 ties between 1+2^-7 (odd) and 1+2^-6 (even): rounds up
    assert lib.synth_f32_to_bf16_rne(1.0 + 3 * 2.0**-8) == 0x3F82
    assert lib.synth_f32_to_bf16_rne(-2.0) == 0xC000


def test_normal_set_statistics():
    w = synth.generate(synth.single_1024x4096()[0])
    x = bf16_to_f64(w)
    assert abs(x.mean()) < 1e-4 and abs(x.std() - 0.02) < 2e-4
    layer = synth.llama_layer()
    assert sum(s.numel for s in layer) == 218_112_000
    down = [s for s in layer if s.name.endswith("down_proj")][0]
    assert abs(down.std - 1 / np.sqrt(14336)) < 1e-12
    norm = synth.generate([s for s in layer if s.name.endswith("input_layernorm")][0])
    assert abs(bf16_to_f64(norm).mean() - 1.0) < 2e-3


def test_heavy_tail_specials():
    spec = synth.heavy_tail_64m()[0]
    assert spec.numel == 67_108_864
    w = synth.generate(spec)
    e = (w >> 7) & 0xFF
    m = w & 0x7F
    assert int(((e == 0xFF) & (m == 0) & (w < 0x8000)).sum()) == 8   # +Inf
    assert int(((e == 0xFF) & (m == 0) & (w >= 0x8000)).sum()) == 8  # -Inf
    nan = (e == 0xFF) & (m != 0)
    assert int(nan.sum()) == 16
    assert int((nan & ((m & 0x40) != 0)).sum()) == 8  # quiet
    assert int(((e == 0) & (m != 0)).sum()) == 64   # subnormals
    zeros = (w == 0) | (w == 0x8000)
    assert 0.009 < zeros.mean() < 0.011
    assert (w == 0x8000).sum() > 0.4 * zeros.sum()
    x = bf16_to_f64(w[(e != 0xFF)])
    assert np.abs(x).max() > 1.0  # outliers x100 of a t(3) tail


def test_weight_set_sizes():
    assert sum(s.numel for s in synth.llama8b_shaped()) == 8_030_257_152
    mixed = synth.mixed_2000()
    sizes = [s.numel for s in mixed]
    assert len(mixed) == 2000 and min(sizes) >= 1 and max(sizes) <= 2**20
    assert 1.0e8 < sum(sizes) < 2.0e8
    assert mixed[1].numel == 65536


def test_threads_do_not_change_bits():
    spec = synth.heavy_tail_64m()[0]
    a = np.empty(300_001, np.uint16)
    b = np.empty(300_001, np.uint16)
    lib = synth._load()
    for arr, th in ((a, 1), (b, 7)):
        lib.synth_fill(spec.kind, spec.seed, spec.mean, spec.std, spec.outlier_p, spec.outlier_mul, spec.zero_p,
                       arr.ctypes.data, arr.size, th)
    assert (a == b).all()

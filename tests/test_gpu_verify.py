"""Checks on the GPU: the device digest against a leaf tree built with
hashlib, the element compare, and verify's three levels with its exit codes
(0 pass, 1 a check fails, 2 could not check) on containers saved to a file and
loaded back, before and after corruptions made on the host."""
import hashlib
import os

import numpy as np
import pytest
import torch

from lossless_bf16_weight_huffman_b200 import api, codec, container_file, synth, verify
from tests.gpu_util import dev_u16

pytestmark = pytest.mark.gpu


def leaf_tree(b: bytes) -> bytes:
    leaves = [hashlib.sha256(b[i: i + 65536]).digest() for i in range(0, len(b), 65536)]
    return hashlib.sha256(b"".join(leaves)).digest()


@pytest.mark.parametrize("n", [0, 1, 63, 64, 65535, 65536, 65537, 1_000_003])
def test_device_digest_matches_leaf_tree(cuda_device, n):
    rng = np.random.default_rng(n)
    a = rng.integers(0, 256, n, dtype=np.uint8)
    d = torch.from_numpy(a).cuda() if n else torch.empty(0, dtype=torch.uint8, device="cuda")
    assert api.df_sha256_device(d) == leaf_tree(a.tobytes())


def test_device_digest_of_unaligned_data(cuda_device):
    """Whole 64 KiB leaves at an odd address take the byte-load path."""
    rng = np.random.default_rng(3)
    a = rng.integers(0, 256, 3 * 65536 + 1001, dtype=np.uint8)
    d = torch.from_numpy(a).cuda()
    assert api.df_sha256_device(d[1:]) == leaf_tree(a[1:].tobytes())


@pytest.mark.parametrize("n", [1, 7, 8, 9, 4095, 1_000_003])
def test_compare_first_difference_sizes_and_alignments(cuda_device, n):
    rng = np.random.default_rng(n)
    base = torch.from_numpy(rng.integers(-32768, 32767, n + 1, dtype=np.int16)).cuda()
    for a_src in (base[:n], base[1:]):  # 16-byte aligned and 2-byte aligned
        a = a_src.contiguous() if a_src.data_ptr() % 16 == 0 else a_src
        b = a.clone()
        out = torch.empty(1, dtype=torch.int64, device="cuda")
        api.df_compare(a, b, out)
        assert int(out.cpu().numpy().view(np.uint64)[0]) == 2**64 - 1
        pos = sorted(set(int(p) for p in rng.integers(0, n, 5)))
        for p in reversed(pos):
            b[p] ^= 1
            api.df_compare(a, b, out)
            assert int(out.item()) == p


def test_compare_finds_the_first_difference(cuda_device):
    a = torch.arange(100_000, dtype=torch.int16, device="cuda")
    b = a.clone()
    out = torch.empty(1, dtype=torch.int64, device="cuda")
    api.df_compare(a, b, out)
    assert int(out.cpu().numpy().view(np.uint64)[0]) == 2**64 - 1
    b[77_777] += 1
    b[91_000] += 1
    api.df_compare(a, b, out)
    assert int(out.item()) == 77_777


@pytest.fixture(scope="module")
def saved(cuda_device, tmp_path_factory):
    specs = synth.llama_layer()[1:3] + [synth.mixed_2000()[5]]
    src = {}
    comps = []
    for s in specs:
        w = synth.generate(s)[:3_000_000]
        x = dev_u16(w)
        src[s.name] = x
        comps.append((s.name, codec.compress(x)))
    hashes = {n: api.df_sha256_device(src[n]) for n, _ in comps}
    path = os.path.join(tmp_path_factory.mktemp("files"), "set.df11")
    container_file.save(path, comps, hashes)
    path_nohash = path + ".nohash"
    container_file.save(path_nohash, comps)
    return path, path_nohash, src


def test_levels_on_a_sound_file(saved):
    path, path_nohash, src = saved
    entries = container_file.load(path)
    assert verify.verify(entries, "structure")[0] == verify.PASS
    assert verify.verify(entries, "sampled", src, samples=200)[0] == verify.PASS
    assert verify.verify(entries, "full", src)[0] == verify.PASS
    assert verify.verify(entries, "full")[0] == verify.PASS  # stored digests
    assert verify.verify(entries, "sampled")[0] == verify.CANNOT
    bare = container_file.load(path_nohash)
    assert verify.verify(bare, "full")[0] == verify.CANNOT
    assert verify.verify(bare, "structure")[0] == verify.PASS


def _entries(path):
    return container_file.load(path)


def test_corrupt_stream_bit_is_caught(saved):
    path, _, src = saved
    entries = _entries(path)
    name, c, _ = entries[0]
    c.stream[1000] ^= 0x10
    code, why = verify.verify(entries, "full", src)
    assert code == verify.FAIL, why
    # every block sampled: the corrupt one is among them
    assert verify.verify(entries, "sampled", src, samples=10**9)[0] == verify.FAIL
    assert verify.verify(entries, "full")[0] == verify.FAIL  # against the stored digest


def test_corrupt_sign_fraction_byte_is_caught_by_the_digest(saved):
    path, _, src = saved
    entries = _entries(path)
    entries[1][1].sm[12345] ^= 0x01  # decodes fine, to the wrong weight
    assert verify.verify(entries, "structure")[0] == verify.PASS
    assert verify.verify(entries, "full")[0] == verify.FAIL
    assert verify.verify(entries, "full", src)[0] == verify.FAIL


def test_corrupt_offsets_fail_the_structure_check(saved):
    path, _, _ = saved
    entries = _entries(path)
    c = entries[0][1]
    o = c.offsets.cpu().numpy().view(np.uint64).copy()
    assert len(o) > 4
    o[len(o) // 2] = o[len(o) // 2 + 1] + 5  # one offset past the next
    c.offsets.copy_(torch.from_numpy(o.view(np.int64)))
    assert verify.verify(entries, "structure")[0] == verify.FAIL


def test_command_line_exit_codes(saved, tmp_path):
    path, path_nohash, src = saved
    npz = os.path.join(tmp_path, "src.npz")
    np.savez(npz, **{k: v.cpu().numpy().view(np.uint16) for k, v in src.items()})
    assert verify.main([path]) == verify.PASS
    assert verify.main([path, "--source", npz]) == verify.PASS
    assert verify.main([path, "--source", npz, "--level", "full"]) == verify.PASS
    assert verify.main([path_nohash, "--level", "full"]) == verify.CANNOT
    raw = open(path, "rb").read()
    broken = os.path.join(tmp_path, "broken.df11")
    open(broken, "wb").write(raw[: len(raw) // 2])
    assert verify.main([broken]) == verify.FAIL


def test_safe_compress_decodes_and_compares(cuda_device):
    w = synth.generate(synth.heavy_tail_64m()[0])[:1_000_001]
    x = dev_u16(w)
    c = codec.compress(x, safe=True)
    out = codec.decompress(c)
    assert torch.equal(out.view(torch.int16).reshape(-1), x)


def test_levels_with_compact_index(cuda_device, tmp_path):
    """Containers that hold the compact block index verify at every level
    (the offsets are expanded on the GPU first); a corrupt delta byte fails
    the structure check or the sampled decode."""
    w = np.concatenate([synth.generate(synth.single_1024x4096()[0])[:900_000], np.full(500_000, 0x3F80, np.uint16),
                        synth.generate(synth.heavy_tail_64m()[0])[:700_001]])
    x = dev_u16(w)
    c = codec.compress(x, index="idx8")
    assert c.index_kind == "idx8" and c.index8_wide >= 1
    path = os.path.join(tmp_path, "ix.df11")
    container_file.save(path, [("t", c)], {"t": api.df_sha256_device(x)})
    entries = container_file.load(path)
    src = {"t": x}
    for level in ("structure", "sampled", "full"):
        assert verify.verify(entries, level, src, samples=10**9)[0] == verify.PASS, level
    nb = entries[0][1].sizes["n_blocks"]
    S = (nb + 63) // 64
    entries[0][1].index8[12 * S + 3] ^= 0x40  # block 3's count off by 64
    code = verify.verify(entries, "structure")[0]
    if code == verify.PASS:
        code = verify.verify(entries, "sampled", src, samples=10**9)[0]
    assert code == verify.FAIL

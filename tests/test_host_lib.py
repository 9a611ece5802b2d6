"""Host side of the CUDA library, on the CPU: the exported symbols, the code
build against the oracle, size planning against the oracle, and the decode
tables (walked here by a plain-Python model of the kernel's table steps)
against the oracle's decoded output. No CUDA call is made.
"""
import math
import os
import re

import numpy as np
import pytest

import oracle
from lossless_bf16_weight_huffman_b200 import _native, api, synth
from tests.cases import long_code_tensor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from lossless_bf16_weight_huffman_b200 import build

    build.build_native()


HEADERS = ("df11.h", "nf12.h")


def header_text() -> str:
    return "\n".join(open(os.path.join(ROOT, "include", h)).read() for h in HEADERS)


def header_functions():
    text = re.sub(r"/\*.*?\*/", "", header_text(), flags=re.S)
    return sorted(set(re.findall(r"\b(df_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    names = header_functions()
    assert len(names) >= 15
    lib = _native.lib()
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(_native.EXPORTS) == names


def test_every_declaration_names_its_source():
    """Each function declared in the header is preceded by a comment that
    names the page passage it follows ("Source: ...") or says that the pages
    have none."""
    text = header_text()
    for name in header_functions():
        m = re.search(r"/\*((?:(?!\*/).)*)\*/\s*(?:#define[^\n]*\n\s*)*[A-Za-z_][A-Za-z_0-9 *]*\b" + name + r"\(",
                      text, flags=re.S)
        assert m, name
        comment = m.group(1)
        assert "Source:" in comment or "no counterpart" in comment, name


def test_struct_sizes_match_header_layout():
    import ctypes

    assert ctypes.sizeof(_native.DfCode) == 16 + 256 + 1024
    assert ctypes.sizeof(_native.DfSizes) == 9 * 8
    assert ctypes.sizeof(_native.DfTensor) == 16 + 16 + 5 * 8 + 256 + 16
    assert ctypes.sizeof(_native.DfBatchPlan) == 8 + 8 * 4 + 8
    assert ctypes.sizeof(_native.DfEncodeTensor) == 4 * 8 + 2 * 4 + 4 * 8
    assert ctypes.sizeof(_native.DfEncodePlan) == 8 + 2 * 4 + 5 * 8
    assert ctypes.sizeof(_native.DfNf12Sizes) == 5 * 8
    assert ctypes.sizeof(_native.DfNf12Tensor) == 16 + 4 * 8 + 8
    assert ctypes.sizeof(_native.DfNf12Plan) == 8 + 8 + 8


@pytest.mark.parametrize("n_blocks,n_wide", [(0, 0), (1, 0), (3, 0), (64, 1), (65, 2), (10**6 + 1, 17)])
def test_index8_bytes_match_the_oracle(n_blocks, n_wide):
    from oracle import index8

    assert api.df_index8_bytes(n_blocks, n_wide) == index8.index_bytes(n_blocks, n_wide)


@pytest.mark.parametrize("n", [0, 1, 7, 8, 9, 16383, 16384, 16385, 10**7 + 3])
def test_nf12_sizes_match_the_oracle(n):
    from oracle import nf12_oracle

    z = api.df_nf12_sizes_for(n).as_dict()
    o = nf12_oracle.sizes(n, 0)
    assert (z["groups"], z["slots_bytes"], z["bitmap_bytes"]) == (o["groups"], o["slots_bytes"], o["bitmap_bytes"])
    assert z["tiles"] == -(-o["groups"] // 2048)
    assert z["encode_ws_bytes"] == 8 * (z["tiles"] + 1)


def _random_hist(rng, kind):
    h = np.zeros(256, np.uint64)
    k = int(rng.integers(1, 257))
    syms = rng.choice(256, size=k, replace=False)
    if kind == 0:
        h[syms] = rng.integers(1, 1000, size=k)
    elif kind == 1:  # heavy tail: long codes
        h[syms] = (rng.pareto(0.5, size=k) * 50).astype(np.uint64) + 1
    elif kind == 2:  # many equal counts: ties everywhere
        h[syms] = rng.integers(1, 4, size=k)
    elif kind == 3:  # geometric, like real exponents
        h[syms] = (2.0 ** rng.uniform(0, 40, size=k)).astype(np.uint64) + 1
    else:  # one dominant symbol and a flat tail
        h[syms] = 1
        h[syms[0]] = int(rng.integers(1, 10**9))
    return h


def test_build_code_matches_oracle_on_many_histograms():
    rng = np.random.default_rng(1234)
    checked = 0
    for trial in range(10000):
        h = _random_hist(rng, trial % 5)
        k = int((h > 0).sum())
        lo = max(1, math.ceil(math.log2(k))) if k > 1 else 1
        max_len = int(rng.integers(lo, 33))
        want = oracle.package_merge(h, max_len)
        code = api.df_build_code(h, max_len)
        got = np.frombuffer(bytes(code.lengths), np.uint8)
        assert (got == want).all(), (trial, max_len)
        codes = np.frombuffer(bytes(code.codes), np.uint32)
        assert (codes == oracle.canonical_codes(want)).all(), trial
        checked += 1
    assert checked == 10000


def test_build_code_limits():
    h = np.ones(256, np.uint64)
    with pytest.raises(_native.DfError):
        api.df_build_code(h, 7)
    with pytest.raises(_native.DfError):
        api.df_build_code(h, 33)
    code = api.df_build_code(np.zeros(256, np.uint64))
    assert code.n_symbols == 0 and code.n_tables == 1
    with pytest.raises(_native.DfError):  # Kraft sum 3/2
        api.df_code_from_lengths(np.array([1, 1, 1] + [0] * 253, np.uint8))


@pytest.mark.parametrize("chunk_bytes,tpb", [(16, 32), (32, 256), (64, 128), (4096, 1024)])
def test_plan_matches_oracle_sizes(chunk_bytes, tpb):
    rng = np.random.default_rng(5)
    for _ in range(200):
        h = _random_hist(rng, 3)
        code = api.df_build_code(h, 32)
        n = int(h.sum())
        z = api.df_plan(code, h, n, chunk_bytes, tpb).as_dict()
        want = oracle.sizes(n, oracle.total_bits(h, oracle.package_merge(h, 32)), chunk_bytes, tpb)
        for key, val in want.items():
            assert z[key] == val, key
    with pytest.raises(_native.DfError):
        api.df_plan(code, h, n + 1, chunk_bytes, tpb)
    with pytest.raises(_native.DfError):
        api.df_plan(code, h, n, 24, tpb)


# ---------------------------------------------------------------- the decode tables


def wide_bits(lut, n_tables):
    """The wide table's window width, from the table sizes (2^W uint64 + 2^W uint16)."""
    words = lut.size - 256 * n_tables - 64 - 4
    W = int(round(np.log2(words / 2.5)))
    assert 5 * (1 << W) // 2 == words
    return W


def wide_entries(lut, W):
    return np.frombuffer(lut[: 2 * (1 << W)].tobytes(), np.uint64)


def wide_masks(lut, W):
    return np.frombuffer(lut[2 * (1 << W): 2 * (1 << W) + (1 << W) // 2].tobytes(), np.uint16)


def table_walk_decode(stream, total_bits, n, gaps_fields, offsets, lut, n_tables, chunk_bytes, tpb):
    """Plain-Python model of the kernel's per-chunk decode: every chunk is
    decoded from its start + gap while the bit position is before its end; a
    wide-table lookup yields every code that lies wholly inside the next W
    bits, a longer code walks the 8-bit tables; the codes of a lookup that
    start at or after the chunk end belong to the next chunk and are dropped
    (the start mask gives their positions); counts are checked against the
    block offsets."""
    WIDE = wide_bits(lut, n_tables)
    wide = wide_entries(lut, WIDE)
    masks = wide_masks(lut, WIDE)
    hier = lut[5 * (1 << WIDE) // 2:]
    assert hier[256 * n_tables + 64 + 3] == 0xDF11DF12
    bits = np.unpackbits(np.asarray(stream, np.uint8))
    cb = 8 * chunk_bytes
    n_chunks = len(gaps_fields)
    out = []
    counts = []

    def window(p):
        w = bits[p:p + 32]
        v = 0
        for b in w:
            v = (v << 1) | int(b)
        return v << (32 - len(w))

    def lookup(p):
        """One table lookup at bit p: (bits used, [(start offset, exponent), ...])."""
        win = window(p)
        e = int(wide[win >> (32 - WIDE)])
        step_word = e >> 32
        used = step_word >> 18
        if used == 0:  # a code longer than the window: the 8-bit tables
            assert step_word == 0
            e = int(hier[win >> 24])
            for lvl in (1, 2, 3):
                if (e >> 24) & 3:
                    break
                t = e & 0xFFFF
                assert t != 0, "unreachable entry"
                e = int(hier[t * 256 + ((win >> (24 - 8 * lvl)) & 0xFF)])
            assert (e >> 24) & 3 == 1
            return (e >> 8) & 63, [(0, e & 0xFF)]
        mask = int(masks[win >> (32 - WIDE)])
        assert bin(mask).count("1") << 3 == step_word & ((1 << 18) - 1)
        starts = [i for i in range(WIDE) if (mask >> i) & 1]
        return used, [(i, ((e & 0xFFFFFFFF) >> (8 * k)) & 0xFF) for k, i in enumerate(starts)]

    for j in range(n_chunks):
        p = j * cb + int(gaps_fields[j])
        end = min((j + 1) * cb, total_bits)
        cnt = 0
        while p < end:
            used, codes = lookup(p)
            for off, sym in codes:
                if p + off < end:
                    out.append(sym)
                    cnt += 1
            p += used
        counts.append(cnt)
    counts = np.array(counts)
    per_block = [int(counts[b * tpb:(b + 1) * tpb].sum()) for b in range(len(offsets) - 1)]
    assert per_block == list(np.diff(offsets.astype(np.int64)))
    assert len(out) == n
    return np.array(out, np.uint8)


@pytest.mark.parametrize("case", ["normal", "heavy12", "single", "all256", "heavy9", "long_codes"])
def test_tables_decode_oracle_streams(case):
    rng = np.random.default_rng(99)
    chunk_bytes, tpb, max_len = 16, 32, 32
    lengths = None
    if case == "normal":
        w = synth.generate(synth.single_1024x4096()[0])[:6000]
    elif case.startswith("heavy"):
        w = synth.generate(synth.heavy_tail_64m()[0])
        # keep rare exponents in the sample so long codes appear
        e = (w >> 7) & 0xFF
        rare = np.nonzero(np.bincount(e, minlength=256)[e] < 2000)[0][:300]
        w = np.concatenate([w[:5000], w[rare]])
        rng.shuffle(w)
        max_len = int(case[5:])
    elif case == "single":
        w = (0x3F80 | rng.integers(0, 128, size=3000)).astype(np.uint16)
    elif case == "long_codes":
        w, lengths = long_code_tensor(20000)
    else:
        w = ((np.arange(4096) % 256) << 7).astype(np.uint16)
    enc = oracle.encode(w, max_len=max_len, chunk_bytes=chunk_bytes, threads_per_block=tpb, lengths=lengths)
    code = api.df_code_from_lengths(enc.lengths, max_len)
    lut = api.df_build_lut(code)
    exps = table_walk_decode(enc.stream, enc.total_bits, enc.n, oracle.unpack_gaps(enc.gaps, enc.sizes["n_chunks"]),
                             enc.offsets, lut, code.n_tables, chunk_bytes, tpb)
    assert (exps == ((w >> 7) & 0xFF)).all()


def test_unreachable_entries_are_zero():
    h = np.zeros(256, np.uint64)
    h[127] = 10  # one symbol: code '0', so every index starting with bit 1 is unreachable
    code = api.df_build_code(h)
    lut = api.df_build_lut(code)
    WIDE = wide_bits(lut, code.n_tables)
    wide = wide_entries(lut, WIDE)
    half = 1 << (WIDE - 1)
    assert (wide[half:] == 0).all() and (wide[:half] != 0).all()
    assert (wide_masks(lut, WIDE)[half:] == 0).all()
    hier = lut[5 * (1 << WIDE) // 2:]
    assert (hier[128:256] == 0).all() and (hier[:128] != 0).all()
    assert list(hier[256 * code.n_tables + 64:]) == [1, 32, code.n_tables, 0xDF11DF12]
    # 256 equally frequent exponents: every code has 8 bits, every entry is reached
    code = api.df_build_code(np.full(256, 7, dtype=np.uint64))
    lut = api.df_build_lut(code)
    wide = wide_entries(lut, WIDE)
    assert ((wide >> np.uint64(32 + 18)) == 8).all()
    hier = lut[5 * (1 << WIDE) // 2:]
    assert (hier[:256] != 0).all()


# ---------------------------------------------------------------- the binding's buffer checks


def test_container_sizes_match_plan_and_oracle():
    """df_container_sizes (the library's layout arithmetic, used by the binding
    to size-check buffers) equals df_plan and the oracle's own size accounting."""
    rng = np.random.default_rng(7)
    for trial in range(400):
        h = _random_hist(rng, trial % 5)
        code = api.df_build_code(h, 32)
        n = int(h.sum())
        C = int(rng.choice([16, 32, 48, 64, 128, 1024, 4096]))
        T = int(rng.choice([32, 64, 96, 256, 1024]))
        z = api.df_plan(code, h, n, C, T).as_dict()
        got = api.df_container_sizes(n, z["total_bits"], C, T).as_dict()
        assert got == z, trial
        ref = oracle.sizes(n, z["total_bits"], C, T)
        for key in ("total_bits", "n_chunks", "stream_bytes", "gap_bytes", "n_blocks", "offsets_bytes", "sm_bytes",
                    "container_bytes"):
            assert got[key] == ref[key], (trial, key)
    z = api.df_plan(api.df_build_code(np.zeros(256, np.uint64)), np.zeros(256, np.uint64), 0, 32, 256).as_dict()
    assert api.df_container_sizes(0, 0, 32, 256).as_dict() == z
    for bad in ((10, 9, 32, 32), (10, 321, 32, 32), (10, 20, 24, 32), (10, 20, 32, 48)):
        with pytest.raises(_native.DfError):
            api.df_container_sizes(*bad)


def test_binding_refuses_wrong_element_sizes():
    import torch

    h = np.zeros(256, np.uint64)
    h[120:124] = [50, 30, 15, 5]
    code = api.df_build_code(h, 32)
    z = api.df_plan(code, h, 100, 32, 32).as_dict()
    bufs = dict(d_stream=torch.empty(z["stream_bytes"], dtype=torch.uint8),
                d_gaps=torch.empty(z["gap_bytes"], dtype=torch.uint8),
                d_block_offsets=torch.empty(z["n_blocks"] + 1, dtype=torch.int64),
                d_sm=torch.empty(100, dtype=torch.uint8))
    with pytest.raises(TypeError, match="d_in"):
        api.df_encode(code, torch.zeros(100, dtype=torch.uint8), z["total_bits"], 32, 32,
                      d_ws=torch.empty(16, dtype=torch.uint8), **bufs)
    with pytest.raises(TypeError, match="d_in"):
        api.df_encode_noalloc(code, torch.zeros(100, dtype=torch.int32), z["total_bits"], 32, 32, **bufs)
    with pytest.raises(TypeError, match="d_in"):
        api.df_histogram(torch.zeros(100, dtype=torch.uint8), torch.empty(256, dtype=torch.int64))
    with pytest.raises(ValueError, match="d_err"):
        api.df_encode(code, torch.zeros(100, dtype=torch.int16), z["total_bits"], 32, 32,
                      d_ws=torch.empty(16, dtype=torch.uint8), d_err=torch.zeros(1, dtype=torch.uint8), **bufs)
    d = _native.DfTensor()
    d.n = 100
    with pytest.raises(ValueError, match="d_err"):
        api.df_decode(d, torch.empty(100, dtype=torch.int16), torch.zeros(2, dtype=torch.int8))


def test_binding_refuses_short_buffers_before_the_library():
    import torch

    h = np.zeros(256, np.uint64)
    h[120:124] = [50, 30, 15, 5]
    code = api.df_build_code(h, 32)
    z = api.df_plan(code, h, 100, 32, 256).as_dict()
    x = torch.zeros(100, dtype=torch.int16)
    bufs = dict(d_stream=torch.empty(z["stream_bytes"], dtype=torch.uint8),
                d_gaps=torch.empty(z["gap_bytes"], dtype=torch.uint8),
                d_block_offsets=torch.empty(z["n_blocks"] + 1, dtype=torch.int64),
                d_sm=torch.empty(100, dtype=torch.uint8))
    for name in bufs:
        short = dict(bufs)
        short[name] = bufs[name][:-1]
        with pytest.raises(ValueError, match=name):
            api.df_encode(code, x, z["total_bits"], 32, 256, d_ws=torch.empty(16, dtype=torch.uint8), **short)
        with pytest.raises(ValueError, match=name):
            api.df_encode_noalloc(code, x, z["total_bits"], 32, 256, **short)
    d = _native.DfTensor()
    d.n = 100
    with pytest.raises(ValueError, match="d_out"):
        api.df_decode(d, torch.empty(99, dtype=torch.int16))
    with pytest.raises(ValueError, match="d_outs"):
        api.df_decode_batch_prepare([d], [torch.empty(50, dtype=torch.int16)], torch.empty(4096, dtype=torch.uint8))


def test_host_sha256_against_hashlib():
    """df_sha256 (host) is plain SHA-256 (FIPS 180-4): the standard's "abc"
    example, the empty message, the padding edge lengths, random data."""
    import hashlib

    assert api.df_sha256(b"abc").hex() == "ba7816bf8f01cfea414140de5dae2223b00361a396177a9cb410ff61f20015ad"
    assert api.df_sha256(b"") == hashlib.sha256(b"").digest()
    rng = np.random.default_rng(8)
    for n in (1, 55, 56, 57, 63, 64, 65, 119, 120, 128, 1000, 65536, 65537):
        data = rng.integers(0, 256, n, dtype=np.uint8).tobytes()
        assert api.df_sha256(data) == hashlib.sha256(data).digest(), n


def test_new_entry_points_refuse_bad_arguments_before_any_device_work():
    """The fixed 12-bit format's and the compact index's calls check their
    arguments on the host and return before touching a device (no GPU here)."""
    import ctypes

    L = _native.lib()
    z = _native.DfNf12Sizes()
    assert L.df_nf12_sizes_for((1 << 48) + 1, ctypes.byref(z)) == _native.DF_ERR_UNSUPPORTED  # DF_MAX_WEIGHTS + 1
    assert L.df_nf12_sizes_for(10, None) == _native.DF_ERR_INVALID_ARG
    # decode: top above 15, a reserved field set, misaligned slots
    t = _native.DfNf12Tensor()
    t.n, t.slots, t.bitmap, t.out, t.top = 16, 256, 512, 1024, 16
    assert L.df_nf12_decode(ctypes.byref(t), None, None) == _native.DF_ERR_INVALID_ARG
    t.top, t.reserved = 7, 1
    assert L.df_nf12_decode(ctypes.byref(t), None, None) == _native.DF_ERR_INVALID_ARG
    t.reserved, t.slots = 0, 258
    assert L.df_nf12_decode(ctypes.byref(t), None, None) == _native.DF_ERR_INVALID_ARG
    # grouped encode: workspace size, then a descriptor with top 16
    e = (_native.DfNf12EncodeTensor * 2)()
    e[0].n, e[1].n = 16384 * 3 + 5, 9  # 4 tiles and 1 tile
    for x in e:
        x.input, x.slots, x.bitmap, x.top = 256, 512, 1024, 7
    ws = L.df_nf12_encode_batch_workspace(e, 2)
    assert ws == 2 * 64 + 8 * 3 + 8 * 5 + 8 * 2
    plan = _native.DfNf12Plan()
    e[1].top = 16
    assert L.df_nf12_encode_batch_prepare(e, 2, 4096, ws, ctypes.byref(plan), None) == _native.DF_ERR_INVALID_ARG
    e[1].top = 7
    assert L.df_nf12_encode_batch_prepare(e, 2, 4096, ws - 8, ctypes.byref(plan), None) == _native.DF_ERR_WORKSPACE
    # compact index: misaligned buffer, too small a buffer, too many blocks
    wide = 4096
    assert L.df_index8_build(256, 10, 260, 76, wide, None, None) == _native.DF_ERR_INVALID_ARG
    assert L.df_index8_build(256, 100, 512, 76, wide, None, None) == _native.DF_ERR_INVALID_ARG  # needs 152
    assert L.df_index8_build(256, 1 << 32, 512, 1 << 40, wide, None, None) == _native.DF_ERR_UNSUPPORTED
    assert L.df_index8_expand(512, 64, 2, 256, None, None) == _native.DF_ERR_INVALID_ARG  # 2 wide of 1 superblock


def test_grouped_encode_refuses_bad_tables_before_any_device_work():
    """df_encode_batch_prepare checks every descriptor, the codes and the
    workspace on the host before it touches a device (no GPU here); the runs
    refuse a plan they cannot use."""
    import ctypes

    L = _native.lib()
    code = api.df_build_code(np.full(256, 1, np.uint64), 32)
    t = (_native.DfEncodeTensor * 2)()
    for x, n in zip(t, (100_000, 4096 * 5)):
        x.input, x.n, x.total_bits, x.chunk_bytes, x.threads_per_block = 256, n, 8 * n, 32, 32
        x.stream, x.gaps, x.block_offsets, x.sm = 4096, 8192, 16384, 32768
    ws_hist = L.df_encode_batch_workspace(t, 2)
    assert ws_hist > 0
    one = L.df_encode_batch_workspace(t, 1)
    assert 0 < one < ws_hist
    plan = _native.DfEncodePlan()
    t[0].code = ctypes.pointer(code)  # a code for one tensor only
    assert L.df_encode_batch_prepare(t, 2, 4096, ws_hist, ctypes.byref(plan), None) == _native.DF_ERR_INVALID_ARG
    t[1].code = ctypes.pointer(code)
    t[1].chunk_bytes = 8  # not a multiple of 16
    assert L.df_encode_batch_prepare(t, 2, 4096, ws_hist, ctypes.byref(plan), None) == _native.DF_ERR_INVALID_ARG
    t[1].chunk_bytes, t[1].stream = 32, 4100  # stream not 16-byte aligned
    assert L.df_encode_batch_prepare(t, 2, 4096, ws_hist, ctypes.byref(plan), None) == _native.DF_ERR_INVALID_ARG
    t[1].stream = 4096
    assert L.df_encode_batch_prepare(t, 2, 4096, ws_hist - 16, ctypes.byref(plan), None) == _native.DF_ERR_WORKSPACE
    assert L.df_encode_batch_prepare(t, 2, 4100, ws_hist, ctypes.byref(plan), None) == _native.DF_ERR_INVALID_ARG
    t[0].input = 257  # input not 2-byte aligned
    assert L.df_encode_batch_prepare(t, 2, 4096, ws_hist, ctypes.byref(plan), None) == _native.DF_ERR_INVALID_ARG
    t[0].input, t[0].n = 256, (1 << 48) + 1  # DF_MAX_WEIGHTS + 1
    assert L.df_encode_batch_prepare(t, 2, 4096, ws_hist, ctypes.byref(plan), None) == _native.DF_ERR_UNSUPPORTED
    # an empty table needs no device: an empty plan, and runs that do nothing
    assert L.df_encode_batch_workspace(t, 0) > 0
    assert L.df_encode_batch_prepare(t, 0, None, 0, ctypes.byref(plan), None) == _native.DF_OK
    assert plan.count == 0 and plan.ranges == 0
    assert L.df_encode_batch_run(ctypes.byref(plan), None, None) == _native.DF_OK
    assert L.df_histogram_batch_run(ctypes.byref(plan), None, None) == _native.DF_OK
    # runs: a plan without codes cannot encode; no histogram buffer
    plan.d_ws, plan.count, plan.has_codes = 4096, 2, 0
    assert L.df_encode_batch_run(ctypes.byref(plan), None, None) == _native.DF_ERR_INVALID_ARG
    assert L.df_histogram_batch_run(ctypes.byref(plan), None, None) == _native.DF_ERR_INVALID_ARG


def test_tensor_level_encoders_refuse_cpu_tensors_and_empty_lists():
    """There is no CPU path: the grouped encoders reject host tensors (and an
    empty list) before any library call."""
    import torch

    from lossless_bf16_weight_huffman_b200 import codec, nf12

    w = torch.zeros(100, dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="CUDA"):
        codec.compress_batch([w])
    with pytest.raises(TypeError, match="CUDA"):
        codec.compress(w)
    with pytest.raises(ValueError, match="no tensors"):
        codec.BatchEncoder([])
    with pytest.raises(ValueError, match="no tensors"):
        nf12.BatchEncoder([])
    with pytest.raises(TypeError):
        nf12.compress(w)
    with pytest.raises(ValueError, match="no tensors"):
        codec.BatchDecoder([])

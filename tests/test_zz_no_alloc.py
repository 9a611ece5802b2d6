"""df_encode_noalloc: the encoder for callers that cannot allocate device
memory at encode time (a runtime that hands out only a fixed arena, a plug-in
that may only touch the buffers its host gives it). It keeps its scratch in a
static device array of the library instead of a caller workspace. Checked
here, through the C ABI, byte for byte against df_encode on two calls in a
row; the second call reuses the array the first one left behind.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from lossless_bf16_weight_huffman_b200 import _native, api, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda(cuda_device):
    from lossless_bf16_weight_huffman_b200 import build

    build.build_native()
    return cuda_device


def _encode_both(w: np.ndarray, chunk_bytes: int, tpb: int):
    x = torch.from_numpy(w.view(np.int16)).cuda()
    h = torch.empty(256, dtype=torch.int64, device="cuda")
    api.df_histogram(x, h)
    hist = h.cpu().numpy().view(np.uint64)
    code = api.df_build_code(hist, 32)
    z = api.df_plan(code, hist, w.size, chunk_bytes, tpb).as_dict()

    def buffers():
        return (torch.full((z["stream_bytes"],), 0x5A, dtype=torch.uint8, device="cuda"),
                torch.full((z["gap_bytes"],), 0x5A, dtype=torch.uint8, device="cuda"),
                torch.full((z["n_blocks"] + 1,), -1, dtype=torch.int64, device="cuda"),
                torch.full((max(w.size, 16),), 0x5A, dtype=torch.uint8, device="cuda"))

    ref = buffers()
    ws = torch.empty(z["encode_ws_bytes"], dtype=torch.uint8, device="cuda")
    err_ref = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.df_encode(code, x, z["total_bits"], chunk_bytes, tpb, *ref, ws, err_ref)
    got = buffers()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.df_encode_noalloc(code, x, z["total_bits"], chunk_bytes, tpb, *got, err)
    assert api.df_read_error(err_ref) == 0 and api.df_read_error(err) == 0
    return ref, got


def test_noalloc_encode_matches_encode_on_two_calls_in_a_row():
    first = synth.generate(synth.heavy_tail_64m()[0])[:3_000_017]
    second = synth.generate(synth.single_1024x4096()[0])[:1_234_567]
    for w, chunk_bytes, tpb in ((first, 32, 256), (second, 16, 64)):
        ref, got = _encode_both(w, chunk_bytes, tpb)
        for a, b in zip(ref, got):
            assert torch.equal(a, b)


def test_noalloc_encode_rejects_oversized_input():
    # the size check comes before any device access
    code = api.df_build_code(np.full(256, 1, np.uint64), 32)
    status = _native.lib().df_encode_noalloc(
        ctypes.byref(code), ctypes.c_void_p(16), _native.DF_ENCODE_NOALLOC_MAX_WEIGHTS + 1, 0, 32, 256,
        ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), None, None)
    assert status == _native.DF_ERR_UNSUPPORTED

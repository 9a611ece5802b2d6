"""Python binding of the C ABI: one function per entry point of include/df11.h
and include/nf12.h, same names, argument marshalling only. Device buffers are torch CUDA tensors
(PyTorch supplies memory and streams); every computation runs in libdf11.so.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from ._native import (DfBatchPlan, DfCode, DfEncodePlan, DfEncodeTensor, DfNf12EncodeTensor, DfNf12Plan,
                      DfNf12Sizes, DfNf12Tensor, DfSizes, DfTensor, check, lib)


def _stream_ptr(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t: torch.Tensor | None, name: str):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, nbytes: int, name: str) -> None:
    """The library writes nbytes through t's pointer: refuse a smaller buffer
    before any device write can run past it."""
    have = t.numel() * t.element_size()
    if have < nbytes:
        raise ValueError(f"{name} holds {have} bytes; the call writes {nbytes}")


def _check_encode_buffers(n, total_bits, chunk_bytes, threads_per_block, d_in, d_stream, d_gaps, d_block_offsets,
                          d_sm, d_err):
    _need_u16(d_in, "d_in")
    _need_err(d_err)
    z = DfSizes()
    if lib().df_container_sizes(n, total_bits, chunk_bytes, threads_per_block, ctypes.byref(z)) != 0:
        return  # the library rejects these arguments itself
    _need(d_stream, z.stream_bytes, "d_stream")
    _need(d_gaps, z.gap_bytes, "d_gaps")
    _need(d_block_offsets, z.offsets_bytes, "d_block_offsets")
    _need(d_sm, z.sm_bytes, "d_sm")


def _need_u16(t: torch.Tensor, name: str) -> None:
    """The library reads 2 bytes per element of a weight buffer."""
    if isinstance(t, torch.Tensor) and t.element_size() != 2:
        raise TypeError(f"{name} must hold 16-bit elements (BF16 bit patterns), got {t.dtype}")


def _need_err(d_err: torch.Tensor | None) -> None:
    """The error word is a 32-bit word the kernels OR flags into."""
    if d_err is not None:
        _need(d_err, 4, "d_err")


def _hist_array(hist) -> np.ndarray:
    h = np.ascontiguousarray(np.asarray(hist, dtype=np.uint64).reshape(-1))
    if h.size != 256:
        raise ValueError("hist must have 256 entries")
    return h


def df_status_string(status: int) -> str:
    return lib().df_status_string(status).decode()


def df_last_cuda_error() -> int:
    return int(lib().df_last_cuda_error())


def df_build_code(hist, max_len: int = 32) -> DfCode:
    h = _hist_array(hist)
    code = DfCode()
    check("df_build_code", lib().df_build_code(h.ctypes.data, max_len, ctypes.byref(code)))
    return code


def df_code_from_lengths(lengths, max_len: int = 32) -> DfCode:
    arr = np.ascontiguousarray(np.asarray(lengths, dtype=np.uint8).reshape(-1))
    if arr.size != 256:
        raise ValueError("lengths must have 256 entries")
    code = DfCode()
    check("df_code_from_lengths", lib().df_code_from_lengths(arr.ctypes.data, max_len, ctypes.byref(code)))
    return code


def df_lut_words(code: DfCode) -> int:
    return int(lib().df_lut_words(ctypes.byref(code)))


def df_build_lut(code: DfCode) -> np.ndarray:
    words = df_lut_words(code)
    out = np.zeros(words, np.uint32)
    check("df_build_lut", lib().df_build_lut(ctypes.byref(code), out.ctypes.data, words))
    return out


def df_container_sizes(n: int, total_bits: int, chunk_bytes: int = 32, threads_per_block: int = 32) -> DfSizes:
    z = DfSizes()
    check("df_container_sizes", lib().df_container_sizes(n, total_bits, chunk_bytes, threads_per_block,
                                                         ctypes.byref(z)))
    return z


def df_plan(code: DfCode, hist, n: int, chunk_bytes: int = 32, threads_per_block: int = 32) -> DfSizes:
    h = _hist_array(hist)
    z = DfSizes()
    check("df_plan", lib().df_plan(ctypes.byref(code), h.ctypes.data, n, chunk_bytes, threads_per_block,
                                   ctypes.byref(z)))
    return z


def df_histogram(d_in: torch.Tensor, d_hist256: torch.Tensor, stream=None) -> None:
    _need_u16(d_in, "d_in")
    _need(d_hist256, 256 * 8, "d_hist256")
    check("df_histogram", lib().df_histogram(_dev(d_in, "d_in"), d_in.numel(), _dev(d_hist256, "d_hist256"),
                                             _stream_ptr(stream)))


def df_encode(code: DfCode, d_in: torch.Tensor, total_bits: int, chunk_bytes: int, threads_per_block: int,
              d_stream: torch.Tensor, d_gaps: torch.Tensor, d_block_offsets: torch.Tensor, d_sm: torch.Tensor,
              d_ws: torch.Tensor, d_err: torch.Tensor | None = None, stream=None) -> None:
    ws_bytes = d_ws.numel() * d_ws.element_size() if d_ws is not None else 0
    _check_encode_buffers(d_in.numel(), total_bits, chunk_bytes, threads_per_block, d_in, d_stream, d_gaps,
                          d_block_offsets, d_sm, d_err)
    check("df_encode", lib().df_encode(
        ctypes.byref(code), _dev(d_in, "d_in"), d_in.numel(), total_bits, chunk_bytes, threads_per_block,
        _dev(d_stream, "d_stream"), _dev(d_gaps, "d_gaps"), _dev(d_block_offsets, "d_block_offsets"),
        _dev(d_sm, "d_sm"), _dev(d_ws, "d_ws"), ws_bytes, _dev(d_err, "d_err"), _stream_ptr(stream)))


def _encode_array(tensors):
    return (DfEncodeTensor * max(1, len(tensors)))(*tensors)


def df_encode_batch_workspace(tensors) -> int:
    return int(lib().df_encode_batch_workspace(_encode_array(tensors), len(tensors)))


def df_encode_batch_prepare(tensors, d_ws: torch.Tensor, stream=None) -> DfEncodePlan:
    """tensors: DfEncodeTensor list (device pointers as ints; `code` a
    pointer to a DfCode the caller keeps alive until the call returns)."""
    _need(d_ws, df_encode_batch_workspace(tensors), "d_ws")
    plan = DfEncodePlan()
    check("df_encode_batch_prepare", lib().df_encode_batch_prepare(
        _encode_array(tensors), len(tensors), _dev(d_ws, "d_ws"), d_ws.numel() * d_ws.element_size(),
        ctypes.byref(plan), _stream_ptr(stream)))
    return plan


def df_histogram_batch_run(plan: DfEncodePlan, d_hist: torch.Tensor, stream=None) -> None:
    _need(d_hist, 2048 * plan.count, "d_hist")
    check("df_histogram_batch_run", lib().df_histogram_batch_run(
        ctypes.byref(plan), _dev(d_hist, "d_hist"), _stream_ptr(stream)))


def df_encode_batch_run(plan: DfEncodePlan, d_err: torch.Tensor | None = None, stream=None) -> None:
    _need_err(d_err)
    check("df_encode_batch_run", lib().df_encode_batch_run(ctypes.byref(plan), _dev(d_err, "d_err"),
                                                           _stream_ptr(stream)))


def df_encode_noalloc(code: DfCode, d_in: torch.Tensor, total_bits: int, chunk_bytes: int, threads_per_block: int,
                      d_stream: torch.Tensor, d_gaps: torch.Tensor, d_block_offsets: torch.Tensor,
                      d_sm: torch.Tensor, d_err: torch.Tensor | None = None, stream=None) -> None:
    """df_encode with the library's static scratch instead of a workspace
    (for callers that cannot allocate device memory; calls on one GPU must not
    overlap)."""
    _check_encode_buffers(d_in.numel(), total_bits, chunk_bytes, threads_per_block, d_in, d_stream, d_gaps,
                          d_block_offsets, d_sm, d_err)
    check("df_encode_noalloc", lib().df_encode_noalloc(
        ctypes.byref(code), _dev(d_in, "d_in"), d_in.numel(), total_bits, chunk_bytes, threads_per_block,
        _dev(d_stream, "d_stream"), _dev(d_gaps, "d_gaps"), _dev(d_block_offsets, "d_block_offsets"),
        _dev(d_sm, "d_sm"), _dev(d_err, "d_err"), _stream_ptr(stream)))


def df_decode(t: DfTensor, d_out: torch.Tensor, d_err: torch.Tensor | None = None, stream=None) -> None:
    if isinstance(d_out, torch.Tensor):
        _need(d_out, 2 * t.n, "d_out")
    _need_err(d_err)
    check("df_decode", lib().df_decode(ctypes.byref(t), _dev(d_out, "d_out"), _dev(d_err, "d_err"),
                                       _stream_ptr(stream)))


def df_decode_batch_workspace(count: int) -> int:
    return int(lib().df_decode_batch_workspace(count))


def _batch_arrays(tensors, d_outs):
    if len(tensors) != len(d_outs):
        raise ValueError("one output per tensor")
    for i, (t, o) in enumerate(zip(tensors, d_outs)):
        if isinstance(o, torch.Tensor):
            _need(o, 2 * t.n, f"d_outs[{i}]")
    arr = (DfTensor * max(1, len(tensors)))(*tensors)
    # an int is a raw device pointer, passed through unchecked
    outs = (ctypes.c_void_p * max(1, len(d_outs)))(
        *[o if isinstance(o, int) else _dev(o, "d_outs[i]").value for o in d_outs])
    return arr, outs


def df_decode_batch_prepare(tensors, d_outs, d_ws: torch.Tensor, stream=None) -> DfBatchPlan:
    arr, outs = _batch_arrays(tensors, d_outs)
    plan = DfBatchPlan()
    ws_bytes = d_ws.numel() * d_ws.element_size()
    check("df_decode_batch_prepare", lib().df_decode_batch_prepare(
        arr, outs, len(tensors), _dev(d_ws, "d_ws"), ws_bytes, ctypes.byref(plan), _stream_ptr(stream)))
    return plan


def df_decode_batch_run(plan: DfBatchPlan, d_err: torch.Tensor | None = None, stream=None) -> None:
    _need_err(d_err)
    check("df_decode_batch_run", lib().df_decode_batch_run(ctypes.byref(plan), _dev(d_err, "d_err"),
                                                           _stream_ptr(stream)))


def df_decode_batch(tensors, d_outs, d_ws: torch.Tensor, d_err: torch.Tensor | None = None, stream=None) -> None:
    arr, outs = _batch_arrays(tensors, d_outs)
    _need_err(d_err)
    ws_bytes = d_ws.numel() * d_ws.element_size()
    check("df_decode_batch", lib().df_decode_batch(arr, outs, len(tensors), _dev(d_ws, "d_ws"), ws_bytes,
                                                   _dev(d_err, "d_err"), _stream_ptr(stream)))


def df_read_error(d_err: torch.Tensor, stream=None) -> int:
    """Return the device error word (0 = clean); waits for the stream."""
    _need_err(d_err)
    flags = ctypes.c_uint32(0)
    status = lib().df_read_error(_dev(d_err, "d_err"), _stream_ptr(stream), ctypes.byref(flags))
    if status not in (0, 3):
        check("df_read_error", status)
    return int(flags.value)


def df_check_structure(t: DfTensor, d_flags: torch.Tensor, stream=None) -> None:
    _need_err(d_flags)
    check("df_check_structure", lib().df_check_structure(ctypes.byref(t), _dev(d_flags, "d_flags"),
                                                         _stream_ptr(stream)))


def df_compare(d_a: torch.Tensor, d_b: torch.Tensor, d_first_diff: torch.Tensor, stream=None) -> None:
    _need_u16(d_a, "d_a")
    _need_u16(d_b, "d_b")
    if d_a.numel() != d_b.numel():
        raise ValueError("d_a and d_b differ in size")
    _need(d_first_diff, 8, "d_first_diff")
    check("df_compare", lib().df_compare(_dev(d_a, "d_a"), _dev(d_b, "d_b"), d_a.numel(),
                                         _dev(d_first_diff, "d_first_diff"), _stream_ptr(stream)))


def df_sha256_workspace(nbytes: int) -> int:
    return int(lib().df_sha256_workspace(nbytes))


def df_sha256_device(d_data: torch.Tensor, d_ws: torch.Tensor | None = None, stream=None) -> bytes:
    """The leaf-tree SHA-256 of a device tensor's bytes (waits for the stream)."""
    nbytes = d_data.numel() * d_data.element_size()
    need = df_sha256_workspace(nbytes)
    if d_ws is None:
        d_ws = torch.empty(need, dtype=torch.uint8, device=d_data.device)
    _need(d_ws, need, "d_ws")
    out = (ctypes.c_uint8 * 32)()
    check("df_sha256_device", lib().df_sha256_device(_dev(d_data, "d_data"), nbytes, _dev(d_ws, "d_ws"),
                                                     d_ws.numel() * d_ws.element_size(), out, _stream_ptr(stream)))
    return bytes(out)


def df_sha256(data) -> bytes:
    """Plain SHA-256 of host bytes (a numpy array or bytes)."""
    arr = np.ascontiguousarray(np.frombuffer(data, np.uint8) if isinstance(data, (bytes, bytearray)) else data)
    buf = arr.view(np.uint8).reshape(-1)
    out = (ctypes.c_uint8 * 32)()
    check("df_sha256", lib().df_sha256(buf.ctypes.data if buf.size else None, buf.size, out))
    return bytes(out)


def df_index8_bytes(n_blocks: int, n_wide: int) -> int:
    return int(lib().df_index8_bytes(n_blocks, n_wide))


def df_index8_build(d_offsets: torch.Tensor, n_blocks: int, d_index8: torch.Tensor, d_n_wide: torch.Tensor,
                    d_err: torch.Tensor | None = None, stream=None) -> None:
    _need(d_offsets, 8 * (n_blocks + 1), "d_offsets")
    _need(d_n_wide, 8, "d_n_wide")
    _need_err(d_err)
    check("df_index8_build", lib().df_index8_build(
        _dev(d_offsets, "d_offsets"), n_blocks, _dev(d_index8, "d_index8"), d_index8.numel() * d_index8.element_size(),
        _dev(d_n_wide, "d_n_wide"), _dev(d_err, "d_err"), _stream_ptr(stream)))


def df_index8_expand(d_index8: torch.Tensor, n_blocks: int, n_wide: int, d_offsets: torch.Tensor,
                     d_err: torch.Tensor | None = None, stream=None) -> None:
    _need(d_index8, df_index8_bytes(n_blocks, n_wide), "d_index8")
    _need(d_offsets, 8 * (n_blocks + 1), "d_offsets")
    _need_err(d_err)
    check("df_index8_expand", lib().df_index8_expand(
        _dev(d_index8, "d_index8"), n_blocks, n_wide, _dev(d_offsets, "d_offsets"), _dev(d_err, "d_err"),
        _stream_ptr(stream)))


# ---------------------------------------------------------------- nf12.h


def df_nf12_sizes_for(n: int) -> DfNf12Sizes:
    z = DfNf12Sizes()
    check("df_nf12_sizes_for", lib().df_nf12_sizes_for(n, ctypes.byref(z)))
    return z


def df_nf12_encode_groups(d_in: torch.Tensor, top: int, d_slots: torch.Tensor, d_bitmap: torch.Tensor,
                          d_ws: torch.Tensor, d_escaped: torch.Tensor, stream=None) -> None:
    _need_u16(d_in, "d_in")
    n = d_in.numel()
    z = df_nf12_sizes_for(n)
    _need(d_slots, z.slots_bytes, "d_slots")
    _need(d_bitmap, z.bitmap_bytes, "d_bitmap")
    _need(d_escaped, 8, "d_escaped")
    check("df_nf12_encode_groups", lib().df_nf12_encode_groups(
        _dev(d_in, "d_in"), n, top, _dev(d_slots, "d_slots"), _dev(d_bitmap, "d_bitmap"), _dev(d_ws, "d_ws"),
        d_ws.numel() * d_ws.element_size(), _dev(d_escaped, "d_escaped"), _stream_ptr(stream)))


def df_nf12_encode_escapes(d_in: torch.Tensor, top: int, d_slots: torch.Tensor, d_bitmap: torch.Tensor,
                           d_ws: torch.Tensor, d_side: torch.Tensor | None, d_err: torch.Tensor | None = None,
                           stream=None) -> None:
    _need_u16(d_in, "d_in")
    _need_err(d_err)
    n = d_in.numel()
    z = df_nf12_sizes_for(n)
    _need(d_slots, z.slots_bytes, "d_slots")
    _need(d_bitmap, z.bitmap_bytes, "d_bitmap")
    cap = 0 if d_side is None else (d_side.numel() * d_side.element_size()) // 16
    check("df_nf12_encode_escapes", lib().df_nf12_encode_escapes(
        _dev(d_in, "d_in"), n, top, _dev(d_slots, "d_slots"), _dev(d_bitmap, "d_bitmap"), _dev(d_ws, "d_ws"),
        d_ws.numel() * d_ws.element_size(), _dev(d_side, "d_side") if cap else None, cap, _dev(d_err, "d_err"),
        _stream_ptr(stream)))


def _nf12_check_tensor(t: DfNf12Tensor, d_out, name: str) -> None:
    if isinstance(d_out, torch.Tensor):
        _need_u16(d_out, name)
        _need(d_out, 2 * t.n, name)


def df_nf12_decode(t: DfNf12Tensor, d_out: torch.Tensor, d_err: torch.Tensor | None = None, stream=None) -> None:
    """Decode one tensor into d_out (t.out is set from d_out)."""
    _nf12_check_tensor(t, d_out, "d_out")
    _need_err(d_err)
    t.out = d_out if isinstance(d_out, int) else _dev(d_out, "d_out").value
    check("df_nf12_decode", lib().df_nf12_decode(ctypes.byref(t), _dev(d_err, "d_err"), _stream_ptr(stream)))


def df_nf12_decode_batch_workspace(count: int) -> int:
    return int(lib().df_nf12_decode_batch_workspace(count))


def df_nf12_decode_batch_prepare(tensors, d_outs, d_ws: torch.Tensor, stream=None) -> DfNf12Plan:
    """tensors: DfNf12Tensor list; d_outs: one output (tensor or raw device pointer) each."""
    if len(tensors) != len(d_outs):
        raise ValueError("one output per tensor")
    for i, (t, o) in enumerate(zip(tensors, d_outs)):
        _nf12_check_tensor(t, o, f"d_outs[{i}]")
        t.out = o if isinstance(o, int) else _dev(o, f"d_outs[{i}]").value
    arr = (DfNf12Tensor * max(1, len(tensors)))(*tensors)
    _need(d_ws, df_nf12_decode_batch_workspace(len(tensors)), "d_ws")
    plan = DfNf12Plan()
    check("df_nf12_decode_batch_prepare", lib().df_nf12_decode_batch_prepare(
        arr, len(tensors), _dev(d_ws, "d_ws"), d_ws.numel() * d_ws.element_size(), ctypes.byref(plan),
        _stream_ptr(stream)))
    return plan


def df_nf12_decode_batch_run(plan: DfNf12Plan, d_err: torch.Tensor | None = None, stream=None) -> None:
    _need_err(d_err)
    check("df_nf12_decode_batch_run", lib().df_nf12_decode_batch_run(ctypes.byref(plan), _dev(d_err, "d_err"),
                                                                     _stream_ptr(stream)))


def _nf12_encode_array(tensors):
    return (DfNf12EncodeTensor * max(1, len(tensors)))(*tensors)


def df_nf12_encode_batch_workspace(tensors) -> int:
    return int(lib().df_nf12_encode_batch_workspace(_nf12_encode_array(tensors), len(tensors)))


def df_nf12_encode_batch_prepare(tensors, d_ws: torch.Tensor, stream=None) -> DfNf12Plan:
    """tensors: DfNf12EncodeTensor list (device pointers as ints)."""
    _need(d_ws, df_nf12_encode_batch_workspace(tensors), "d_ws")
    plan = DfNf12Plan()
    check("df_nf12_encode_batch_prepare", lib().df_nf12_encode_batch_prepare(
        _nf12_encode_array(tensors), len(tensors), _dev(d_ws, "d_ws"), d_ws.numel() * d_ws.element_size(),
        ctypes.byref(plan), _stream_ptr(stream)))
    return plan


def df_nf12_encode_batch_groups(plan: DfNf12Plan, d_escaped: torch.Tensor, stream=None) -> None:
    _need(d_escaped, 8 * plan.count, "d_escaped")
    check("df_nf12_encode_batch_groups", lib().df_nf12_encode_batch_groups(
        ctypes.byref(plan), _dev(d_escaped, "d_escaped"), _stream_ptr(stream)))


def df_nf12_encode_batch_escapes(plan: DfNf12Plan, d_err: torch.Tensor | None = None, stream=None) -> None:
    _need_err(d_err)
    check("df_nf12_encode_batch_escapes", lib().df_nf12_encode_batch_escapes(
        ctypes.byref(plan), _dev(d_err, "d_err"), _stream_ptr(stream)))

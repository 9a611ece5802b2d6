"""ctypes view of libdf11.so (the C ABI declared in include/df11.h and
include/nf12.h).

The library is loaded on first use. There is no fallback: if the CUDA library
has not been built, every call raises ``NativeLibraryMissing``.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdf11.so")

DF_OK = 0
DF_ERR_INVALID_ARG = 1
DF_ERR_CUDA = 2
DF_ERR_CORRUPT = 3
DF_ERR_UNSUPPORTED = 4
DF_ERR_WORKSPACE = 5

DF_EFLAG_BAD_CODE = 1
DF_EFLAG_COUNT = 2
DF_EFLAG_OFFSETS = 4
DF_EFLAG_TABLES = 8
DF_EFLAG_ENC_TOTAL = 16
DF_EFLAG_ENC_SYMBOL = 32
DF_EFLAG_ENC_WAIT = 64
DF_EFLAG_NF12_SIDE = 128
DF_EFLAG_INDEX8 = 256

DF_NF12_TOP = 7
DF_NF12_TILE_GROUPS = 2048

DF_ENCODE_NOALLOC_MAX_WEIGHTS = 1 << 29

# every function declared in include/df11.h and include/nf12.h
EXPORTS = (
    "df_status_string", "df_last_cuda_error", "df_build_code", "df_code_from_lengths", "df_lut_words", "df_build_lut", "df_plan",
    "df_container_sizes",
    "df_histogram", "df_encode", "df_encode_noalloc", "df_encode_batch_workspace", "df_encode_batch_prepare",
    "df_histogram_batch_run", "df_encode_batch_run", "df_decode", "df_decode_batch_workspace",
    "df_decode_batch_prepare", "df_decode_batch_run", "df_decode_batch", "df_read_error", "df_check_structure", "df_compare",
    "df_sha256_workspace", "df_sha256_device", "df_sha256", "df_index8_bytes", "df_index8_build",
    "df_index8_expand",
    "df_nf12_sizes_for", "df_nf12_encode_groups", "df_nf12_encode_escapes", "df_nf12_decode",
    "df_nf12_decode_batch_workspace", "df_nf12_decode_batch_prepare", "df_nf12_decode_batch_run",
    "df_nf12_encode_batch_workspace", "df_nf12_encode_batch_prepare", "df_nf12_encode_batch_groups",
    "df_nf12_encode_batch_escapes",
)


class NativeLibraryMissing(RuntimeError):
    pass


class DfError(RuntimeError):
    def __init__(self, func: str, status: int, detail: str = ""):
        self.status = status
        name = _status_name(status)
        super().__init__(f"{func} failed: {name}{(' ' + detail) if detail else ''}")


class DfCode(ctypes.Structure):
    _fields_ = [
        ("max_len", ctypes.c_uint32),
        ("n_symbols", ctypes.c_uint32),
        ("min_len", ctypes.c_uint32),
        ("n_tables", ctypes.c_uint32),
        ("lengths", ctypes.c_uint8 * 256),
        ("codes", ctypes.c_uint32 * 256),
    ]


class DfSizes(ctypes.Structure):
    _fields_ = [(name, ctypes.c_uint64) for name in (
        "total_bits", "n_chunks", "stream_bytes", "gap_bytes", "n_blocks", "offsets_bytes", "sm_bytes",
        "container_bytes", "encode_ws_bytes")]

    def as_dict(self) -> dict:
        return {name: int(getattr(self, name)) for name, _ in self._fields_}


class DfTensor(ctypes.Structure):
    _fields_ = [
        ("n", ctypes.c_uint64),
        ("total_bits", ctypes.c_uint64),
        ("chunk_bytes", ctypes.c_uint32),
        ("threads_per_block", ctypes.c_uint32),
        ("max_len", ctypes.c_uint32),
        ("n_tables", ctypes.c_uint32),
        ("stream", ctypes.c_void_p),
        ("gaps", ctypes.c_void_p),
        ("block_offsets", ctypes.c_void_p),
        ("sm", ctypes.c_void_p),
        ("lut", ctypes.c_void_p),
        ("lengths", ctypes.c_uint8 * 256),
        ("index8", ctypes.c_void_p),
        ("index8_wide", ctypes.c_uint64),
    ]


class DfBatchPlan(ctypes.Structure):
    _fields_ = [
        ("d_ws", ctypes.c_void_p),
        ("count", ctypes.c_uint32),
        ("cta_threads", ctypes.c_uint32),
        ("words_per_chunk", ctypes.c_uint32),
        ("region_bytes", ctypes.c_uint32),
        ("max_groups", ctypes.c_uint32),
        ("smem_bytes", ctypes.c_uint32),
        ("max_ctas", ctypes.c_uint32),
        ("reserved", ctypes.c_uint32),
        ("total_blocks", ctypes.c_uint64),
    ]


class DfEncodeTensor(ctypes.Structure):
    _fields_ = [
        ("input", ctypes.c_void_p),
        ("n", ctypes.c_uint64),
        ("code", ctypes.POINTER(DfCode)),
        ("total_bits", ctypes.c_uint64),
        ("chunk_bytes", ctypes.c_uint32),
        ("threads_per_block", ctypes.c_uint32),
        ("stream", ctypes.c_void_p),
        ("gaps", ctypes.c_void_p),
        ("block_offsets", ctypes.c_void_p),
        ("sm", ctypes.c_void_p),
    ]


class DfEncodePlan(ctypes.Structure):
    _fields_ = [
        ("d_ws", ctypes.c_void_p),
        ("count", ctypes.c_uint32),
        ("has_codes", ctypes.c_uint32),
        ("sum_tiles", ctypes.c_uint64),
        ("hist_tiles", ctypes.c_uint64),
        ("hist_tile_weights", ctypes.c_uint64),
        ("ranges", ctypes.c_uint64),
        ("zero_tiles", ctypes.c_uint64),
    ]


class DfNf12Sizes(ctypes.Structure):
    _fields_ = [(name, ctypes.c_uint64) for name in ("groups", "slots_bytes", "bitmap_bytes", "tiles", "encode_ws_bytes")]

    def as_dict(self) -> dict:
        return {name: int(getattr(self, name)) for name, _ in self._fields_}


class DfNf12Tensor(ctypes.Structure):
    _fields_ = [
        ("n", ctypes.c_uint64),
        ("n_escaped", ctypes.c_uint64),
        ("slots", ctypes.c_void_p),
        ("bitmap", ctypes.c_void_p),
        ("side", ctypes.c_void_p),
        ("out", ctypes.c_void_p),
        ("top", ctypes.c_uint32),
        ("reserved", ctypes.c_uint32),
    ]


class DfNf12EncodeTensor(ctypes.Structure):
    _fields_ = [
        ("input", ctypes.c_void_p),
        ("n", ctypes.c_uint64),
        ("slots", ctypes.c_void_p),
        ("bitmap", ctypes.c_void_p),
        ("side", ctypes.c_void_p),
        ("side_capacity", ctypes.c_uint64),
        ("top", ctypes.c_uint32),
        ("reserved", ctypes.c_uint32),
        ("reserved2", ctypes.c_uint64),
    ]


class DfNf12Plan(ctypes.Structure):
    _fields_ = [
        ("d_ws", ctypes.c_void_p),
        ("count", ctypes.c_uint32),
        ("reserved", ctypes.c_uint32),
        ("total_tiles", ctypes.c_uint64),
    ]


_lib = None


def _status_name(status: int) -> str:
    names = {0: "DF_OK", 1: "DF_ERR_INVALID_ARG", 2: "DF_ERR_CUDA", 3: "DF_ERR_CORRUPT", 4: "DF_ERR_UNSUPPORTED",
             5: "DF_ERR_WORKSPACE"}
    return names.get(status, f"status {status}")


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise NativeLibraryMissing(
            f"{LIB_PATH} is missing: build it with `python -m lossless_bf16_weight_huffman_b200.build` "
            "(there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    vp, u64, u32, i32, sz = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int, ctypes.c_size_t
    L.df_status_string.argtypes = [i32]
    L.df_status_string.restype = ctypes.c_char_p
    L.df_last_cuda_error.argtypes = []
    L.df_last_cuda_error.restype = i32
    L.df_build_code.argtypes = [vp, u32, ctypes.POINTER(DfCode)]
    L.df_build_code.restype = i32
    L.df_code_from_lengths.argtypes = [vp, u32, ctypes.POINTER(DfCode)]
    L.df_code_from_lengths.restype = i32
    L.df_lut_words.argtypes = [ctypes.POINTER(DfCode)]
    L.df_lut_words.restype = sz
    L.df_build_lut.argtypes = [ctypes.POINTER(DfCode), vp, sz]
    L.df_build_lut.restype = i32
    L.df_plan.argtypes = [ctypes.POINTER(DfCode), vp, u64, u32, u32, ctypes.POINTER(DfSizes)]
    L.df_plan.restype = i32
    L.df_container_sizes.argtypes = [u64, u64, u32, u32, ctypes.POINTER(DfSizes)]
    L.df_container_sizes.restype = i32
    L.df_histogram.argtypes = [vp, u64, vp, vp]
    L.df_histogram.restype = i32
    L.df_encode.argtypes = [ctypes.POINTER(DfCode), vp, u64, u64, u32, u32, vp, vp, vp, vp, vp, sz, vp, vp]
    L.df_encode.restype = i32
    L.df_encode_noalloc.argtypes = [ctypes.POINTER(DfCode), vp, u64, u64, u32, u32, vp, vp, vp, vp, vp, vp]
    L.df_encode_noalloc.restype = i32
    L.df_encode_batch_workspace.argtypes = [ctypes.POINTER(DfEncodeTensor), u32]
    L.df_encode_batch_workspace.restype = sz
    L.df_encode_batch_prepare.argtypes = [ctypes.POINTER(DfEncodeTensor), u32, vp, sz, ctypes.POINTER(DfEncodePlan),
                                          vp]
    L.df_encode_batch_prepare.restype = i32
    L.df_histogram_batch_run.argtypes = [ctypes.POINTER(DfEncodePlan), vp, vp]
    L.df_histogram_batch_run.restype = i32
    L.df_encode_batch_run.argtypes = [ctypes.POINTER(DfEncodePlan), vp, vp]
    L.df_encode_batch_run.restype = i32
    L.df_decode.argtypes = [ctypes.POINTER(DfTensor), vp, vp, vp]
    L.df_decode.restype = i32
    L.df_decode_batch_workspace.argtypes = [u32]
    L.df_decode_batch_workspace.restype = sz
    L.df_decode_batch_prepare.argtypes = [ctypes.POINTER(DfTensor), vp, u32, vp, sz, ctypes.POINTER(DfBatchPlan), vp]
    L.df_decode_batch_prepare.restype = i32
    L.df_decode_batch_run.argtypes = [ctypes.POINTER(DfBatchPlan), vp, vp]
    L.df_decode_batch_run.restype = i32
    L.df_decode_batch.argtypes = [ctypes.POINTER(DfTensor), vp, u32, vp, sz, vp, vp]
    L.df_decode_batch.restype = i32
    L.df_read_error.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    L.df_read_error.restype = i32
    L.df_check_structure.argtypes = [ctypes.POINTER(DfTensor), vp, vp]
    L.df_check_structure.restype = i32
    L.df_compare.argtypes = [vp, vp, u64, vp, vp]
    L.df_compare.restype = i32
    L.df_sha256_workspace.argtypes = [u64]
    L.df_sha256_workspace.restype = sz
    L.df_sha256_device.argtypes = [vp, u64, vp, sz, vp, vp]
    L.df_sha256_device.restype = i32
    L.df_sha256.argtypes = [vp, u64, vp]
    L.df_sha256.restype = i32
    L.df_index8_bytes.argtypes = [u64, u64]
    L.df_index8_bytes.restype = u64
    L.df_index8_build.argtypes = [vp, u64, vp, sz, vp, vp, vp]
    L.df_index8_build.restype = i32
    L.df_index8_expand.argtypes = [vp, u64, u64, vp, vp, vp]
    L.df_index8_expand.restype = i32
    L.df_nf12_sizes_for.argtypes = [u64, ctypes.POINTER(DfNf12Sizes)]
    L.df_nf12_sizes_for.restype = i32
    L.df_nf12_encode_groups.argtypes = [vp, u64, u32, vp, vp, vp, sz, vp, vp]
    L.df_nf12_encode_groups.restype = i32
    L.df_nf12_encode_escapes.argtypes = [vp, u64, u32, vp, vp, vp, sz, vp, u64, vp, vp]
    L.df_nf12_encode_escapes.restype = i32
    L.df_nf12_decode.argtypes = [ctypes.POINTER(DfNf12Tensor), vp, vp]
    L.df_nf12_decode.restype = i32
    L.df_nf12_decode_batch_workspace.argtypes = [u32]
    L.df_nf12_decode_batch_workspace.restype = sz
    L.df_nf12_decode_batch_prepare.argtypes = [ctypes.POINTER(DfNf12Tensor), u32, vp, sz, ctypes.POINTER(DfNf12Plan), vp]
    L.df_nf12_decode_batch_prepare.restype = i32
    L.df_nf12_decode_batch_run.argtypes = [ctypes.POINTER(DfNf12Plan), vp, vp]
    L.df_nf12_decode_batch_run.restype = i32
    L.df_nf12_encode_batch_workspace.argtypes = [ctypes.POINTER(DfNf12EncodeTensor), u32]
    L.df_nf12_encode_batch_workspace.restype = sz
    L.df_nf12_encode_batch_prepare.argtypes = [ctypes.POINTER(DfNf12EncodeTensor), u32, vp, sz,
                                               ctypes.POINTER(DfNf12Plan), vp]
    L.df_nf12_encode_batch_prepare.restype = i32
    L.df_nf12_encode_batch_groups.argtypes = [ctypes.POINTER(DfNf12Plan), vp, vp]
    L.df_nf12_encode_batch_groups.restype = i32
    L.df_nf12_encode_batch_escapes.argtypes = [ctypes.POINTER(DfNf12Plan), vp, vp]
    L.df_nf12_encode_batch_escapes.restype = i32
    _lib = L
    return L


def check(func: str, status: int) -> None:
    if status != DF_OK:
        detail = ""
        if status == DF_ERR_CUDA:
            detail = f"(cudaError {lib().df_last_cuda_error()})"
        raise DfError(func, status, detail)

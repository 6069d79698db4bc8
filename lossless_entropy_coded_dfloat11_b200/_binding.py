"""ctypes binding of libdf11.so: argument marshalling only.

Every computation happens in the library (CUDA kernels and its host code);
this module converts Python values to the C ABI of include/df11.h.  There is
no fallback: if the library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

DF11_MAX_SEGMENTS = 64
STATUS_NAMES = {0: "DF11_OK", 1: "DF11_ERR_INVALID", 2: "DF11_ERR_CUDA", 3: "DF11_ERR_CORRUPT",
                4: "DF11_ERR_TOO_LARGE", 5: "DF11_ERR_CAPACITY"}
DF11_OK, DF11_ERR_INVALID, DF11_ERR_CUDA, DF11_ERR_CORRUPT, DF11_ERR_TOO_LARGE, DF11_ERR_CAPACITY = range(6)

EXPORTED = ["df11_version", "df11_last_error", "df11_code_lengths", "df11_header_init", "df11_build_lut",
            "df11_compress_workspace_size", "df11_compress_plan", "df11_compress_encode", "df11_decompress",
            "df11_compress_encode_static", "df11_decompress_sms", "df11_compress_plan_u8",
            "df11_compress_encode_u8", "df11_decompress_u8", "df11_compress_encode_chunked",
            "df11_decompress_chunked", "df11_decompress_blocks", "df11_decompress_u8_blocks",
            "df11_decode_kernel_info", "df11_decompress_opts"]


class Header(ctypes.Structure):
    """Mirror of df11_header."""
    _fields_ = [
        ("version", ctypes.c_uint32),
        ("window_bytes", ctypes.c_uint32),
        ("threads_per_block", ctypes.c_uint32),
        ("max_code_len", ctypes.c_uint32),
        ("n_elems", ctypes.c_uint64),
        ("total_bits", ctypes.c_uint64),
        ("n_threads", ctypes.c_uint64),
        ("n_blocks", ctypes.c_uint64),
        ("code_len", ctypes.c_uint8 * 256),
        ("n_segments", ctypes.c_uint32),
        ("plan_token", ctypes.c_uint32),
        ("seg_elem_off", ctypes.c_uint64 * (DF11_MAX_SEGMENTS + 1)),
        ("bytes_exp", ctypes.c_uint64),
        ("bytes_sm", ctypes.c_uint64),
        ("bytes_gaps", ctypes.c_uint64),
        ("bytes_off", ctypes.c_uint64),
        ("bytes_lut", ctypes.c_uint64),
    ]


class DecodeOptions(ctypes.Structure):
    """Mirror of df11_decode_options."""
    _fields_ = [
        ("peek_bits", ctypes.c_uint32),
        ("max_sms", ctypes.c_uint32),
        ("max_warps_per_cta", ctypes.c_uint32),
        ("ctas", ctypes.c_uint32),
        ("block_begin", ctypes.c_uint32),
        ("block_end", ctypes.c_uint32),
        ("early_staging", ctypes.c_uint32),
        ("reserved", ctypes.c_uint32),
    ]


class KernelInfo(ctypes.Structure):
    """Mirror of df11_kernel_info."""
    _fields_ = [
        ("kernel", ctypes.c_char * 64),
        ("grid", ctypes.c_uint32),
        ("block", ctypes.c_uint32),
        ("smem_bytes", ctypes.c_uint32),
        ("peek_bits", ctypes.c_uint32),
        ("table_copies", ctypes.c_uint32),
        ("reserved", ctypes.c_uint32),
        ("thread_blocks", ctypes.c_uint64),
    ]


class DF11Error(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} -> {STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


_lib = None


def library_path() -> str:
    return _build.LIB_PATH


def load(build_if_missing: bool = True):
    """Load libdf11.so (building it first if it is missing or stale and nvcc
    is available).  Raises if the library cannot be loaded."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.LIB_PATH
    if build_if_missing:
        try:
            _build.build()
        except (OSError, RuntimeError) as exc:
            if not os.path.exists(path):
                raise RuntimeError(f"libdf11.so is missing and could not be built: {exc}") from exc
    if not os.path.exists(path):
        raise RuntimeError(f"libdf11.so not found at {path}; run lossless_entropy_coded_dfloat11_b200/build.py")
    lib = ctypes.CDLL(path)
    vp, u64, u32 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32
    hp = ctypes.POINTER(Header)
    lib.df11_version.argtypes = []
    lib.df11_version.restype = ctypes.c_int
    lib.df11_last_error.argtypes = []
    lib.df11_last_error.restype = ctypes.c_char_p
    lib.df11_code_lengths.argtypes = [vp, u32, vp]
    lib.df11_header_init.argtypes = [hp, vp, u64, u64, u32, u32, vp, u32]
    lib.df11_build_lut.argtypes = [hp, vp, u64]
    lib.df11_compress_workspace_size.argtypes = [u64, ctypes.POINTER(u64)]
    lib.df11_compress_plan.argtypes = [vp, vp, u32, u32, u32, vp, u64, hp, vp]
    lib.df11_compress_encode.argtypes = [vp, hp, vp, u64, vp, vp, vp, vp, vp, vp]
    lib.df11_decompress.argtypes = [hp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.df11_decompress_sms.argtypes = [hp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_uint32, vp]
    lib.df11_compress_encode_static.argtypes = [vp, hp, vp, vp, vp, vp, vp, vp]
    lib.df11_compress_plan_u8.argtypes = [vp, vp, u32, u32, u32, vp, u64, hp, vp]
    lib.df11_compress_encode_u8.argtypes = [vp, hp, vp, u64, vp, vp, vp, vp, vp]
    lib.df11_decompress_u8.argtypes = [hp, vp, vp, vp, vp, vp, vp, vp]
    lib.df11_compress_encode_chunked.argtypes = [vp, hp, vp, u64, vp, vp, vp, vp, vp]
    lib.df11_decompress_chunked.argtypes = [hp, vp, vp, vp, vp, vp, vp, vp]
    lib.df11_decompress_blocks.argtypes = [hp, vp, vp, vp, vp, vp, vp, u64, u64, vp, vp]
    lib.df11_decompress_u8_blocks.argtypes = [hp, vp, vp, vp, vp, vp, u64, u64, vp, vp]
    lib.df11_decode_kernel_info.argtypes = [hp, u32, ctypes.POINTER(DecodeOptions), ctypes.POINTER(KernelInfo)]
    lib.df11_decompress_opts.argtypes = [hp, vp, vp, vp, vp, vp, vp, u32, ctypes.POINTER(DecodeOptions), vp, vp]
    for name in EXPORTED[2:]:
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def check(fn: str, rc: int) -> None:
    if rc != DF11_OK:
        msg = load().df11_last_error().decode(errors="replace")
        raise DF11Error(fn, rc, msg)


def call(fn: str, *args) -> None:
    check(fn, getattr(load(), fn)(*args))

"""DF11 oracle -- test infrastructure only.

A plain, slow, single-threaded CPU encoder/decoder for the DFloat11 container
(``df11_oracle.c``), loaded with ctypes.  Only the tests, the smoke check and the
benchmark's CPU-baseline / reference arm may import this package.  The CUDA
library never imports, links or calls it, and the two share no code: they meet
only through the byte layout of the container and the seeded inputs.

Sources: "DFloat11: compressao sem perda para inferencia em GPU que reduz LLMs
para 70% do tamanho" (sections "O formato DFloat11", "Decodificacao com LUT
hierarquica", "Kernel de GPU em 2 etapas e metadados auxiliares"), and the
abstract "70% Size, 100% Accuracy: Lossless LLM Compression for Efficient GPU
Inference via Dynamic-Length Float".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "df11_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

OK, ERR_ARG, ERR_CORRUPT, ERR_TOO_LARGE, ERR_CAPACITY = 0, 1, 3, 4, 5


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, one thread, no vector tuning)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    # a test may point at a deliberately broken build of the oracle to show
    # that the pins catch it
    lib = ctypes.CDLL(os.environ.get("DF11_ORACLE_LIB") or build())
    u8p = ctypes.POINTER(ctypes.c_uint8)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    u32p = ctypes.POINTER(ctypes.c_uint32)
    u64p = ctypes.POINTER(ctypes.c_uint64)
    c_u32, c_u64, c_int = ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int
    lib.oracle_exponent.argtypes = [c_u32]; lib.oracle_exponent.restype = c_u32
    lib.oracle_sign_mantissa.argtypes = [c_u32]; lib.oracle_sign_mantissa.restype = c_u32
    lib.oracle_merge.argtypes = [c_u32, c_u32]; lib.oracle_merge.restype = c_u32
    lib.oracle_histogram.argtypes = [u16p, c_u64, u64p]; lib.oracle_histogram.restype = None
    lib.oracle_entropy_bits.argtypes = [u64p]; lib.oracle_entropy_bits.restype = ctypes.c_double
    lib.oracle_code_lengths.argtypes = [u64p, c_int, u8p]; lib.oracle_code_lengths.restype = c_int
    lib.oracle_canonical_codes.argtypes = [u8p, u32p]; lib.oracle_canonical_codes.restype = c_int
    lib.oracle_sizes_for.argtypes = [u64p, u8p, c_u32, u64p]; lib.oracle_sizes_for.restype = c_int
    lib.oracle_read_gap.argtypes = [u8p, c_u64]; lib.oracle_read_gap.restype = c_u32
    lib.oracle_encode.argtypes = [u16p, c_u64, u8p, c_u32, u8p, c_u64, u8p, c_u64,
                                  u8p, c_u64, u32p, c_u64]
    lib.oracle_encode.restype = c_int
    lib.oracle_decode.argtypes = [u8p, u8p, c_u64, u8p, c_u64, u16p]
    lib.oracle_decode.restype = c_int
    lib.oracle_decode_windowed.argtypes = [u8p, u8p, c_u64, u8p, u8p, u32p, c_u32, c_u64,
                                           c_u64, c_u64, u16p]
    lib.oracle_decode_windowed.restype = c_int
    _lib = lib
    return lib


def _ptr(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be contiguous"
    return a.ctypes.data_as(ctypes.POINTER(ctype))


class OracleError(RuntimeError):
    def __init__(self, what: str, code: int):
        super().__init__(f"{what} failed with status {code}")
        self.code = code


def _check(what: str, rc: int) -> None:
    if rc != OK:
        raise OracleError(what, rc)


# --------------------------------------------------------------------------- #
# Field split and statistics                                                  #
# --------------------------------------------------------------------------- #
def exponent(x: int) -> int:
    return _load().oracle_exponent(x)


def sign_mantissa(x: int) -> int:
    return _load().oracle_sign_mantissa(x)


def merge(e: int, sm: int) -> int:
    return _load().oracle_merge(e, sm)


def histogram(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.uint16).reshape(-1)
    h = np.zeros(256, dtype=np.uint64)
    _load().oracle_histogram(_ptr(x, ctypes.c_uint16), x.size, _ptr(h, ctypes.c_uint64))
    return h


def entropy_bits(hist: np.ndarray) -> float:
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    return float(_load().oracle_entropy_bits(_ptr(h, ctypes.c_uint64)))


def code_lengths(hist: np.ndarray, max_len: int = 32) -> np.ndarray:
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    assert h.size == 256
    out = np.zeros(256, dtype=np.uint8)
    _check("oracle_code_lengths",
           _load().oracle_code_lengths(_ptr(h, ctypes.c_uint64), max_len, _ptr(out, ctypes.c_uint8)))
    return out


def canonical_codes(lengths: np.ndarray) -> np.ndarray:
    ln = np.ascontiguousarray(lengths, dtype=np.uint8)
    out = np.zeros(256, dtype=np.uint32)
    _check("oracle_canonical_codes",
           _load().oracle_canonical_codes(_ptr(ln, ctypes.c_uint8), _ptr(out, ctypes.c_uint32)))
    return out


# --------------------------------------------------------------------------- #
# Container                                                                   #
# --------------------------------------------------------------------------- #
@dataclass
class Stream:
    """One DF11 stream as the oracle writes it (all arrays on the host)."""
    code_len: np.ndarray   # uint8[256]
    n_elems: int
    total_bits: int
    threads_per_block: int
    n_threads: int
    n_blocks: int
    exp: np.ndarray        # uint8[bytes_exp]   EncodedExponent
    sm: np.ndarray         # uint8[bytes_sm]    PackedSignMantissa
    gaps: np.ndarray       # uint8[bytes_gaps]  5-bit Gaps
    block_off: np.ndarray  # uint32[n_blocks+1] per-thread-block output positions

    def compressed_bytes(self) -> int:
        """Bytes of the arrays the format defines, without padding: the code
        bits, one byte per element, 5 bits per thread, 4 bytes per block
        position, and the 256-byte code-length table."""
        return ((self.total_bits + 7) // 8 + self.n_elems + (5 * self.n_threads + 7) // 8
                + 4 * (self.n_blocks + 1) + 256)


def sizes(hist: np.ndarray, lengths: np.ndarray, threads_per_block: int) -> dict:
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    ln = np.ascontiguousarray(lengths, dtype=np.uint8)
    out = np.zeros(8, dtype=np.uint64)
    _check("oracle_sizes_for", _load().oracle_sizes_for(
        _ptr(h, ctypes.c_uint64), _ptr(ln, ctypes.c_uint8), threads_per_block,
        _ptr(out, ctypes.c_uint64)))
    keys = ["n_elems", "total_bits", "n_threads", "n_blocks", "bytes_exp", "bytes_sm",
            "bytes_gaps", "bytes_off"]
    return {k: int(v) for k, v in zip(keys, out)}


def encode(x: np.ndarray, threads_per_block: int = 256, max_len: int = 32,
           lengths: np.ndarray | None = None) -> Stream:
    """Encode BF16 bit patterns (uint16) with a table built from their own
    histogram (or the given code lengths)."""
    x = np.ascontiguousarray(x, dtype=np.uint16).reshape(-1)
    hist = histogram(x)
    ln = code_lengths(hist, max_len) if lengths is None else np.ascontiguousarray(lengths, dtype=np.uint8)
    sz = sizes(hist, ln, threads_per_block)
    exp = np.zeros(sz["bytes_exp"], dtype=np.uint8)
    sm = np.zeros(sz["bytes_sm"], dtype=np.uint8)
    gaps = np.zeros(sz["bytes_gaps"], dtype=np.uint8)
    off = np.zeros(sz["n_blocks"] + 1, dtype=np.uint32)
    _check("oracle_encode", _load().oracle_encode(
        _ptr(x, ctypes.c_uint16), x.size, _ptr(ln, ctypes.c_uint8), threads_per_block,
        _ptr(exp, ctypes.c_uint8), exp.size, _ptr(sm, ctypes.c_uint8), sm.size,
        _ptr(gaps, ctypes.c_uint8), gaps.size, _ptr(off, ctypes.c_uint32), off.size))
    return Stream(code_len=ln, n_elems=x.size, total_bits=sz["total_bits"],
                  threads_per_block=threads_per_block, n_threads=sz["n_threads"],
                  n_blocks=sz["n_blocks"], exp=exp, sm=sm, gaps=gaps, block_off=off)


def decode(s: Stream) -> np.ndarray:
    """Bit-serial decode (walks the code trie one bit at a time)."""
    out = np.zeros(s.n_elems, dtype=np.uint16)
    ln = np.ascontiguousarray(s.code_len, dtype=np.uint8)
    exp = np.ascontiguousarray(s.exp, dtype=np.uint8)
    sm = np.ascontiguousarray(s.sm, dtype=np.uint8)
    _check("oracle_decode", _load().oracle_decode(
        _ptr(ln, ctypes.c_uint8), _ptr(exp, ctypes.c_uint8), s.total_bits,
        _ptr(sm, ctypes.c_uint8), s.n_elems, _ptr(out, ctypes.c_uint16)))
    return out


def decode_windowed(s: Stream, b0: int = 0, b1: int | None = None) -> np.ndarray:
    """Decode thread blocks [b0, b1) through Gaps and block offsets, checking
    that the auxiliary arrays are consistent.  Returns elements
    block_off[b0] .. block_off[b1]."""
    if b1 is None:
        b1 = s.n_blocks
    lo = int(s.block_off[b0]) if b0 < b1 else 0
    hi = int(s.block_off[b1]) if b0 < b1 else 0
    out = np.zeros(max(hi - lo, 1), dtype=np.uint16)
    ln = np.ascontiguousarray(s.code_len, dtype=np.uint8)
    exp = np.ascontiguousarray(s.exp, dtype=np.uint8)
    sm = np.ascontiguousarray(s.sm, dtype=np.uint8)
    gaps = np.ascontiguousarray(s.gaps, dtype=np.uint8)
    off = np.ascontiguousarray(s.block_off, dtype=np.uint32)
    _check("oracle_decode_windowed", _load().oracle_decode_windowed(
        _ptr(ln, ctypes.c_uint8), _ptr(exp, ctypes.c_uint8), s.total_bits,
        _ptr(sm, ctypes.c_uint8), _ptr(gaps, ctypes.c_uint8), _ptr(off, ctypes.c_uint32),
        s.threads_per_block, s.n_threads, b0, b1, _ptr(out, ctypes.c_uint16)))
    return out[: hi - lo]


def read_gap(gaps: np.ndarray, t: int) -> int:
    g = np.ascontiguousarray(gaps, dtype=np.uint8)
    return int(_load().oracle_read_gap(_ptr(g, ctypes.c_uint8), t))


def chunk_starts(x: np.ndarray, code_len: np.ndarray, chunk: int) -> np.ndarray:
    """Start bit of the code of element k*chunk, k = 0 .. ceil(n/chunk) - 1,
    then total_bits: the table of the independent-chunk variant of the
    container (segments that decode on their own, "EntroLLM: Compressao de
    Pesos Codificada por Entropia ...", section "Metodologia", item 3).  By
    definition the prefix sums of the code lengths of the elements' exponent
    fields (summed per chunk first)."""
    x = np.ascontiguousarray(x, dtype=np.uint16).reshape(-1)
    n = x.size
    ln = np.ascontiguousarray(code_len, dtype=np.uint8)[(x >> 7) & 0xFF]
    if n == 0:
        return np.zeros(1, dtype=np.uint64)
    per_chunk = np.add.reduceat(ln.astype(np.uint64), np.arange(0, n, chunk))
    return np.concatenate([[0], np.cumsum(per_chunk)]).astype(np.uint64)

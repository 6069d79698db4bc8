"""CPU checks of the C ABI's argument validation on the decode entry points.

Every call here is rejected (or is a no-op) on the host before any CUDA call:
the header, the block range, SM caps, null and misaligned device pointers are
all checked first, so no GPU is needed.  The device pointers passed are
well-formed but fake; a rejected call never dereferences them.
"""
import ctypes

import numpy as np
import pytest

import oracle
import lossless_entropy_coded_dfloat11_b200 as df11
from lossless_entropy_coded_dfloat11_b200 import _binding as B

FAKE = 0x7F0000001000  # 16-byte aligned, never dereferenced
MISALIGNED = FAKE + 8


@pytest.fixture(scope="module")
def hdr():
    x = np.random.default_rng(5).normal(0, 0.02, size=50000).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    s = oracle.encode(bits, threads_per_block=64)
    h = df11.make_header(s.code_len, s.n_elems, s.total_bits, 64)
    assert int(h.n_blocks) > 4
    return h


def status_of(fn, *args) -> int:
    lib = B.load()
    return int(getattr(lib, fn)(*args))


def ptrs(n, bad_index=None, bad_value=0):
    p = [ctypes.c_void_p(FAKE) for _ in range(n)]
    if bad_index is not None:
        p[bad_index] = ctypes.c_void_p(bad_value) if bad_value else ctypes.c_void_p(None)
    return p


def blocks_call(h, b0, b1, bad_index=None, bad_value=0):
    p = ptrs(6, bad_index, bad_value)  # exp, sm, gaps, off, lut, out
    return status_of("df11_decompress_blocks", ctypes.byref(h), *p, ctypes.c_uint64(b0), ctypes.c_uint64(b1),
                     ctypes.c_void_p(None), ctypes.c_void_p(None))


def test_block_ranges_outside_the_stream_are_rejected(hdr):
    nb = int(hdr.n_blocks)
    for b0, b1 in [(3, 2), (0, nb + 1), (nb + 1, nb + 2), (nb, nb - 1)]:
        assert blocks_call(hdr, b0, b1) == B.DF11_ERR_INVALID, (b0, b1)
        assert "block range" in B.load().df11_last_error().decode()


def test_empty_block_ranges_are_no_ops_before_any_pointer_check(hdr):
    nb = int(hdr.n_blocks)
    for b in (0, 1, nb):
        assert blocks_call(hdr, b, b, bad_index=0) == B.DF11_OK  # null exp, but nothing to do


@pytest.mark.parametrize("which", range(6))
def test_null_and_misaligned_pointers_are_rejected(hdr, which):
    assert blocks_call(hdr, 0, 1, bad_index=which) == B.DF11_ERR_INVALID
    assert "null device pointer" in B.load().df11_last_error().decode()
    assert blocks_call(hdr, 0, 1, bad_index=which, bad_value=MISALIGNED) == B.DF11_ERR_INVALID
    assert "16-byte aligned" in B.load().df11_last_error().decode()


def test_whole_stream_calls_validate_the_same_way(hdr):
    p = ptrs(6)
    st = ctypes.c_void_p(None)
    assert status_of("df11_decompress_sms", ctypes.byref(hdr), *p, st, ctypes.c_uint32(0), st) == B.DF11_ERR_INVALID
    assert "max_sms" in B.load().df11_last_error().decode()
    q = ptrs(6, bad_index=2)  # null gaps
    assert status_of("df11_decompress", ctypes.byref(hdr), *q, st, st) == B.DF11_ERR_INVALID
    # 8-bit symbols take no sign+mantissa array: exp, gaps, off, lut, out
    u = ptrs(5, bad_index=4, bad_value=MISALIGNED)
    assert status_of("df11_decompress_u8", ctypes.byref(hdr), *u, st, st) == B.DF11_ERR_INVALID
    assert status_of("df11_decompress_u8_blocks", ctypes.byref(hdr), *ptrs(5), ctypes.c_uint64(2),
                     ctypes.c_uint64(1), st, st) == B.DF11_ERR_INVALID


def test_a_header_that_disagrees_with_its_sizes_is_rejected_first(hdr):
    bad = B.Header.from_buffer_copy(hdr)
    bad.bytes_exp += 16
    assert blocks_call(bad, 0, 1) == B.DF11_ERR_INVALID
    assert "header sizes" in B.load().df11_last_error().decode()
    bad = B.Header.from_buffer_copy(hdr)
    bad.version = 99
    assert status_of("df11_decompress", ctypes.byref(bad), *ptrs(6), ctypes.c_void_p(None),
                     ctypes.c_void_p(None)) == B.DF11_ERR_INVALID


def test_empty_stream_is_a_no_op(hdr):
    ln = np.zeros(256, dtype=np.uint8)
    ln[[1, 2]] = 1
    empty = df11.make_header(ln, 0, 0, 64)
    st = ctypes.c_void_p(None)
    nulls = [ctypes.c_void_p(None)] * 6
    assert status_of("df11_decompress", ctypes.byref(empty), *nulls, st, st) == B.DF11_OK
    assert status_of("df11_decompress_blocks", ctypes.byref(empty), *nulls, ctypes.c_uint64(0),
                     ctypes.c_uint64(int(empty.n_blocks)), st, st) == B.DF11_OK

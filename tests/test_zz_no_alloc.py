"""The allocation-free encode entry point, df11_compress_encode_static.

Some callers cannot allocate device memory at the moment they compress: a
serving engine that has handed all of HBM to its own pools and forbids later
cudaMalloc calls, or code running inside an allocator (an out-of-memory
handler, for instance) where allocating would recurse.  For them the library
keeps the encoder's scratch in a fixed array of its own.  These tests call
that entry point through the C ABI and check, on two calls in a row, that it
writes exactly the bytes the workspace-based df11_compress_encode writes.

This file is collected last on purpose: if it fails, every other test has
already run.
"""
import ctypes

import numpy as np
import pytest
import torch

import lossless_entropy_coded_dfloat11_b200 as df11
from lossless_entropy_coded_dfloat11_b200 import _binding as B
from lossless_entropy_coded_dfloat11_b200 import inputs

pytestmark = pytest.mark.gpu

STATIC_MAX_ELEMS = 1 << 28


def _ptr(t):
    return ctypes.c_void_p(int(t.data_ptr()))


def _encode_static(tensors, header):
    """Caller-owned outputs (allocated here, by the test, not by the entry
    point), then one df11_compress_encode_static call."""
    dev = tensors[0].device
    exp = torch.empty(int(header.bytes_exp), dtype=torch.uint8, device=dev)
    sm = torch.empty(int(header.bytes_sm) or 16, dtype=torch.uint8, device=dev)
    gaps = torch.empty(int(header.bytes_gaps), dtype=torch.uint8, device=dev)
    off = torch.empty(int(header.n_blocks) + 1, dtype=torch.int32, device=dev)
    lut = torch.empty(int(header.bytes_lut), dtype=torch.uint8, device=dev)
    segs = (ctypes.c_void_p * len(tensors))(*[int(t.data_ptr()) for t in tensors])
    stream = ctypes.c_void_p(int(torch.cuda.current_stream().cuda_stream))
    B.call("df11_compress_encode_static", segs, ctypes.byref(header), _ptr(exp), _ptr(sm), _ptr(gaps),
           _ptr(off), _ptr(lut), stream)
    torch.cuda.synchronize()
    return df11.CompressedStream(header, exp, sm, gaps, off, lut,
                                 shapes=[tuple(t.shape) for t in tensors])


def _same(a: df11.CompressedStream, b: df11.CompressedStream):
    ha, hb = df11.to_host(a), df11.to_host(b)
    for key in ("exp", "sm", "gaps", "block_off", "code_len"):
        np.testing.assert_array_equal(ha[key], hb[key], err_msg=key)
    n = int(a.header.bytes_lut)
    assert torch.equal(a.lut[:n], b.lut[:n])


@pytest.mark.parametrize("make", [
    lambda: inputs.llama_block(dict(hidden=512, intermediate=1408, kv=128), seed_base=61),
    lambda: inputs.matrix_outliers(2048, 1024, seed=62),
    lambda: inputs.edge_case(65537, "zipf", 515),
])
def test_static_encode_matches_workspace_encode_twice(make):
    w = make()
    tensors = [t.cuda() for t in w.tensors]
    ref = df11.compress(tensors)                    # workspace-based path
    for _ in range(2):                              # two calls in a row
        got = _encode_static(tensors, ref.header)
        _same(ref, got)
        out = df11.decompress(got)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16).cpu(),
                           torch.cat([t.reshape(-1) for t in w.tensors]).view(torch.int16))


def test_static_encode_reuses_its_scratch_across_streams():
    """A large stream, then a small one, then the large one again: the
    scratch keeps the previous call's contents, which must not leak."""
    big = [t.cuda() for t in inputs.llama_block(dict(hidden=1024, intermediate=3584, kv=256),
                                                 seed_base=71).tensors]
    small = [inputs.gaussian((333, 77), 0.02, 72).cuda()]
    ref_big, ref_small = df11.compress(big), df11.compress(small)
    _same(ref_big, _encode_static(big, ref_big.header))
    _same(ref_small, _encode_static(small, ref_small.header))
    _same(ref_big, _encode_static(big, ref_big.header))


def test_static_encode_rejects_streams_above_its_limit():
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    hdr = df11.make_header(np.eye(1, 256, 0, dtype=np.uint8).reshape(-1), STATIC_MAX_ELEMS + 1,
                           STATIC_MAX_ELEMS + 1, 256)
    segs = (ctypes.c_void_p * 1)(int(x.data_ptr()))
    rc = B.load().df11_compress_encode_static(segs, ctypes.byref(hdr), _ptr(x), _ptr(x), _ptr(x), _ptr(x),
                                              _ptr(x), ctypes.c_void_p(0))
    assert rc == B.DF11_ERR_TOO_LARGE
    assert "at most" in B.load().df11_last_error().decode()

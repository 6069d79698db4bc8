"""The encode kernel learns each chunk range's code bits in one of two ways:
from the per-range histograms that df11_compress_plan leaves in its workspace
(named by the header's plan_token), or by counting them itself in a pass
over the range (any other workspace, a header the plan did not fill, the
allocation-free entry point).  Both must give the same stream, byte for
byte, and the oracle's.  Ragged segments put the ranges' edges at unaligned
offsets inside segments, where the histogram kernel counts element by
element.
"""
import ctypes

import numpy as np
import pytest
import torch

import lossless_entropy_coded_dfloat11_b200 as df11
import oracle
from lossless_entropy_coded_dfloat11_b200 import _binding as B

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(int(t.data_ptr()))


def _plan(tensors, u8: bool):
    n = sum(t.numel() for t in tensors)
    ws = torch.empty(max(df11.workspace_bytes(n), 16), dtype=torch.uint8, device="cuda")
    ptrs = (ctypes.c_void_p * len(tensors))(*[int(t.data_ptr()) for t in tensors])
    counts = (ctypes.c_uint64 * len(tensors))(*[t.numel() for t in tensors])
    hdr = B.Header()
    stream = ctypes.c_void_p(int(torch.cuda.current_stream().cuda_stream))
    B.call("df11_compress_plan_u8" if u8 else "df11_compress_plan", ptrs, counts, len(tensors), 32 if u8 else 64,
           32, _ptr(ws), ws.numel(), ctypes.byref(hdr), stream)
    return hdr, ws


def _encode(tensors, hdr, ws, u8: bool) -> dict:
    ptrs = (ctypes.c_void_p * len(tensors))(*[int(t.data_ptr()) for t in tensors])
    stream = ctypes.c_void_p(int(torch.cuda.current_stream().cuda_stream))
    exp = torch.empty(int(hdr.bytes_exp), dtype=torch.uint8, device="cuda")
    sm = torch.empty(int(hdr.bytes_sm) or 16, dtype=torch.uint8, device="cuda")
    gaps = torch.empty(int(hdr.bytes_gaps), dtype=torch.uint8, device="cuda")
    off = torch.empty(int(hdr.n_blocks) + 1, dtype=torch.int32, device="cuda")
    lut = torch.empty(int(hdr.bytes_lut), dtype=torch.uint8, device="cuda")
    if u8:
        B.call("df11_compress_encode_u8", ptrs, ctypes.byref(hdr), _ptr(ws), ws.numel(), _ptr(exp), _ptr(gaps),
               _ptr(off), _ptr(lut), stream)
    else:
        B.call("df11_compress_encode", ptrs, ctypes.byref(hdr), _ptr(ws), ws.numel(), _ptr(exp), _ptr(sm),
               _ptr(gaps), _ptr(off), _ptr(lut), stream)
    torch.cuda.synchronize()
    got = dict(exp=exp.cpu().numpy()[: int(hdr.bytes_exp)], gaps=gaps.cpu().numpy()[: int(hdr.bytes_gaps)],
               off=off.cpu().numpy().view(np.uint32)[: int(hdr.n_blocks) + 1], lut=lut.cpu().numpy())
    if not u8:
        got["sm"] = sm.cpu().numpy()[: int(hdr.bytes_sm)]
    return got


def _three_ways(tensors, u8: bool) -> dict:
    hdr, ws = _plan(tensors, u8)
    assert hdr.plan_token != 0 or hdr.n_elems == 0
    a = _encode(tensors, hdr, ws, u8)                     # the plan's histograms
    other = torch.full_like(ws, 0xA5)                      # another workspace: stale bytes
    b = _encode(tensors, hdr, other, u8)
    h2 = B.Header.from_buffer_copy(hdr)                    # a header the plan did not fill
    h2.plan_token ^= 0x5A5A5A5A
    c = _encode(tensors, h2, ws, u8)
    for key in a:
        np.testing.assert_array_equal(a[key], b[key], err_msg=f"other workspace: {key}")
        np.testing.assert_array_equal(a[key], c[key], err_msg=f"other token: {key}")
    return a


def _bf16_ragged(sizes, seed):
    g = torch.Generator().manual_seed(seed)
    return [(torch.randn(n, generator=g) * 0.02).to(torch.bfloat16) for n in sizes]


@pytest.mark.parametrize("sizes", [
    [1, 7, 4097, 13, 100003, 9],             # one range, every segment edge unaligned
    [1000003, 999999, 1500001],              # many ranges, range edges inside segments
    [3 * 4096 * 600 + 5],                    # one segment, the last range short
])
def test_bf16_range_histograms_match_counting(sizes):
    ts = _bf16_ragged(sizes, 40 + len(sizes))
    got = _three_ways([t.cuda() for t in ts], u8=False)
    x = torch.cat(ts).view(torch.int16).numpy().view(np.uint16)
    s = oracle.encode(x, threads_per_block=64)
    np.testing.assert_array_equal(got["exp"], s.exp)
    np.testing.assert_array_equal(got["sm"], s.sm)
    np.testing.assert_array_equal(got["gaps"], s.gaps)
    np.testing.assert_array_equal(got["off"], s.block_off)


def test_bf16_sixty_four_ragged_segments():
    """The most segments a stream may have, of random sizes: segment edges
    fall anywhere inside the encode ranges, several segments per range."""
    rng = np.random.default_rng(77)
    sizes = [int(v) for v in rng.integers(1, 150_000, size=B.DF11_MAX_SEGMENTS)]
    ts = _bf16_ragged(sizes, 78)
    got = _three_ways([t.cuda() for t in ts], u8=False)
    x = torch.cat(ts).view(torch.int16).numpy().view(np.uint16)
    s = oracle.encode(x, threads_per_block=64)
    np.testing.assert_array_equal(got["exp"], s.exp)
    np.testing.assert_array_equal(got["sm"], s.sm)
    np.testing.assert_array_equal(got["gaps"], s.gaps)
    np.testing.assert_array_equal(got["off"], s.block_off)


@pytest.mark.parametrize("sizes", [[3, 15, 16, 17, 70001], [2000001, 1999999]])
def test_u8_range_histograms_match_counting(sizes):
    rng = np.random.default_rng(50 + len(sizes))
    ts = [torch.from_numpy(np.clip(np.round(rng.normal(120, 9, n)), 0, 255).astype(np.uint8)) for n in sizes]
    got = _three_ways([t.cuda() for t in ts], u8=True)
    x = torch.cat(ts).numpy()
    s = oracle.encode(x.astype(np.uint16) << 7, threads_per_block=32)  # the byte as a BF16 exponent
    np.testing.assert_array_equal(got["exp"], s.exp)
    np.testing.assert_array_equal(got["gaps"], s.gaps)
    np.testing.assert_array_equal(got["off"], s.block_off)


def test_plan_tokens_differ_between_plans():
    t = _bf16_ragged([5000], 60)[0].cuda()
    h1, _ = _plan([t], False)
    h2, _ = _plan([t], False)
    assert h1.plan_token != 0 and h2.plan_token != 0 and h1.plan_token != h2.plan_token

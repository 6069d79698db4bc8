"""GPU: decoding a range of thread blocks (df11_decompress_blocks and its
8-bit twin) and the pipelined end-to-end decode from host buffers built on it
(HostStream.run), against the CPU oracle.

* Any partition of a stream into block ranges, decoded piece by piece into
  one buffer, equals the oracle's decode; elements outside a piece's range are
  left untouched.
* A piece decodes correctly when the device arrays hold garbage everywhere
  except the bytes `piece_ranges` lists for it (the read contract, checked
  on the kernels themselves: T = 32 and 64 warp kernels, T = 256 block kernel).
* HostStream.run gives the original weights for any number of pieces.
"""
import numpy as np
import pytest
import torch

import oracle
import lossless_entropy_coded_dfloat11_b200 as df11
from lossless_entropy_coded_dfloat11_b200 import _binding as B
from lossless_entropy_coded_dfloat11_b200 import inputs

pytestmark = pytest.mark.gpu

SMALL_BLOCK = dict(hidden=512, intermediate=1408, kv=128)
SENTINEL = 0x7FC1  # a NaN pattern no decode produces here


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().reshape(-1).view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_stream(T: int, seed: int):
    w = inputs.llama_block(SMALL_BLOCK, seed_base=seed)
    x = w.flat_u16()
    s = oracle.encode(x, threads_per_block=T)
    cs = df11.from_arrays(s.code_len, s.n_elems, s.total_bits, T, s.exp, s.sm, s.gaps, s.block_off,
                          seg_counts=[t.numel() for t in w.tensors])
    return x, s, cs


def cut_points(n_blocks: int, seed: int):
    rng = np.random.default_rng(seed)
    k = min(9, n_blocks)
    return sorted(set(rng.integers(0, n_blocks + 1, size=k).tolist()) | {0, n_blocks})


@pytest.mark.parametrize("T", [32, 64, 256])
def test_pieces_in_any_order_rebuild_the_stream(T):
    x, s, cs = oracle_stream(T, seed=80 + T)
    cuts = cut_points(s.n_blocks, seed=T)
    out = torch.full((s.n_elems,), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pieces = list(zip(cuts[:-1], cuts[1:]))
    for b0, b1 in reversed(pieces):  # order does not matter
        df11.decompress_blocks(cs, b0, b1, out, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    np.testing.assert_array_equal(u16(out), x)


@pytest.mark.parametrize("T", [32, 64, 256])
def test_a_piece_writes_only_its_own_elements(T):
    x, s, cs = oracle_stream(T, seed=90 + T)
    nb = s.n_blocks
    for b0, b1 in [(0, 1), (nb // 3, nb // 3 + 1), (nb // 4, (3 * nb) // 4), (nb - 1, nb), (5, 5)]:
        out = torch.full((s.n_elems,), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        df11.decompress_blocks(cs, b0, b1, out)
        torch.cuda.synchronize()
        got = u16(out)
        lo, hi = int(s.block_off[b0]), int(s.block_off[b1])
        np.testing.assert_array_equal(got[lo:hi], x[lo:hi])
        assert (got[:lo] == SENTINEL).all() and (got[hi:] == SENTINEL).all(), (b0, b1)


def fill_garbage_except(cs, r: dict):
    """Overwrite every byte of the stream's device arrays outside r."""
    for k in ("exp", "sm", "gaps", "block_off"):
        if k not in r:
            continue
        t = getattr(cs, k).view(torch.uint8)
        lo, hi = r[k]
        t[:lo] = 0xA5
        t[hi:] = 0x5A


@pytest.mark.parametrize("T", [32, 64, 256])
def test_a_piece_needs_only_the_bytes_piece_ranges_lists(T):
    x, s, _ = oracle_stream(T, seed=100 + T)
    hdr = df11.make_header(s.code_len, s.n_elems, s.total_bits, T)
    for b0, b1 in [(0, 2), (s.n_blocks // 2, s.n_blocks // 2 + 3), (s.n_blocks - 2, s.n_blocks)]:
        cs = df11.from_arrays(s.code_len, s.n_elems, s.total_bits, T, s.exp, s.sm, s.gaps, s.block_off)
        fill_garbage_except(cs, df11.piece_ranges(hdr, s.block_off, b0, b1))
        out = torch.full((s.n_elems,), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        df11.decompress_blocks(cs, b0, b1, out, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        lo, hi = int(s.block_off[b0]), int(s.block_off[b1])
        np.testing.assert_array_equal(u16(out)[lo:hi], x[lo:hi])


@pytest.mark.parametrize("T", [32, 64])
def test_8bit_symbol_pieces(T):
    w = inputs.llama_block_u8(SMALL_BLOCK, seed_base=110 + T)
    v = np.concatenate([t.reshape(-1).numpy() for t in w.tensors])
    s = oracle.encode(v.astype(np.uint16) << 7, threads_per_block=T)
    hdr = df11.make_header(s.code_len, s.n_elems, s.total_bits, T)
    cuts = cut_points(s.n_blocks, seed=T + 5)
    out = torch.full((s.n_elems,), 0xEE, dtype=torch.uint8, device="cuda")
    for b0, b1 in zip(cuts[:-1], cuts[1:]):
        cs = df11.from_arrays(s.code_len, s.n_elems, s.total_bits, T, s.exp, None, s.gaps, s.block_off,
                              symbols="u8")
        fill_garbage_except(cs, df11.piece_ranges(hdr, s.block_off, b0, b1, u8=True))
        df11.decompress_blocks(cs, b0, b1, out)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.cpu().numpy(), v)


def test_block_range_errors():
    _, s, cs = oracle_stream(64, seed=120)
    out = torch.empty(s.n_elems, dtype=torch.bfloat16, device="cuda")
    for b0, b1 in [(3, 2), (0, s.n_blocks + 1), (s.n_blocks + 1, s.n_blocks + 1)]:
        with pytest.raises(B.DF11Error) as e:
            df11.decompress_blocks(cs, b0, b1, out)
        assert e.value.code == B.DF11_ERR_INVALID
    df11.decompress_blocks(cs, s.n_blocks, s.n_blocks, out)  # empty: no-op


@pytest.mark.parametrize("pieces", [1, 2, 3, 17, None, 10 ** 6])
def test_host_stream_pipelined_is_exact(pieces):
    w = inputs.llama_block(SMALL_BLOCK, seed_base=130)
    cs = df11.compress([t.cuda() for t in w.tensors])
    hs = df11.HostStream(cs)
    hs.PIECE_OUT_BYTES = 256 << 10  # several pieces by default on this small block
    for _ in range(2):  # reuse of the buffers across runs
        res = hs.run(pieces=pieces)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(res.view(torch.int16).numpy().view(np.uint16), w.flat_u16())
    n_arrays = sum(v.numel() * v.element_size() for v in hs.host.values())
    assert n_arrays <= hs.h2d_bytes() <= n_arrays + 256 * min(pieces or 64, cs.header.n_blocks)


def test_host_stream_on_a_side_stream_and_8bit_symbols():
    w = inputs.llama_block_u8(SMALL_BLOCK, seed_base=140)
    cs = df11.compress_u8([t.cuda() for t in w.tensors])
    hs = df11.HostStream(cs)
    s = torch.cuda.Stream()
    res = hs.run(stream=s, pieces=5)
    s.synchronize()
    np.testing.assert_array_equal(res.numpy(), np.concatenate([t.reshape(-1).numpy() for t in w.tensors]))

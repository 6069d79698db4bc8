"""CPU checks of the piece contract behind df11_decompress_blocks: the byte
ranges `piece_ranges` lists for thread blocks [b0, b1) are all a decoder
needs.  The oracle's windowed decode of [b0, b1), run on copies of the arrays
whose every other byte is overwritten with garbage, must still return the
original elements off[b0] .. off[b1]; the ranges stay inside the arrays and
together cover them.  No kernel runs here.
"""
import numpy as np
import pytest

import oracle
import lossless_entropy_coded_dfloat11_b200 as df11
from lossless_entropy_coded_dfloat11_b200 import inputs

GARBAGE = 0xA5


def sample(n: int, seed: int) -> np.ndarray:
    w = inputs.matrix_outliers(rows=n // 512, cols=512, seed=seed)
    return w.flat_u16()


def header_of(s: oracle.Stream):
    return df11.make_header(s.code_len, s.n_elems, s.total_bits, s.threads_per_block)


def masked(s: oracle.Stream, r: dict) -> oracle.Stream:
    """Copies of the stream's arrays with every byte outside r replaced."""
    def keep(a: np.ndarray, lo: int, hi: int) -> np.ndarray:
        b = np.full(a.view(np.uint8).size, GARBAGE, dtype=np.uint8)
        b[lo:hi] = a.view(np.uint8)[lo:hi]
        return b.view(a.dtype)
    return oracle.Stream(code_len=s.code_len, n_elems=s.n_elems, total_bits=s.total_bits,
                         threads_per_block=s.threads_per_block, n_threads=s.n_threads, n_blocks=s.n_blocks,
                         exp=keep(s.exp, *r["exp"]), sm=keep(s.sm, *r["sm"]), gaps=keep(s.gaps, *r["gaps"]),
                         block_off=keep(s.block_off, *r["block_off"]))


def partitions(n_blocks: int, seed: int):
    rng = np.random.default_rng(seed)
    yield [0, n_blocks]
    yield list(range(0, n_blocks + 1))  # one block per piece
    cuts = sorted(set(rng.integers(0, n_blocks + 1, size=min(7, n_blocks)).tolist()) | {0, n_blocks})
    yield cuts


@pytest.mark.parametrize("T", [32, 64, 256])
def test_each_piece_decodes_from_its_ranges_alone(T):
    x = sample(96 * 512, seed=40 + T)
    s = oracle.encode(x, threads_per_block=T)
    hdr = header_of(s)
    assert int(hdr.n_blocks) == s.n_blocks
    for cuts in partitions(s.n_blocks, seed=T):
        for b0, b1 in zip(cuts[:-1], cuts[1:]):
            if b0 == b1:
                continue
            r = df11.piece_ranges(hdr, s.block_off, b0, b1)
            got = oracle.decode_windowed(masked(s, r), b0, b1)
            lo, hi = int(s.block_off[b0]), int(s.block_off[b1])
            np.testing.assert_array_equal(got, x[lo:hi])


@pytest.mark.parametrize("T", [32, 64, 1024])
def test_ranges_stay_inside_the_arrays_and_cover_them(T):
    x = sample(64 * 512, seed=7 + T)
    s = oracle.encode(x, threads_per_block=T)
    hdr = header_of(s)
    sizes = {"exp": int(hdr.bytes_exp), "sm": int(hdr.bytes_sm), "gaps": int(hdr.bytes_gaps),
             "block_off": 4 * (s.n_blocks + 1)}
    for cuts in partitions(s.n_blocks, seed=T + 1):
        covered = {k: np.zeros(v, bool) for k, v in sizes.items()}
        for b0, b1 in zip(cuts[:-1], cuts[1:]):
            r = df11.piece_ranges(hdr, s.block_off, b0, b1)
            assert set(r) == set(sizes)
            for k, (lo, hi) in r.items():
                assert 0 <= lo <= hi <= sizes[k], (k, lo, hi)
                covered[k][lo:hi] = True
            # every window, gap field and element of the piece is included
            assert r["exp"][0] == 8 * T * b0 and r["exp"][1] >= min(8 * T * b1 + 4, sizes["exp"])
            assert r["gaps"][0] * 8 <= 5 * T * b0 and r["gaps"][1] * 8 >= 5 * T * b1
            assert r["sm"][0] <= int(s.block_off[b0]) and r["sm"][1] >= int(s.block_off[b1])
            assert r["block_off"] == (4 * b0, 4 * (b1 + 1))
        # the pieces together hold every byte of the data the format defines
        assert covered["exp"][: (s.total_bits + 7) // 8].all()
        assert covered["sm"][: s.n_elems].all()
        assert covered["gaps"][: (5 * s.n_threads + 7) // 8].all()
        assert covered["block_off"].all()


def test_ranges_for_8bit_symbols_have_no_side_array():
    v = np.random.default_rng(3).integers(0, 40, size=20000).astype(np.uint16)
    s = oracle.encode(v << 7, threads_per_block=64)
    hdr = header_of(s)
    r = df11.piece_ranges(hdr, s.block_off, 0, s.n_blocks, u8=True)
    assert set(r) == {"exp", "gaps", "block_off"}
    assert r["exp"] == (0, int(hdr.bytes_exp))

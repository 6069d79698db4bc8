"""GPU parity: the CUDA library against the CPU oracle, bit for bit.

Both directions on the same seeded inputs:
  * oracle-encoded streams decoded by the library's kernel == the input;
  * library-encoded streams are byte-identical to the oracle's (same code
    lengths, codes, bit packing, Gaps and block offsets) and the oracle
    decodes them back to the input.
Sizes span many thread blocks and ragged tails; the full-size workloads run in
the launch configuration the benchmark times (the default T, one launch per
stream).
"""
import numpy as np
import pytest
import torch

import oracle
import lossless_entropy_coded_dfloat11_b200 as df11
from lossless_entropy_coded_dfloat11_b200 import _binding as B
from lossless_entropy_coded_dfloat11_b200 import inputs

pytestmark = pytest.mark.gpu


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().reshape(-1).view(torch.int16).cpu().numpy().view(np.uint16)


def to_device(w: inputs.Workload):
    return [t.cuda() for t in w.tensors]


def lib_stream_from_oracle(s: oracle.Stream, seg_counts=None) -> df11.CompressedStream:
    return df11.from_arrays(s.code_len, s.n_elems, s.total_bits, s.threads_per_block, s.exp, s.sm,
                            s.gaps, s.block_off, seg_counts=seg_counts)


def decode_on_gpu(cs: df11.CompressedStream) -> np.ndarray:
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = df11.decompress(cs, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return u16(out)


def assert_same_stream(cs: df11.CompressedStream, s: oracle.Stream):
    h = df11.to_host(cs)
    np.testing.assert_array_equal(h["code_len"], s.code_len)
    assert h["total_bits"] == s.total_bits and h["n_threads"] == s.n_threads and h["n_blocks"] == s.n_blocks
    np.testing.assert_array_equal(h["exp"], s.exp)
    np.testing.assert_array_equal(h["sm"], s.sm)
    np.testing.assert_array_equal(h["gaps"], s.gaps)
    np.testing.assert_array_equal(h["block_off"], s.block_off)


def both_directions(w: inputs.Workload, T=df11.DEFAULT_THREADS_PER_BLOCK, L=32):
    x = w.flat_u16()
    s = oracle.encode(x, threads_per_block=T, max_len=L)
    # oracle stream -> library kernel
    counts = [t.numel() for t in w.tensors]
    np.testing.assert_array_equal(decode_on_gpu(lib_stream_from_oracle(s, counts)), x)
    # library encoder -> identical bytes -> oracle decoder
    cs = df11.compress(to_device(w), threads_per_block=T, max_code_len=L)
    assert_same_stream(cs, s)
    lib = df11.to_host(cs)
    back = oracle.decode(oracle.Stream(code_len=lib["code_len"], n_elems=lib["n_elems"],
                                       total_bits=lib["total_bits"], threads_per_block=T,
                                       n_threads=lib["n_threads"], n_blocks=lib["n_blocks"],
                                       exp=lib["exp"], sm=lib["sm"], gaps=lib["gaps"],
                                       block_off=lib["block_off"]))
    np.testing.assert_array_equal(back, x)
    # library encoder -> library decoder
    np.testing.assert_array_equal(decode_on_gpu(cs), x)
    return cs, s


def test_matrix_1k():
    both_directions(inputs.matrix_1k())


@pytest.mark.parametrize("T", [32, 64, 128, 256, 512, 1024])
def test_threads_per_block_variants(T):
    both_directions(inputs.matrix_1k(), T=T)
    both_directions(inputs.edge_case(65537, "zipf", 515), T=T)


@pytest.mark.parametrize("dist", inputs.EDGE_DISTS)
@pytest.mark.parametrize("idx", range(len(inputs.EDGE_SIZES)))
def test_edge_sweep(idx, dist):
    n = inputs.EDGE_SIZES[idx]
    both_directions(inputs.edge_case(n, dist, 500 + idx))


@pytest.mark.parametrize("dist", inputs.EDGE_DISTS)
@pytest.mark.parametrize("n", [1, 33, 127, 4097, 65537, (1 << 20) + 7, (1 << 24) + 3])
def test_edge_cases_four_windows_per_lane(n, dist):
    both_directions(inputs.edge_case(n, dist, 950 + n % 97), T=128)


def test_llama8b_block_four_windows_per_lane():
    w = inputs.llama_block(inputs.LLAMA_8B, seed_base=3)
    x = w.flat_u16()
    cs = df11.compress(to_device(w), threads_per_block=128)
    assert cs.kernel_info()["kernel"].startswith("decode_warp_kernel")
    np.testing.assert_array_equal(decode_on_gpu(cs), x)
    s = oracle.encode(x, threads_per_block=128)
    assert_same_stream(cs, s)


@pytest.mark.parametrize("dist", inputs.EDGE_DISTS)
@pytest.mark.parametrize("n", [1, 33, 127, 4097, 65537, (1 << 20) + 7])
def test_edge_cases_one_window_per_lane(n, dist):
    # the sweep above runs the default T = 64 (two windows per lane when every
    # code has 2 bits or more, the block kernel when a code is 1 bit long);
    # T = 32 streams take the one-window warp kernel, whose 1-bit-code variant
    # the 99.9%-one-exponent distribution reaches
    both_directions(inputs.edge_case(n, dist, 900 + n % 97), T=32)


def test_all_bf16_patterns():
    both_directions(inputs.all_patterns())


def test_fibonacci_counts_bind_the_32_bit_limit():
    cs, s = both_directions(inputs.fibonacci())
    assert int(s.code_len.max()) == 32


def test_matrix_outliers_full_size():
    cs, s = both_directions(inputs.matrix_outliers())
    assert 20 <= int(s.code_len.max()) <= 32        # long codes (level-2 path)
    assert s.code_len[0] > 0                        # zero exponent present


@pytest.mark.parametrize("L", [9, 12, 16])
def test_length_limit_variants(L):
    # the limit binds: the unrestricted code is longer than L
    both_directions(inputs.matrix_outliers(1024, 2048, seed=21), L=L)


def test_ragged_segments():
    """Segments whose sizes are not multiples of 16 (misaligned concatenation
    offsets in the encoder)."""
    g = torch.Generator().manual_seed(31)
    sizes = [1, 17, 4099, 33, 1000003, 5, 257]
    ts = [(torch.randn(n, generator=g) * 0.02).to(torch.bfloat16) for n in sizes]
    w = inputs.Workload("ragged", [f"s{k}" for k in range(len(ts))], ts)
    cs, _ = both_directions(w)
    out = df11.decompress(cs)
    for v, t in zip(cs.views(out), ts):
        assert torch.equal(v.cpu().view(torch.int16), t.view(torch.int16))


def test_llama8b_block_single_launch():
    """One Llama-3.1-8B-shaped block, one shared table, one launch."""
    w = inputs.llama_block()
    assert w.n_elems == 218_112_000
    cs, s = both_directions(w)
    out = df11.decompress(cs)
    torch.cuda.synchronize()
    for name, v, t in zip(w.names, cs.views(out), w.tensors):
        assert v.shape == t.shape
        assert torch.equal(v.cpu().view(torch.int16), t.view(torch.int16)), name
    ratio = cs.compressed_bytes() / (2 * cs.n_elems)
    assert 0.65 <= ratio <= 0.72


def test_llama70b_block_reused_buffer():
    """A 70B-shaped block (855,654,400 elements): library round trip, the
    oracle's table and sampled thread blocks decoded by the oracle from the
    library's stream; then a second block decoded into the same buffer."""
    w = inputs.llama70b_block(0)
    assert w.n_elems == 855_654_400
    x = w.flat_u16()
    cs = df11.compress(to_device(w))
    hist = oracle.histogram(x)
    np.testing.assert_array_equal(cs.code_len, oracle.code_lengths(hist))
    buf = torch.empty(cs.n_elems, dtype=torch.bfloat16, device="cuda")
    out = df11.decompress(cs, out=buf)
    torch.cuda.synchronize()
    assert np.array_equal(u16(out), x)
    lib = df11.to_host(cs)
    ls = oracle.Stream(code_len=lib["code_len"], n_elems=lib["n_elems"], total_bits=lib["total_bits"],
                       threads_per_block=cs.threads_per_block, n_threads=lib["n_threads"], n_blocks=lib["n_blocks"],
                       exp=lib["exp"], sm=lib["sm"], gaps=lib["gaps"], block_off=lib["block_off"])
    rng = np.random.default_rng(70)
    for b in list(rng.integers(0, ls.n_blocks, size=48)) + [0, ls.n_blocks - 1]:
        b = int(b)
        lo, hi = int(ls.block_off[b]), int(ls.block_off[b + 1])
        np.testing.assert_array_equal(oracle.decode_windowed(ls, b, b + 1), x[lo:hi])
    del cs
    w2 = inputs.llama70b_block(1, device="cuda")
    cs2 = df11.compress(w2.tensors)
    out2 = df11.decompress(cs2, out=buf)
    torch.cuda.synchronize()
    for v, t in zip(cs2.views(out2), w2.tensors):
        assert torch.equal(v.view(torch.int16), t.view(torch.int16))


# --------------------------------------------------------------------------- #
# Degenerate inputs and failure reporting                                     #
# --------------------------------------------------------------------------- #
def test_empty_and_single_element():
    cs = df11.from_arrays(np.zeros(256, np.uint8), 0, 0, 256, np.zeros(16, np.uint8),
                          np.zeros(0, np.uint8), np.zeros(16, np.uint8), np.zeros(1, np.uint32))
    out = df11.decompress(cs)
    torch.cuda.synchronize()
    assert out.numel() == 0
    both_directions(inputs.edge_case(1, "uniform", 500))
    x = np.full(100_000, 0x3F80, dtype=np.uint16)          # one exponent value
    w = inputs.Workload("const", ["x"], [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)])
    both_directions(w)


@pytest.mark.parametrize("T", [64, 128])
def test_corrupt_block_offsets_are_reported_not_trapped(T):
    x = inputs.matrix_1k().flat_u16()
    s = oracle.encode(x, threads_per_block=T)
    guard = 4096
    for b, delta in ((5, 1), (100, -3), (s.n_blocks, 1000)):
        off = s.block_off.copy()
        off[b] = np.uint32(int(off[b]) + delta)
        cs = df11.from_arrays(s.code_len, s.n_elems, s.total_bits, T, s.exp, s.sm, s.gaps, off)
        buf = torch.full((s.n_elems + guard,), 7.0, dtype=torch.bfloat16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        df11.decompress(cs, out=buf[: s.n_elems], status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == B.DF11_ERR_CORRUPT
        assert bool((buf[s.n_elems:] == 7.0).all())       # nothing written past the output


@pytest.mark.parametrize("T", [64, 128])
def test_corrupt_gaps_and_bits_terminate(T):
    x = inputs.matrix_outliers(512, 512, seed=5).flat_u16()
    s = oracle.encode(x, threads_per_block=T)
    gaps = s.gaps.copy()
    gaps[40] ^= 0x1F
    cs = df11.from_arrays(s.code_len, s.n_elems, s.total_bits, T, s.exp, s.sm, gaps, s.block_off)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.decompress(cs, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == B.DF11_ERR_CORRUPT
    rng = np.random.default_rng(9)
    for _ in range(8):                      # random bit flips: must end, flag or not
        exp = s.exp.copy()
        idx = rng.integers(0, (s.total_bits + 7) // 8, size=16)
        exp[idx] ^= rng.integers(1, 256, size=16).astype(np.uint8)
        cs = df11.from_arrays(s.code_len, s.n_elems, s.total_bits, T, exp, s.sm, s.gaps, s.block_off)
        status.zero_()
        out = df11.decompress(cs, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) in (0, B.DF11_ERR_CORRUPT)
        assert out.numel() == s.n_elems


@pytest.mark.parametrize("T", [32, 64, 256])
def test_tables_without_the_magic_word_are_reported(T):
    """Decode tables whose magic word is not the library's (a table buffer
    never filled, or the tables of an encode that gave up waiting): every
    decode kernel reports the stream corrupt and writes nothing."""
    x = inputs.matrix_1k().flat_u16()
    s = oracle.encode(x, threads_per_block=T)
    cs = lib_stream_from_oracle(s)
    cs.lut[:4] = 0
    buf = torch.full((s.n_elems,), 7.0, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.decompress(cs, out=buf, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == B.DF11_ERR_CORRUPT
    assert bool((buf == 7.0).all())


def test_host_side_argument_checks():
    s = oracle.encode(inputs.matrix_1k().flat_u16(), threads_per_block=df11.DEFAULT_THREADS_PER_BLOCK)
    cs = lib_stream_from_oracle(s)
    out = torch.empty(s.n_elems + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(df11.DF11Error) as e:
        df11.decompress(cs, out=out[1:1 + s.n_elems])          # misaligned output
    assert e.value.code == B.DF11_ERR_INVALID
    cs.header.n_blocks += 1                                     # inconsistent header
    with pytest.raises(df11.DF11Error):
        df11.decompress(cs)
    cs.header.n_blocks -= 1
    with pytest.raises(TypeError):
        df11.compress([torch.zeros(16, dtype=torch.float16, device="cuda")])


def test_decompress_on_a_side_stream():
    w = inputs.matrix_1k()
    cs = df11.compress(to_device(w))
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        out = df11.decompress(cs, stream=side)
    side.synchronize()
    assert np.array_equal(u16(out), w.flat_u16())


def test_end_to_end_host_buffers():
    w = inputs.matrix_1k()
    hs = df11.HostStream(df11.compress(to_device(w)))
    res = hs.run()
    torch.cuda.synchronize()
    assert np.array_equal(res.view(torch.int16).numpy().view(np.uint16), w.flat_u16())
    assert hs.d2h_bytes() == 2 * w.n_elems

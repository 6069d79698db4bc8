"""GPU parity for the independent-chunk variant of the container (the
ablation of the Gaps-and-block-offsets design): the same code stream and
PackedSignMantissa as a DF11 stream, plus the start bit of every 64 elements.

Both directions against the CPU oracle: library-encoded arrays and chunk
table equal the oracle's stream and `oracle.chunk_starts`; the library's
chunk decoder rebuilds the input from the oracle's arrays and from its own.
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


def decode(cs) -> np.ndarray:
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = df11.decompress_chunked(cs, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return u16(out)


def both_directions(w: inputs.Workload):
    x = w.flat_u16()
    counts = [t.numel() for t in w.tensors]
    s = oracle.encode(x)
    starts = oracle.chunk_starts(x, s.code_len, df11.IND_CHUNK)
    # oracle arrays -> library chunk decoder
    ocs = df11.chunked_from_arrays(s.code_len, s.n_elems, s.total_bits, s.exp, s.sm, starts, seg_counts=counts)
    np.testing.assert_array_equal(decode(ocs), x)
    # library encoder == oracle arrays and chunk table
    cs = df11.compress_chunked([t.cuda() for t in w.tensors])
    np.testing.assert_array_equal(np.frombuffer(bytes(cs.header.code_len), np.uint8), s.code_len)
    assert int(cs.header.total_bits) == s.total_bits
    nb = (s.total_bits + 7) // 8  # the code bytes (the padding after them depends on T)
    np.testing.assert_array_equal(cs.exp.cpu().numpy()[:nb], s.exp[:nb])
    np.testing.assert_array_equal(cs.sm.cpu().numpy()[: x.size], s.sm[: x.size])
    np.testing.assert_array_equal(cs.chunk_bit.cpu().numpy().view(np.uint32)[: starts.size], starts)
    # library encoder -> library decoder
    np.testing.assert_array_equal(decode(cs), x)
    return cs


def test_matrix_1k():
    cs = both_directions(inputs.matrix_1k())
    assert cs.compressed_bytes() / (2 * cs.n_elems) < 0.70


@pytest.mark.parametrize("dist", inputs.EDGE_DISTS)
@pytest.mark.parametrize("n", [1, 2, 63, 64, 65, 127, 4097, 65537, (1 << 20) + 7])
def test_edge_cases(n, dist):
    both_directions(inputs.edge_case(n, dist, 700 + n % 83))


def test_fibonacci_32_bit_codes():
    both_directions(inputs.fibonacci())


def test_ragged_segments():
    parts = [inputs.gaussian((k,), 0.02, 50 + k) for k in (1, 65, 4096, 7, 70003, 2)]
    both_directions(inputs.Workload("ragged", [f"s{k}" for k in range(len(parts))], parts))


def test_matrix_outliers():
    both_directions(inputs.matrix_outliers())


def test_llama8b_block():
    w = inputs.llama_block(inputs.LLAMA_8B, seed_base=3)
    x = w.flat_u16()
    cs = df11.compress_chunked([t.cuda() for t in w.tensors], names=w.names)
    np.testing.assert_array_equal(decode(cs), x)
    code_len = oracle.code_lengths(oracle.histogram(x))
    np.testing.assert_array_equal(np.frombuffer(bytes(cs.header.code_len), np.uint8), code_len)
    want = oracle.chunk_starts(x, code_len, df11.IND_CHUNK)
    np.testing.assert_array_equal(cs.chunk_bit.cpu().numpy().view(np.uint32)[: want.size], want)
    assert int(want[-1]) == int(cs.header.total_bits)


def test_corrupt_chunk_table_is_reported_not_trapped():
    w = inputs.matrix_1k()
    cs = df11.compress_chunked([t.cuda() for t in w.tensors])
    for k, delta in ((5, 3), (100, -7), (7000, 1 << 20)):
        bad = df11.ChunkedStream(cs.header, cs.exp, cs.sm, cs.chunk_bit.clone(), cs.lut, cs.names, cs.shapes)
        bad.chunk_bit[k] += delta
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        df11.decompress_chunked(bad, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) & B.DF11_ERR_CORRUPT, (k, delta)

"""GPU parity for streams of 8-bit symbols coded whole (EntroLLM-style
Huffman coding of quantized integer weights on this library's container).

The oracle needs no new arithmetic: a byte v is the exponent field of the
BF16 pattern v << 7 (sign and mantissa zero), so the oracle's stream for those
patterns has exactly the u8 stream's code bits, Gaps, block offsets and code
table, and its decode gives v back in the exponent field.  Both directions:
oracle stream -> library u8 decoder, and library u8 encoder -> identical
bytes -> oracle decoder.
"""
import numpy as np
import pytest
import torch

import oracle
import lossless_entropy_coded_dfloat11_b200 as df11
from lossless_entropy_coded_dfloat11_b200 import _binding as B
from lossless_entropy_coded_dfloat11_b200 import inputs

pytestmark = pytest.mark.gpu


def flat_u8(w: inputs.Workload) -> np.ndarray:
    parts = [t.reshape(-1).cpu().numpy() for t in w.tensors]
    return np.concatenate(parts) if parts else np.zeros(0, np.uint8)


def oracle_stream(v: np.ndarray, T: int) -> oracle.Stream:
    return oracle.encode(v.astype(np.uint16) << 7, threads_per_block=T)


def decode_u8(cs) -> np.ndarray:
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = df11.decompress_u8(cs, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out.cpu().numpy()


def both_directions(w: inputs.Workload, T: int = df11.DEFAULT_THREADS_PER_BLOCK):
    v = flat_u8(w)
    counts = [t.numel() for t in w.tensors]
    # library encoder (T = 128 falls back to 32 when a code is 1 bit long)
    cs = df11.compress_u8([t.cuda() for t in w.tensors], threads_per_block=T)
    s = oracle_stream(v, cs.threads_per_block)
    # oracle stream -> library u8 kernel
    ocs = df11.from_arrays(s.code_len, s.n_elems, s.total_bits, s.threads_per_block, s.exp, None, s.gaps,
                           s.block_off, seg_counts=counts, symbols="u8")
    np.testing.assert_array_equal(decode_u8(ocs), v)
    # library stream == oracle stream, byte for byte
    h = df11.to_host(cs)
    np.testing.assert_array_equal(h["code_len"], s.code_len)
    assert h["total_bits"] == s.total_bits and h["n_blocks"] == s.n_blocks
    np.testing.assert_array_equal(h["exp"], s.exp)
    np.testing.assert_array_equal(h["gaps"], s.gaps)
    np.testing.assert_array_equal(h["block_off"], s.block_off)
    back = oracle.decode(oracle.Stream(code_len=h["code_len"], n_elems=h["n_elems"], total_bits=h["total_bits"],
                                       threads_per_block=h["threads_per_block"], n_threads=h["n_threads"],
                                       n_blocks=h["n_blocks"], exp=h["exp"],
                                       sm=np.zeros(max(s.sm.size, 16), np.uint8), gaps=h["gaps"],
                                       block_off=h["block_off"]))
    np.testing.assert_array_equal((back >> 7).astype(np.uint8), v)
    # library encoder -> library decoder
    np.testing.assert_array_equal(decode_u8(cs), v)
    return cs


@pytest.mark.parametrize("T", [32, 64, 128])
def test_quantized_matrix(T):
    w = inputs.Workload("q", ["w"], [inputs.quantize_u8(inputs.gaussian((1024, 1024), 0.02, 1))])
    cs = both_directions(w, T)
    # ~6.74 code bits per symbol (entropy 6.71) plus a 5-bit gap per 64-bit
    # window: ~7.3 bits, i.e. ~0.92 of the uint8 size
    assert 0.88 < cs.compressed_bytes() / cs.n_elems < 0.95


@pytest.mark.parametrize("T", [32, 64, 128])
def test_uint4_values_one_per_byte(T):
    """uint4 weights (the other alphabet the EntroLLM page codes), one value
    per byte: a 16-symbol alphabet on the same streams and kernels."""
    w = inputs.Workload("q4", ["w"], [inputs.quantize_u4(inputs.gaussian((1024, 1024), 0.02, 1))])
    cs = both_directions(w, T)
    # ~2.69 code bits per value (entropy 2.65) plus a 5-bit gap per 64-bit
    # window: ~0.365 bytes per value
    assert 0.34 < cs.compressed_bytes() / cs.n_elems < 0.40


def test_uint4_block():
    both_directions(inputs.llama_block_u4(dict(hidden=512, intermediate=1408, kv=128), seed_base=150))


@pytest.mark.parametrize("dist", inputs.EDGE_DISTS)
@pytest.mark.parametrize("n", [1, 2, 31, 33, 255, 4097, 65537, (1 << 20) + 7])
def test_edge_cases(n, dist):
    both_directions(inputs.edge_case_u8(n, dist, 600 + n % 89))


@pytest.mark.parametrize("dist", inputs.EDGE_DISTS)
@pytest.mark.parametrize("n", [1, 33, 4097, 65537, (1 << 20) + 7])
def test_edge_cases_four_windows_per_lane(n, dist):
    both_directions(inputs.edge_case_u8(n, dist, 700 + n % 89), T=128)


def test_llama8b_block_quantized_four_windows_per_lane():
    w = inputs.llama_block_u8(inputs.LLAMA_8B, seed_base=3)
    v = flat_u8(w)
    cs = df11.compress_u8([t.cuda() for t in w.tensors], names=w.names, threads_per_block=128)
    assert cs.threads_per_block == 128
    np.testing.assert_array_equal(decode_u8(cs), v)


def test_ragged_segments():
    parts = [inputs.quantize_u8(inputs.gaussian((k,), 0.02, 40 + k)) for k in (1, 17, 4096, 5, 70001, 3)]
    both_directions(inputs.Workload("ragged", [f"s{k}" for k in range(len(parts))], parts))


def test_llama8b_block_quantized_one_launch():
    w = inputs.llama_block_u8(inputs.LLAMA_8B, seed_base=3)
    v = flat_u8(w)
    cs = df11.compress_u8([t.cuda() for t in w.tensors], names=w.names)
    np.testing.assert_array_equal(decode_u8(cs), v)
    # the views give back each quantized matrix
    out = df11.decompress_u8(cs)
    for ref, got in zip(w.tensors, cs.views(out)):
        assert torch.equal(got.cpu(), ref)


def test_one_bit_code_decodes_at_t64_and_is_refused_at_t128():
    """A 1-bit code puts up to 128 codes in a lane's two windows (T = 64: the
    kernel instance with buffers for them) and 256 in four (T = 128: no
    8-bit-symbol decoder, an argument error)."""
    v = flat_u8(inputs.edge_case_u8(5000, "one_value", 3))
    s = oracle_stream(v, 64)
    assert s.code_len[s.code_len > 0].min() == 1
    cs = df11.from_arrays(s.code_len, s.n_elems, s.total_bits, 64, s.exp, None, s.gaps, s.block_off,
                          symbols="u8")
    np.testing.assert_array_equal(decode_u8(cs), v)
    s = oracle_stream(v, 128)
    cs = df11.from_arrays(s.code_len, s.n_elems, s.total_bits, 128, s.exp, None, s.gaps, s.block_off,
                          symbols="u8")
    with pytest.raises(B.DF11Error) as e:
        df11.decompress_u8(cs)
    assert e.value.code == B.DF11_ERR_INVALID

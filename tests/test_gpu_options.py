"""GPU: df11_decompress_opts -- the first-level table width and the launch
shape -- against the CPU oracle, bit for bit.

The pages' first level is a 256-entry table per 8 code bits ("Decodificacao
com LUT hierarquica"); the library's default is a 12-bit multi-symbol table.
peek_bits = 8, 9, 10 decode with a narrow table kept in 16 copies in shared
memory; every width must give the same output.  Launch shapes (CTA count,
warps per CTA, SM cap) only move work between warps and must not change a
bit either.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import lossless_entropy_coded_dfloat11_b200 as df11
from lossless_entropy_coded_dfloat11_b200 import _binding as B
from lossless_entropy_coded_dfloat11_b200 import inputs

pytestmark = pytest.mark.gpu

SMALL_BLOCK = dict(hidden=512, intermediate=1408, kv=128)


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().reshape(-1).view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_stream_on_gpu(w: inputs.Workload, T=64):
    x = w.flat_u16()
    s = oracle.encode(x, threads_per_block=T)
    cs = df11.from_arrays(s.code_len, s.n_elems, s.total_bits, T, s.exp, s.sm, s.gaps, s.block_off,
                          seg_counts=[t.numel() for t in w.tensors])
    return x, cs


def decode_with(cs, opts) -> np.ndarray:
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = df11.decompress(cs, status=status, options=opts)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return u16(out)


WORKLOADS = {
    "block": lambda: inputs.llama_block(SMALL_BLOCK, seed_base=90),
    "outliers": lambda: inputs.matrix_outliers(2048, 1024, seed=91),      # codes up to ~26 bits
    "zipf": lambda: inputs.edge_case(65537, "zipf", 92),
    "uniform": lambda: inputs.edge_case((1 << 20) + 7, "uniform", 93),
    "fibonacci": lambda: inputs.fibonacci(),                               # a 32-bit code
    "patterns": lambda: inputs.all_patterns(),
}


@pytest.mark.parametrize("peek_bits", [8, 9, 10, 12])
@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_narrow_first_level_tables_are_exact(name, peek_bits):
    x, cs = oracle_stream_on_gpu(WORKLOADS[name]())
    np.testing.assert_array_equal(decode_with(cs, df11.decode_options(peek_bits=peek_bits)), x)
    info = cs.kernel_info(options=df11.decode_options(peek_bits=peek_bits))
    assert info["peek_bits"] == peek_bits
    assert info["table_copies"] == (1 if peek_bits == 12 else 16)


@pytest.mark.parametrize("peek_bits", [8, 10])
def test_narrow_tables_full_llama8b_block(peek_bits):
    w = inputs.llama_block(inputs.LLAMA_8B, seed_base=3)
    cs = df11.compress([t.cuda() for t in w.tensors])
    out = df11.decompress(cs, options=df11.decode_options(peek_bits=peek_bits))
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16).cpu(), torch.cat([t.reshape(-1) for t in w.tensors]).view(torch.int16))


@pytest.mark.parametrize("shape", [dict(ctas=1), dict(ctas=1, max_warps_per_cta=1), dict(ctas=7, max_warps_per_cta=3),
                                   dict(ctas=2000, max_warps_per_cta=4), dict(max_sms=5), dict(max_warps_per_cta=2)])
@pytest.mark.parametrize("T", [32, 64, 128, 256])
def test_launch_shapes_are_exact(T, shape):
    x, cs = oracle_stream_on_gpu(inputs.llama_block(SMALL_BLOCK, seed_base=94), T=T)
    np.testing.assert_array_equal(decode_with(cs, df11.decode_options(**shape)), x)
    info = cs.kernel_info(options=df11.decode_options(**shape))
    if "ctas" in shape:
        assert info["grid"] <= shape["ctas"]
    if "max_warps_per_cta" in shape and info["kernel"].startswith("decode_warp"):
        assert info["block"] <= 32 * shape["max_warps_per_cta"]


def test_many_small_ctas_on_a_full_size_block():
    w = inputs.llama_block(inputs.LLAMA_8B, seed_base=3)
    cs = df11.compress([t.cuda() for t in w.tensors])
    opts = df11.decode_options(ctas=4 * 148 * 4, max_warps_per_cta=4)
    out = df11.decompress(cs, options=opts)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16).cpu(), torch.cat([t.reshape(-1) for t in w.tensors]).view(torch.int16))
    assert cs.kernel_info(options=opts)["grid"] == 4 * 148 * 4


@pytest.mark.parametrize("T", [32, 64, 256])
def test_block_ranges_write_only_their_elements(T):
    """A block range in the options decodes exactly as df11_decompress_blocks:
    output elements [off[b0], off[b1]) and nothing else; ranges that tile the
    stream rebuild it, on any launch shape."""
    x, cs = oracle_stream_on_gpu(inputs.llama_block(SMALL_BLOCK, seed_base=97), T=T)
    nb = int(cs.header.n_blocks)
    off = cs.block_off.cpu().numpy().view(np.uint32)
    cuts = [0, 1, nb // 3, nb // 3 + 1, nb - 1, nb]
    out = torch.full((cs.n_elems,), 3.0, dtype=torch.bfloat16, device="cuda")
    for b0, b1 in zip(cuts[:-1], cuts[1:]):
        before = u16(out)
        opts = df11.decode_options(block_begin=b0, block_end=b1, max_sms=7 if b0 % 2 else 0)
        df11.decompress(cs, out=out, options=opts)
        torch.cuda.synchronize()
        after = u16(out)
        e0, e1 = int(off[b0]), int(off[b1])
        np.testing.assert_array_equal(after[e0:e1], x[e0:e1])
        np.testing.assert_array_equal(np.delete(after, np.s_[e0:e1]), np.delete(before, np.s_[e0:e1]))
    np.testing.assert_array_equal(u16(out), x)
    with pytest.raises(df11.DF11Error):
        df11.decompress(cs, out=out, options=df11.decode_options(block_begin=2, block_end=1))


def test_u8_streams_take_launch_shapes():
    w = inputs.Workload("q", ["w"], [inputs.quantize_u8(inputs.gaussian((1024, 1024), 0.02, 95))])
    cs = df11.compress_u8([t.cuda() for t in w.tensors])
    ref = w.tensors[0].reshape(-1)
    out = df11.decompress_u8(cs, options=df11.decode_options(ctas=50, max_warps_per_cta=2))
    torch.cuda.synchronize()
    assert torch.equal(out.cpu(), ref)


def test_bad_options_are_rejected_on_the_host():
    x, cs = oracle_stream_on_gpu(inputs.matrix_1k())
    for opts in (df11.decode_options(peek_bits=7), df11.decode_options(peek_bits=11),
                 df11.decode_options(peek_bits=13)):
        with pytest.raises(df11.DF11Error) as e:
            df11.decompress(cs, options=opts)
        assert e.value.code == B.DF11_ERR_INVALID
    bad = df11.decode_options()
    bad.reserved = 1
    with pytest.raises(df11.DF11Error):
        df11.decompress(cs, options=bad)
    bad = df11.decode_options()
    bad.early_staging = 2
    with pytest.raises(df11.DF11Error):
        df11.decompress(cs, options=bad)
    # narrow tables: BF16 streams with T = 64 only
    _, cs32 = oracle_stream_on_gpu(inputs.matrix_1k(), T=32)
    with pytest.raises(df11.DF11Error):
        df11.decompress(cs32, options=df11.decode_options(peek_bits=10))
    q = df11.compress_u8([inputs.quantize_u8(inputs.gaussian((256, 256), 0.02, 96)).cuda()])
    with pytest.raises(df11.DF11Error):
        df11.decompress_u8(q, options=df11.decode_options(peek_bits=10))


def test_early_staging_back_to_back():
    """Consecutive decodes with early staging (each stages its tables and
    first loads while the previous one finishes): bit-exact, through one
    reused output buffer and through alternating streams' buffers."""
    w1 = inputs.llama_block(dict(hidden=512, intermediate=1408, kv=128), seed_base=131)
    w2 = inputs.llama_block(dict(hidden=512, intermediate=1408, kv=128), seed_base=137)
    c1 = df11.compress([t.cuda() for t in w1.tensors])
    c2 = df11.compress([t.cuda() for t in w2.tensors])
    opts = df11.decode_options(early_staging=True)
    out = torch.empty(max(c1.n_elems, c2.n_elems), dtype=torch.bfloat16, device="cuda")
    r1 = torch.cat([t.reshape(-1) for t in w1.tensors]).view(torch.int16)
    r2 = torch.cat([t.reshape(-1) for t in w2.tensors]).view(torch.int16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for k in range(6):
        cs, ref = (c1, r1) if k % 2 == 0 else (c2, r2)
        got = df11.decompress(cs, out=out[: cs.n_elems], status=status, options=opts)
        if k >= 4:  # the last two: check each after its own launch
            torch.cuda.synchronize()
            assert torch.equal(got.view(torch.int16).cpu(), ref)
    assert int(status.item()) == 0
    q = df11.compress_u8([inputs.quantize_u8(inputs.gaussian((512, 384), 0.02, 138)).cuda()])
    ref8 = inputs.quantize_u8(inputs.gaussian((512, 384), 0.02, 138)).reshape(-1)
    for _ in range(3):
        got8 = df11.decompress_u8(q, options=opts)
    torch.cuda.synchronize()
    assert torch.equal(got8.cpu(), ref8)

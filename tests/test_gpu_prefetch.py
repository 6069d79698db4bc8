"""GPU: decompress on a capped number of SMs, and blocks decompressed ahead
of their use on a side stream (BlockPrefetcher), against the CPU oracle.

Every result is compared bit for bit with the original weights, which the
oracle round trip also reproduces; the prefetcher test runs a matrix
multiplication on each block while the next one decodes, so the two streams
really overlap.
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


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().reshape(-1).view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("T", [32, 256])
@pytest.mark.parametrize("max_sms", [1, 3, 17, 148, 100000])
def test_decompress_on_capped_sms(T, max_sms):
    w = inputs.llama_block(SMALL_BLOCK, seed_base=70)
    x = w.flat_u16()
    s = oracle.encode(x, threads_per_block=T)
    cs = df11.from_arrays(s.code_len, s.n_elems, s.total_bits, T, s.exp, s.sm, s.gaps, s.block_off,
                          seg_counts=[t.numel() for t in w.tensors])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = df11.decompress(cs, status=status, max_sms=max_sms)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    np.testing.assert_array_equal(u16(out), x)


def test_zero_sm_cap_is_rejected():
    w = inputs.matrix_1k()
    cs = df11.compress([t.cuda() for t in w.tensors])
    with pytest.raises(B.DF11Error) as e:
        df11.decompress(cs, max_sms=0)
    assert e.value.code == B.DF11_ERR_INVALID


@pytest.mark.parametrize("n_buffers,max_sms,split", [(2, None, None), (2, 8, None), (3, 31, None),
                                                    (2, None, 0.0), (2, None, 0.35), (3, None, 1.0)])
def test_block_prefetcher_overlaps_and_is_exact(n_buffers, max_sms, split):
    blocks = [inputs.llama_block(SMALL_BLOCK, seed_base=200 + 16 * b) for b in range(5)]
    streams = [df11.compress([t.cuda() for t in w.tensors], names=w.names) for w in blocks]
    # the oracle agrees with every input (the reference the GPU results are held to)
    for w in blocks[:2]:
        x = w.flat_u16()
        np.testing.assert_array_equal(oracle.decode(oracle.encode(x, threads_per_block=32)), x)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    act = torch.randn(64, SMALL_BLOCK["intermediate"], device="cuda").to(torch.bfloat16)
    copies, sums = [], []
    pf = df11.BlockPrefetcher(streams, n_buffers=n_buffers, max_sms=max_sms, status=status, split=split,
                              side_sms=5)
    for i, views in pf:
        acc = torch.zeros((), dtype=torch.float32, device="cuda")
        for v in views:
            if v.dim() == 2:  # the consumer: activations times the weight matrix
                acc += (act[:, : v.shape[1]] @ v.t()).float().sum()
        sums.append(acc)
        copies.append([v.clone() for v in views])
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert len(copies) == len(blocks)
    for w, got, acc in zip(blocks, copies, sums):
        for ref, v in zip(w.tensors, got):
            np.testing.assert_array_equal(u16(v), u16(ref))
        assert torch.isfinite(acc)


def test_block_prefetcher_matches_direct_decode_sums():
    """The same consumer computation gives the same result with and without
    the prefetcher (same kernels, same inputs, same order)."""
    blocks = [inputs.llama_block(SMALL_BLOCK, seed_base=300 + 16 * b) for b in range(3)]
    streams = [df11.compress([t.cuda() for t in w.tensors]) for w in blocks]
    act = torch.randn(32, SMALL_BLOCK["hidden"], device="cuda").to(torch.bfloat16)

    def consume(views):
        return [act @ v.t() for v in views if v.dim() == 2 and v.shape[1] == SMALL_BLOCK["hidden"]]

    direct = [consume(cs.views(df11.decompress(cs))) for cs in streams]
    pre = [[y.clone() for y in consume(views)] for _, views in df11.BlockPrefetcher(streams)]
    torch.cuda.synchronize()
    for a, b in zip(direct, pre):
        for ya, yb in zip(a, b):
            assert torch.equal(ya, yb)

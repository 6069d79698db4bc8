"""CPU checks of the uint4 workload (per-tensor 4-bit quantisation, one value
per byte) against the oracle: the values fill the 16-symbol alphabet, the
oracle's stream round-trips them, and its code meets the Shannon bounds the
pages' entropy argument rests on (H <= mean code length < H + 1)."""
import numpy as np
import torch

import oracle
from lossless_entropy_coded_dfloat11_b200 import inputs


def test_quantize_u4_range_and_rounding():
    t = torch.tensor([-1.0, -0.5, 0.1, 0.49, 1.0])
    q = inputs.quantize_u4(t)
    assert q.dtype == torch.uint8
    # [min, max] = [-1, 1] onto 0..15: (x + 1) * 7.5 = 0, 3.75, 8.25, 11.175, 15
    assert q.tolist() == [0, 4, 8, 11, 15]
    assert inputs.quantize_u4(torch.zeros(7)).tolist() == [0] * 7


def test_uint4_block_round_trips_through_the_oracle():
    w = inputs.llama_block_u4(dict(hidden=512, intermediate=1408, kv=128), seed_base=150)
    v = np.concatenate([t.reshape(-1).numpy() for t in w.tensors])
    assert v.max() == 15 and v.min() == 0
    for T in (32, 64):
        s = oracle.encode(v.astype(np.uint16) << 7, threads_per_block=T)
        np.testing.assert_array_equal((oracle.decode(s) >> 7).astype(np.uint8), v)
        np.testing.assert_array_equal((oracle.decode_windowed(s) >> 7).astype(np.uint8), v)
    hist = np.bincount(v, minlength=256)
    assert np.count_nonzero(hist) == 16
    p = hist[hist > 0] / v.size
    H = float(-(p * np.log2(p)).sum())
    mean = s.total_bits / v.size
    assert H <= mean < H + 1
    assert 2.5 < H < 3.0  # ~0.6 sigma bins over the tensor's range
    assert int(s.code_len[s.code_len > 0].min()) >= 2  # the two-window kernel applies

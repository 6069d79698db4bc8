"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test ties one part of the oracle to something independent: the BF16
bit layout, a hand-worked stream (tests/golden/df11_tiny_stream.txt),
brute-force optimal code lengths, the textbook Huffman cost, Kraft's equality,
Shannon's bound, the statistics the pages report for BF16 weights, and the
self-consistency of the auxiliary arrays under a windowed re-decode.
"""
import heapq
import itertools
import os

import numpy as np
import pytest
import torch

import oracle
from lossless_entropy_coded_dfloat11_b200 import inputs
from tests.conftest import parse_golden


def bf16_bits(values):
    t = torch.tensor(values, dtype=torch.float32).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# --------------------------------------------------------------------------- #
# Field split ("O espaco de compressao ainda disponivel no expoente": 1 sign, #
# 8 exponent, 7 mantissa bits)                                                #
# --------------------------------------------------------------------------- #
KNOWN = [  # value, exponent field, sign<<7 | mantissa
    (1.0, 127, 0x00), (-2.0, 128, 0x80), (0.5, 126, 0x00), (-0.75, 126, 0xC0),
    (0.375, 125, 0x40), (-3.5, 128, 0xE0), (3.0, 128, 0x40), (0.0, 0, 0x00),
    (-0.0, 0, 0x80), (float("inf"), 255, 0x00), (float("-inf"), 255, 0x80),
    (2.0 ** -126, 1, 0x00), (2.0 ** -133, 0, 0x01), (65280.0, 142, 0x7F),
]


@pytest.mark.parametrize("value,e,sm", KNOWN)
def test_split_known_values(value, e, sm):
    (x,) = bf16_bits([value])
    assert oracle.exponent(int(x)) == e
    assert oracle.sign_mantissa(int(x)) == sm
    assert oracle.merge(e, sm) == int(x)


def test_split_merge_exhaustive():
    """All 65536 patterns (zeros, subnormals, infinities, NaN payloads): the
    split must lose nothing and merge must invert it."""
    for x in range(0, 65536, 1):
        e, sm = oracle.exponent(x), oracle.sign_mantissa(x)
        assert 0 <= e < 256 and 0 <= sm < 256
        assert oracle.merge(e, sm) == x
    # the exponent field is what numpy's frexp sees for normal numbers
    xs = np.arange(0x0080, 0x7F80, 97, dtype=np.uint16)
    f = torch.from_numpy(xs.view(np.int16)).view(torch.bfloat16).float().numpy()
    _, ex = np.frexp(f)
    assert all(oracle.exponent(int(x)) == int(k) + 126 for x, k in zip(xs, ex))


def test_round_trip_all_patterns():
    x = inputs.all_patterns().flat_u16()
    s = oracle.encode(x)
    assert (oracle.histogram(x) == 256).all()
    np.testing.assert_array_equal(oracle.decode(s), x)
    np.testing.assert_array_equal(oracle.decode_windowed(s), x)


# --------------------------------------------------------------------------- #
# Hand-worked stream                                                          #
# --------------------------------------------------------------------------- #
def _golden(golden_dir):
    return parse_golden(os.path.join(golden_dir, "df11_tiny_stream.txt"))


def _kv(text, conv=int):
    return {int(k): conv(v) for k, v in (item.split("=") for item in text.split())}


def _golden_input(g, n=None):
    vals = _kv(g["value_of_exponent"], float)
    ex = [int(v) for v in g["A.exponents"].split()]
    if n is not None:
        ex = ex[:n]
    return np.array(ex), bf16_bits([vals[e] for e in ex])


def test_golden_stream_A(golden_dir):
    g = _golden(golden_dir)
    ex, x = _golden_input(g)
    sm_of = _kv(g["sm_of_exponent"], lambda v: int(v, 16))
    assert [oracle.exponent(int(v)) for v in x] == list(ex)

    lengths = oracle.code_lengths(oracle.histogram(x))
    assert {s: int(lengths[s]) for s in np.nonzero(lengths)[0]} == _kv(g["A.code_len"])
    codes = oracle.canonical_codes(lengths)
    want_codes = _kv(g["A.codes"], str)
    for sym, bits in want_codes.items():
        assert format(int(codes[sym]), "0%db" % len(bits)) == bits

    bits = g["A.bits"]
    assert bits == "10" + "00101100010111" * 5
    assert len(bits) == int(g["A.total_bits"])
    # the exponent stream, read MSB first, is the bit string
    packed = bytes(int(bits[i:i + 8].ljust(8, "0"), 2) for i in range(0, len(bits), 8))
    assert packed == bytes.fromhex(g["A.exp_head"])

    for T in (1, 2):
        s = oracle.encode(x, threads_per_block=T)
        assert s.total_bits == int(g["A.total_bits"])
        assert s.n_threads == int(g["A.n_threads"])
        assert s.n_blocks == int(g[f"A.T{T}.n_blocks"])
        assert s.exp.size == int(g[f"A.T{T}.bytes_exp"])
        assert bytes(s.exp[:9]) == bytes.fromhex(g["A.exp_head"])
        assert not s.exp[9:].any()
        assert [oracle.read_gap(s.gaps, t) for t in range(s.n_threads)] == [int(v) for v in g["A.gaps"].split()]
        assert bytes(s.gaps[:2]) == bytes.fromhex(g["A.gaps_head"])
        assert list(s.block_off) == [int(v) for v in g[f"A.T{T}.block_off"].split()]
        assert list(s.sm[:x.size]) == [sm_of[e] for e in ex]
        assert s.sm.size == 48 and not s.sm[x.size:].any()
        np.testing.assert_array_equal(oracle.decode(s), x)
        np.testing.assert_array_equal(oracle.decode_windowed(s), x)


def test_chunk_starts_golden_stream_A(golden_dir):
    # every chunk start is where that element's hand-written code sits in the
    # hand-derived bit string, and the table ends at total_bits
    g = _golden(golden_dir)
    ex, x = _golden_input(g)
    bits = g["A.bits"]
    want_codes = _kv(g["A.codes"], str)
    lengths = np.zeros(256, np.uint8)
    for sym, code in want_codes.items():
        lengths[sym] = len(code)
    starts = oracle.chunk_starts(x, lengths, 1)
    assert starts.size == x.size + 1 and starts[-1] == int(g["A.total_bits"])
    for i, e in enumerate(ex):
        code = want_codes[int(e)]
        assert bits[int(starts[i]): int(starts[i]) + len(code)] == code, i
    # the leading 126 takes bits 0..1, then groups of 8 elements take 14 bits
    assert list(oracle.chunk_starts(x, lengths, 8)) == [0, 13, 27, 41, 55, 69, 72]
    for chunk in (2, 3, 5, 64):
        np.testing.assert_array_equal(oracle.chunk_starts(x, lengths, chunk),
                                      np.append(starts[:-1][::chunk], starts[-1]))
    assert list(oracle.chunk_starts(x[:0], lengths, 4)) == [0]


def test_golden_stream_B_empty_last_window(golden_dir):
    g = _golden(golden_dir)
    n = int(g["B.n_elems"])
    ex, x = _golden_input(g, n)
    s = oracle.encode(x, threads_per_block=1)
    assert s.total_bits == int(g["B.total_bits"])
    assert bytes(s.exp[:9]) == bytes.fromhex(g["B.exp_head"])
    assert [oracle.read_gap(s.gaps, t) for t in range(s.n_threads)] == [int(v) for v in g["B.gaps"].split()]
    assert list(s.block_off) == [int(v) for v in g["B.T1.block_off"].split()]
    np.testing.assert_array_equal(oracle.decode_windowed(s), x)


# --------------------------------------------------------------------------- #
# Code lengths: optimality, Kraft, length limit                               #
# --------------------------------------------------------------------------- #
def kraft_units(lengths):
    """sum 2^(32-l): equals 2^32 exactly when the code is complete."""
    return sum(1 << (32 - int(l)) for l in lengths if l > 0)


def cost(hist, lengths):
    return int(sum(int(h) * int(l) for h, l in zip(hist, lengths)))


def brute_force_min_cost(weights, L):
    m = len(weights)
    best = None
    for vec in itertools.product(range(1, L + 1), repeat=m):
        if sum(2.0 ** -l for l in vec) <= 1.0 + 1e-12:
            c = sum(w * l for w, l in zip(weights, vec))
            best = c if best is None else min(best, c)
    return best


def huffman_cost_and_depth(weights):
    """Textbook Huffman with a heap: cost = sum of all merged weights."""
    heap = [(w, 0, i) for i, w in enumerate(weights)]
    heapq.heapify(heap)
    total, uid = 0, len(weights)
    while len(heap) > 1:
        a, da, _ = heapq.heappop(heap)
        b, db, _ = heapq.heappop(heap)
        total += a + b
        heapq.heappush(heap, (a + b, max(da, db) + 1, uid))
        uid += 1
    return total, heap[0][1]


def hist_of(weights, symbols=None):
    h = np.zeros(256, dtype=np.uint64)
    symbols = symbols if symbols is not None else range(len(weights))
    for s, w in zip(symbols, weights):
        h[s] = w
    return h


def test_lengths_brute_force_small_alphabets():
    rng = np.random.default_rng(1234)
    cases = 0
    for m in range(2, 8):
        for L in range(2, 6):
            if (1 << L) < m:
                continue
            for _ in range(3 if m < 7 else 1):
                w = [int(v) for v in rng.integers(1, 60, size=m)]
                if rng.random() < 0.5:  # skewed weights make the limit bind
                    w = sorted(int(v) for v in rng.geometric(0.3, size=m) ** 3)
                syms = sorted(rng.choice(256, size=m, replace=False).tolist())
                h = hist_of(w, syms)
                ln = oracle.code_lengths(h, L)
                assert ln.max() <= L
                assert kraft_units(ln) <= 1 << 32
                assert cost(h, ln) == brute_force_min_cost(w, L), (w, L, ln[syms])
                cases += 1
    assert cases > 40


def test_lengths_match_textbook_huffman_when_unconstrained():
    rng = np.random.default_rng(99)
    for m in list(range(2, 13)) + [40, 100, 256]:
        for _ in range(4):
            w = [int(v) for v in rng.integers(1, 10_000, size=m)]
            syms = sorted(rng.choice(256, size=m, replace=False).tolist())
            h = hist_of(w, syms)
            hc, depth = huffman_cost_and_depth(w)
            assert depth <= 32
            ln = oracle.code_lengths(h, 32)
            assert cost(h, ln) == hc
            assert kraft_units(ln) == 1 << 32  # complete code: Kraft equality


def test_shannon_bound():
    rng = np.random.default_rng(5)
    for m in (2, 3, 17, 64, 255):
        w = rng.integers(1, 1_000_000, size=m)
        h = hist_of(w, rng.choice(256, size=m, replace=False))
        ln = oracle.code_lengths(h, 32)
        H = oracle.entropy_bits(h)
        mean = cost(h, ln) / int(h.sum())
        assert H - 1e-9 <= mean < H + 1


def test_entropy_closed_forms():
    assert oracle.entropy_bits(hist_of([5] * 8)) == pytest.approx(3.0, abs=1e-12)
    assert oracle.entropy_bits(hist_of([2, 1, 1])) == pytest.approx(1.5, abs=1e-12)
    assert oracle.entropy_bits(hist_of([7])) == 0.0
    assert oracle.entropy_bits(np.zeros(256, dtype=np.uint64)) == 0.0
    assert oracle.entropy_bits(hist_of([1] * 256)) == pytest.approx(8.0, abs=1e-12)


def fibonacci(k):
    f = [1, 1]
    while len(f) < k:
        f.append(f[-1] + f[-2])
    return f[:k]


def clamp_and_repair(weights, L):
    """A simple feasible length limiter (not optimal): clamp the Huffman
    depths at L, then lengthen the lightest codes shorter than L until Kraft
    holds again."""
    # Huffman depths by a heap over (weight, node)
    n = len(weights)
    parent = {}
    heap = [(w, i) for i, w in enumerate(weights)]
    heapq.heapify(heap)
    nxt = n
    while len(heap) > 1:
        a, ia = heapq.heappop(heap)
        b, ib = heapq.heappop(heap)
        parent[ia] = parent[ib] = nxt
        heapq.heappush(heap, (a + b, nxt))
        nxt += 1
    depth = []
    for i in range(n):
        d, j = 0, i
        while j in parent:
            j = parent[j]
            d += 1
        depth.append(min(d, L))
    order = sorted(range(n), key=lambda i: weights[i])
    while sum(2.0 ** -d for d in depth) > 1.0:
        for i in order:
            if depth[i] < L:
                depth[i] += 1
                break
    return depth


def test_length_limit_binds_on_fibonacci_counts():
    w = fibonacci(34)
    h = hist_of(w, range(100, 134))
    _, depth = huffman_cost_and_depth(w)
    assert depth == 33                      # unconstrained tree is too deep
    ln = oracle.code_lengths(h, 32)
    assert ln.max() == 32
    assert kraft_units(ln) == 1 << 32
    hc, _ = huffman_cost_and_depth(w)
    assert cost(h, ln) >= hc
    assert cost(h, ln) <= sum(a * b for a, b in zip(w, clamp_and_repair(w, 32)))
    # small Fibonacci alphabets against brute force with a binding limit
    for k, L in ((7, 4), (6, 3), (7, 3), (5, 3)):
        wk = fibonacci(k)
        hk = hist_of(wk)
        lk = oracle.code_lengths(hk, L)
        assert lk.max() <= L
        assert cost(hk, lk) == brute_force_min_cost(wk, L)


def test_single_and_empty_alphabets():
    h = hist_of([10], [77])
    ln = oracle.code_lengths(h)
    assert ln[77] == 1 and ln.sum() == 1
    assert (oracle.code_lengths(np.zeros(256, dtype=np.uint64)) == 0).all()


def test_tie_rule_leaf_before_package_golden(golden_dir):
    """Hand-worked example C: on a leaf/package tie the leaf comes first."""
    g = _golden(golden_dir)
    h = np.zeros(256, dtype=np.uint64)
    for sym, cnt in _kv(g["C.counts"]).items():
        h[sym] = cnt
    ln = oracle.code_lengths(h, int(g["C.max_len"]))
    assert {s: int(ln[s]) for s in np.nonzero(ln)[0]} == _kv(g["C.code_len"])


def test_tie_rule_orders_equal_counts_by_value():
    # three equal weights: one symbol gets 1 bit, two get 2 bits.  The tie
    # rule orders leaves by (count, value), so among equal counts the lower
    # values count as the lighter symbols and take the longer codes.
    ln = oracle.code_lengths(hist_of([4, 4, 4], [9, 3, 200]))
    assert (ln[3], ln[9], ln[200]) == (2, 2, 1)


# --------------------------------------------------------------------------- #
# Canonical codes                                                             #
# --------------------------------------------------------------------------- #
def test_canonical_codes_properties():
    rng = np.random.default_rng(8)
    for m in (2, 5, 22, 36, 255, 256):
        w = rng.integers(1, 2 ** 20, size=m) if m < 250 else rng.zipf(1.3, size=m).clip(max=2 ** 30)
        syms = rng.choice(256, size=m, replace=False)
        h = hist_of(w, syms)
        ln = oracle.code_lengths(h, 32)
        codes = oracle.canonical_codes(ln)
        present = sorted((int(ln[s]), int(s)) for s in syms)
        strs = [format(int(codes[s]), "0%db" % l) for l, s in present]
        # prefix-free
        for a, b in itertools.combinations(strs, 2):
            assert not a.startswith(b) and not b.startswith(a)
        # left-justified values increase along the (length, value) order,
        # starting from all zeros and, for a complete code, ending all ones
        lj = [int(s, 2) << (32 - len(s)) for s in strs]
        assert lj == sorted(lj) and len(set(lj)) == len(lj)
        assert set(strs[0]) == {"0"}
        assert set(strs[-1]) == {"1"}


# --------------------------------------------------------------------------- #
# Whole codec on the workloads                                               #
# --------------------------------------------------------------------------- #
def test_gaussian_statistics_match_the_pages():
    """Exponent entropy about 2.6 bits, about 11 bits per weight and about 70%
    of the BF16 size ("O espaco de compressao ..." and "O formato DFloat11";
    abstract: 30% smaller)."""
    x = inputs.matrix_1k().flat_u16()
    s = oracle.encode(x)
    h = oracle.histogram(x)
    H = oracle.entropy_bits(h)
    assert 2.4 <= H <= 2.8
    mean = s.total_bits / x.size
    assert H <= mean < H + 1
    ratio = s.compressed_bytes() / (2 * x.size)
    assert 0.65 <= ratio <= 0.72
    assert 10.4 <= 16 * ratio <= 11.6
    np.testing.assert_array_equal(oracle.decode(s), x)


@pytest.mark.parametrize("dist", inputs.EDGE_DISTS)
@pytest.mark.parametrize("n", [1, 2, 3, 7, 8, 9, 31, 33, 63, 65, 127, 255, 257, 1023, 4097, 65537])
def test_round_trip_edge_sweep(n, dist):
    x = inputs.edge_case(n, dist, 500 + inputs.EDGE_SIZES.index(n)).flat_u16()
    for T in (1, 32, 256):
        s = oracle.encode(x, threads_per_block=T)
        assert s.code_len.max() <= 32
        np.testing.assert_array_equal(oracle.decode(s), x)
        np.testing.assert_array_equal(oracle.decode_windowed(s), x)


def test_round_trip_fibonacci_limit():
    x = inputs.fibonacci().flat_u16()
    s = oracle.encode(x)
    assert s.code_len.max() == 32
    np.testing.assert_array_equal(oracle.decode(s), x)


def test_empty_and_constant_inputs():
    s = oracle.encode(np.zeros(0, dtype=np.uint16))
    assert s.n_elems == 0 and s.total_bits == 0 and s.n_blocks == 0
    assert list(s.block_off) == [0]
    x = np.full(1000, 0x3F80, dtype=np.uint16)  # one exponent value
    s = oracle.encode(x, threads_per_block=4)
    assert s.total_bits == 1000 and s.code_len[127] == 1
    assert not s.exp.any()                        # the one code is "0"
    np.testing.assert_array_equal(oracle.decode_windowed(s), x)


# --------------------------------------------------------------------------- #
# Gaps and block offsets                                                      #
# --------------------------------------------------------------------------- #
def starts_by_brute_force(x, lengths):
    ln = [int(lengths[oracle.exponent(int(v))]) for v in x]
    return list(itertools.accumulate([0] + ln[:-1])), sum(ln)


@pytest.mark.parametrize("seed", range(6))
def test_aux_arrays_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 400))
    dist = ["uniform", "zipf", "one_value"][seed % 3]
    x = inputs.edge_case(n, dist, 900 + seed).flat_u16()
    T = int(rng.choice([1, 2, 3, 32]))
    s = oracle.encode(x, threads_per_block=T, max_len=int(rng.choice([12, 32])))
    starts, total = starts_by_brute_force(x, s.code_len)
    assert s.total_bits == total
    for w in range(s.n_threads):
        first = min([p for p in starts if p >= 64 * w] + [total])
        assert oracle.read_gap(s.gaps, w) == first - 64 * w < 32
    for b in range(s.n_blocks + 1):
        assert int(s.block_off[b]) == sum(1 for p in starts if p < 64 * T * b)


def test_corrupted_aux_arrays_are_detected():
    x = inputs.matrix_1k().flat_u16()[:20000]
    s = oracle.encode(x, threads_per_block=32)
    bad = oracle.Stream(**{**s.__dict__, "block_off": s.block_off.copy()})
    bad.block_off[3] += 1
    with pytest.raises(oracle.OracleError):
        oracle.decode_windowed(bad)
    bad = oracle.Stream(**{**s.__dict__, "gaps": s.gaps.copy()})
    bad.gaps[10] ^= 0x04
    with pytest.raises(oracle.OracleError):
        oracle.decode_windowed(bad)

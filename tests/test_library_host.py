"""CPU-only checks of the C-ABI library: it loads, exports every entry point
that include/df11.h declares, and its host logic (code builder, header
validation, decode tables) agrees with the oracle.  No kernel runs here."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import lossless_entropy_coded_dfloat11_b200 as df11
from lossless_entropy_coded_dfloat11_b200 import _binding as B
from lossless_entropy_coded_dfloat11_b200 import inputs
from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "df11.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(df11_[a-z0-9_]+)\s*\(", text)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = df11.load_library()
    names = declared_functions()
    assert len(names) >= 9
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(B.EXPORTED)
    assert lib.df11_version() == 1


def test_header_struct_layout_matches_c():
    assert ctypes.sizeof(B.Header) == 872
    assert B.Header.code_len.offset == 48
    assert B.Header.seg_elem_off.offset == 312
    assert B.Header.bytes_lut.offset == 864


def hist_of(weights, symbols):
    h = np.zeros(256, dtype=np.uint64)
    h[list(symbols)] = weights
    return h


@pytest.mark.parametrize("seed", range(12))
def test_code_lengths_identical_to_oracle(seed):
    """The library and the oracle implement package-merge separately with the
    same tie rule, so their lengths must be identical, not just equally good."""
    rng = np.random.default_rng(seed)
    m = int(rng.integers(1, 257))
    syms = rng.choice(256, size=m, replace=False)
    kind = seed % 4
    if kind == 0:
        w = rng.integers(1, 10, size=m)          # many ties
    elif kind == 1:
        w = rng.zipf(1.1, size=m).clip(max=10 ** 12)
    elif kind == 2:
        w = rng.integers(1, 2 ** 40, size=m)
    else:
        w = np.full(m, 7)
    h = hist_of(w, syms)
    minL = max(1, int(np.ceil(np.log2(max(m, 2)))))
    for L in sorted({minL, minL + 1, 12, 16, 24, 32}):
        if L > 32:
            continue
        np.testing.assert_array_equal(df11.code_lengths(h, L), oracle.code_lengths(h, L))


def test_code_lengths_fibonacci_and_workloads():
    fib = [1, 1]
    while len(fib) < 40:
        fib.append(fib[-1] + fib[-2])
    h = hist_of(fib, range(200, 240))
    for L in (6, 12, 20, 32):
        np.testing.assert_array_equal(df11.code_lengths(h, L), oracle.code_lengths(h, L))
    for w in (inputs.matrix_1k(), inputs.edge_case(65537, "zipf", 515), inputs.all_patterns()):
        h = oracle.histogram(w.flat_u16())
        np.testing.assert_array_equal(df11.code_lengths(h, 32), oracle.code_lengths(h, 32))


def test_code_lengths_tie_rule_golden(golden_dir):
    """The hand-worked tie case (tests/golden, example C)."""
    from tests.conftest import parse_golden
    g = parse_golden(os.path.join(golden_dir, "df11_tiny_stream.txt"))
    h = np.zeros(256, dtype=np.uint64)
    for item in g["C.counts"].split():
        k, v = item.split("=")
        h[int(k)] = int(v)
    ln = df11.code_lengths(h, int(g["C.max_len"]))
    want = {int(k): int(v) for k, v in (i.split("=") for i in g["C.code_len"].split())}
    assert {s: int(ln[s]) for s in np.nonzero(ln)[0]} == want


def test_code_lengths_rejects_bad_limits():
    h = hist_of([1] * 5, range(5))
    with pytest.raises(df11.DF11Error):
        df11.code_lengths(h, 2)        # 5 values do not fit 2-bit codes
    with pytest.raises(df11.DF11Error):
        df11.code_lengths(h, 33)


@pytest.mark.parametrize("T", [64, 256, 1024])
def test_header_sizes_match_oracle(T):
    x = inputs.edge_case(4097, "zipf", 514).flat_u16()
    s = oracle.encode(x, threads_per_block=T)
    hdr = df11.make_header(s.code_len, s.n_elems, s.total_bits, T)
    sz = oracle.sizes(oracle.histogram(x), s.code_len, T)
    assert (hdr.n_threads, hdr.n_blocks) == (sz["n_threads"], sz["n_blocks"])
    assert (hdr.bytes_exp, hdr.bytes_sm, hdr.bytes_gaps, hdr.bytes_off) == (
        sz["bytes_exp"], sz["bytes_sm"], sz["bytes_gaps"], sz["bytes_off"])


def test_header_validation():
    ln = np.zeros(256, dtype=np.uint8)
    ln[[1, 2, 3]] = [1, 2, 2]
    df11.make_header(ln, 10, 15, 256)
    bad = ln.copy()
    bad[4] = 3                                   # Kraft sum above 1
    with pytest.raises(df11.DF11Error):
        df11.make_header(bad, 10, 15, 256)
    bad = ln.copy()
    bad[3] = 3                                   # incomplete code
    with pytest.raises(df11.DF11Error):
        df11.make_header(bad, 10, 15, 256)
    with pytest.raises(df11.DF11Error):
        df11.make_header(ln, 10, 15, 96)         # T not a power of two
    with pytest.raises(df11.DF11Error) as e:
        df11.make_header(ln, 2 ** 32, 2 ** 33, 256)
    assert e.value.code == B.DF11_ERR_TOO_LARGE
    with pytest.raises(df11.DF11Error):
        df11.make_header(ln, 10, 5, 256)         # fewer bits than elements
    one = np.zeros(256, dtype=np.uint8)
    one[9] = 1
    df11.make_header(one, 3, 3, 64)              # single value: code "0"
    one[9] = 2
    with pytest.raises(df11.DF11Error):
        df11.make_header(one, 3, 6, 64)


PEEK_BITS = 12
ESCAPE = 512
# table offsets: 64-byte header, lj_end u64[33], delta u32[33], syms u8[256],
# then count u32[4096], mask u16[4096], decode (u32, u32)[4096]
OFF_COUNT = 736
OFF_MASK = OFF_COUNT + 4 * 4096
OFF_DECODE = OFF_MASK + 2 * 4096
OFF_LONG = OFF_DECODE + 8 * 4096
# then the narrow sections for K = 10, 9, 8: mask u16[2^K], long u16[4096
# (8192 for K = 8)], decode (u32, u32)[2^K], each rounded up to 16 bytes
OFF_NARROW = OFF_LONG + 2 * 4096


def narrow_long_entries(k):
    return 8192 if k == 8 else 4096


def narrow_bytes(k):
    return -(-(2 * 2 ** k + 2 * narrow_long_entries(k) + 8 * 2 ** k) // 16) * 16


def narrow_off(k):
    return OFF_NARROW + sum(narrow_bytes(j) for j in range(10, k, -1))


LUT_BYTES = narrow_off(8) + narrow_bytes(8)


def _oracle_prefix_decoder(code_len):
    codes = oracle.canonical_codes(code_len)
    table = {format(int(codes[s]), "0%db" % int(code_len[s])): int(s)
             for s in range(256) if code_len[s]}
    return table


def _decode_bits(table, bits, limit):
    """Complete codes at the front of the bit string (oracle codes)."""
    out, pos = [], 0
    while True:
        for l in range(1, len(bits) - pos + 1):
            sym = table.get(bits[pos:pos + l])
            if sym is not None:
                break
        else:
            return out, pos
        if len(out) == limit:
            return out, pos
        out.append((sym, pos))
        pos += l


@pytest.mark.parametrize("source", ["matrix_1k", "zipf", "one_value", "fibonacci"])
def test_decode_tables_agree_with_oracle_codes(source):
    """Every level-1 entry must describe exactly the complete oracle codes at
    the front of its 12-bit index."""
    if source == "matrix_1k":
        x = inputs.matrix_1k().flat_u16()
    elif source == "fibonacci":
        x = inputs.fibonacci().flat_u16()
    else:
        x = inputs.edge_case(65537, source, 515).flat_u16()
    s = oracle.encode(x)
    hdr = df11.make_header(s.code_len, s.n_elems, s.total_bits, 256)
    lut = df11.build_lut(hdr)
    assert lut.size == LUT_BYTES == int(hdr.bytes_lut)
    assert lut[:4].tobytes() == b"DF11"
    ctab = lut[OFF_COUNT:OFF_MASK].view(np.uint32)
    mtab = lut[OFF_MASK:OFF_DECODE].view(np.uint16)
    dtab = lut[OFF_DECODE:OFF_LONG].view(np.uint32).reshape(-1, 2)
    table = _oracle_prefix_decoder(s.code_len)
    rng = np.random.default_rng(3)
    for v in list(range(64)) + list(rng.integers(0, 4096, size=400)) + list(range(4032, 4096)):
        bits = format(int(v), "012b")
        codes, used = _decode_bits(table, bits, None)
        mask = sum(1 << p for _, p in codes)
        assert int(mtab[v]) == mask, (v, bits)
        assert int(ctab[v]) == ((used << 16) | len(codes) if codes else ESCAPE << 16), (v, bits)
        codes4, used4 = _decode_bits(table, bits, 4)
        x, y = int(dtab[v, 0]), int(dtab[v, 1])
        if not codes4:
            assert (x, y) == (0, ESCAPE << 16)
            continue
        assert y == (used4 << 16) | (8 * len(codes4))
        assert len(codes4) == 4 or x >> (8 * len(codes4)) == 0   # unused symbol bytes are zero
        for k, (sym, _) in enumerate(codes4):   # staged rotated right by one bit
            assert (x >> (8 * k)) & 0xFF == ((sym >> 1) | (sym << 7)) & 0xFF


@pytest.mark.parametrize("k", [10, 9, 8])
@pytest.mark.parametrize("source", ["matrix_1k", "zipf", "fibonacci"])
def test_narrow_tables_agree_with_oracle_codes(source, k):
    """The narrow first levels (a K-bit peek, K = 10, 9 and the pages' 8-bit
    256-entry table): every mask and decode entry describes exactly the
    complete oracle codes at the front of its K-bit index, and entry i of the
    section's long table the code at the top of the 20-bit prefix
    long_base + i when that code is longer than K and at most 20 bits."""
    if source == "matrix_1k":
        x = inputs.matrix_1k().flat_u16()
    elif source == "fibonacci":
        x = inputs.fibonacci().flat_u16()
    else:
        x = inputs.edge_case(65537, source, 515).flat_u16()
    s = oracle.encode(x)
    hdr = df11.make_header(s.code_len, s.n_elems, s.total_bits, 64)
    lut = df11.build_lut(hdr)
    assert lut.size == LUT_BYTES == int(hdr.bytes_lut)
    sec = lut[narrow_off(k):narrow_off(k) + narrow_bytes(k)]
    mtab = sec[: 2 * 2 ** k].view(np.uint16)
    nl = narrow_long_entries(k)
    ltab = sec[2 * 2 ** k: 2 * 2 ** k + 2 * nl].view(np.uint16)
    dtab = sec[2 * 2 ** k + 2 * nl: 2 * 2 ** k + 2 * nl + 8 * 2 ** k].view(np.uint32).reshape(-1, 2)
    table = _oracle_prefix_decoder(s.code_len)
    for v in range(2 ** k):
        bits = format(v, "0%db" % k)
        codes, _ = _decode_bits(table, bits, None)
        assert int(mtab[v]) == sum(1 << p for _, p in codes), (v, bits)
        codes4, used4 = _decode_bits(table, bits, 4)
        x_, y = int(dtab[v, 0]), int(dtab[v, 1])
        if not codes4:
            assert (x_, y) == (0, ESCAPE << 16)
            continue
        assert y == (used4 << 16) | (8 * len(codes4))
        assert len(codes4) == 4 or x_ >> (8 * len(codes4)) == 0
        for j, (sym, _) in enumerate(codes4):
            assert (x_ >> (8 * j)) & 0xFF == ((sym >> 1) | (sym << 7)) & 0xFF
    row = 10 - k   # LutHeader: 8 words, then (long_base, long_count) per narrow K
    long_base, long_count = (int(v) for v in lut[32 + 8 * row: 40 + 8 * row].view(np.uint32))
    short_space = sum(1 << (32 - int(l)) for l in s.code_len if 0 < l <= k)
    assert long_base == short_space >> 12
    need = -(-((1 << 32) - short_space) // 4096)
    assert long_count == (need if short_space < (1 << 32) and need <= nl else 0)
    rng = np.random.default_rng(k)
    picks = range(long_count) if long_count <= 600 else rng.integers(0, long_count, size=600)
    for i in picks:
        bits = format(long_base + int(i), "020b")
        codes, _ = _decode_bits(table, bits, 1)
        e = int(ltab[i])
        if not codes:
            assert e == 0
            continue
        sym, _ = codes[0]
        length = next(len(c) for c, v in table.items() if v == sym)
        assert length > k
        assert e == (((sym >> 1) | (sym << 7)) & 0xFF) | (length << 8)


@pytest.mark.parametrize("source", ["outliers", "fibonacci", "matrix_1k"])
def test_long_code_table_agrees_with_oracle_codes(source):
    """Level 2: entry i of the long table describes the code at the top of the
    20-bit prefix long_base + i (rotated symbol | length << 8, 0 if longer)."""
    if source == "outliers":
        x = inputs.matrix_outliers(1024, 1024, seed=21).flat_u16()
    elif source == "fibonacci":
        x = inputs.fibonacci().flat_u16()
    else:
        x = inputs.matrix_1k().flat_u16()
    s = oracle.encode(x)
    hdr = df11.make_header(s.code_len, s.n_elems, s.total_bits, 32)
    lut = df11.build_lut(hdr)
    long_base, long_count = (int(v) for v in lut[24:32].view(np.uint32))
    assert 0 < long_count <= 4096
    ltab = lut[OFF_LONG:OFF_NARROW].view(np.uint16)
    table = _oracle_prefix_decoder(s.code_len)
    # the first long prefix is where the codes of more than 12 bits begin
    short_space = sum(1 << (32 - int(l)) for l in s.code_len if 0 < l <= 12)
    assert long_base == short_space >> 12
    for i in range(long_count):
        bits = format(long_base + i, "020b")
        codes, _ = _decode_bits(table, bits, 1)
        e = int(ltab[i])
        if not codes:
            assert e == 0                       # longer than 20 bits: ladder
            continue
        sym, _ = codes[0]
        length = next(len(k) for k, v in table.items() if v == sym)
        assert length > 12
        assert e == (((sym >> 1) | (sym << 7)) & 0xFF) | (length << 8)

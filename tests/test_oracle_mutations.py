"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of oracle/df11_oracle.c (a dropped
term, a wrong shift, sign or index, a transposed field), builds it, and runs
the pin suite (tests/test_oracle_pins.py) against that build: the suite must
fail.  The Python part of the oracle (the chunk start table) gets the same
treatment through a mutated copy of the package, imported ahead of the real
one.  Nothing here touches the real oracle or the CUDA library.
"""
import os
import shutil
import subprocess
import sys

import pytest

from tests.conftest import ROOT

SRC = os.path.join(ROOT, "oracle", "df11_oracle.c")

MUTATIONS = [
    ("LSB-first exponent bits", "a[p >> 3] |= (uint8_t)(0x80u >> (p & 7));", "a[p >> 3] |= (uint8_t)(1u << (p & 7));"),
    ("sign bit at 6", "return (sign << 7) | mant;", "return (sign << 6) | mant;"),
    ("exponent field off by one bit", "uint32_t oracle_exponent(uint32_t x) { return (x >> 7) & 0xFFu; }",
     "uint32_t oracle_exponent(uint32_t x) { return (x >> 8) & 0xFFu; }"),
    ("merge shifts exponent by 8", "return (sign << 15) | ((e & 0xFFu) << 7) | mant;",
     "return (sign << 15) | ((e & 0xFFu) << 8) | mant;"),
    ("canonical codes drop the +1", "if (k > 0) code = (code + 1) << (l - prev_len);",
     "if (k > 0) code = code << (l - prev_len);"),
    ("package-merge ties favour packages", "else take_leaf = (hist[syms[li]] <= pw); /* leaf first on ties */",
     "else take_leaf = (hist[syms[li]] < pw);"),
    ("package-merge takes one item too many", "int take = 2 * (m - 1);", "int take = 2 * m - 1;"),
    ("leaf order by descending symbol", "(hist[syms[j]] == hist[v] && syms[j] > v))) {",
     "(hist[syms[j]] == hist[v] && syms[j] < v))) {"),
    ("gap one bit late", "uint64_t g = start - 64 * w;\n            if (g > 31) return ORC_ERR_ARG;",
     "uint64_t g = start - 64 * w + 1;\n            if (g > 32) return ORC_ERR_ARG;"),
    ("empty last window gap = 0", "uint64_t g = sz.total_bits - 64 * w;", "uint64_t g = 0 * sz.total_bits;"),
    ("block offset counts codes at the boundary", "while (b <= sz.n_blocks && 64 * (uint64_t)T * b <= start) {",
     "while (b <= sz.n_blocks && 64 * (uint64_t)T * b < start) {"),
    ("gap fields MSB-first", "if ((g >> k) & 1) gaps[q >> 3] |= (uint8_t)(1u << (q & 7));",
     "if ((g >> k) & 1) gaps[q >> 3] |= (uint8_t)(0x80u >> (q & 7));"),
    ("smaller exponent guard", "out->bytes_exp = 8 * (uint64_t)T * out->n_blocks + 16;",
     "out->bytes_exp = 8 * (uint64_t)T * out->n_blocks + 8;"),
    ("entropy drops the probability weight", "h -= p * log2(p);", "h -= log2(p);"),
    ("histogram counts twice", "for (uint64_t i = 0; i < n; i++) hist[oracle_exponent(x[i])] += 1;",
     "for (uint64_t i = 0; i < n; i++) hist[oracle_exponent(x[i])] += 2;"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(name, old, new, tmp_path):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not found: {name}"
    bad = tmp_path / "df11_oracle_mutant.c"
    bad.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-o", str(lib), str(bad), "-lm"])
    env = dict(os.environ, DF11_ORACLE_LIB=str(lib))
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                         capture_output=True, text=True, env=env, cwd=ROOT, timeout=600)
    assert res.returncode != 0, f"pins did not catch: {name}\n{res.stdout[-1500:]}"


PY_SRC = os.path.join(ROOT, "oracle", "__init__.py")

PY_MUTATIONS = [
    ("chunk table without its leading zero", "return np.concatenate([[0], np.cumsum(per_chunk)]).astype(np.uint64)",
     "return np.concatenate([np.cumsum(per_chunk), [per_chunk.sum()]]).astype(np.uint64)"),
    ("chunk lengths from the wrong field", "ln = np.ascontiguousarray(code_len, dtype=np.uint8)[(x >> 7) & 0xFF]",
     "ln = np.ascontiguousarray(code_len, dtype=np.uint8)[(x >> 8) & 0xFF]"),
    ("chunks start one element late", "per_chunk = np.add.reduceat(ln.astype(np.uint64), np.arange(0, n, chunk))",
     "per_chunk = np.add.reduceat(ln.astype(np.uint64), np.minimum(np.arange(0, n, chunk) + 1, n - 1))"),
]


@pytest.mark.parametrize("name,old,new", PY_MUTATIONS, ids=[m[0] for m in PY_MUTATIONS])
def test_pins_catch_planted_mistake_in_python_oracle(name, old, new, tmp_path):
    src = open(PY_SRC).read()
    assert src.count(old) == 1, f"mutation site not found: {name}"
    pkg = tmp_path / "oracle"
    pkg.mkdir()
    (pkg / "__init__.py").write_text(src.replace(old, new))
    shutil.copy(os.path.join(ROOT, "oracle", "df11_oracle.c"), pkg / "df11_oracle.c")
    import oracle
    env = dict(os.environ, DF11_ORACLE_LIB=oracle.build())  # the real C part
    pins = os.path.join(ROOT, "tests", "test_oracle_pins.py")
    code = (f"import sys; sys.path.insert(0, {str(tmp_path)!r}); import oracle; "
            f"assert oracle.__file__.startswith({str(tmp_path)!r}); import pytest; "
            f"sys.exit(pytest.main(['-x', '-q', '-p', 'no:cacheprovider', {pins!r}]))")
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env, cwd=ROOT,
                         timeout=600)
    assert res.returncode != 0, f"pins did not catch: {name}\n{res.stdout[-1500:]}"
    assert "failed" in res.stdout, res.stdout[-800:] + res.stderr[-800:]

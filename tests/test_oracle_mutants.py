"""Plant plausible mistakes in copies of the oracle (CPU only) and check that
the pins catch every one of them."""
import os
import shutil
import subprocess
import sys

import pytest

import oracle
from oracle_pins import ALL_PINS

# (description, text in mla_oracle.c, replacement); each text must occur once.
MUTANTS = [
    ("dropped softmax scale", "dot += qv[d] * bf16_to_double(k[d]);\n            s[j] = scale * dot;",
     "dot += qv[d] * bf16_to_double(k[d]);\n            s[j] = dot;"),
    ("wrong sign in the exponent",
     "const uint16_t *k = token_row(&p, b, j);\n            const double w = exp(s[j] - m);",
     "const uint16_t *k = token_row(&p, b, j);\n            const double w = exp(m - s[j]);"),
    ("value read from the wrong columns", "o[c] += w * bf16_to_double(k[c]);",
     "o[c] += w * bf16_to_double(k[c + 64]);"),
    ("causal window off by one", "int64_t n = seqlen - s_q + 1 + i;", "int64_t n = seqlen - s_q + i;"),
    ("lse in base 2", "*ls = m + log(l);\n        free(s);\n    }\n    return failed ? ORC_NO_MEMORY : ORC_OK;\n}\n\n/* ---",
     "*ls = m + log2(l);\n        free(s);\n    }\n    return failed ? ORC_NO_MEMORY : ORC_OK;\n}\n\n/* ---"),
    ("page and in-page offset swapped", "int64_t page = j / ORC_PAGE;", "int64_t page = j % ORC_PAGE;"),
    ("rope part of the score dropped",
     "for (int d = 0; d < ORC_DQK; ++d) dot += qv[d] * bf16_to_double(k[d]);\n            s[j] = scale * dot;",
     "for (int d = 0; d < ORC_DV; ++d) dot += qv[d] * bf16_to_double(k[d]);\n            s[j] = scale * dot;"),
    ("output not normalised", "for (int c = 0; c < ORC_DV; ++c) o[c] /= l;\n        *ls",
     "*ls"),
    ("head index ignored", "return p->q + (((int64_t)b * p->s_q + i) * p->H + h) * ORC_DQK;",
     "return p->q + (((int64_t)b * p->s_q + i) * p->H + 0) * ORC_DQK;"),
    ("query position ignored", "return p->q + (((int64_t)b * p->s_q + i) * p->H + h) * ORC_DQK;",
     "return p->q + (((int64_t)b * p->s_q + 0) * p->H + h) * ORC_DQK;"),
    ("merged states weighted by the max, not the total",
     "const double wt = exp(lse_parts[(int64_t)w * rows + r] - total);",
     "const double wt = exp(lse_parts[(int64_t)w * rows + r] - M);"),
    ("merged lse without the max", "        lse[r] = total;\n    }\n    return ORC_OK;",
     "        lse[r] = log(sum);\n    }\n    return ORC_OK;"),
    ("merge reads the wrong state's rows", "const double *po = out_parts + ((int64_t)w * rows + r) * ORC_DV;",
     "const double *po = out_parts + r * ORC_DV;"),
    ("e4m3 exponent bias off by one", "else mag = ldexp(1.0 + mant / 8.0, ex - 7);",
     "else mag = ldexp(1.0 + mant / 8.0, ex - 8);"),
    ("e4m3 subnormals scaled wrongly", "if (ex == 0) mag = ldexp((double)mant, -9);",
     "if (ex == 0) mag = ldexp((double)mant, -10);"),
    ("fp8 token scale dropped", "row[j * ORC_DQK + d] = table[kv_codes[tok * ORC_DQK + d]] * ks;",
     "row[j * ORC_DQK + d] = table[kv_codes[tok * ORC_DQK + d]];"),
    ("non-absorbed: key matrix read transposed", "ke += c[x] * wk[(int64_t)e * ORC_DV + x];",
     "ke += c[x] * wk[(int64_t)x * ORC_DNOPE + e];"),
    ("non-absorbed: value decompressed with the key matrix", "ve += c[x] * wv[(int64_t)e * ORC_DV + x];",
     "ve += c[x] * wk[(int64_t)e * ORC_DV + x];"),
    ("non-absorbed: rope part of the score dropped",
     "for (int x = 0; x < ORC_DROPE; ++x) dot += qv[ORC_DNOPE + x] * bf16_to_double(row[ORC_DV + x]);", ""),
    ("non-absorbed: head of the up-projections ignored",
     "const uint16_t *wkh = w_uk + (int64_t)h * ORC_DNOPE * ORC_DV;", "const uint16_t *wkh = w_uk;"),
]


@pytest.fixture(scope="module")
def source_text():
    with open(oracle.SOURCE) as f:
        return f.read()


_RUNNER = """
import sys
sys.path[:0] = {paths!r}
import oracle
from oracle_pins import ALL_PINS
m = oracle.Oracle(library={lib!r}, source={src!r})
caught = []
for pin in ALL_PINS:
    try:
        pin(m)
    except (AssertionError, ValueError):
        caught.append(pin.__name__)
print("CAUGHT", len(caught), " ".join(caught))
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("desc,find,repl", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, source_text, desc, find, repl):
    assert source_text.count(find) == 1, f"mutation site for {desc!r} not unique"
    src = tmp_path / "mutant.c"
    src.write_text(source_text.replace(find, repl))
    lib = tmp_path / "libmutant.so"
    oracle.compile_oracle(str(src), str(lib))
    here = os.path.dirname(os.path.abspath(__file__))
    code = _RUNNER.format(paths=[os.path.dirname(here), here], lib=str(lib), src=str(src))
    # A separate process: a planted indexing mistake may crash outright,
    # which also counts as caught.
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                         env=dict(os.environ, OMP_NUM_THREADS="2"), timeout=600)
    if res.returncode != 0:
        return
    line = [l for l in res.stdout.splitlines() if l.startswith("CAUGHT")][-1]
    assert int(line.split()[1]) > 0, f"no pin caught the planted mistake: {desc}"

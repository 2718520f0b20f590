"""The pins catch plausible mistakes: each test compiles a copy of the oracle
with one planted mistake (on the CPU, in a temporary directory) and requires
at least one pin of tests/pins.py to fail on it."""
import os
import shutil

import pytest

import oracle
from tests import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "hils_oracle.c")

# (name, text in the oracle, planted replacement)
MUTANTS = [
    ("own_chunk_drops_diagonal", "own * C, t + 1, acc", "own * C, t, acc"),
    ("selects_lowest_scores", "if (a->s32 > b->s32) return -1;", "if (a->s32 > b->s32) return 1;"),
    ("ties_favour_high_index",
     "  return (a->c > b->c) - (a->c < b->c);\n}\nstatic int by_chunk_asc",
     "  return (a->c < b->c) - (a->c > b->c);\n}\nstatic int by_chunk_asc"),
    ("own_logit_zero", "g[nsel] = chunk_attend(", "g[nsel] = 0.0 * chunk_attend("),
    ("landmark_unscaled", "s = P->scale * dot(qt, P->lmk", "s = dot(qt, P->lmk"),
    ("fusion_not_normalised", "const double wi = exp(g[i] - lse_row);",
     "const double wi = exp(g[i] - m);"),
    ("normaliser_no_shift", "for (int c = 0; c < n_c; ++c) l += exp(cs[c].s - m);",
     "for (int c = 0; c < n_c; ++c) l += exp(cs[c].s);"),
    ("values_read_from_keys", "o[i] += p * ld(P->v,", "o[i] += p * ld(P->k,"),
    ("gqa_head_interleaved", "const int hkv = hq / (P->Hq / P->Hkv);",
     "const int hkv = hq % P->Hkv;"),
    ("chunk_lse_unshifted", "for (int j = j0; j < j1; ++j) l += exp(xbuf[j - j0] - m);",
     "for (int j = j0; j < j1; ++j) l += exp(xbuf[j - j0]);"),
    ("token_scale_dropped", "xbuf[j - j0] = P->scale * dot(", "xbuf[j - j0] = dot("),
    ("union_misses_own", "    mark[t / C] = 1;\n", "\n"),
    ("selection_off_by_one", "nsel = n_c < k ? n_c : k;", "nsel = n_c < k ? n_c : k - (k > 1);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation anchor not unique/found: {old!r}"
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    lib = oracle.compile_source(str(src), str(tmp_path / "libmutant.so"))
    orc = oracle.Oracle(lib)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"planted mistake {name} passed every pin"
    shutil.rmtree(tmp_path, ignore_errors=True)

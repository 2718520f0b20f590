"""The pins catch plausible mistakes: each test compiles a copy of the oracle
with one planted mistake (on the CPU, in a temporary directory), or swaps one
of the oracle's Python functions for a broken version, and requires a pin of
tests/pins.py to fail on it."""
import os
import shutil

import numpy as np
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


# ---------------------------------------------------------------------------
# The Python parts of the oracle (paged-cache gather, HoPE, Q-Cal): each
# planted mistake replaces one function for the duration of the test, and
# the pin written for that function must fail.

def _gather_ignores_table(pages, page_table, L):
    pg, _ = oracle._as_array(pages)
    tab = np.asarray(page_table)
    num_pages, Hkv, C, d = pg.shape
    B, npg = tab.shape[0], -(-L // C)
    out = np.empty((B, Hkv, L, d), pg.dtype)
    for b in range(B):
        for c in range(npg):
            n = min(C, L - c * C)
            out[b, :, c * C:c * C + n] = pg[b * npg + c, :, :n]
    return out


def _gather_token_major_pages(pages, page_table, L):
    pg, _ = oracle._as_array(pages)
    tab = np.asarray(page_table)
    num_pages, Hkv, C, d = pg.shape
    flat = pg.reshape(num_pages, C, Hkv, d)
    out = np.empty((tab.shape[0], Hkv, L, d), pg.dtype)
    for b in range(tab.shape[0]):
        for c in range(-(-L // C)):
            n = min(C, L - c * C)
            out[b, :, c * C:c * C + n] = flat[int(tab[b, c])].transpose(1, 0, 2)[:, :n]
    return out


def _hope_variant(kind):
    def hope(x, positions, n_rope_pairs, base=10000.0):
        a, bf16 = oracle._as_array(x)
        a = a.astype(np.float64)
        d = a.shape[-1]
        half = d // 2
        t = np.asarray(positions, dtype=np.float64).reshape(-1)
        out = a.copy()
        for i in range(n_rope_pairs):
            theta = base ** ((-1.0 if kind == "frequency_exponent" else -2.0) * i / d)
            j = half - 1 - i if kind == "last_pairs_rotated" else i
            p0, p1 = (2 * i, 2 * i + 1) if kind == "interleaved_pairs" else (j, j + half)
            s = np.sin(t * theta)[:, None] * (-1.0 if kind == "sign" else 1.0)
            c = np.cos(t * theta)[:, None]
            xi, xj = a[..., :, p0:p0 + 1], a[..., :, p1:p1 + 1]
            out[..., :, p0:p0 + 1] = xi * c - xj * s
            out[..., :, p1:p1 + 1] = xi * s + xj * c
        return out
    return hope


def _qcal_everywhere(self, p, q, k, v, lmk, qs, rows, nthreads=0):
    k32, v32, l32 = (oracle._widen32(a) for a in (k, v, lmk))
    return self.rows(p, oracle._widen32(qs), k32, v32, l32, rows)


def _qcal_ignored(self, p, q, k, v, lmk, qs, rows, nthreads=0):
    return self.rows(p, q, k, v, lmk, rows)


def _split_on_frequency(d, base, train_len):
    # compares the angular frequency instead of the wavelength
    return sum(1 for i in range(d // 2) if base ** (-2.0 * i / d) <= train_len)


def _split_without_two_pi(d, base, train_len):
    n = 0
    while n < d // 2 and base ** (2.0 * n / d) <= train_len:
        n += 1
    return n


PY_MUTANTS = [
    ("gather_ignores_table", oracle, "gather_pages", _gather_ignores_table,
     pins.pin_paged_decode_is_dense_decode),
    ("gather_token_major_pages", oracle, "gather_pages", _gather_token_major_pages,
     pins.pin_paged_decode_is_dense_decode),
    ("hope_frequency_exponent", oracle, "hope", _hope_variant("frequency_exponent"),
     pins.pin_hope_rotation_properties),
    ("hope_last_pairs_rotated", oracle, "hope", _hope_variant("last_pairs_rotated"),
     pins.pin_hope_rotation_properties),
    ("hope_interleaved_pairs", oracle, "hope", _hope_variant("interleaved_pairs"),
     pins.pin_hope_rotation_properties),
    ("hope_sign", oracle, "hope", _hope_variant("sign"), pins.pin_hope_rotation_properties),
    ("qcal_query_used_for_attention", oracle.Oracle, "rows_qcal", _qcal_everywhere,
     pins.pin_qcal_scoring_query),
    ("qcal_query_ignored", oracle.Oracle, "rows_qcal", _qcal_ignored, pins.pin_qcal_scoring_query),
    ("split_on_frequency", oracle, "rope_pairs", _split_on_frequency, pins.pin_hope_split_rule),
    ("split_without_two_pi", oracle, "rope_pairs", _split_without_two_pi, pins.pin_hope_split_rule),
]


@pytest.mark.parametrize("name,owner,attr,bad,pin", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_python_mutant_is_caught(monkeypatch, name, owner, attr, bad, pin):
    monkeypatch.setattr(owner, attr, bad)
    with pytest.raises((AssertionError, ValueError, IndexError)):
        pin(oracle.default())

"""Parity helpers: compare CUDA results with the oracle on the same inputs.

Selection indices must match the oracle exactly, except at near-ties: a row
whose k-th and (k+1)-th landmark logits lie within 1e-4 * max(1, |s_k|) of
each other admits several top-k sets.  For such a row the oracle enumerates
every admissible set itself (from its own logits) and computes the output of
each; the GPU row must equal one of those sets and match that set's output.
No value computed by the CUDA path is ever fed to the oracle.
"""
from __future__ import annotations

import itertools
import math

import numpy as np

import oracle

NEAR_TIE_REL = 1e-4
MAX_ALTERNATIVES = 64


def tolerances(dtype: str) -> dict:
    """Output tolerances: bf16 inputs max-abs 1e-2 / mean-abs 1e-3; fp32 1e-5.
    Logits (chunk_w, lse, lse_lmk) are computed in fp32 on both dtypes."""
    if dtype == "f32":
        return dict(out_max=1e-5, out_mean=1e-5, lse=1e-5, w=1e-5, lse_lmk=1e-5, wfin=1e-5)
    return dict(out_max=1e-2, out_mean=1e-3, lse=5e-4, w=1e-4, lse_lmk=1e-4, wfin=1e-3)


def admissible_sets(scores: np.ndarray, k: int):
    """All top-k sets consistent with one row's oracle logits up to the
    near-tie band.  `scores` holds the logits of the completed chunks."""
    n = scores.shape[0]
    if n <= k:
        return [tuple(range(n))]
    s32 = scores.astype(np.float32)
    order = sorted(range(n), key=lambda c: (-float(s32[c]), c))
    sk = float(scores[order[k - 1]])
    tol = NEAR_TIE_REL * max(1.0, abs(sk))
    band = [c for c in range(n) if abs(float(scores[c]) - sk) < tol]
    must = [c for c in range(n) if float(scores[c]) >= sk + tol]
    r = k - len(must)
    if r < 0 or r > len(band):
        return [tuple(sorted(order[:k]))]
    if math.comb(len(band), r) > MAX_ALTERNATIVES:
        raise AssertionError(f"{math.comb(len(band), r)} admissible top-k sets: too many near-ties")
    return [tuple(sorted(must + list(extra))) for extra in itertools.combinations(band, r)]


def compare_rows(p: oracle.Problem, inputs, rows, gpu: dict, ref: dict, dtype: str,
                 decode: bool = False, orc=None, score_q=None) -> dict:
    """Compare GPU outputs of `rows` (numbered as in oracle rows(); decode
    heads when decode=True) with the oracle's result `ref` for the same rows.
    gpu/ref: dicts of numpy arrays sel [n,k], w [n,k], out [n,d], lse [n],
    optional lse_lmk [n] and wfin [n,k+1].  score_q: the query of the
    landmark scores when it is not q (Q-Cal).  Raises AssertionError on a
    mismatch; returns statistics."""
    orc = orc or oracle.default()
    tol = tolerances(dtype)
    q, k, v, lmk = inputs
    n, K = ref["sel"].shape
    rows = np.asarray(rows, np.int64).reshape(-1)
    same = (gpu["sel"] == ref["sel"]).all(axis=1)
    exp_out = ref["out"].copy()
    exp_lse = ref["lse"].copy()
    exp_w = ref["w"].copy()
    exp_wfin = ref["wfin"].copy() if gpu.get("wfin") is not None else None
    near_ties = 0
    for i in np.nonzero(~same)[0]:
        t = p.L - 1 if decode else int(rows[i] % p.L)
        sc = orc.scores(p, q if score_q is None else score_q, lmk, [rows[i]],
                        decode=decode)[0][: t // p.C]
        alts = admissible_sets(sc, K)
        got = tuple(int(c) for c in gpu["sel"][i] if c >= 0)
        if got not in alts:
            raise AssertionError(
                f"row {rows[i]}: GPU selection {got} is not an admissible top-{K} "
                f"(oracle {tuple(int(c) for c in ref['sel'][i] if c >= 0)})")
        near_ties += 1
        # the oracle evaluates every admissible set of its own enumeration;
        # the GPU row is compared with the one it chose
        for alt in alts:
            sel_in = np.array([list(alt) + [-1] * (K - len(alt))], np.int32)
            w_in = np.array([[sc[c] for c in alt] + [-np.inf] * (K - len(alt))])
            r = orc.rows(p, q, k, v, lmk, [rows[i]], mode="given", sel_in=sel_in, w_in=w_in,
                         decode=decode)
            if alt == got:
                exp_out[i], exp_lse[i], exp_w[i] = r["out"][0], r["lse"][0], w_in[0]
                if exp_wfin is not None:
                    exp_wfin[i] = r["wfin"][0]
    valid = gpu["sel"] >= 0
    assert (np.isneginf(gpu["w"]) == ~valid).all(), "chunk_w padding must be -inf"
    dw = np.abs(np.where(valid, gpu["w"], 0.0) - np.where(valid, exp_w, 0.0))
    w_tol = tol["w"] * np.maximum(1.0, np.abs(np.where(valid, exp_w, 0.0)))
    assert (dw <= w_tol).all(), f"chunk_w error {dw.max():.3g}"
    out = gpu["out"].astype(np.float64)
    assert np.isfinite(out).all(), "non-finite output"
    err = np.abs(out - exp_out)
    assert err.max() <= tol["out_max"], f"out max-abs error {err.max():.3g}"
    assert err.mean() <= tol["out_mean"], f"out mean-abs error {err.mean():.3g}"
    le = np.abs(gpu["lse"] - exp_lse) / np.maximum(1.0, np.abs(exp_lse))
    assert le.max() <= tol["lse"], f"lse error {le.max():.3g}"
    if gpu.get("lse_lmk") is not None:
        a, b = gpu["lse_lmk"], ref["lse_lmk"]
        assert (np.isneginf(a) == np.isneginf(b)).all(), "lse_lmk -inf pattern"
        fin = np.isfinite(b)
        e = np.abs(a[fin] - b[fin]) / np.maximum(1.0, np.abs(b[fin]))
        assert e.size == 0 or e.max() <= tol["lse_lmk"], f"lse_lmk error {e.max():.3g}"
    if exp_wfin is not None:
        e = np.abs(gpu["wfin"] - exp_wfin)
        assert e.max() <= tol["wfin"], f"w_final error {e.max():.3g}"
    return dict(rows=n, near_ties=near_ties, out_max=float(err.max()),
                out_mean=float(err.mean()))


def sample_rows(B, Hq, L, C, n, seed):
    """Seeded sample of flat prefill rows that always includes chunk-boundary
    positions, rows in chunk 0, rows with few completed chunks and the last
    row of every head."""
    rng = np.random.default_rng(seed)
    heads = rng.integers(0, B * Hq, size=n)
    t = rng.integers(0, L, size=n)
    special = [0, 1, C - 1, C, C + 1, 2 * C - 1, 3 * C, L - 1, L - C, L - C - 1, L // 2]
    special = [x for x in special if 0 <= x < L]
    t[: len(special)] = special
    rows = heads.astype(np.int64) * L + t
    last = np.arange(B * Hq, dtype=np.int64) * L + (L - 1)
    return np.unique(np.concatenate([rows, last]))

"""Pins for the CPU oracle: checks against what the pages and mathematics fix.

Each pin takes an ``oracle.Oracle`` and raises AssertionError when the
oracle's result disagrees with a value fixed independently of the oracle's
code: hand-derived numbers, closed forms written as one dense matrix
expression in numpy, textbook causal attention, or a library primitive.
``test_oracle_pins.py`` runs them on the real oracle; ``test_oracle_mutants.py``
runs them on deliberately broken copies of it and requires each copy to fail
at least one pin.

Passages (pages on HiLS attention):
  [MC] model card "HiLS-Attention", section "What HiLS-Attention is";
  [AW] aiweekly.co article on HiLS, paragraph on the mechanism;
  [KR] molayo1419.me article, sections "Core idea" and "Hardware-efficient kernel".
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

from oracle import Problem

_GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_cases.json")


def _golden(name):
    with open(_GOLDEN) as f:
        return json.load(f)[name]


def _rng(seed):
    return np.random.default_rng(seed)


def _f32(*shape, rng, scale=1.0):
    return (scale * rng.standard_normal(shape)).astype(np.float32)


def _lse(x, axis=-1):
    m = np.max(x, axis=axis, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    with np.errstate(divide="ignore"):
        return np.squeeze(m, axis) + np.log(np.sum(np.exp(x - m), axis=axis))


def causal_attention(q, k, v, scale):
    """Textbook causal softmax attention for one head: q, k, v [L, d] fp64."""
    L = q.shape[0]
    X = scale * q @ k.T
    X = np.where(np.arange(L)[None, :] <= np.arange(L)[:, None], X, -np.inf)
    lse = _lse(X)
    return np.exp(X - lse[:, None]) @ v, lse


def all_selected_closed_form(q, k, v, lmk, C, scale, qs=None):
    """HiLS output when every completed chunk is selected, written as ONE
    masked softmax over keys ([MC]: inter-chunk softmax times intra-chunk
    softmax): key j of a completed chunk c gets logit
    scale*<q,k_j> + s_c - lse_c with s_c = scale*<q, lmk_c> and lse_c the
    log-sum-exp of chunk c's token logits; own-chunk keys (j <= t) keep their
    token logit.  q, k, v [L, d], lmk [L//C, d] fp64 for one head; qs, when
    given, replaces q in the landmark logits s_c only (Q-Cal)."""
    L = q.shape[0]
    nfull = L // C
    X = scale * q @ k.T                                # [L, L]
    S = scale * (q if qs is None else qs) @ lmk.T      # [L, nfull]
    chunk_lse = _lse(X[:, :nfull * C].reshape(L, nfull, C), axis=2) if nfull else np.zeros((L, 0))
    t = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    cj = j // C
    own = t // C
    bias = np.zeros((L, L))
    completed = cj < own
    cj_clip = np.minimum(cj, max(nfull - 1, 0))
    if nfull:
        bias = np.where(completed, np.take_along_axis(S, np.broadcast_to(cj_clip, (L, L)), 1)
                        - np.take_along_axis(chunk_lse, np.broadcast_to(cj_clip, (L, L)), 1), 0.0)
    allowed = completed | ((cj == own) & (j <= t))
    Z = np.where(allowed, X + bias, -np.inf)
    lse = _lse(Z)
    return np.exp(Z - lse[:, None]) @ v, lse


def block_sparse_exact_mass(q, k, v, C, scale, topk):
    """The naive selector of [MC]: rank completed chunks by their exact mass
    (log-sum-exp of the chunk's token logits), keep the top-k, and run plain
    softmax attention over the keys of those chunks plus the causal own chunk."""
    L = q.shape[0]
    X = scale * q @ k.T
    nfull = L // C
    out = np.empty_like(q)
    lse = np.empty(L)
    for t in range(L):
        own = t // C
        mass = np.array([_lse(X[t, c * C:(c + 1) * C]) for c in range(own)])
        keep = np.argsort(-mass, kind="stable")[:topk] if own else np.array([], int)
        mask = np.zeros(L, bool)
        for c in keep:
            mask[c * C:(c + 1) * C] = True
        mask[own * C:t + 1] = True
        z = np.where(mask, X[t], -np.inf)
        lse[t] = _lse(z)
        out[t] = np.exp(z - lse[t]) @ v
    assert nfull >= 0
    return out, lse


# ----------------------------------------------------------------------------------------
# pins


def pin_landmark_logit_and_normaliser(orc):
    """Hand values (tests/golden/hand_cases.json "landmark_logits"): d=4
    (scale 1/2), q_t = (2,0,0,0), landmarks (3,0,0,0) and (1,0,0,0) give
    logits 3 and 1 [KR step 1]; the inter-chunk normaliser is log(e^3 + e^1)
    [MC]."""
    g = _golden("landmark_logits")
    d, C, L, t = g["d"], g["C"], g["L"], g["row"]
    p = Problem(B=1, Hq=1, Hkv=1, L=L, d=d, C=C, topk=g["topk"], scale=1 / math.sqrt(d))
    q = np.zeros((1, 1, L, d), np.float32)
    q[0, 0, t] = g["q_row"]
    kv = np.zeros((1, 1, L, d), np.float32)
    lmk = np.array(g["landmarks"], np.float32).reshape(1, 1, L // C, d)
    r = orc.rows(p, q, kv, kv, lmk, [t])
    assert r["sel"][0].tolist() == g["expect_sel"], r["sel"]
    assert np.allclose(r["w"][0], g["expect_logits"], rtol=0, atol=1e-15), r["w"]
    assert abs(r["lse_lmk"][0] - g["expect_lse_lmk"]) < 1e-14, r["lse_lmk"]
    s = orc.scores(p, q, lmk, [t])
    assert s.shape == (1, L // C)
    assert np.allclose(s[0, :2], g["expect_logits"], rtol=0, atol=1e-15) and s[0, 2] == -np.inf, s


def pin_topk_planted_ties(orc):
    """Hand values (tests/golden/hand_cases.json "planted_ties"): with q = e_0
    and landmark first coordinates (0.1, 0.5, 0.5, 0.9, 0.5, 0.2) the top-2 are
    {3, 1} and the top-3 {3, 1, 2}: equal scores go to the lower chunk index;
    the selection is reported in ascending chunk order ([MC]: the top-k
    chunks are kept)."""
    g = _golden("planted_ties")
    d, C, L, t = g["d"], g["C"], g["L"], g["row"]
    vals = g["landmark_first_coord"]
    for topk_s, want in g["expect"].items():
        topk = int(topk_s)
        p = Problem(B=1, Hq=1, Hkv=1, L=L, d=d, C=C, topk=topk, scale=1 / math.sqrt(d))
        q = np.zeros((1, 1, L, d), np.float32)
        q[0, 0, t, 0] = 1.0  # own chunk t // C, completed chunks 0..len(vals)-1
        lmk = np.zeros((1, 1, L // C, d), np.float32)
        lmk[0, 0, :len(vals), 0] = vals
        kv = np.zeros((1, 1, L, d), np.float32)
        r = orc.rows(p, q, kv, kv, lmk, [t])
        assert r["sel"][0].tolist() == want, (topk, r["sel"][0])


def pin_zero_query_closed_form(orc):
    """Closed form: with q = 0 every token and landmark logit is 0, so all
    chunks tie and the lowest indices are selected; a full chunk has log mass
    log C and the own chunk log(r+1) (r = t mod C).  Fusion [AW] then gives
    out_t = (sum_{c in S} mean(V_c) + sum_{own keys} v_j) / (|S| + r + 1),
    lse_t = log(|S| + r + 1), lse_lmk = log(n_c).  Ragged L exercises a
    partial last chunk."""
    rng = _rng(3)
    L, C, d, topk = 37, 8, 5, 2
    p = Problem(B=1, Hq=1, Hkv=1, L=L, d=d, C=C, topk=topk, scale=1 / math.sqrt(d))
    q = np.zeros((1, 1, L, d), np.float32)
    k = _f32(1, 1, L, d, rng=rng)
    v = _f32(1, 1, L, d, rng=rng)
    lmk = _f32(1, 1, L // C, d, rng=rng)
    r = orc.rows(p, q, k, v, lmk, np.arange(L))
    V = v[0, 0].astype(np.float64)
    for t in range(L):
        n_c, rr = t // C, t % C
        S = list(range(min(topk, n_c)))
        assert r["sel"][t].tolist() == S + [-1] * (topk - len(S)), (t, r["sel"][t])
        num = sum(V[c * C:(c + 1) * C].mean(0) for c in S) + V[n_c * C:t + 1].sum(0)
        den = len(S) + rr + 1
        assert np.allclose(r["out"][t], num / den, rtol=0, atol=1e-12), t
        assert abs(r["lse"][t] - math.log(den)) < 1e-12, t
        want = math.log(n_c) if n_c else -math.inf
        assert r["lse_lmk"][t] == want or abs(r["lse_lmk"][t] - want) < 1e-12, t
        assert np.allclose(r["wfin"][t][:len(S)], 1 / den) and abs(r["wfin"][t][-1] - (rr + 1) / den) < 1e-12


def pin_first_chunk_is_causal_attention(orc):
    """One chunk: rows t < C have no completed chunk, so HiLS reduces to
    standard causal softmax attention [KR step 2] (own chunk only)."""
    rng = _rng(5)
    L, C, d = 24, 32, 6  # L < C: a single partial chunk
    p = Problem(B=1, Hq=2, Hkv=1, L=L, d=d, C=C, topk=3, scale=1 / math.sqrt(d))
    q = _f32(1, 2, L, d, rng=rng)
    k = _f32(1, 1, L, d, rng=rng)
    v = _f32(1, 1, L, d, rng=rng)
    lmk = np.zeros((1, 1, 0, d), np.float32)
    r = orc.rows(p, q, k, v, lmk, np.arange(2 * L))
    for h in range(2):
        o, lse = causal_attention(q[0, h].astype(float), k[0, 0].astype(float),
                                  v[0, 0].astype(float), p.scale)
        assert np.allclose(r["out"][h * L:(h + 1) * L], o, rtol=0, atol=1e-12)
        assert np.allclose(r["lse"][h * L:(h + 1) * L], lse, rtol=0, atol=1e-12)
        assert (r["sel"][h * L:(h + 1) * L] == -1).all()


def pin_all_selected_closed_form(orc):
    """top-k >= number of completed chunks: the output must equal the dense
    closed form sum_c softmax(landmark logits + own log mass)_c * attn_c
    ([MC] factorisation, [AW] fusion), evaluated as one masked matrix softmax.
    GQA (4 query heads on 2 KV heads), batch 2, ragged last chunk."""
    rng = _rng(7)
    B, Hq, Hkv, L, d, C = 2, 4, 2, 45, 8, 4
    p = Problem(B=B, Hq=Hq, Hkv=Hkv, L=L, d=d, C=C, topk=L // C + 1, scale=1 / math.sqrt(d))
    q = _f32(B, Hq, L, d, rng=rng)
    k = _f32(B, Hkv, L, d, rng=rng)
    v = _f32(B, Hkv, L, d, rng=rng)
    lmk = _f32(B, Hkv, L // C, d, rng=rng, scale=0.7)
    r = orc.rows(p, q, k, v, lmk, np.arange(B * Hq * L))
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            o, lse = all_selected_closed_form(q[b, h].astype(float), k[b, g].astype(float),
                                              v[b, g].astype(float), lmk[b, g].astype(float),
                                              C, p.scale)
            s = slice((b * Hq + h) * L, (b * Hq + h + 1) * L)
            assert np.allclose(r["out"][s], o, rtol=0, atol=1e-11), (b, h)
            assert np.allclose(r["lse"][s], lse, rtol=0, atol=1e-11), (b, h)


def pin_exact_mass_is_block_sparse_attention(orc):
    """Exact-mass scores ([MC]'s naive selector): with landmark logits replaced
    by each chunk's exact log mass, fusion reproduces plain softmax attention
    restricted to the selected chunks plus the own chunk; with top-k covering
    all completed chunks it is full causal attention."""
    rng = _rng(11)
    L, C, d = 50, 5, 6
    q = _f32(1, 1, L, d, rng=rng)
    k = _f32(1, 1, L, d, rng=rng)
    v = _f32(1, 1, L, d, rng=rng)
    lmk = np.zeros((1, 1, L // C, d), np.float32)
    Q, K, V = (x[0, 0].astype(float) for x in (q, k, v))
    sc = 1 / math.sqrt(d)
    full = Problem(B=1, Hq=1, Hkv=1, L=L, d=d, C=C, topk=L // C, scale=sc)
    r = orc.rows(full, q, k, v, lmk, np.arange(L), mode="exact_mass")
    o, lse = causal_attention(Q, K, V, sc)
    assert np.allclose(r["out"], o, rtol=0, atol=1e-11)
    assert np.allclose(r["lse"], lse, rtol=0, atol=1e-11)
    for topk in (1, 3):
        p = Problem(B=1, Hq=1, Hkv=1, L=L, d=d, C=C, topk=topk, scale=sc)
        r = orc.rows(p, q, k, v, lmk, np.arange(L), mode="exact_mass")
        o, lse = block_sparse_exact_mass(Q, K, V, C, sc, topk)
        assert np.allclose(r["out"], o, rtol=0, atol=1e-11), topk
        assert np.allclose(r["lse"], lse, rtol=0, atol=1e-11), topk


def pin_constant_key_chunk(orc):
    """Closed form: a chunk whose keys all equal kappa has log mass
    scale*<q,kappa> + log(n) over its n visible keys and output mean(V).
    With the selection {c} given (logit s), lse = log(e^s + e^{lse_own}) and
    out = w_c mean(V_c) + w_own mean(V_own)."""
    rng = _rng(13)
    L, C, d = 24, 8, 4
    sc = 0.5
    p = Problem(B=1, Hq=1, Hkv=1, L=L, d=d, C=C, topk=1, scale=sc)
    q = _f32(1, 1, L, d, rng=rng)
    k = _f32(1, 1, L, d, rng=rng)
    v = _f32(1, 1, L, d, rng=rng)
    kappa_own = np.array([0.5, -1.0, 0.25, 2.0], np.float32)
    k[0, 0, 16:24] = kappa_own
    k[0, 0, 0:8] = np.array([1.0, 0.0, -0.5, 0.0], np.float32)
    t = 21  # own chunk 2 with r = 5 -> 6 visible keys
    s = 0.75
    r = orc.rows(p, q, k, v, np.zeros((1, 1, 3, d), np.float32), [t], mode="given",
                 sel_in=[[0]], w_in=[[s]])
    qt = q[0, 0, t].astype(float)
    lse_own = sc * qt @ kappa_own.astype(float) + math.log(6)
    lse = math.log(math.exp(s) + math.exp(lse_own))
    wc, wo = math.exp(s - lse), math.exp(lse_own - lse)
    V = v[0, 0].astype(float)
    want = wc * V[0:8].mean(0) + wo * V[16:22].mean(0)
    assert abs(r["lse"][0] - lse) < 1e-12
    assert np.allclose(r["out"][0], want, rtol=0, atol=1e-12)
    assert np.allclose(r["wfin"][0], [wc, wo], rtol=0, atol=1e-14)


def pin_weights_and_lse_bounds(orc):
    """Fusion weights form a distribution (sum to 1); lse lies between the
    largest fused logit and that plus log(#attended chunks)."""
    rng = _rng(17)
    B, Hq, Hkv, L, d, C, topk = 1, 2, 1, 96, 8, 8, 3
    p = Problem(B=B, Hq=Hq, Hkv=Hkv, L=L, d=d, C=C, topk=topk, scale=1 / math.sqrt(d))
    q = _f32(B, Hq, L, d, rng=rng)
    k = _f32(B, Hkv, L, d, rng=rng)
    v = _f32(B, Hkv, L, d, rng=rng)
    lmk = _f32(B, Hkv, L // C, d, rng=rng)
    r = orc.rows(p, q, k, v, lmk, np.arange(B * Hq * L))
    assert np.allclose(r["wfin"].sum(1), 1.0, rtol=0, atol=1e-12)
    assert (r["wfin"] >= 0).all()
    nsel = (r["sel"] >= 0).sum(1)
    wmax = np.where(r["sel"] >= 0, r["w"], -np.inf).max(1)
    own_logit = r["lse"] + np.log(r["wfin"][:, -1])
    gmax = np.maximum(wmax, own_logit)
    assert (r["lse"] >= gmax - 1e-12).all()
    assert (r["lse"] <= gmax + np.log(nsel + 1) + 1e-12).all()
    n_c = np.tile(np.arange(L) // C, B * Hq)
    assert (np.isfinite(r["lse_lmk"]) == (n_c > 0)).all()
    assert (nsel == np.minimum(n_c, topk)).all()


def pin_invariances(orc):
    """Permuting the keys and values inside a completed chunk leaves every
    later row unchanged (a chunk is a set [KR step 2]); the output is linear
    in V for a fixed selection."""
    rng = _rng(19)
    L, C, d, topk = 64, 8, 6, 2
    p = Problem(B=1, Hq=1, Hkv=1, L=L, d=d, C=C, topk=topk, scale=1 / math.sqrt(d))
    q = _f32(1, 1, L, d, rng=rng)
    k = _f32(1, 1, L, d, rng=rng)
    v = _f32(1, 1, L, d, rng=rng)
    lmk = _f32(1, 1, L // C, d, rng=rng)
    rows = np.arange(24, L)
    base = orc.rows(p, q, k, v, lmk, rows)
    perm = rng.permutation(C)
    k2, v2 = k.copy(), v.copy()
    k2[0, 0, 8:16] = k[0, 0, 8 + perm]
    v2[0, 0, 8:16] = v[0, 0, 8 + perm]
    r2 = orc.rows(p, q, k2, v2, lmk, rows)
    assert (r2["sel"] == base["sel"]).all()
    assert np.allclose(r2["out"], base["out"], rtol=0, atol=1e-12)
    va = _f32(1, 1, L, d, rng=rng)
    comb = (2.0 * v.astype(np.float64) - 0.5 * va.astype(np.float64)).astype(np.float32)
    ra = orc.rows(p, q, k, va, lmk, rows)
    rc = orc.rows(p, q, k, comb, lmk, rows)
    assert np.allclose(rc["out"], 2.0 * base["out"] - 0.5 * ra["out"], rtol=0, atol=1e-5)


def pin_decode_is_last_prefill_row(orc):
    """Decode: the cache of length N holds the new token, so the decode output
    equals the prefill output of row N-1 (for every head, GQA)."""
    rng = _rng(23)
    B, Hq, Hkv, N, d, C, topk = 2, 4, 2, 70, 8, 8, 3
    p = Problem(B=B, Hq=Hq, Hkv=Hkv, L=N, d=d, C=C, topk=topk, scale=1 / math.sqrt(d))
    q = _f32(B, Hq, N, d, rng=rng)
    k = _f32(B, Hkv, N, d, rng=rng)
    v = _f32(B, Hkv, N, d, rng=rng)
    lmk = _f32(B, Hkv, N // C, d, rng=rng)
    rows = [(b * Hq + h) * N + N - 1 for b in range(B) for h in range(Hq)]
    pre = orc.rows(p, q, k, v, lmk, rows)
    dec = orc.decode(p, np.ascontiguousarray(q[:, :, N - 1]), k, v, lmk)
    for key in ("sel", "w", "out", "lse", "lse_lmk", "wfin"):
        assert np.array_equal(pre[key], dec[key]), key


def pin_bf16_bits_widen_exactly(orc):
    """bf16 inputs are read as raw bits and widened exactly: feeding the same
    values as fp32 gives identical results."""
    rng = _rng(29)
    L, d, C = 40, 8, 8
    p = Problem(B=1, Hq=1, Hkv=1, L=L, d=d, C=C, topk=2, scale=1 / math.sqrt(d))
    arrs = [_f32(1, 1, L, d, rng=rng) for _ in range(3)] + [_f32(1, 1, L // C, d, rng=rng)]
    bits = [(a.view(np.uint32) >> 16).astype(np.uint16) for a in arrs]
    wide = [(b.astype(np.uint32) << 16).view(np.float32) for b in bits]
    r1 = orc.rows(p, *bits, np.arange(L))
    r2 = orc.rows(p, *wide, np.arange(L))
    for key in ("sel", "out", "lse"):
        assert np.array_equal(r1[key], r2[key]), key


def pin_union_is_set_union(orc):
    """Chunk union of a group [KR "hardware-efficient kernel"]: equals
    Python's set union of the rows' selections and own chunks."""
    rng = _rng(31)
    L, C, topk, M = 200, 8, 3, 16
    sel = rng.integers(-1, L // C, size=(2 * L, topk)).astype(np.int32)
    for head in range(2):
        for g in range((L + M - 1) // M):
            want = set()
            for t in range(g * M, min((g + 1) * M, L)):
                want |= {int(c) for c in sel[head * L + t] if c >= 0}
                want.add(t // C)
            got = orc.union(L, C, topk, M, head, g, sel)
            assert got.tolist() == sorted(want), (head, g)


def pin_paged_decode_is_dense_decode(orc):
    """A paged cache is another layout of the dense cache: the decode step
    over pages in shuffled order (with unused pages, unused table columns and
    the tail of a partial last page all NaN) equals the decode over the dense
    cache exactly; two sequences sharing every page equal two sequences with
    identical dense caches."""
    rng = _rng(37)
    B, Hq, Hkv, N, d, C, topk = 2, 4, 2, 70, 8, 8, 3
    npg = -(-N // C)
    p = Problem(B=B, Hq=Hq, Hkv=Hkv, L=N, d=d, C=C, topk=topk, scale=1 / math.sqrt(d))
    q = _f32(B, Hq, d, rng=rng)
    k = _f32(B, Hkv, N, d, rng=rng)
    v = _f32(B, Hkv, N, d, rng=rng)
    lmk = _f32(B, Hkv, N // C, d, rng=rng)
    num_pages = B * npg + 3
    perm = rng.permutation(num_pages)[:B * npg]
    table = np.full((B, npg + 2), -1, np.int64)
    kp = np.full((num_pages, Hkv, C, d), np.nan, np.float32)
    vp = np.full((num_pages, Hkv, C, d), np.nan, np.float32)
    for b in range(B):
        for c in range(npg):
            page = int(perm[b * npg + c])
            table[b, c] = page
            n = min(C, N - c * C)
            # the page holds [Hkv][C][d]: head-major, the chunk's tokens in order
            kp[page, :, :n] = k[b, :, c * C:c * C + n]
            vp[page, :, :n] = v[b, :, c * C:c * C + n]
    dense = orc.decode(p, q, k, v, lmk)
    paged = orc.decode_paged(p, q, kp, vp, table, lmk)
    for key in ("sel", "w", "out", "lse", "lse_lmk", "wfin"):
        assert np.array_equal(dense[key], paged[key]), key
    # shared pages: sequence 1 reads sequence 0's pages
    shared = table.copy()
    shared[1] = table[0]
    k2, v2, lmk2 = k.copy(), v.copy(), lmk.copy()
    k2[1], v2[1], lmk2[1] = k[0], v[0], lmk[0]
    dense2 = orc.decode(p, q, k2, v2, lmk2)
    paged2 = orc.decode_paged(p, q, kp, vp, shared, lmk2)
    for key in ("sel", "out", "lse"):
        assert np.array_equal(dense2[key], paged2[key]), key
    assert np.isfinite(paged["out"]).all()


def pin_hope_rotation_properties(orc):
    """HoPE [KR "Engineering details", HoPE]: on the rotated pairs a rotary
    embedding, on the others the identity.  Checked against what rotations
    fix: norms are kept; position 0 and n_rope_pairs = 0 are the identity;
    the NoPE half of the pairs is untouched; rotating by t1 then by t2 equals
    rotating by t1 + t2; the dot product of a rotated query and key depends
    on their positions only through t - s; one pair at one position equals a
    hand-computed 2-d rotation."""
    from oracle import hope
    rng = _rng(41)
    d, n = 16, 9
    x = rng.standard_normal((2, n, d))
    pos = rng.integers(0, 5000, size=n)
    y = hope(x.astype(np.float32), pos, 5, 500.0)
    x32 = x.astype(np.float32).astype(np.float64)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x32, axis=-1), rtol=1e-12)
    assert np.array_equal(hope(x32.astype(np.float32), np.zeros(n), 8, 500.0), x32)
    assert np.array_equal(hope(x32.astype(np.float32), pos, 0, 500.0), x32)
    nope = [i for i in range(d // 2) if i >= 5]
    for i in nope:
        assert np.array_equal(y[..., i], x32[..., i]) and np.array_equal(y[..., i + d // 2], x32[..., i + d // 2])
    # group property, with the rotation written out as a matrix per pair
    t1, t2 = 1234, 777
    def rot(v, t, pairs, base):
        out = v.copy()
        for i in range(pairs):
            th = base ** (-2.0 * i / d) * t
            m = np.array([[math.cos(th), -math.sin(th)], [math.sin(th), math.cos(th)]])
            u = np.stack([v[..., i], v[..., i + d // 2]], -1) @ m.T
            out[..., i], out[..., i + d // 2] = u[..., 0], u[..., 1]
        return out
    v = rng.standard_normal((n, d)).astype(np.float32)
    a1 = hope(v, np.full(n, t1 + t2), 6, 10000.0)
    a2 = rot(rot(v.astype(np.float64), t1, 6, 10000.0), t2, 6, 10000.0)
    assert np.allclose(a1, a2, atol=1e-9)
    # relative positions: <R(t) q, R(s) k> is a function of t - s
    q = rng.standard_normal((1, d)).astype(np.float32)
    k = rng.standard_normal((1, d)).astype(np.float32)
    dots = [float((hope(q, [t], 8, 10000.0) @ hope(k, [s], 8, 10000.0).T)[0, 0])
            for t, s in ((50, 20), (1030, 1000), (900030, 900000))]
    assert np.allclose(dots, dots[0], atol=1e-8)
    # hand value: d = 4, pair 0 has theta 1; x = (1, 0, 0, 0) at position t -> (cos t, 0, sin t, 0)
    h = hope(np.array([[1.0, 0.0, 0.0, 0.0]], np.float32), [3], 1, 10000.0)
    assert np.allclose(h, [[math.cos(3.0), 0.0, math.sin(3.0), 0.0]], atol=1e-15)


def pin_qcal_scoring_query(orc):
    """Q-Cal [KR "Engineering details", Q-Cal]: the offset W_up W_down h
    changes the query of the chunk scores only.  A hand value of the offset;
    no offset reproduces the plain oracle; with every chunk selected the
    output is the dense closed form whose chunk logits use the calibrated
    query and whose token logits use the plain one; an offset along one
    landmark makes k = 1 pick that chunk on every row that can."""
    from oracle import qcal_query
    # hand value: D = 2, r = 1, d = 2, h_t = (1, 1): z = 1 + 2 = 3, dq = (3*3, 4*3)
    qs = qcal_query(np.zeros((1, 1, 1, 2), np.float32), np.ones((1, 1, 2)),
                    np.array([[1.0, 2.0]]), np.array([[[3.0], [4.0]]]))
    assert np.array_equal(qs.reshape(-1), np.array([9.0, 12.0], np.float32))
    # the fixed fp32 order: 1 + 2^-24 + 2^-24 is 1 summed left to right (each
    # partial sum rounds back to 1), but 1 + 2^-23 summed the other way round
    one = np.float32(1.0)
    eps = np.float32(2.0 ** -24)
    qs = qcal_query(np.zeros((1, 1, 1, 1), np.float32), np.array([[[1.0, 1.0, 1.0]]]),
                    np.array([[one, eps, eps]]), np.array([[[1.0]]]))
    assert qs.reshape(-1)[0] == one
    qs = qcal_query(np.zeros((1, 1, 1, 1), np.float32), np.array([[[1.0, 1.0, 1.0]]]),
                    np.array([[eps, eps, one]]), np.array([[[1.0]]]))
    assert qs.reshape(-1)[0] == np.float32(1.0 + 2.0 ** -23)
    # a bf16 query gets a bf16 scoring query (spacing 2^-7 above 1): 1 + 2^-9
    # is below the halfway point 1 + 2^-8 and rounds to 1, 1 + 3*2^-9 rounds up
    import torch
    qb = torch.zeros((1, 1, 2, 1), dtype=torch.bfloat16) + 1.0
    qs = qcal_query(qb, np.ones((1, 2, 1)), np.array([[1.0]]),
                    np.array([[[2.0 ** -9]]]))
    assert np.array_equal(qs.reshape(-1), np.array([1.0, 1.0], np.float32))
    qs = qcal_query(qb, np.ones((1, 2, 1)), np.array([[3.0]]), np.array([[[2.0 ** -9]]]))
    assert np.array_equal(qs.reshape(-1), np.array([1.0 + 2.0 ** -7] * 2, np.float32))
    rng = _rng(43)
    B, Hq, Hkv, L, d, C, D, r = 1, 4, 2, 45, 8, 4, 12, 3
    q = _f32(B, Hq, L, d, rng=rng)
    k = _f32(B, Hkv, L, d, rng=rng)
    v = _f32(B, Hkv, L, d, rng=rng)
    lmk = _f32(B, Hkv, L // C, d, rng=rng, scale=0.7)
    h = rng.standard_normal((B, L, D))
    wd = rng.standard_normal((r, D)) * 0.3
    wu = rng.standard_normal((Hq, d, r)) * 0.3
    rows = np.arange(B * Hq * L)
    p = Problem(B=B, Hq=Hq, Hkv=Hkv, L=L, d=d, C=C, topk=3, scale=1 / math.sqrt(d))
    plain = orc.rows(p, q, k, v, lmk, rows)
    same = orc.rows_qcal(p, q, k, v, lmk, qcal_query(q, h, wd, 0 * wu), rows)
    for key in ("sel", "w", "out", "lse", "lse_lmk"):
        assert np.array_equal(plain[key], same[key]), key
    pa = Problem(B=B, Hq=Hq, Hkv=Hkv, L=L, d=d, C=C, topk=L // C + 1, scale=1 / math.sqrt(d))
    qs = qcal_query(q, h, wd, wu)
    res = orc.rows_qcal(pa, q, k, v, lmk, qs, rows)
    for hq in range(Hq):
        g = hq // (Hq // Hkv)
        o, lse = all_selected_closed_form(q[0, hq].astype(float), k[0, g].astype(float),
                                          v[0, g].astype(float), lmk[0, g].astype(float), C,
                                          pa.scale, qs=qs[0, hq].astype(float))
        sl = slice(hq * L, (hq + 1) * L)
        assert np.allclose(res["out"][sl], o, rtol=0, atol=1e-11), hq
        assert np.allclose(res["lse"][sl], lse, rtol=0, atol=1e-11), hq
    star = 2
    pull = qs.copy()
    for hq in range(Hq):
        pull[0, hq] += 40.0 * lmk[0, hq // (Hq // Hkv), star] / np.linalg.norm(lmk[0, hq // (Hq // Hkv), star])
    p1 = Problem(B=B, Hq=Hq, Hkv=Hkv, L=L, d=d, C=C, topk=1, scale=1 / math.sqrt(d))
    got = orc.rows_qcal(p1, q, k, v, lmk, pull, rows)
    t = rows % L
    can = t // C > star
    assert (got["sel"][can, 0] == star).all()


def pin_hope_split_rule(orc):
    """The HoPE split [KR "Engineering details", HoPE]: pairs whose wavelength
    fits the pre-training length are rotated.  Hand values: d = 128, base
    10^4, window 4096 -- the wavelength 2 pi 10^4^(i/64) is about 4080 at
    i = 45 and 4710 at i = 46, so 46 pairs; base 5*10^5, window 65536 --
    about 63 900 at i = 45 and 78 400 at i = 46, so 46 again; a window below
    2 pi rotates nothing, exactly 2 pi rotates pair 0; a window beyond the
    longest wavelength rotates every pair."""
    from oracle import rope_pairs
    assert 4000 < 2 * math.pi * 1e4 ** (45 / 64) < 4096 < 2 * math.pi * 1e4 ** (46 / 64) < 4800
    assert rope_pairs(128, 1e4, 4096) == 46
    assert 63000 < 2 * math.pi * 5e5 ** (45 / 64) < 65536 < 2 * math.pi * 5e5 ** (46 / 64)
    assert rope_pairs(128, 5e5, 65536) == 46
    assert rope_pairs(64, 1e4, 6.0) == 0
    assert rope_pairs(64, 1e4, 2 * math.pi) == 1
    assert rope_pairs(64, 1e4, 1e12) == 32


ALL_PINS = [
    pin_landmark_logit_and_normaliser,
    pin_topk_planted_ties,
    pin_zero_query_closed_form,
    pin_first_chunk_is_causal_attention,
    pin_all_selected_closed_form,
    pin_exact_mass_is_block_sparse_attention,
    pin_constant_key_chunk,
    pin_weights_and_lse_bounds,
    pin_invariances,
    pin_decode_is_last_prefill_row,
    pin_bf16_bits_widen_exactly,
    pin_union_is_set_union,
    pin_paged_decode_is_dense_decode,
    pin_hope_rotation_properties,
    pin_qcal_scoring_query,
    pin_hope_split_rule,
]

"""The backward-pass oracle (oracle/backward.py) against its pins.

Its forward is a second, independent statement of the HiLS forward (plain
PyTorch fp64, per row) and must equal the C oracle's; its gradients are
torch.autograd's and must equal central finite differences of that forward
(torch.autograd.gradcheck) on inputs whose top-k choice has a margin, and
closed forms for the gradient of lse; keys, values and landmarks that no row
uses get exactly zero gradient."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob


def inputs(B, Hq, Hkv, L, d, C, seed, scale_lmk=1.0):
    rng = np.random.default_rng(seed)
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    return f(B, Hq, L, d), f(B, Hkv, L, d), f(B, Hkv, L, d), (scale_lmk * f(B, Hkv, L // C, d)).astype(np.float32)


def margin_ok(p, q, lmk, margin=1e-3):
    """Every row's k-th and (k+1)-th fp32 scores differ by more than margin."""
    B, Hq, L, d = q.shape
    G = Hq // lmk.shape[1]
    for b in range(B):
        for hq in range(Hq):
            for t in range(L):
                n = t // p.C
                if n <= p.topk:
                    continue
                s = np.sort((p.scale * (lmk[b, hq // G, :n].astype(np.float64) @ q[b, hq, t])).astype(np.float32))[::-1]
                if s[p.topk - 1] - s[p.topk] <= margin:
                    return False
    return True


@pytest.mark.parametrize("B,Hq,Hkv,L,d,C,topk", [(1, 2, 1, 40, 4, 8, 2), (2, 4, 2, 37, 8, 4, 3),
                                                  (1, 2, 2, 19, 4, 4, 8)])
def test_forward_equals_c_oracle(B, Hq, Hkv, L, d, C, topk):
    p = oracle.Problem(B=B, Hq=Hq, Hkv=Hkv, L=L, d=d, C=C, topk=topk, scale=1 / math.sqrt(d))
    q, k, v, lmk = inputs(B, Hq, Hkv, L, d, C, seed=L)
    out, lse, sels = ob.forward(p, *(torch.from_numpy(a).double() for a in (q, k, v, lmk)))
    ref = oracle.rows(p, q, k, v, lmk, np.arange(B * Hq * L))
    assert np.abs(out.numpy().reshape(-1, d) - ref["out"]).max() <= 1e-12
    assert np.abs(lse.numpy().reshape(-1) - ref["lse"]).max() <= 1e-12
    for r, s in enumerate(sels):
        want = [int(c) for c in ref["sel"][r] if c >= 0]
        assert s == want, r


def test_gradients_equal_finite_differences():
    B, Hq, Hkv, L, d, C, topk = 1, 2, 1, 24, 4, 4, 2
    p = oracle.Problem(B=B, Hq=Hq, Hkv=Hkv, L=L, d=d, C=C, topk=topk, scale=1 / math.sqrt(d))
    seed = 0
    while True:
        q, k, v, lmk = inputs(B, Hq, Hkv, L, d, C, seed, scale_lmk=2.0)
        if margin_ok(p, q, lmk):
            break
        seed += 1
    xs = [torch.from_numpy(a).double().requires_grad_(True) for a in (q, k, v, lmk)]

    def f(*ts):
        out, lse, _ = ob.forward(p, *ts)
        return out, lse
    assert torch.autograd.gradcheck(f, xs, eps=1e-6, atol=1e-6, rtol=1e-5)


def test_lse_gradient_closed_form():
    """With dout = 0 and dlse = 1: d lse_t / d s_c = w_c (the fusion weight),
    so dlmk_c = sum over rows that selected c of w_c * scale * q_t, and
    dq_t = scale * (sum_c w_c lmk_c + w_own * sum_j p_j k_j) over the own
    chunk's causal keys j with p = softmax of their logits; dv = 0.  The
    weights come from the C oracle's selected logits and lse."""
    B, Hq, Hkv, L, d, C, topk = 1, 4, 2, 33, 4, 4, 2
    p = oracle.Problem(B=B, Hq=Hq, Hkv=Hkv, L=L, d=d, C=C, topk=topk, scale=1 / math.sqrt(d))
    q, k, v, lmk = inputs(B, Hq, Hkv, L, d, C, seed=5)
    r = ob.backward(p, q, k, v, lmk, np.zeros((B, Hq, L, d)), np.ones((B, Hq, L)))
    ref = oracle.rows(p, q, k, v, lmk, np.arange(B * Hq * L))
    G = Hq // Hkv
    dlmk = np.zeros(lmk.shape)
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    for hq in range(Hq):
        hk = hq // G
        for t in range(L):
            row = hq * L + t
            qt = q[0, hq, t].astype(np.float64)
            lse = ref["lse"][row]
            for c, s in zip(ref["sel"][row], ref["w"][row]):
                if c < 0:
                    continue
                w = math.exp(s - lse)
                dlmk[0, hk, c] += w * p.scale * qt
                dq[0, hq, t] += w * p.scale * lmk[0, hk, c].astype(np.float64)
            oc = t // C
            keys = k[0, hk, oc * C:t + 1].astype(np.float64)
            x = p.scale * keys @ qt
            pj = np.exp(x - x.max())
            pj /= pj.sum()
            w_own = math.exp(np.log(np.exp(x - x.max()).sum()) + x.max() - lse)
            dq[0, hq, t] += w_own * p.scale * (pj @ keys)
            dk[0, hk, oc * C:t + 1] += w_own * p.scale * pj[:, None] * qt[None, :]
    assert np.abs(r["dlmk"] - dlmk).max() <= 1e-12
    assert np.abs(r["dq"] - dq).max() <= 1e-12
    assert np.abs(r["dk"] - dk).max() <= 1e-12
    assert not r["dv"].any()


def test_unused_inputs_get_no_gradient():
    """k = 1 over 10 chunks: landmarks of chunks no row selects, and keys and
    values of chunks no row attends, get exactly zero gradient."""
    B, Hq, Hkv, L, d, C, topk = 1, 1, 1, 80, 4, 8, 1
    p = oracle.Problem(B=B, Hq=Hq, Hkv=Hkv, L=L, d=d, C=C, topk=topk, scale=1 / math.sqrt(d))
    q, k, v, lmk = inputs(B, Hq, Hkv, L, d, C, seed=9)
    rng = np.random.default_rng(10)
    r = ob.backward(p, q, k, v, lmk, rng.standard_normal((B, Hq, L, d)), rng.standard_normal((B, Hq, L)))
    used = set()
    for t, s in enumerate(r["sel"]):
        used.update(s)
        used.add(t // C)
    chosen = {c for s in r["sel"] for c in s}
    for c in range(L // C):
        if c not in chosen:
            assert not r["dlmk"][0, 0, c].any(), c
        if c not in used:
            assert not r["dk"][0, 0, c * C:(c + 1) * C].any(), c
            assert not r["dv"][0, 0, c * C:(c + 1) * C].any(), c
    assert len(chosen) < L // C  # the case is not vacuous


@pytest.mark.parametrize("B,Hq,Hkv,L,d,C,topk,with_dlse", [(1, 2, 1, 40, 4, 8, 2, True),
                                                            (2, 4, 2, 37, 8, 4, 3, False),
                                                            (1, 2, 2, 19, 4, 4, 8, True)])
def test_explicit_formulas_equal_autograd(B, Hq, Hkv, L, d, C, topk, with_dlse):
    """The per-chunk backward formulas (the quantities a kernel would form)
    give autograd's gradients: GQA, a ragged last chunk, k >= n_c, with and
    without an lse gradient."""
    p = oracle.Problem(B=B, Hq=Hq, Hkv=Hkv, L=L, d=d, C=C, topk=topk, scale=1 / math.sqrt(d))
    q, k, v, lmk = inputs(B, Hq, Hkv, L, d, C, seed=L + 1)
    rng = np.random.default_rng(L + 2)
    dout = rng.standard_normal((B, Hq, L, d))
    dlse = rng.standard_normal((B, Hq, L)) if with_dlse else None
    a = ob.backward(p, q, k, v, lmk, dout, dlse)
    e = ob.backward_explicit(p, q, k, v, lmk, dout, dlse)
    for key in ("dq", "dk", "dv", "dlmk"):
        assert np.abs(a[key] - e[key]).max() <= 1e-12, key

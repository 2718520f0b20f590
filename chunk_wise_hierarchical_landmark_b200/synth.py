"""Seeded synthetic inputs for HiLS attention (shared by the CUDA path's tests,
the benchmark and the CPU oracle).

This module holds no part of the method's arithmetic: it only draws q, k, v
and landmark keys with the shapes and statistics of the workloads in
``workloads.py``.  Recipes:

* k, v ~ N(0, 1) i.i.d.
* q ~ N(0, 1) i.i.d., or a stationary AR(1) walk per head,
  q_t = rho * q_{t-1} + sigma * eps_t with rho = sqrt(1 - sigma^2), which keeps
  the N(0, 1) marginal while adjacent queries stay close (a raw random walk
  with step sigma would grow without bound over 10^5 steps).
* needle chunks: per KV head a random unit direction u_h and `needles`
  distinct random chunks whose keys are shifted by needle_amp * sqrt(d) * u_h.
* landmark keys: mean of the chunk's (shifted) keys + N(0, lmk_noise^2), one
  per complete chunk; lmk_noise == 0 draws them i.i.d. N(0, 1) instead.

All draws come from one torch.Generator seeded with the workload seed on the
requested device; values are produced in fp32 and rounded to the workload
dtype at the end.
"""
from __future__ import annotations

import math

import torch

from .workloads import Workload


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def _ar1(n_heads, L, d, sigma, g, device, block=64):
    """Stationary AR(1) walk of length L for n_heads independent heads, [n, L, d] fp32.

    Blocked evaluation of the linear recurrence: inside a block of `block`
    steps the walk is a lower-triangular Toeplitz combination of the
    innovations; the blocks are then chained through their carries."""
    rho = math.sqrt(1.0 - sigma * sigma)
    out = torch.empty((n_heads, L, d), dtype=torch.float32, device=device)
    T = block
    i = torch.arange(T, device=device, dtype=torch.float64)
    W = torch.where(i[:, None] >= i[None, :], rho ** (i[:, None] - i[None, :]),
                    torch.zeros((), dtype=torch.float64, device=device)).float()
    powers = (rho ** (i + 1)).float()  # rho^(i+1) for the carry term
    for h in range(n_heads):
        q0 = _randn((d,), g, device)
        eps = _randn((L, d), g, device) * sigma
        nb = (L + T - 1) // T
        pad = nb * T - L
        if pad:
            eps = torch.cat([eps, torch.zeros((pad, d), device=device)], 0)
        inner = torch.matmul(W, eps.view(nb, T, d))  # [nb, T, d]
        carry = q0
        qh = torch.empty((nb, T, d), dtype=torch.float32, device=device)
        # chain the blocks: q[b, i] = inner[b, i] + rho^(i+1) * carry_{b-1}
        # (the first block's carry is q_{-1} := q0, so q_0 = rho*q0 + sigma*eps_0)
        for b in range(nb):
            qh[b] = inner[b] + powers[:, None] * carry[None, :]
            carry = qh[b, T - 1]
        out[h] = qh.view(nb * T, d)[:L]
    return out


def _finish(x, dtype):
    return x.to(torch.bfloat16) if dtype == "bf16" else x.contiguous()


def make_kv_lmk(w: Workload, device="cpu", seed=None):
    """Keys, values and landmark keys for workload w: k, v [B,Hkv,L,d] and
    lmk [B,Hkv,L//C,d] in the workload dtype."""
    g = _gen(device, w.seed if seed is None else seed)
    B, H, L, d, C = w.B, w.Hkv, w.L, w.d, w.C
    nl = L // C
    k = torch.empty((B, H, L, d), dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32,
                    device=device)
    v = torch.empty_like(k)
    lmk = torch.empty((B, H, nl, d), dtype=k.dtype, device=device)
    for b in range(B):
        for h in range(H):
            kh = _randn((L, d), g, device)
            if w.needles:
                u = _randn((d,), g, device)
                u = u / u.norm()
                n = min(w.needles, nl)
                chunks = torch.randperm(nl, generator=g, device=device)[:n]
                for c in chunks.tolist():
                    kh[c * C:(c + 1) * C] += w.needle_amp * math.sqrt(d) * u
            if w.lmk_noise > 0:
                mean = kh[:nl * C].view(nl, C, d).mean(dim=1)
                lh = mean + w.lmk_noise * _randn((nl, d), g, device)
            else:
                lh = _randn((nl, d), g, device)
            k[b, h] = _finish(kh, w.dtype)
            lmk[b, h] = _finish(lh, w.dtype)
            v[b, h] = _finish(_randn((L, d), g, device), w.dtype)
    return k, v, lmk


def make_q(w: Workload, device="cpu", seed=None):
    """Queries: [B,Hq,L,d] for prefill, [B,Hq,d] for decode."""
    g = _gen(device, (w.seed if seed is None else seed) + 7919)
    B, H, L, d = w.B, w.Hq, w.L, w.d
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    if w.decode:
        return _finish(_randn((B, H, d), g, device), w.dtype)
    q = torch.empty((B, H, L, d), dtype=dt, device=device)
    for b in range(B):
        if w.q_kind == "ar1":
            for h in range(H):
                q[b, h] = _finish(_ar1(1, L, d, w.q_sigma, g, device)[0], w.dtype)
        else:
            for h in range(H):
                q[b, h] = _finish(_randn((L, d), g, device), w.dtype)
    return q


def make_inputs(w: Workload, device="cpu", seed=None):
    """(q, k, v, lmk) for workload w on `device`."""
    k, v, lmk = make_kv_lmk(w, device, seed)
    q = make_q(w, device, seed)
    return q, k, v, lmk

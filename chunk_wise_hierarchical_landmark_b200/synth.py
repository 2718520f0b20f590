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


def _ar1(n_heads, L, d, sigma, g, device):
    """Stationary AR(1) walk of length L for n_heads independent heads, [n, L, d] fp32.

    q_t = rho * q_{t-1} + sigma * eps_t with q_{-1} ~ N(0, 1), evaluated as a
    log-depth scan of the linear recurrence (each doubling step adds the
    contribution of the element 2^s positions back, weighted by rho^(2^s))."""
    rho = math.sqrt(1.0 - sigma * sigma)
    q0 = _randn((n_heads, 1, d), g, device)
    x = _randn((n_heads, L, d), g, device) * sigma
    span = 1
    while span < L:
        x[:, span:] += (rho ** span) * x[:, :-span].clone()
        span *= 2
    t = torch.arange(1, L + 1, device=device, dtype=torch.float64)
    x += (rho ** t).float()[None, :, None] * q0
    return x


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
            for h0 in range(0, H, 8):
                hs = min(8, H - h0)
                q[b, h0:h0 + hs] = _finish(_ar1(hs, L, d, w.q_sigma, g, device), w.dtype)
        else:
            for h in range(H):
                q[b, h] = _finish(_randn((L, d), g, device), w.dtype)
    return q


def make_inputs(w: Workload, device="cpu", seed=None):
    """(q, k, v, lmk) for workload w on `device`."""
    k, v, lmk = make_kv_lmk(w, device, seed)
    q = make_q(w, device, seed)
    return q, k, v, lmk

"""Backward pass of the HiLS forward -- TEST INFRASTRUCTURE ONLY (oracle).

Only ``tests/`` may import this module; the CUDA library never calls it.

The pages put the chunk scores inside the forward computation so that the
language-modelling loss reaches them (aiweekly.co, the paragraph on the
mechanism: outputs fused by the retrieval scores, which therefore receive
gradient; molayo1419.me, "Core idea": the landmark keys take part in the
forward pass and gradients flow into them).  The top-k choice itself is a
discrete decision and carries no gradient.

This module restates the forward pass once more, in plain PyTorch fp64 and
independently of ``hils_oracle.c`` (one query row at a time):

  s_c   = scale * <q_t, lmk_c>            c < n_c = floor(t / C)
  sel   = the k best s_c (decided on the fp32-rounded score, ties to the
          lower chunk id; every completed chunk when n_c <= k)
  own chunk o = floor(t / C): x_j = scale * <q_t, k_j>, j = oC .. t,
          l_own = logsumexp(x), a_own = softmax(x) V
  chunk c in sel: x_j over the C keys of c, a_c = softmax(x) V
  w     = softmax over (s_c for c in sel, l_own)
  out_t = sum_c w_c a_c + w_own a_own,   lse_t = logsumexp(s_sel, l_own)

and obtains dq, dk, dv and dlmk with torch.autograd for given output
gradients.  Pinned in ``tests/test_oracle_backward.py``: its forward equals
the C oracle's, its gradients equal finite differences of its forward, and
closed forms for the landmark gradient.
"""
from __future__ import annotations

import numpy as np
import torch


def _f64(x):
    """fp64 tensor from fp32 / bf16 data (numpy bits as uint16 = bf16)."""
    if isinstance(x, np.ndarray):
        if x.dtype == np.uint16:
            x = (x.astype(np.uint32) << 16).view(np.float32)
        return torch.from_numpy(np.ascontiguousarray(x)).to(torch.float64)
    return x.detach().to(torch.float64)


def select(s: torch.Tensor, topk: int) -> list[int]:
    """Indices of the k best scores in ascending id order; the decision is
    taken on the fp32-rounded scores, ties going to the lower id."""
    n = s.shape[0]
    if n <= topk:
        return list(range(n))
    s32 = s.detach().to(torch.float32).tolist()
    order = sorted(range(n), key=lambda c: (-s32[c], c))
    return sorted(order[:topk])


def forward(p, q, k, v, lmk):
    """Prefill forward over every row.  q [B,Hq,L,d], k/v [B,Hkv,L,d],
    lmk [B,Hkv,L//C,d] as fp64 tensors (gradients flow through them).
    Returns out [B,Hq,L,d], lse [B,Hq,L], sel (list of lists per row)."""
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    C, scale = p.C, p.scale
    outs, lses, sels = [], [], []
    for b in range(B):
        for hq in range(Hq):
            hk = hq // G
            for t in range(L):
                qt = q[b, hq, t]
                oc = t // C
                s = scale * (lmk[b, hk, :oc] @ qt) if oc > 0 else q.new_zeros(0)
                pick = select(s, p.topk)
                logits, parts = [], []
                for c in pick:
                    x = scale * (k[b, hk, c * C:(c + 1) * C] @ qt)
                    parts.append(torch.softmax(x, 0) @ v[b, hk, c * C:(c + 1) * C])
                    logits.append(s[c])
                x = scale * (k[b, hk, oc * C:t + 1] @ qt)
                parts.append(torch.softmax(x, 0) @ v[b, hk, oc * C:t + 1])
                logits.append(torch.logsumexp(x, 0))
                lg = torch.stack(logits)
                w = torch.softmax(lg, 0)
                outs.append((w[:, None] * torch.stack(parts)).sum(0))
                lses.append(torch.logsumexp(lg, 0))
                sels.append(pick)
    out = torch.stack(outs).reshape(B, Hq, L, d)
    lse = torch.stack(lses).reshape(B, Hq, L)
    return out, lse, sels


def backward(p, q, k, v, lmk, dout, dlse=None) -> dict:
    """Gradients of sum(out * dout) + sum(lse * dlse) with respect to q, k, v
    and lmk (numpy fp64 arrays), plus the forward's out, lse and selection."""
    xs = [_f64(a).requires_grad_(True) for a in (q, k, v, lmk)]
    out, lse, sels = forward(p, *xs)
    loss = (out * _f64(dout)).sum()
    if dlse is not None:
        loss = loss + (lse * _f64(dlse)).sum()
    g = torch.autograd.grad(loss, xs, allow_unused=True)
    g = [torch.zeros_like(x) if gi is None else gi for x, gi in zip(xs, g)]
    return {"dq": g[0].numpy(), "dk": g[1].numpy(), "dv": g[2].numpy(), "dlmk": g[3].numpy(),
            "out": out.detach().numpy(), "lse": lse.detach().numpy(), "sel": sels}


def backward_explicit(p, q, k, v, lmk, dout, dlse=None) -> dict:
    """The same gradients from explicit formulas (numpy fp64, one row at a
    time), in the quantities a kernel forms per (row, attended chunk):

      P_j   = w_c p_{c,j}        the fused weight of key j of chunk c
                                 (p: softmax inside the chunk, w: fusion)
      dP_j  = <dout, v_j>        g_c = sum_j p_{c,j} dP_j = <dout, a_c>
      D     = <dout, out>        (the row's output-gradient dot product)
      dv_j += P_j dout
      dx_j  = P_j (dP_j - g_c)                  token logit x_j = scale <q, k_j>
            + p_{own,j} w_own (g_own - D + dlse)   (own chunk: through l_own)
      ds_c  = w_c (g_c - D + dlse)                chunk logit s_c of a selected c
      dq   += scale (sum_j dx_j k_j + sum_c ds_c lmk_c)
      dk_j += scale dx_j q,   dlmk_c += scale ds_c q
    The selection is the forward's (no gradient through the choice)."""
    q, k, v, lmk = (_f64(a).numpy() for a in (q, k, v, lmk))
    dout = np.asarray(dout, np.float64)
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    C, scale = p.C, p.scale
    dq, dk, dv, dl = (np.zeros_like(a) for a in (q, k, v, lmk))
    for b in range(B):
        for hq in range(Hq):
            hk = hq // G
            for t in range(L):
                qt, dot = q[b, hq, t], dout[b, hq, t]
                dls = 0.0 if dlse is None else float(np.asarray(dlse)[b, hq, t])
                oc = t // C
                s = scale * (lmk[b, hk, :oc] @ qt) if oc else np.zeros(0)
                pick = select(torch.from_numpy(s), p.topk)
                spans = [(c * C, c * C + C) for c in pick] + [(oc * C, t + 1)]
                pc, ac = [], []
                for j0, j1 in spans:
                    x = scale * (k[b, hk, j0:j1] @ qt)
                    e = np.exp(x - x.max())
                    pc.append(e / e.sum())
                    ac.append(pc[-1] @ v[b, hk, j0:j1])
                x_own = scale * (k[b, hk, oc * C:t + 1] @ qt)
                logits = np.array([s[c] for c in pick] + [x_own.max() + np.log(np.exp(x_own - x_own.max()).sum())])
                w = np.exp(logits - logits.max())
                w /= w.sum()
                out = sum(wi * ai for wi, ai in zip(w, ac))
                D = float(dot @ out)
                for i, (j0, j1) in enumerate(spans):
                    dP = v[b, hk, j0:j1] @ dot
                    g = float(pc[i] @ dP)
                    P = w[i] * pc[i]
                    dv[b, hk, j0:j1] += P[:, None] * dot[None, :]
                    dx = P * (dP - g)
                    if i == len(spans) - 1:  # own chunk: its logit is l_own
                        dx = dx + pc[i] * w[i] * (g - D + dls)
                    else:
                        ds = w[i] * (g - D + dls)
                        c = pick[i]
                        dq[b, hq, t] += scale * ds * lmk[b, hk, c]
                        dl[b, hk, c] += scale * ds * qt
                    dq[b, hq, t] += scale * (dx @ k[b, hk, j0:j1])
                    dk[b, hk, j0:j1] += scale * dx[:, None] * qt[None, :]
    return {"dq": dq, "dk": dk, "dv": dv, "dlmk": dl}

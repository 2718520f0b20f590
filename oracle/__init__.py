"""CPU oracle for the HiLS attention forward pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and it
imports nothing from the CUDA package: the two sides share only the seeded
input generator.

The arithmetic lives in ``hils_oracle.c`` (plain C, fp64, OpenMP over rows),
which follows the pages on HiLS attention step by step:

* model card "HiLS-Attention" (axforge.ai), section "What HiLS-Attention is":
  landmark-key chunk-mass surrogate, inter-/intra-chunk softmax factorisation,
  top-k chunk selection, and the naive exact-chunk-mass selector;
* "HiLS Attention Extrapolates 64x at 90% Retrieval Accuracy" (aiweekly.co):
  each retrieved chunk attended independently, outputs fused by chunk scores;
* "HiLS Attention: ..." (molayo1419.me), section "Core idea": the two-step
  factorisation (inter-chunk attention over landmarks, then standard attention
  inside the selected chunks) and section "Hardware-efficient kernel": the
  union of the chunks of M adjacent queries.

``gather_pages`` turns a paged KV cache (one chunk of every KV head per page,
as an inference engine's attention backend receives it; the same page's
section "Converting existing models" has HiLS served as such a backend) back
into the dense cache it describes; ``decode_paged`` is the decode step on that
dense cache.

``hope`` is the hierarchical positional encoding of the same page, section
"Engineering details" (HoPE): rotary position embedding on the dimensions
that fall inside the pre-training window, no positional encoding on the rest.

``qcal_query`` and ``Oracle.rows_qcal`` follow the Q-Cal item of the same
section: a low-rank offset W_up W_down h added to the query for the chunk
scores only (selection and chunk logits); attention inside the chunks keeps
the plain query.

``oracle.backward`` (plain PyTorch fp64) states the forward a second time and
differentiates it with autograd: the reference for a backward pass.

Every entry point is pinned in ``tests/test_oracle_pins.py`` against closed
forms, hand-derived values and brute force; none is "parity unpinned".

This module compiles the C source with gcc on first use (``build()``).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hils_oracle.c")
_LIB = os.path.join(_HERE, "libhils_oracle.so")

MODES = {"landmark": 0, "given": 1, "exact_mass": 2}


def compile_source(src: str, lib: str) -> str:
    """Compile one oracle C source into a shared library (gcc, -O2, OpenMP)."""
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
                           "-o", tmp, src, "-lm"])
    os.replace(tmp, lib)
    return lib


def build(force: bool = False) -> str:
    """Compile ``hils_oracle.c`` into ``libhils_oracle.so`` when it is stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB)
    return _LIB


def _bind(path):
    lib = ctypes.CDLL(path)
    P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.hils_oracle_rows.argtypes = [I, I, I, I, I, I, I, D, I, I, P, P, P, P, I64, P, I, P, P,
                                     P, P, P, P, P, P, I]
    lib.hils_oracle_rows.restype = I
    lib.hils_oracle_union.argtypes = [I, I, I, I, I64, I64, P, P, I64]
    lib.hils_oracle_union.restype = I64
    lib.hils_oracle_scores.argtypes = [I, I, I, I, I, I, D, I, I, P, P, I64, P, P, I, I]
    lib.hils_oracle_scores.restype = I
    return lib


@dataclass
class Problem:
    """Shapes of one HiLS problem (BHLD layout, chunk size C, top-k)."""
    B: int
    Hq: int
    Hkv: int
    L: int
    d: int
    C: int
    topk: int
    scale: float


def _as_array(x):
    """Accept numpy arrays or CPU torch tensors (fp32, or bf16 kept as raw bits).

    Returns (contiguous numpy array, is_bf16)."""
    if hasattr(x, "detach"):  # torch tensor, imported lazily
        import torch
        x = x.detach()
        if x.device.type != "cpu":
            raise ValueError("oracle inputs must live in host memory")
        if x.dtype == torch.bfloat16:
            return np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16)), True
        if x.dtype == torch.float32:
            return np.ascontiguousarray(x.contiguous().numpy()), False
        raise TypeError(f"unsupported oracle input dtype {x.dtype}")
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), True
    if x.dtype == np.float32:
        return np.ascontiguousarray(x), False
    if x.dtype == np.float64:
        # fp64 inputs are rounded to fp32 storage: the oracle reads fp32 or bf16.
        return np.ascontiguousarray(x.astype(np.float32)), False
    raise TypeError(f"unsupported oracle input dtype {x.dtype}")


def _inputs(q, k, v, lmk):
    arrs = [_as_array(a) for a in (q, k, v, lmk)]
    fmts = {b for _, b in arrs}
    if len(fmts) != 1:
        raise TypeError("q, k, v and lmk must share one element format")
    return [a for a, _ in arrs], fmts.pop()


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _outputs(n, p):
    return {
        "sel": np.empty((n, p.topk), np.int32),
        "w": np.empty((n, p.topk), np.float64),
        "lse_lmk": np.empty((n,), np.float64),
        "out": np.empty((n, p.d), np.float64),
        "lse": np.empty((n,), np.float64),
        "wfin": np.empty((n, p.topk + 1), np.float64),
    }


class Oracle:
    """The oracle bound to one compiled library (the default one, or a test's
    deliberately broken copy)."""

    def __init__(self, lib_path: str | None = None):
        self.lib = _bind(lib_path or build())

    def rows(self, p: Problem, q, k, v, lmk, rows, mode: str = "landmark", sel_in=None,
             w_in=None, nthreads: int = 0, decode: bool = False) -> dict:
        """Prefill rows (flat indices (b*Hq + hq)*L + t), or with decode=True
        decode heads (flat b*Hq + hq, q [B,Hq,d], position t = L-1).

        Returns numpy arrays: sel [n,k] int32 (ascending, -1 pad), w [n,k]
        (selected logits, -inf pad), lse_lmk [n], out [n,d], lse [n],
        wfin [n,k+1] (fusion weights in sel order, own chunk last)."""
        (qa, ka, va, la), bf16 = _inputs(q, k, v, lmk)
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
        n = r.shape[0]
        res = _outputs(n, p)
        si = wi = None
        if mode == "given":
            si = np.ascontiguousarray(np.asarray(sel_in, dtype=np.int32).reshape(n, p.topk))
            wi = np.ascontiguousarray(np.asarray(w_in, dtype=np.float64).reshape(n, p.topk))
        rc = self.lib.hils_oracle_rows(
            p.B, p.Hq, p.Hkv, p.L, p.d, p.C, p.topk, p.scale, int(bf16), int(decode), _ptr(qa), _ptr(ka),
            _ptr(va), _ptr(la), n, _ptr(r), MODES[mode], _ptr(si), _ptr(wi), _ptr(res["sel"]),
            _ptr(res["w"]), _ptr(res["lse_lmk"]), _ptr(res["out"]), _ptr(res["lse"]),
            _ptr(res["wfin"]), int(nthreads))
        if rc != 0:
            raise ValueError("oracle rejected its arguments")
        return res

    def decode(self, p: Problem, q, k, v, lmk, heads=None, nthreads: int = 0) -> dict:
        """Decode step: q is [B,Hq,d], the cache length is p.L and the query
        position is p.L - 1.  heads: flat b*Hq + hq (default: all)."""
        h = np.arange(p.B * p.Hq, dtype=np.int64) if heads is None else heads
        return self.rows(p, q, k, v, lmk, h, nthreads=nthreads, decode=True)

    def decode_paged(self, p: Problem, q, k_pages, v_pages, page_table, lmk, heads=None,
                     nthreads: int = 0) -> dict:
        """Decode step over a paged cache: the dense-cache decode of the caches
        that ``gather_pages`` rebuilds from the pages and the table."""
        k = gather_pages(k_pages, page_table, p.L)
        v = gather_pages(v_pages, page_table, p.L)
        return self.decode(p, q, k, v, lmk, heads, nthreads)

    def rows_qcal(self, p: Problem, q, k, v, lmk, qs, rows, nthreads: int = 0) -> dict:
        """Prefill rows with a separate scoring query qs [B,Hq,L,d] (fp32):
        landmark scores, top-k, chunk logits and lse_lmk come from qs; the
        attention inside the chunks and the own chunk's logit from q.  Two
        calls of the same oracle: landmark mode on qs, then given mode on q
        with that selection and those logits (all inputs widened to fp32)."""
        k32, v32, l32, q32 = (_widen32(a) for a in (k, v, lmk, q))
        sc = self.rows(p, _widen32(qs), k32, v32, l32, rows, nthreads=nthreads)
        res = self.rows(p, q32, k32, v32, l32, rows, mode="given", sel_in=sc["sel"],
                        w_in=sc["w"], nthreads=nthreads)
        res["lse_lmk"] = sc["lse_lmk"]
        return res

    def scores(self, p: Problem, q, lmk, rows, nthreads: int = 0,
               decode: bool = False) -> np.ndarray:
        """Landmark logits of every completed chunk for the rows (numbered as in
        rows()): [n, L//C] fp64, -inf for chunks that are not completed."""
        qa, bf16 = _as_array(q)
        la, bf16_l = _as_array(lmk)
        if bf16 != bf16_l:
            raise TypeError("q and lmk must share one element format")
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
        ncols = max(p.L // p.C, 1)
        s = np.empty((r.shape[0], ncols), np.float64)
        rc = self.lib.hils_oracle_scores(p.B, p.Hq, p.Hkv, p.L, p.d, p.C, p.scale, int(bf16),
                                         int(decode), _ptr(qa), _ptr(la), r.shape[0], _ptr(r), _ptr(s), ncols,
                                         int(nthreads))
        if rc != 0:
            raise ValueError("oracle rejected its arguments")
        return s[:, :p.L // p.C]

    def union(self, L: int, C: int, topk: int, M: int, head: int, g: int, sel) -> np.ndarray:
        """Sorted chunk union of query group g (rows [g*M, (g+1)*M)) of flat
        head `head`, from a full selection array sel [B*Hq*L, topk]."""
        s = np.ascontiguousarray(np.asarray(sel, dtype=np.int32))
        cap = (L + C - 1) // C
        u = np.empty((cap,), np.int32)
        n = self.lib.hils_oracle_union(L, C, topk, M, head, g, _ptr(s), _ptr(u), cap)
        if n < 0:
            raise ValueError("union capacity exceeded")
        return u[:n].copy()


def _widen32(x) -> np.ndarray:
    """fp32 copy of fp32 / bf16 input (bf16 widens exactly)."""
    a, bf16 = _as_array(x)
    if bf16:
        a = (a.astype(np.uint32) << 16).view(np.float32)
    return np.ascontiguousarray(a, dtype=np.float32)


def _bf16_round(x: np.ndarray) -> np.ndarray:
    """fp32 values rounded to the nearest bf16 (ties to even), as fp32."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return (r.astype(np.uint32) << 16).view(np.float32)


def qcal_query(q, h, w_down, w_up) -> np.ndarray:
    """Q-Cal scoring query: q_t + W_up[hq] (W_down h_t) for every head and
    position (molayo1419.me, "Engineering details", Q-Cal: a low-rank learnable
    offset of the query used for the chunk-mass estimate).

    q [B,Hq,L,d], h [B,L,D] hidden states, w_down [r,D] (shared by the heads),
    w_up [Hq,d,r]; each fp32 or bf16 (widened exactly), fp64 data is first
    rounded to fp32.  The pages fix no precision; the reading taken here is
    the query's own: everything in fp32, every product and every partial sum
    rounded (no fused multiply-add), in a fixed order --
      z_r  = sum over i = 0 .. D-1 of w_down[r, i] * h_t[i]
      dq_e = sum over j = 0 .. r-1 of w_up[hq, e, j] * z_j
      q_cal = q + dq, rounded to bf16 (nearest even) when q is bf16
    -- so that a scoring pass fed this query sees exactly these values.
    Returns fp32 [B,Hq,L,d] (bf16 values widened exactly)."""
    qa, q_bf16 = _as_array(q)
    q32 = _widen32(q)
    h32, wd32, wu32 = (_widen32(a) for a in (h, w_down, w_up))
    B, Hq, L, d = q32.shape
    r, D = wd32.shape
    z = np.zeros((B, L, r), np.float32)
    for i in range(D):
        z = (z + (h32[:, :, None, i] * wd32[None, None, :, i]).astype(np.float32)).astype(np.float32)
    dq = np.zeros((B, Hq, L, d), np.float32)
    for j in range(r):
        dq = (dq + (wu32[None, :, None, :, j] * z[:, None, :, j, None]).astype(np.float32)).astype(np.float32)
    qc = (q32 + dq).astype(np.float32)
    return _bf16_round(qc) if q_bf16 else qc


def gather_pages(pages, page_table, L: int) -> np.ndarray:
    """Dense cache [B, Hkv, L, d] from a paged one.

    pages [num_pages, Hkv, C, d] (fp32, or bf16 as raw bits / a bf16 tensor);
    page_table [B, max_pages] integers.  Token t = c*C + r (r < C) of sequence
    b and KV head h is row r of KV head h of page page_table[b, c]; only the
    ceil(L/C) first entries of a table row are read, and rows r with
    c*C + r >= L are not.  Returns numpy (uint16 bits for bf16 input)."""
    pg, _ = _as_array(pages)
    tab = np.asarray(page_table.cpu() if hasattr(page_table, "cpu") else page_table)
    num_pages, Hkv, C, d = pg.shape
    B = tab.shape[0]
    out = np.empty((B, Hkv, L, d), pg.dtype)
    for b in range(B):
        for c in range(-(-L // C)):
            page = int(tab[b, c])
            if not 0 <= page < num_pages:
                raise ValueError(f"page table entry ({b}, {c}) = {page} outside the pool")
            n = min(C, L - c * C)
            out[b, :, c * C:c * C + n, :] = pg[page, :, :n, :]
    return out


def hope(x, positions, n_rope_pairs: int, base: float = 10000.0) -> np.ndarray:
    """HoPE applied to x [..., n, d] at integer positions [n], in fp64.

    Dimensions pair up as (i, i + d/2) (the rotate-half convention); pair i
    has angular frequency theta_i = base ** (-2 i / d), so the wavelength
    grows with i.  Pairs i < n_rope_pairs (the short wavelengths, inside the
    pre-training window) are rotated by the angle t * theta_i:
        x'_i       = x_i cos - x_{i+d/2} sin
        x'_{i+d/2} = x_i sin + x_{i+d/2} cos
    and the other pairs are left as they are (NoPE).  Returns fp64; bf16
    input (raw bits or a bf16 tensor) is widened exactly first."""
    a, bf16 = _as_array(x)
    if bf16:
        a = (a.astype(np.uint32) << 16).view(np.float32)
    a = a.astype(np.float64)
    d = a.shape[-1]
    half = d // 2
    if not 0 <= n_rope_pairs <= half:
        raise ValueError("n_rope_pairs must lie in [0, d/2]")
    t = np.asarray(positions, dtype=np.float64).reshape(-1)
    if t.shape[0] != a.shape[-2]:
        raise ValueError("one position per row")
    out = a.copy()
    for i in range(n_rope_pairs):
        theta = float(base) ** (-2.0 * i / d)
        ang = t * theta
        c, s = np.cos(ang)[:, None], np.sin(ang)[:, None]
        xi = a[..., :, i:i + 1]
        xj = a[..., :, i + half:i + half + 1]
        out[..., :, i:i + 1] = xi * c - xj * s
        out[..., :, i + half:i + half + 1] = xi * s + xj * c
    return out


def rope_pairs(d: int, base: float, train_len: float) -> int:
    """The HoPE split (molayo1419.me, "Engineering details", HoPE: rotary
    embedding on the dimensions that fall inside the pre-training window,
    none on the others): the number of rotate-half pairs i whose wavelength
    2 pi base^(2i/d) -- the positions one full turn of pair i takes -- is at
    most the pre-training length.  The wavelength grows with i, so these are
    the pairs 0 .. n-1."""
    n = 0
    for i in range(d // 2):
        if 2.0 * math.pi * float(base) ** (2.0 * i / d) <= float(train_len):
            n = i + 1
        else:
            break
    return n


_default = None


def default() -> Oracle:
    """The oracle compiled from ``hils_oracle.c``."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def rows(*a, **kw):
    return default().rows(*a, **kw)


def decode(*a, **kw):
    return default().decode(*a, **kw)


def union(*a, **kw):
    return default().union(*a, **kw)


def scores(*a, **kw):
    return default().scores(*a, **kw)


def decode_paged(*a, **kw):
    return default().decode_paged(*a, **kw)

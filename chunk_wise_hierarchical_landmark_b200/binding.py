"""Thin Python binding of libhils.so (include/hils.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI.  Tensors are torch CUDA tensors (torch provides
device memory and the current stream); outputs are allocated here with torch
and passed to the library as device pointers.  There is no fallback: if
libhils.so is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhils.so")

HILS_OK = 0
HILS_F32, HILS_BF16 = 0, 1
HILS_OP_PREFILL, HILS_OP_DECODE = 0, 1


class HilsError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"hils status {status}: {msg}")
        self.status = status


class Params(ctypes.Structure):
    """Mirror of hils_params."""
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("L", ctypes.c_int), ("d", ctypes.c_int), ("chunk", ctypes.c_int),
                ("topk", ctypes.c_int), ("M", ctypes.c_int), ("scale", ctypes.c_float),
                ("dtype", ctypes.c_int), ("debug_checks", ctypes.c_int)]


_lib = None
EXPORTS = ["hils_workspace_size", "hils_select", "hils_union_capacity", "hils_union",
           "hils_attn_fwd", "hils_prefill", "hils_decode_fwd", "hils_decode_fwd_paged",
           "hils_decode_fwd_noalloc", "hils_hope", "hils_qcal_workspace_size", "hils_qcal_query",
           "hils_prefill_qcal", "hils_hope_rope_pairs", "hils_test_set_wait_limit",
           "hils_attn_bwd_workspace_size", "hils_attn_bwd", "hils_prefill_hope",
           "hils_status_string", "hils_last_error", "hils_launch_count"]


def lib():
    """Load libhils.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m chunk_wise_hierarchical_landmark_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, PP, I, I64, SZ = ctypes.c_void_p, ctypes.POINTER(Params), ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        L.hils_workspace_size.argtypes = [PP, I]
        L.hils_workspace_size.restype = SZ
        L.hils_select.argtypes = [PP, P, P, P, P, P, P, SZ, P]
        L.hils_union_capacity.argtypes = [PP]
        L.hils_union_capacity.restype = I64
        L.hils_union.argtypes = [PP, P, P, P, I64, P, SZ, P]
        L.hils_attn_fwd.argtypes = [PP, P, P, P, P, P, P, P, P, P, SZ, P]
        L.hils_prefill.argtypes = [PP, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.hils_decode_fwd.argtypes = [PP, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.hils_decode_fwd_paged.argtypes = [PP, P, P, P, I64, P, I, P, P, P, P, P, P, P, SZ, P]
        L.hils_decode_fwd_noalloc.argtypes = [PP, P, P, P, P, P, P, P, P, P, P]
        L.hils_hope.argtypes = [P, I, I, I, I, I, I, I, ctypes.c_double, P]
        L.hils_prefill_hope.argtypes = [PP, P, P, P, P, I, I, ctypes.c_double, P, P, P, P, P, P,
                                        SZ, P]
        L.hils_prefill_hope.restype = I
        L.hils_attn_bwd_workspace_size.argtypes = [PP]
        L.hils_attn_bwd_workspace_size.restype = SZ
        L.hils_attn_bwd.argtypes = [PP, P, P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.hils_attn_bwd.restype = I
        L.hils_test_set_wait_limit.argtypes = [ctypes.c_uint64, I]
        L.hils_test_set_wait_limit.restype = None
        L.hils_hope_rope_pairs.argtypes = [I, ctypes.c_double, ctypes.c_double]
        L.hils_hope_rope_pairs.restype = I
        L.hils_qcal_workspace_size.argtypes = [PP, I]
        L.hils_qcal_workspace_size.restype = SZ
        L.hils_qcal_query.argtypes = [PP, P, P, P, P, I, I, P, P, SZ, P]
        L.hils_prefill_qcal.argtypes = [PP, P, P, P, P, P, P, P, I, I, P, P, P, P, P, P, P, SZ, P]
        for f in ("hils_select", "hils_union", "hils_attn_fwd", "hils_prefill", "hils_decode_fwd",
                  "hils_decode_fwd_paged", "hils_decode_fwd_noalloc", "hils_hope",
                  "hils_qcal_query", "hils_prefill_qcal"):
            getattr(L, f).restype = I
        L.hils_status_string.argtypes = [I]
        L.hils_status_string.restype = ctypes.c_char_p
        L.hils_last_error.argtypes = []
        L.hils_last_error.restype = ctypes.c_char_p
        L.hils_launch_count.argtypes = []
        L.hils_launch_count.restype = I64
        _lib = L
    return _lib


def _check(status):
    if status != HILS_OK:
        L = lib()
        raise HilsError(status, f"{L.hils_status_string(status).decode()}: "
                                f"{L.hils_last_error().decode()}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def make_params(B, Hq, Hkv, L, d, topk, M=64, chunk=64, scale=None, dtype=torch.bfloat16,
                debug_checks=False) -> Params:
    return Params(B, Hq, Hkv, L, d, chunk, topk, M,
                  float(scale if scale is not None else 1.0 / d ** 0.5),
                  HILS_BF16 if dtype == torch.bfloat16 else HILS_F32, int(bool(debug_checks)))


def params_for(q, k, topk, M=64, chunk=64, scale=None, debug_checks=False, decode=False):
    """hils_params from tensors: prefill q [B,Hq,L,d] or decode q [B,Hq,d];
    k [B,Hkv,L,d]."""
    B, Hkv, L, d = k.shape
    Hq = q.shape[1]
    return make_params(B, Hq, Hkv, L, d, topk, M, chunk, scale, q.dtype, debug_checks)


def workspace(p: Params, op: int, device=None) -> torch.Tensor | None:
    n = lib().hils_workspace_size(ctypes.byref(p), op)
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def _ws_args(ws):
    return (_ptr(ws), 0 if ws is None else ws.numel())


def hils_select(p: Params, q, lmk_k, sel_idx, chunk_w, lse_lmk=None, ws=None, stream=None):
    _check(lib().hils_select(ctypes.byref(p), _ptr(q), _ptr(lmk_k), _ptr(sel_idx), _ptr(chunk_w),
                             _ptr(lse_lmk), *_ws_args(ws), _stream(stream)))


def hils_union_capacity(p: Params) -> int:
    return int(lib().hils_union_capacity(ctypes.byref(p)))


def hils_union(p: Params, sel_idx, u_off, u_idx, ws=None, stream=None):
    _check(lib().hils_union(ctypes.byref(p), _ptr(sel_idx), _ptr(u_off), _ptr(u_idx),
                            u_idx.numel(), *_ws_args(ws), _stream(stream)))


def hils_attn_fwd(p: Params, q, k, v, sel_idx, chunk_w, out, lse, w_final=None, ws=None,
                  stream=None):
    _check(lib().hils_attn_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(sel_idx),
                               _ptr(chunk_w), _ptr(out), _ptr(lse), _ptr(w_final),
                               *_ws_args(ws), _stream(stream)))


def hils_prefill(p: Params, q, k, v, lmk_k, sel_idx, chunk_w, lse_lmk, out, lse, ws=None,
                 stream=None):
    _check(lib().hils_prefill(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(lmk_k),
                              _ptr(sel_idx), _ptr(chunk_w), _ptr(lse_lmk), _ptr(out), _ptr(lse),
                              *_ws_args(ws), _stream(stream)))


def hils_decode_fwd(p: Params, q, k_cache, v_cache, lmk_k, sel_idx, chunk_w, lse_lmk, out, lse,
                    ws=None, stream=None):
    _check(lib().hils_decode_fwd(ctypes.byref(p), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                 _ptr(lmk_k), _ptr(sel_idx), _ptr(chunk_w), _ptr(lse_lmk),
                                 _ptr(out), _ptr(lse), *_ws_args(ws), _stream(stream)))


def hils_decode_fwd_paged(p: Params, q, k_pages, v_pages, page_table, lmk_k, sel_idx, chunk_w,
                          lse_lmk, out, lse, ws=None, stream=None):
    """k_pages / v_pages [num_pages, Hkv, C, d]; page_table [B, max_pages] int32."""
    _check(lib().hils_decode_fwd_paged(ctypes.byref(p), _ptr(q), _ptr(k_pages), _ptr(v_pages),
                                       int(k_pages.shape[0]), _ptr(page_table),
                                       int(page_table.shape[1]), _ptr(lmk_k), _ptr(sel_idx),
                                       _ptr(chunk_w), _ptr(lse_lmk), _ptr(out), _ptr(lse),
                                       *_ws_args(ws), _stream(stream)))


def hils_decode_fwd_noalloc(p: Params, q, k_cache, v_cache, lmk_k, sel_idx, chunk_w, lse_lmk,
                            out, lse, stream=None):
    _check(lib().hils_decode_fwd_noalloc(ctypes.byref(p), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                         _ptr(lmk_k), _ptr(sel_idx), _ptr(chunk_w), _ptr(lse_lmk),
                                         _ptr(out), _ptr(lse), _stream(stream)))


def hils_hope(x, n_rope_pairs: int, pos0: int = 0, base: float = 10000.0, stream=None):
    """HoPE in place on x [B,H,L,d] (or a decode query [B,H,d], one position)."""
    if x.dim() == 3:
        B, H, d = x.shape
        L = 1
    else:
        B, H, L, d = x.shape
    dt = HILS_BF16 if x.dtype == torch.bfloat16 else HILS_F32
    _check(lib().hils_hope(_ptr(x), dt, B, H, L, d, int(pos0), int(n_rope_pairs), float(base),
                           _stream(stream)))


def qcal_workspace(p: Params, r: int, device=None) -> torch.Tensor:
    n = lib().hils_qcal_workspace_size(ctypes.byref(p), int(r))
    if n == 0:
        raise HilsError(1, "hils_qcal_workspace_size rejected the parameters")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def hils_qcal_query(p: Params, q, h, w_down, w_up, q_cal, ws, stream=None):
    r, D = w_down.shape
    _check(lib().hils_qcal_query(ctypes.byref(p), _ptr(q), _ptr(h), _ptr(w_down), _ptr(w_up),
                                 int(D), int(r), _ptr(q_cal), *_ws_args(ws), _stream(stream)))


def hils_prefill_qcal(p: Params, q, k, v, lmk_k, h, w_down, w_up, q_cal, sel_idx, chunk_w,
                      lse_lmk, out, lse, ws, stream=None):
    r, D = w_down.shape
    _check(lib().hils_prefill_qcal(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(lmk_k),
                                   _ptr(h), _ptr(w_down), _ptr(w_up), int(D), int(r), _ptr(q_cal),
                                   _ptr(sel_idx), _ptr(chunk_w), _ptr(lse_lmk), _ptr(out),
                                   _ptr(lse), *_ws_args(ws), _stream(stream)))


def prefill_qcal(q, k, v, lmk_k, h, w_down, w_up, topk, M=64, scale=None, debug_checks=False):
    """Prefill with the Q-Cal scoring query (h [B,L,D], w_down [r,D], w_up
    [Hq,d,r]): returns dict(out, lse, sel_idx, chunk_w, lse_lmk, q_cal)."""
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    p = make_params(B, Hq, Hkv, L, d, topk, M, 64, scale, q.dtype, debug_checks)
    dev = q.device
    sel = torch.empty((B, Hq, L, topk), dtype=torch.int32, device=dev)
    w = torch.empty((B, Hq, L, topk), dtype=torch.float32, device=dev)
    lse_lmk = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    q_cal = torch.empty_like(q)
    ws = qcal_workspace(p, w_down.shape[0], dev)
    hils_prefill_qcal(p, q, k, v, lmk_k, h, w_down, w_up, q_cal, sel, w, lse_lmk, out, lse, ws)
    return dict(out=out, lse=lse, sel_idx=sel, chunk_w=w, lse_lmk=lse_lmk, q_cal=q_cal)


def hils_attn_bwd(p: Params, q, k, v, lmk_k, sel_idx, chunk_w, lse, dout, dlse, dq, dk, dv,
                  dlmk, ws, stream=None):
    _check(lib().hils_attn_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(lmk_k),
                               _ptr(sel_idx), _ptr(chunk_w), _ptr(lse), _ptr(dout), _ptr(dlse),
                               _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlmk), *_ws_args(ws),
                               _stream(stream)))


def attn_bwd(q, k, v, lmk_k, sel_idx, chunk_w, lse, dout, dlse=None, scale=None,
             debug_checks=False):
    """Backward pass for a forward's selection: returns fp32 (dq, dk, dv, dlmk)."""
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    topk = sel_idx.shape[-1]
    p = make_params(B, Hq, Hkv, L, d, topk, 64, 64, scale, q.dtype, debug_checks)
    dev = q.device
    dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
    dk = torch.empty(k.shape, dtype=torch.float32, device=dev)
    dv = torch.empty(v.shape, dtype=torch.float32, device=dev)
    dl = torch.empty(lmk_k.shape, dtype=torch.float32, device=dev)
    n = lib().hils_attn_bwd_workspace_size(ctypes.byref(p))
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    hils_attn_bwd(p, q, k, v, lmk_k, sel_idx, chunk_w, lse, dout, dlse, dq, dk, dv, dl, ws)
    return dq, dk, dv, dl


def hils_prefill_hope(p: Params, q, k, v, lmk_k, pos0, n_rope_pairs, base, sel_idx, chunk_w,
                      lse_lmk, out, lse, ws=None, stream=None):
    _check(lib().hils_prefill_hope(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(lmk_k),
                                   int(pos0), int(n_rope_pairs), float(base), _ptr(sel_idx),
                                   _ptr(chunk_w), _ptr(lse_lmk), _ptr(out), _ptr(lse),
                                   *_ws_args(ws), _stream(stream)))


def prefill_hope(q, k, v, lmk_k, topk, n_rope_pairs, base, pos0=0, M=64, scale=None,
                 debug_checks=False):
    """Prefill with HoPE applied to the (unrotated) queries inside the kernels;
    k holds rotated keys.  Returns dict(out, lse, sel_idx, chunk_w, lse_lmk)."""
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    p = make_params(B, Hq, Hkv, L, d, topk, M, 64, scale, q.dtype, debug_checks)
    dev = q.device
    sel = torch.empty((B, Hq, L, topk), dtype=torch.int32, device=dev)
    w = torch.empty((B, Hq, L, topk), dtype=torch.float32, device=dev)
    lse_lmk = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    hils_prefill_hope(p, q, k, v, lmk_k, pos0, n_rope_pairs, base, sel, w, lse_lmk, out, lse,
                      workspace(p, HILS_OP_PREFILL, dev))
    return dict(out=out, lse=lse, sel_idx=sel, chunk_w=w, lse_lmk=lse_lmk)


def rope_pairs_for(d: int, base: float, train_len: int) -> int:
    """The HoPE split of the library (hils_hope_rope_pairs): the pairs whose
    wavelength fits in the pre-training length get RoPE."""
    n = lib().hils_hope_rope_pairs(int(d), float(base), float(train_len))
    if n < 0:
        raise HilsError(1, "hils_hope_rope_pairs rejected its arguments")
    return n


def launch_count() -> int:
    return int(lib().hils_launch_count())


# ---------------------------------------------------------------------------
# allocation helpers (outputs allocated with torch, then one C-ABI call)

def select(q, lmk_k, topk, M=64, scale=None, with_lse_lmk=True, debug_checks=False, k_shape=None):
    """Landmark scoring + top-k for a prefill: returns (sel_idx, chunk_w, lse_lmk)."""
    B, Hq, L, d = q.shape
    Hkv = lmk_k.shape[1]
    p = make_params(B, Hq, Hkv, L, d, topk, M, 64, scale, q.dtype, debug_checks)
    sel = torch.empty((B, Hq, L, topk), dtype=torch.int32, device=q.device)
    w = torch.empty((B, Hq, L, topk), dtype=torch.float32, device=q.device)
    lse_lmk = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device) if with_lse_lmk else None
    hils_select(p, q, lmk_k, sel, w, lse_lmk, workspace(p, HILS_OP_PREFILL, q.device))
    return sel, w, lse_lmk


def attn_fwd(q, k, v, sel_idx, chunk_w, M=64, scale=None, with_w_final=False, debug_checks=False):
    """Intra-chunk attention + fusion: returns (out, lse, w_final or None)."""
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    topk = sel_idx.shape[-1]
    p = make_params(B, Hq, Hkv, L, d, topk, M, 64, scale, q.dtype, debug_checks)
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    wf = torch.empty((B, Hq, L, topk + 1), dtype=torch.float32, device=q.device) if with_w_final else None
    hils_attn_fwd(p, q, k, v, sel_idx, chunk_w, out, lse, wf, workspace(p, HILS_OP_PREFILL, q.device))
    return out, lse, wf


def prefill(q, k, v, lmk_k, topk, M=64, scale=None, debug_checks=False):
    """Full prefill forward: returns dict(out, lse, sel_idx, chunk_w, lse_lmk)."""
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    p = make_params(B, Hq, Hkv, L, d, topk, M, 64, scale, q.dtype, debug_checks)
    dev = q.device
    sel = torch.empty((B, Hq, L, topk), dtype=torch.int32, device=dev)
    w = torch.empty((B, Hq, L, topk), dtype=torch.float32, device=dev)
    lse_lmk = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    hils_prefill(p, q, k, v, lmk_k, sel, w, lse_lmk, out, lse, workspace(p, HILS_OP_PREFILL, dev))
    return dict(out=out, lse=lse, sel_idx=sel, chunk_w=w, lse_lmk=lse_lmk)


def decode(q, k_cache, v_cache, lmk_k, topk, scale=None, debug_checks=False):
    """One decode step (q [B,Hq,d], cache [B,Hkv,N,d]): returns dict(out, lse, sel_idx, chunk_w, lse_lmk)."""
    B, Hq, d = q.shape
    _, Hkv, N, _ = k_cache.shape
    p = make_params(B, Hq, Hkv, N, d, topk, 64, 64, scale, q.dtype, debug_checks)
    dev = q.device
    sel = torch.empty((B, Hq, topk), dtype=torch.int32, device=dev)
    w = torch.empty((B, Hq, topk), dtype=torch.float32, device=dev)
    lse_lmk = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    hils_decode_fwd(p, q, k_cache, v_cache, lmk_k, sel, w, lse_lmk, out, lse,
                    workspace(p, HILS_OP_DECODE, dev))
    return dict(out=out, lse=lse, sel_idx=sel, chunk_w=w, lse_lmk=lse_lmk)


def decode_paged(q, k_pages, v_pages, page_table, lmk_k, N, topk, scale=None,
                 debug_checks=False):
    """One decode step over a paged cache (q [B,Hq,d]; pages [num_pages,Hkv,64,d];
    page_table [B, max_pages] int32; N tokens per sequence): returns
    dict(out, lse, sel_idx, chunk_w, lse_lmk)."""
    B, Hq, d = q.shape
    Hkv = k_pages.shape[1]
    p = make_params(B, Hq, Hkv, N, d, topk, 64, 64, scale, q.dtype, debug_checks)
    dev = q.device
    sel = torch.empty((B, Hq, topk), dtype=torch.int32, device=dev)
    w = torch.empty((B, Hq, topk), dtype=torch.float32, device=dev)
    lse_lmk = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    hils_decode_fwd_paged(p, q, k_pages, v_pages, page_table, lmk_k, sel, w, lse_lmk, out, lse,
                          workspace(p, HILS_OP_DECODE, dev))
    return dict(out=out, lse=lse, sel_idx=sel, chunk_w=w, lse_lmk=lse_lmk)


def union(sel_idx, M=64, debug_checks=False):
    """Chunk union per group of M rows in CSR form: returns (u_off, u_idx)."""
    B, Hq, L, topk = sel_idx.shape
    p = make_params(B, Hq, Hq, L, 64, topk, M, 64, None, torch.bfloat16, debug_checks)
    cap = hils_union_capacity(p)
    G = B * Hq * ((L + M - 1) // M)
    u_off = torch.empty(G + 1, dtype=torch.int32, device=sel_idx.device)
    u_idx = torch.empty(max(cap, 4), dtype=torch.int32, device=sel_idx.device)
    hils_union(p, sel_idx, u_off, u_idx, workspace(p, HILS_OP_PREFILL, sel_idx.device))
    return u_off, u_idx[:int(u_off[-1].item())]

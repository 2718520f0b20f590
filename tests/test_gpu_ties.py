"""GPU selection under exact ties.

The landmark keys repeat a few distinct rows, so every query sees each
landmark logit on many chunks at once and the k-th best value is shared by
more chunks than the top-k has room for.  The selection order (logit
descending, chunk index ascending) then fixes a unique set: the lowest chunk
ids among the tied ones.  Both the prefill scoring kernel (seeded top-k over
six launch levels) and the decode top-k (radix select) must return exactly
the oracle's set, and the outputs must match the oracle's."""
import numpy as np
import pytest
import torch

import oracle
from chunk_wise_hierarchical_landmark_b200 import binding as hb
from chunk_wise_hierarchical_landmark_b200 import workloads as W
from tests.parity import compare_rows
from tests.test_gpu_decode import problem, to_np
from tests.test_gpu_prefill import gather, gpu_prefill

pytestmark = pytest.mark.gpu


def tied_inputs(w, n_distinct, seed, decode=False):
    """q, k, v ~ N(0,1); the landmark of chunk c is row c mod n_distinct of a
    small random table (bf16), so logits repeat exactly across chunks."""
    g = torch.Generator().manual_seed(seed)
    nl = w.L // w.C
    qshape = (w.B, w.Hq, w.d) if decode else (w.B, w.Hq, w.L, w.d)
    q = torch.randn(qshape, generator=g).to(torch.bfloat16)
    k = torch.randn((w.B, w.Hkv, w.L, w.d), generator=g).to(torch.bfloat16)
    v = torch.randn((w.B, w.Hkv, w.L, w.d), generator=g).to(torch.bfloat16)
    table = torch.randn((w.B, w.Hkv, n_distinct, w.d), generator=g).to(torch.bfloat16)
    idx = torch.arange(nl) % n_distinct
    lmk = table[:, :, idx, :].contiguous()
    return q, k, v, lmk


def test_prefill_exact_ties_pick_lowest_ids():
    # 64 chunks, 8 distinct landmark rows, k = 12: the best value covers 8
    # chunks, the second best 8 more, of which the 4 lowest ids are kept
    w = W.PREFILL_128K.with_(B=1, Hq=2, Hkv=1, L=4096, topk=12, M=64)
    q, k, v, lmk = tied_inputs(w, 8, seed=4242)
    res = gpu_prefill(q.cuda(), k.cuda(), v.cuda(), lmk.cuda(), w, with_wfin=True)
    rows = np.arange(w.B * w.Hq * w.L)
    ref = oracle.rows(problem(w), q, k, v, lmk, rows)
    got = gather(res, torch.from_numpy(rows), w.topk, w.d)
    assert (got["sel"] == ref["sel"]).all(), "tied selection differs from the lowest-id rule"
    compare_rows(problem(w), (q, k, v, lmk), rows, got, ref, w.dtype)


def test_decode_exact_ties_pick_lowest_ids():
    w = W.DECODE_512K.with_(B=2, Hq=8, Hkv=2, L=4096 + 37, topk=12)
    q, k, v, lmk = tied_inputs(w, 8, seed=4243, decode=True)
    res = hb.decode(q.cuda(), k.cuda(), v.cuda(), lmk.cuda(), w.topk)
    torch.cuda.synchronize()
    heads = np.arange(w.B * w.Hq)
    ref = oracle.decode(problem(w), q, k, v, lmk, heads)
    got = to_np(res, w.d)
    assert (got["sel"] == ref["sel"]).all(), "tied selection differs from the lowest-id rule"
    compare_rows(problem(w), (q, k, v, lmk), heads, got, ref, w.dtype, decode=True)

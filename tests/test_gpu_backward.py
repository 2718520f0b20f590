"""GPU parity of the backward pass (hils_attn_bwd) against the oracle's
explicit per-chunk gradient formulas (oracle/backward.py, itself pinned to
autograd and finite differences): dq, dk, dv and dlmk for the forward's
selection, on GQA, ragged-length, k >= n_c, k > 32 and fp32 (d = 64 and 128)
cases."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as obwd
from chunk_wise_hierarchical_landmark_b200 import binding as hb
from chunk_wise_hierarchical_landmark_b200 import synth
from chunk_wise_hierarchical_landmark_b200 import workloads as W

pytestmark = pytest.mark.gpu

CASES = [
    # bf16, d=128, GQA 8/2, random-walk queries, ragged length (a partial last chunk)
    (W.PREFILL_128K.with_(Hq=8, Hkv=2, L=700, topk=4), 2e-3),
    # fp32, d=64, k larger than every row's completed chunks (all selected)
    (W.TINY_F32.with_(Hq=2, Hkv=1, L=300, topk=8), 1e-4),
    # bf16, d=64, one query head per KV head, k=3, two sequences
    (W.SMALL_32K.with_(B=2, Hq=2, Hkv=2, L=520, topk=3), 2e-3),
    # fp32, d=128, k=2 of up to 5 completed chunks (smallest gap at the k-th
    # logit 8e-4 relative in fp64)
    (W.TINY_F32.with_(d=128, Hq=2, Hkv=1, L=400, topk=2), 1e-4),
    # bf16, d=64, k=40: more selected slots than a warp has lanes, ragged
    # length (smallest gap at the k-th logit 2.6e-4 relative in fp64)
    (W.SMALL_32K.with_(B=1, Hq=2, Hkv=1, L=64 * 44 + 17, topk=40), 2e-3),
]


@pytest.mark.parametrize("w,tol", CASES, ids=["bf16_gqa_ragged", "f32_all_selected", "bf16_d64_b2",
                                              "f32_d128_k2", "bf16_k40"])
def test_backward_matches_oracle(w, tol):
    q, k, v, lmk = synth.make_inputs(w, "cpu")
    g = torch.Generator().manual_seed(w.seed + 5)
    dout = torch.randn(q.shape, generator=g).to(q.dtype)
    dlse = torch.randn(q.shape[:3], generator=g)
    dq_, dk_, dv_, dl_ = (x.cuda() for x in (q, k, v, lmk))
    sel, cw, _ = hb.select(dq_, dl_, w.topk, w.M, debug_checks=True)
    _, lse, _ = hb.attn_fwd(dq_, dk_, dv_, sel, cw, w.M, debug_checks=True)
    gq, gk, gv, gl = hb.attn_bwd(dq_, dk_, dv_, dl_, sel, cw, lse, dout.cuda(), dlse.cuda(),
                                 debug_checks=True)
    torch.cuda.synchronize()
    p = oracle.Problem(w.B, w.Hq, w.Hkv, w.L, w.d, w.C, w.topk, w.scale)
    rows = np.arange(w.B * w.Hq * w.L)
    want_sel = oracle.rows(p, q, k, v, lmk, rows)["sel"]
    # the gradients follow the forward's selection: these inputs have no near-tie
    assert np.array_equal(sel.reshape(-1, w.topk).cpu().numpy(), want_sel)
    ref = obwd.backward_explicit(p, q, k, v, lmk, dout.float().numpy(), dlse.numpy())
    for name, got in (("dq", gq), ("dk", gk), ("dv", gv), ("dlmk", gl)):
        r = ref[name]
        e = np.abs(got.cpu().numpy().astype(np.float64) - r).max()
        scale = max(np.abs(r).max(), 1e-30)
        assert e <= tol * scale, f"{name}: max error {e:.3g} against max |grad| {scale:.3g}"


def test_backward_without_dlse_and_run_to_run():
    """dlse = NULL is the zero gradient; dq is deterministic, dk/dv/dlmk agree
    to rounding between two runs."""
    w = W.PREFILL_128K.with_(Hq=4, Hkv=1, L=640, topk=4)
    q, k, v, lmk = (x.cuda() for x in synth.make_inputs(w, "cpu"))
    g = torch.Generator(device="cuda").manual_seed(9)
    dout = torch.randn(q.shape, generator=g, device="cuda").to(q.dtype)
    sel, cw, _ = hb.select(q, lmk, w.topk, w.M)
    _, lse, _ = hb.attn_fwd(q, k, v, sel, cw, w.M)
    a = hb.attn_bwd(q, k, v, lmk, sel, cw, lse, dout, None)
    b = hb.attn_bwd(q, k, v, lmk, sel, cw, lse, dout, torch.zeros_like(lse))
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0])
    for x, y in zip(a[1:], b[1:]):
        assert (x - y).abs().max().item() <= 1e-5 * max(y.abs().max().item(), 1e-30)

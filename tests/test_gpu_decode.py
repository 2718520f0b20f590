"""GPU parity of the decode step (hils_decode_fwd) against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from chunk_wise_hierarchical_landmark_b200 import binding as hb
from chunk_wise_hierarchical_landmark_b200 import synth
from chunk_wise_hierarchical_landmark_b200 import workloads as W
from tests.parity import compare_rows

pytestmark = pytest.mark.gpu


def problem(w):
    return oracle.Problem(w.B, w.Hq, w.Hkv, w.L, w.d, w.C, w.topk, w.scale)


def to_np(res, d):
    return {
        "sel": res["sel_idx"].reshape(-1, res["sel_idx"].shape[-1]).cpu().numpy(),
        "w": res["chunk_w"].reshape(-1, res["chunk_w"].shape[-1]).cpu().numpy().astype(np.float64),
        "lse_lmk": res["lse_lmk"].reshape(-1).cpu().numpy().astype(np.float64),
        "out": res["out"].reshape(-1, d).float().cpu().numpy(),
        "lse": res["lse"].reshape(-1).cpu().numpy().astype(np.float64),
    }


def check_decode(w, device="cpu"):
    dq, dk, dv, dl = synth.make_inputs(w, device)
    dq, dk, dv, dl = (x.cuda() for x in (dq, dk, dv, dl))
    res = hb.decode(dq, dk, dv, dl, w.topk)
    torch.cuda.synchronize()
    q, k, v, lmk = (x.cpu() for x in (dq, dk, dv, dl))
    heads = np.arange(w.B * w.Hq)
    ref = oracle.decode(problem(w), q, k, v, lmk, heads)
    return compare_rows(problem(w), (q, k, v, lmk), heads, to_np(res, w.d), ref, w.dtype,
                        decode=True)


@pytest.mark.parametrize("N", [1, 64, 65, 3000, 4096])
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("f32", 64)])
def test_decode_small(N, dtype, d):
    w = W.DECODE_512K.with_(B=2, L=N, d=d, dtype=dtype, topk=16, seed=300 + N)
    check_decode(w)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 2), (6, 3)])
def test_decode_group_sizes(Hq, Hkv):
    """G = Hq / Hkv of 1, 8 (the most one decode CTA serves) and 2 with an
    odd head count."""
    w = W.DECODE_512K.with_(B=2, Hq=Hq, Hkv=Hkv, L=3000 + Hq, topk=16, seed=400 + Hq)
    check_decode(w)


def test_decode_equals_last_prefill_row():
    """The decode step equals row N-1 of a prefill over the same cache."""
    w = W.PREFILL_128K.with_(Hq=8, Hkv=2, L=1000, topk=8)
    q, k, v, lmk = (x.cuda() for x in synth.make_inputs(w, "cpu"))
    pre = hb.prefill(q, k, v, lmk, w.topk, w.M)
    dec = hb.decode(q[:, :, -1].contiguous(), k, v, lmk, w.topk)
    assert torch.equal(pre["sel_idx"][:, :, -1], dec["sel_idx"])
    assert (pre["out"][:, :, -1].float() - dec["out"].float()).abs().max().item() <= 1e-2
    assert (pre["lse"][:, :, -1] - dec["lse"]).abs().max().item() <= 1e-3


def test_decode_full_size():
    """The full batched-decode workload (B=16, N=524288, k=64), every head."""
    st = check_decode(W.DECODE_512K, device="cuda")
    assert st["near_ties"] <= 0.02 * W.DECODE_512K.B * W.DECODE_512K.Hq

"""GPU parity of the Q-Cal path (hils_qcal_query, hils_prefill_qcal) against
the oracle: the calibrated scoring query bit for bit, then the prefill whose
chunk scores use it (selection, chunk logits, lse_lmk) while attention keeps
q (molayo1419.me, "Engineering details", Q-Cal)."""
import numpy as np
import pytest
import torch

import oracle
from chunk_wise_hierarchical_landmark_b200 import binding as hb
from chunk_wise_hierarchical_landmark_b200 import synth
from chunk_wise_hierarchical_landmark_b200 import workloads as W
from tests.parity import compare_rows

pytestmark = pytest.mark.gpu


def qcal_inputs(w, D, r, seed):
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    h = torch.randn((w.B, w.L, D), generator=g).to(dt)
    wd = (torch.randn((r, D), generator=g) / D ** 0.5).to(dt)
    wu = (torch.randn((w.Hq, w.d, r), generator=g) * 0.5).to(dt)
    return h, wd, wu


CASES = [
    # bf16, d=128, GQA 8/2, random-walk queries, ragged length
    (W.PREFILL_128K.with_(Hq=8, Hkv=2, L=1000, topk=8), 256, 16),
    # bf16, d=64, MHA, k larger than most rows' completed chunks
    (W.SMALL_32K.with_(B=2, Hq=2, Hkv=2, L=700, topk=16), 96, 8),
    # fp32 workload, odd D, rank 64 (the largest)
    (W.TINY_F32.with_(Hq=2, Hkv=1, L=650), 130, 64),
    # an odd rank and an odd hidden size
    (W.PREFILL_128K.with_(Hq=4, Hkv=2, L=333, topk=4), 37, 5),
]


@pytest.mark.parametrize("w,D,r", CASES, ids=["bf16_gqa", "bf16_d64", "f32_r64", "bf16_r5"])
def test_qcal_prefill_matches_oracle(w, D, r):
    q, k, v, lmk = synth.make_inputs(w, "cpu")
    h, wd, wu = qcal_inputs(w, D, r, seed=w.seed + D)
    res = hb.prefill_qcal(q.cuda(), k.cuda(), v.cuda(), lmk.cuda(), h.cuda(), wd.cuda(), wu.cuda(),
                          w.topk, w.M, debug_checks=True)
    torch.cuda.synchronize()
    qs = oracle.qcal_query(q, h, wd, wu)
    # the calibrated query: bit for bit
    got_q = res["q_cal"].float().cpu().numpy()
    assert np.array_equal(got_q, qs), f"q_cal differs in {(got_q != qs).sum()} elements"
    p = oracle.Problem(w.B, w.Hq, w.Hkv, w.L, w.d, w.C, w.topk, w.scale)
    rows = np.arange(w.B * w.Hq * w.L)
    ref = oracle.default().rows_qcal(p, q, k, v, lmk, qs, rows)
    gpu = {
        "sel": res["sel_idx"].reshape(-1, w.topk).cpu().numpy(),
        "w": res["chunk_w"].reshape(-1, w.topk).cpu().double().numpy(),
        "lse_lmk": res["lse_lmk"].reshape(-1).cpu().double().numpy(),
        "out": res["out"].reshape(-1, w.d).float().cpu().numpy(),
        "lse": res["lse"].reshape(-1).cpu().double().numpy(),
    }
    score_q = torch.from_numpy(qs).to(q.dtype)
    st = compare_rows(p, (q, k, v, lmk), rows, gpu, ref, w.dtype, score_q=score_q)
    assert st["near_ties"] <= 0.01 * len(rows)


def test_qcal_zero_offset_is_the_plain_prefill():
    """W_up = 0: the calibrated query is q itself and every output equals the
    plain prefill's, bit for bit."""
    w = W.PREFILL_128K.with_(Hq=4, Hkv=1, L=900, topk=8)
    q, k, v, lmk = (x.cuda() for x in synth.make_inputs(w, "cpu"))
    h, wd, wu = (x.cuda() for x in qcal_inputs(w, 64, 4, seed=3))
    a = hb.prefill_qcal(q, k, v, lmk, h, wd, torch.zeros_like(wu), w.topk, w.M)
    b = hb.prefill(q, k, v, lmk, w.topk, w.M)
    torch.cuda.synchronize()
    assert torch.equal(a["q_cal"], q)
    for key in ("sel_idx", "chunk_w", "lse_lmk", "out", "lse"):
        assert torch.equal(a[key], b[key]), key

"""GPU parity of the prefill path (hils_select + hils_attn_fwd, and
hils_union) against the CPU oracle on the same seeded inputs.

Small cases compare every row; full-size workloads compare a seeded sample
of rows (chunk boundaries, first chunk, last row of every head included)."""
import numpy as np
import pytest
import torch

import oracle
from chunk_wise_hierarchical_landmark_b200 import binding as hb
from chunk_wise_hierarchical_landmark_b200 import synth
from chunk_wise_hierarchical_landmark_b200 import workloads as W
from tests.parity import compare_rows, sample_rows

pytestmark = pytest.mark.gpu


def problem(w):
    return oracle.Problem(w.B, w.Hq, w.Hkv, w.L, w.d, w.C, w.topk, w.scale)


def gpu_prefill(dq, dk, dv, dl, w, with_wfin=False):
    # debug mode: a device-side check or a bounded wait that gave up raises
    sel, cw, lse_lmk = hb.select(dq, dl, w.topk, w.M, debug_checks=True)
    out, lse, wf = hb.attn_fwd(dq, dk, dv, sel, cw, w.M, with_w_final=with_wfin, debug_checks=True)
    torch.cuda.synchronize()
    return dict(sel=sel, w=cw, lse_lmk=lse_lmk, out=out, lse=lse, wfin=wf)


def gather(res, rows, K, d):
    g = {
        "sel": res["sel"].reshape(-1, K)[rows].cpu().numpy(),
        "w": res["w"].reshape(-1, K)[rows].cpu().numpy().astype(np.float64),
        "lse_lmk": res["lse_lmk"].reshape(-1)[rows].cpu().numpy().astype(np.float64),
        "out": res["out"].reshape(-1, d)[rows].float().cpu().numpy(),
        "lse": res["lse"].reshape(-1)[rows].cpu().numpy().astype(np.float64),
    }
    if res.get("wfin") is not None:
        g["wfin"] = res["wfin"].reshape(-1, K + 1)[rows].cpu().numpy().astype(np.float64)
    return g


def check_all_rows(w, with_wfin=True):
    q, k, v, lmk = synth.make_inputs(w, "cpu")
    res = gpu_prefill(q.cuda(), k.cuda(), v.cuda(), lmk.cuda(), w, with_wfin)
    rows = torch.arange(w.B * w.Hq * w.L)
    ref = oracle.rows(problem(w), q, k, v, lmk, rows.numpy())
    return compare_rows(problem(w), (q, k, v, lmk), rows.numpy(),
                        gather(res, rows, w.topk, w.d), ref, w.dtype)


def test_tiny_f32_all_rows():
    """fp32 workload (L=4096, k=8, M=16): every row, tolerance 1e-5."""
    st = check_all_rows(W.TINY_F32)
    assert st["near_ties"] <= 4


def test_small_bf16_all_rows():
    """bf16, d=64, 4 planted needles per head, every row."""
    w = W.SMALL_32K.with_(B=2, Hq=4, Hkv=4, L=2048)
    st = check_all_rows(w)
    assert st["near_ties"] <= 0.01 * w.B * w.Hq * w.L


def test_gqa_d128_random_walk_all_rows():
    """bf16, d=128, GQA 8/2, AR(1) queries, M=64, every row."""
    w = W.PREFILL_128K.with_(Hq=8, Hkv=2, L=1536)
    st = check_all_rows(w)
    assert st["near_ties"] <= 0.01 * w.B * w.Hq * w.L


@pytest.mark.parametrize("L", [1, 37, 64, 65, 127, 128, 1000, 1088])
@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("bf16", 128), ("f32", 128)])
def test_ragged_lengths(L, dtype, d):
    """Lengths that are not a multiple of the chunk or of the tile."""
    w = W.Workload("ragged", B=1, Hq=4, Hkv=2, L=L, d=d, C=64, topk=4, M=128, dtype=dtype,
                   lmk_noise=0.5, seed=77 + L)
    check_all_rows(w)


@pytest.mark.parametrize("topk", [1, 3, 64])
def test_topk_edges(topk):
    """k = 1, an odd k, and the maximum k = 64 (more than the completed
    chunks of most rows)."""
    w = W.Workload("topk", B=1, Hq=2, Hkv=1, L=64 * 70 + 17, d=128, C=64, topk=topk, M=64,
                   dtype="bf16", q_kind="ar1", q_sigma=0.05, lmk_noise=0.5, seed=5)
    check_all_rows(w, with_wfin=True)


def test_staged_epilogue_k32_all_rows():
    """bf16, d=128, k=32 on rows with more than 32 completed chunks (the
    selection's rows leave through the per-warp staging blocks for K = 32),
    and a ragged last tile (29 rows) whose warps past L write nothing."""
    w = W.PREFILL_128K.with_(Hq=4, Hkv=2, L=64 * 40 + 29)
    st = check_all_rows(w)
    assert st["near_ties"] <= 0.01 * w.B * w.Hq * w.L


def test_deterministic():
    w = W.PREFILL_128K.with_(Hq=4, Hkv=1, L=2048)
    q, k, v, lmk = (x.cuda() for x in synth.make_inputs(w, "cpu"))
    a = gpu_prefill(q, k, v, lmk, w)
    b = gpu_prefill(q, k, v, lmk, w)
    for key in ("sel", "w", "lse_lmk", "out", "lse"):
        assert torch.equal(a[key], b[key]), key


def test_group_size_does_not_change_results():
    """The prefill kernels always walk 128-row tiles; M only sets the groups
    hils_union reports.  Every output is therefore bit-identical across M."""
    w = W.PREFILL_128K.with_(Hq=4, Hkv=1, L=2048)
    q, k, v, lmk = (x.cuda() for x in synth.make_inputs(w, "cpu"))
    outs = [gpu_prefill(q, k, v, lmk, w.with_(M=m)) for m in (16, 32, 64, 128)]
    for o in outs[1:]:
        for key in ("sel", "w", "lse_lmk", "out", "lse"):
            assert torch.equal(o[key], outs[0][key]), key


def test_union_matches_oracle():
    """hils_union: the CSR union of every group equals the oracle's set union
    bit for bit."""
    w = W.PREFILL_128K.with_(Hq=4, Hkv=2, L=1000, topk=8)
    q, k, v, lmk = synth.make_inputs(w, "cpu")
    sel, _, _ = hb.select(q.cuda(), lmk.cuda(), w.topk, w.M)
    for M in (16, 64, 128):
        u_off, u_idx = hb.union(sel, M=M)
        u_off, u_idx = u_off.cpu().numpy(), u_idx.cpu().numpy()
        s = sel.reshape(-1, w.topk).cpu().numpy()
        gph = (w.L + M - 1) // M
        for head in range(w.B * w.Hq):
            for g in range(gph):
                gid = head * gph + g
                want = oracle.union(w.L, w.C, w.topk, M, head, g, s)
                assert np.array_equal(u_idx[u_off[gid]:u_off[gid + 1]], want), (M, head, g)


def test_debug_checks_report_bad_selection():
    """A corrupted selection (a chunk that is not completed for its row) is
    reported as HILS_ERR_DEVICE_CHECK by the debug mode; nothing faults."""
    w = W.PREFILL_128K.with_(Hq=2, Hkv=1, L=512, topk=4)
    q, k, v, lmk = (x.cuda() for x in synth.make_inputs(w, "cpu"))
    sel, cw, _ = hb.select(q, lmk, w.topk, w.M)
    bad = sel.clone()
    bad[0, 0, 300, 0] = 300 // 64  # the row's own chunk: not a completed chunk
    with pytest.raises(hb.HilsError) as ei:
        hb.attn_fwd(q, k, v, bad, cw, w.M, debug_checks=True)
    assert ei.value.status == 5
    hb.attn_fwd(q, k, v, sel, cw, w.M, debug_checks=True)  # the intact selection passes


@pytest.mark.parametrize("w", [W.SMALL_32K, W.PREFILL_128K, W.PREFILL_512K], ids=lambda w: w.name)
def test_full_size_sampled_rows(w):
    """The full workloads, in the launch configuration the benchmark times,
    checked on a seeded sample of rows."""
    dq, dk, dv, dl = synth.make_inputs(w, "cuda")
    res = gpu_prefill(dq, dk, dv, dl, w)
    rows = sample_rows(w.B, w.Hq, w.L, w.C, 320, seed=w.seed)
    q, k, v, lmk = (x.cpu() for x in (dq, dk, dv, dl))
    del dq, dk, dv, dl
    ref = oracle.rows(problem(w), q, k, v, lmk, rows)
    st = compare_rows(problem(w), (q, k, v, lmk), rows,
                      gather(res, torch.from_numpy(rows).cuda(), w.topk, w.d), ref, w.dtype)
    assert st["near_ties"] <= 0.02 * len(rows)

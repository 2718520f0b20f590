"""Host-side arithmetic of bench.py on CPU: the algorithmic work and bytes
the roofline divides by, and the rule that a DRAM-traffic record is used only
while the kernel's sources are the ones it was captured from."""
import json

import torch

import bench
from chunk_wise_hierarchical_landmark_b200 import workloads as W


def test_prefill_work_counts_rows_one_by_one():
    w = W.PREFILL_128K.with_(B=2, Hq=3, Hkv=1, L=300, d=8, topk=2)
    score = attn = 0
    for t in range(w.L):
        n_c = t // w.C
        score += 2 * w.d * n_c
        attn += 4 * w.d * (min(w.topk, n_c) * w.C + t - (t // w.C) * w.C + 1)
    got = bench.prefill_work(w)
    assert got["score_flop"] == score * w.B * w.Hq
    assert got["attn_flop"] == attn * w.B * w.Hq


def test_decode_bytes_counts_the_union_once():
    # N = 200: own chunk 3 holds 8 keys; 3 landmark rows per KV head
    w = W.DECODE_512K.with_(B=1, Hq=4, Hkv=2, L=200, d=8, topk=2, dtype="bf16")
    sel = torch.tensor([[[0, 1], [1, -1], [2, 0], [2, 3 - 1]]], dtype=torch.int32)
    # KV head 0 (query heads 0, 1): {0, 1} + own -> 2 full chunks + 8 own keys
    # KV head 1 (query heads 2, 3): {0, 2} + own -> 2 full chunks + 8 own keys
    keys = (2 * 64 + 8) + (2 * 64 + 8)
    want = 2 * 3 * 8 * 2 + 2 * keys * 8 * 2
    assert bench.decode_bytes(w, sel) == want


def test_traffic_record_follows_its_sources(tmp_path, monkeypatch):
    files = ["attn_sm100.cu", "kernels.h"]
    rec = {"hils_attn_fwd": {"workload": "wl", "bytes_per_launch": 123, "sources": files,
                             "source_hash": bench.source_hash(files)}}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.load_traffic("hils_attn_fwd", "wl") == 123
    assert bench.load_traffic("hils_attn_fwd", "other workload") is None
    rec["hils_attn_fwd"]["source_hash"] = "0" * 16
    path.write_text(json.dumps(rec))
    assert bench.load_traffic("hils_attn_fwd", "wl") is None


def test_select_executed_flop_counts_mma_tiles():
    w = W.PREFILL_128K.with_(B=1, Hq=2, Hkv=1, L=64 * 300 + 5, d=64, topk=4)
    want = 0
    for t0 in range(0, w.L, 128):
        t_last = min(t0 + 127, w.L - 1)
        n = min(t_last // w.C, w.L // w.C)
        if n > 0:
            want += 2 * 128 * 64 * w.d                          # seed tile
        if n > w.topk:
            want += -(-n // 64) * 2 * 128 * 64 * (w.d + 16)     # scan with the masking step
    assert bench.select_executed_flop(w) == want * w.B * w.Hq


def test_near_tie_sample_flags_a_wrong_selection():
    """The bench's sampled selection check agrees with the oracle's top-k and
    counts a planted wrong index outside any near-tie."""
    import numpy as np
    import oracle
    from chunk_wise_hierarchical_landmark_b200 import synth
    w = W.PREFILL_128K.with_(Hq=2, Hkv=1, L=640, topk=3)
    q, k, v, lmk = synth.make_inputs(w, "cpu")
    p = oracle.Problem(w.B, w.Hq, w.Hkv, w.L, w.d, w.C, w.topk, w.scale)
    rows = np.arange(w.B * w.Hq * w.L)
    ref = oracle.rows(p, q, k, v, lmk, rows)
    sel = torch.from_numpy(np.ascontiguousarray(ref["sel"])).reshape(w.B, w.Hq, w.L, w.topk)
    st = bench.near_tie_sample(w, q, lmk, sel, n_rows=200, seed=3)
    assert st["index_mismatches"] == st["mismatches_outside_near_ties"] == 0
    # plant a wrong chunk in every sampled row that has more than k candidates
    rs = np.random.default_rng(3).integers(0, w.B * w.Hq * w.L, size=200)
    bad = sel.clone()
    planted = 0
    for r in set(rs.tolist()):
        bh, t = divmod(r, w.L)
        if t // w.C > w.topk:
            row = bad[0, bh, t]
            unused = [c for c in range(t // w.C) if c not in row.tolist()]
            row[0] = unused[0]
            planted += 1
    st = bench.near_tie_sample(w, q, lmk, bad, n_rows=200, seed=3)
    assert planted > 0 and st["index_mismatches"] >= planted - st["near_ties"]


def test_backward_work_counts_rows_one_by_one():
    w = W.PREFILL_128K.with_(B=1, Hq=2, Hkv=1, L=200, d=8, topk=2)
    want = 0
    for t in range(w.L):
        n_c = t // w.C
        keys = min(w.topk, n_c) * w.C + t % w.C + 1
        want += 10 * w.d * keys + 4 * w.d * min(w.topk, n_c)
    assert bench.backward_work(w) == want * w.B * w.Hq

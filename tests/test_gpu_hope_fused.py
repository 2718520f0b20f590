"""The fused HoPE prefill (hils_prefill_hope: the queries are rotated while the
scoring and attention kernels stage them) against the two-step path it
replaces, hils_hope on the queries followed by hils_prefill: every output
bit for bit.  The two-step path's pieces are each checked against the
oracle (the rotation in the HoPE tests, the prefill in the prefill tests),
and the fused kernels use the same rotation arithmetic, so equality here
carries that parity over without feeding a kernel's output to the oracle."""
import pytest
import torch

from chunk_wise_hierarchical_landmark_b200 import binding as hb
from chunk_wise_hierarchical_landmark_b200 import synth
from chunk_wise_hierarchical_landmark_b200 import workloads as W

pytestmark = pytest.mark.gpu

CASES = [
    # d=128 GQA 8/2, ragged length, the split rule's pair count at base 5e5
    (W.PREFILL_128K.with_(Hq=8, Hkv=2, L=1000, topk=8), 46, 500000.0, 0),
    # positions far from zero (a suffix of a long prompt), every pair rotating
    (W.PREFILL_128K.with_(Hq=4, Hkv=4, L=777, topk=4), 64, 500000.0, 3_000_000),
    # d=64 MHA, two batches, one rotating pair only
    (W.SMALL_32K.with_(B=2, Hq=2, Hkv=2, L=700, topk=16), 1, 10000.0, 17),
    # shorter than a chunk: no landmark, attention over the prefix only
    (W.PREFILL_128K.with_(Hq=2, Hkv=1, L=50, topk=4), 40, 500000.0, 5),
    # zero pairs: NoPE throughout, the fused call must equal the plain prefill
    (W.PREFILL_128K.with_(Hq=4, Hkv=2, L=300, topk=4), 0, 500000.0, 0),
]


@pytest.mark.parametrize("w,n_pairs,base,pos0", CASES,
                         ids=["gqa_46", "far_pos0", "d64_1pair", "short", "zero_pairs"])
def test_fused_hope_equals_prepass(w, n_pairs, base, pos0):
    q, k, v, lmk = (t.cuda() for t in synth.make_inputs(w, "cpu"))
    # keys enter the cache rotated, once
    k_rot = k.clone()
    hb.hils_hope(k_rot, n_pairs, pos0, base)
    q_rot = q.clone()
    hb.hils_hope(q_rot, n_pairs, pos0, base)
    ref = hb.prefill(q_rot, k_rot, v, lmk, w.topk, w.M, debug_checks=True)
    got = hb.prefill_hope(q, k_rot, v, lmk, w.topk, n_pairs, base, pos0, w.M, debug_checks=True)
    torch.cuda.synchronize()
    for name in ("sel_idx", "chunk_w", "lse_lmk", "out", "lse"):
        a, b = got[name], ref[name]
        if name == "out":
            a, b = a.view(torch.int16), b.view(torch.int16)
        elif a.dtype == torch.float32:
            a, b = a.view(torch.int32), b.view(torch.int32)
        assert torch.equal(a, b), f"{name}: {(a != b).sum().item()} elements differ"
    # the caller's q is not modified
    assert torch.equal(q, synth.make_inputs(w, "cpu")[0].cuda())


def test_fused_hope_rejects_f32_and_bad_args():
    w = W.TINY_F32.with_(L=200)
    q, k, v, lmk = (t.cuda() for t in synth.make_inputs(w, "cpu"))
    with pytest.raises(hb.HilsError):
        hb.prefill_hope(q, k, v, lmk, w.topk, 8, 10000.0)
    wb = W.PREFILL_128K.with_(Hq=2, Hkv=1, L=200, topk=4)
    q, k, v, lmk = (t.cuda() for t in synth.make_inputs(wb, "cpu"))
    for bad in (dict(n_rope_pairs=65, base=1e4), dict(n_rope_pairs=8, base=1.0),
                dict(n_rope_pairs=-1, base=1e4), dict(n_rope_pairs=8, base=1e4, pos0=-3)):
        with pytest.raises(hb.HilsError):
            hb.prefill_hope(q, k, v, lmk, wb.topk, **bad)

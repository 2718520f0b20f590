"""The failure path of the bounded device waits, made to run out on purpose
without any fault: the scoring kernel keeps back one arrival on its first
landmark tile (hils_test_set_wait_limit), the MMA issuer's wait gives up
after a short limit, every role of every CTA unwinds through the common
teardown, and the call reports HILS_ERR_TIMEOUT in debug mode.  A normal call
right afterwards must be exact again (the context stays usable)."""
import pytest
import torch

from chunk_wise_hierarchical_landmark_b200 import binding as hb
from chunk_wise_hierarchical_landmark_b200 import synth
from chunk_wise_hierarchical_landmark_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_withheld_arrival_times_out_and_the_next_call_is_exact():
    w = W.PREFILL_128K.with_(Hq=4, Hkv=1, L=2048, topk=8)
    q, k, v, lmk = (x.cuda() for x in synth.make_inputs(w, "cpu"))
    ref = hb.prefill(q, k, v, lmk, w.topk, w.M)
    torch.cuda.synchronize()
    try:
        hb.lib().hils_test_set_wait_limit(20_000_000, 1)  # 20 ms, first arrival withheld
        with pytest.raises(hb.HilsError) as ei:
            hb.select(q, lmk, w.topk, w.M, debug_checks=True)
        assert ei.value.status == 6, str(ei.value)
        # the short limit alone (nothing withheld) does not fire on a normal call
        hb.lib().hils_test_set_wait_limit(20_000_000, 0)
        sel, cw, lse_lmk = hb.select(q, lmk, w.topk, w.M, debug_checks=True)
    finally:
        hb.lib().hils_test_set_wait_limit(0, 0)
    again = hb.prefill(q, k, v, lmk, w.topk, w.M, debug_checks=True)
    torch.cuda.synchronize()
    assert torch.equal(sel, ref["sel_idx"]) and torch.equal(cw, ref["chunk_w"])
    for key in ("sel_idx", "chunk_w", "lse_lmk", "out", "lse"):
        assert torch.equal(again[key], ref[key]), key

"""The allocation-free decode entry point, hils_decode_fwd_noalloc.

It serves callers that cannot allocate device memory (a framework that owns
the whole GPU's memory through its own pool, or a per-token loop where a
cudaMalloc/cudaFree pair would synchronise the device): its scratch lives in
a fixed 32 MiB array inside the library.  This file is collected last so
that a failure here does not hide the results of the other tests."""
import ctypes

import pytest
import torch

from chunk_wise_hierarchical_landmark_b200 import binding as hb
from chunk_wise_hierarchical_landmark_b200 import synth
from chunk_wise_hierarchical_landmark_b200 import workloads as W
from tests.parity import tolerances

pytestmark = pytest.mark.gpu


def _outputs(w, dev):
    return dict(
        sel=torch.full((w.B, w.Hq, w.topk), -7, dtype=torch.int32, device=dev),
        w=torch.full((w.B, w.Hq, w.topk), 7.0, dtype=torch.float32, device=dev),
        lse_lmk=torch.full((w.B, w.Hq), 7.0, dtype=torch.float32, device=dev),
        out=torch.full((w.B, w.Hq, w.d), 7.0, dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32, device=dev),
        lse=torch.full((w.B, w.Hq), 7.0, dtype=torch.float32, device=dev),
    )


@pytest.mark.parametrize("w,debug", [
    (W.DECODE_512K.with_(B=2, L=3000, topk=16), False),
    (W.DECODE_512K.with_(B=2, Hq=8, Hkv=2, L=2500, d=64, topk=8, dtype="f32"), False),
    # debug mode: the error word sits at the start of the library's array
    (W.DECODE_512K.with_(B=2, L=3000, topk=16), True),
    (W.DECODE_512K.with_(B=16, L=524288), False),  # the full decode workload (17.6 MB of scratch)
], ids=["small", "small_f32", "small_debug", "full"])
def test_noalloc_matches_workspace_decode_twice(w, debug):
    dev = torch.device("cuda")
    q, k, v, lmk = synth.make_inputs(w, "cuda")
    p = hb.make_params(w.B, w.Hq, w.Hkv, w.L, w.d, w.topk, w.M, w.C, w.scale, q.dtype,
                       debug_checks=debug)
    ref = _outputs(w, dev)
    hb.hils_decode_fwd(p, q, k, v, lmk, ref["sel"], ref["w"], ref["lse_lmk"], ref["out"],
                       ref["lse"], hb.workspace(p, hb.HILS_OP_DECODE, dev))
    tol = tolerances(w.dtype)
    for _ in range(2):  # two calls in a row share (and reuse) the library's scratch array
        got = _outputs(w, dev)
        hb.hils_decode_fwd_noalloc(p, q, k, v, lmk, got["sel"], got["w"], got["lse_lmk"],
                                   got["out"], got["lse"])
        torch.cuda.synchronize()
        assert torch.equal(got["sel"], ref["sel"])
        assert (got["w"] - ref["w"]).nan_to_num(0.0).abs().max().item() <= tol["w"]
        assert torch.equal(torch.isneginf(got["w"]), torch.isneginf(ref["w"]))
        err = (got["out"].float() - ref["out"].float()).abs()
        assert err.max().item() <= tol["out_max"] and err.mean().item() <= tol["out_mean"]
        assert (got["lse"] - ref["lse"]).abs().max().item() <= tol["lse"]
        assert (got["lse_lmk"] - ref["lse_lmk"]).abs().max().item() <= tol["lse_lmk"]


def test_noalloc_rejects_shapes_beyond_its_scratch():
    p = hb.make_params(B=64, Hq=32, Hkv=8, L=524288, d=128, topk=64)  # needs ~70 MB of scratch
    fake = ctypes.c_void_p(1 << 20)
    rc = hb.lib().hils_decode_fwd_noalloc(ctypes.byref(p), fake, fake, fake, fake, fake, fake,
                                         None, fake, fake, None)
    assert rc == 3  # HILS_ERR_WORKSPACE, before any launch
    assert b"32 MiB" in hb.lib().hils_last_error()

"""GPU parity of the decode step over a paged KV cache (hils_decode_fwd_paged).

A page holds one 64-token chunk of every KV head ([num_pages, Hkv, 64, d]).
The pool is shuffled, unused pages, unused page-table columns and the tail of
a partial last page hold NaN, so a read of anything the table does not
describe shows up in the outputs.  The results must equal the dense decode
over the same caches bit for bit (the same kernels, the same data) and match
the oracle's paged decode."""
import numpy as np
import pytest
import torch

import oracle
from chunk_wise_hierarchical_landmark_b200 import binding as hb
from chunk_wise_hierarchical_landmark_b200 import synth
from chunk_wise_hierarchical_landmark_b200 import workloads as W
from tests.parity import compare_rows
from tests.test_gpu_decode import problem, to_np

pytestmark = pytest.mark.gpu

C = 64


def paginate(k, v, seed, spare_pages=5, spare_cols=3):
    """Pools [B*npg + spare, Hkv, C, d] in a shuffled order, and the table."""
    B, Hkv, N, d = k.shape
    npg = -(-N // C)
    g = torch.Generator().manual_seed(seed)
    num_pages = B * npg + spare_pages
    perm = torch.randperm(num_pages, generator=g)[:B * npg]
    table = torch.full((B, npg + spare_cols), -1, dtype=torch.int32)
    kp = torch.full((num_pages, Hkv, C, d), float("nan"), dtype=k.dtype)
    vp = torch.full((num_pages, Hkv, C, d), float("nan"), dtype=v.dtype)
    for b in range(B):
        for c in range(npg):
            page = int(perm[b * npg + c])
            table[b, c] = page
            n = min(C, N - c * C)
            kp[page, :, :n] = k[b, :, c * C:c * C + n]
            vp[page, :, :n] = v[b, :, c * C:c * C + n]
    return kp, vp, table


@pytest.mark.parametrize("N", [1, 65, 3000 + 37])
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_paged_equals_dense_and_oracle(N, dtype, d):
    w = W.DECODE_512K.with_(B=2, Hq=8, Hkv=2, L=N, d=d, dtype=dtype, topk=16, seed=500 + N)
    q, k, v, lmk = synth.make_inputs(w, "cpu")
    kp, vp, table = paginate(k, v, seed=N)
    got = hb.decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), lmk.cuda(), N, w.topk)
    dense = hb.decode(q.cuda(), k.cuda(), v.cuda(), lmk.cuda(), w.topk)
    torch.cuda.synchronize()
    for key in ("sel_idx", "chunk_w", "lse_lmk", "out", "lse"):
        assert torch.equal(got[key], dense[key]), key
    heads = np.arange(w.B * w.Hq)
    ref = oracle.decode_paged(problem(w), q, kp, vp, table, lmk, heads)
    compare_rows(problem(w), (q, k, v, lmk), heads, to_np(got, w.d), ref, w.dtype, decode=True)


def test_paged_shared_pages():
    """Two sequences whose tables name the same pages give the same result."""
    w = W.DECODE_512K.with_(B=2, Hq=8, Hkv=2, L=2000, topk=16, seed=601)
    q, k, v, lmk = synth.make_inputs(w, "cpu")
    kp, vp, table = paginate(k, v, seed=7)
    table[1] = table[0]
    lmk[1] = lmk[0]
    q[1] = q[0]
    got = hb.decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), lmk.cuda(), w.L, w.topk)
    torch.cuda.synchronize()
    for key in ("sel_idx", "out", "lse"):
        assert torch.equal(got[key][0], got[key][1]), key


def test_paged_entry_outside_pool_is_reported():
    """With debug checks, a table entry outside [0, num_pages) is caught by the
    kernel's own bounds check (no copy is issued for it) and reported."""
    w = W.DECODE_512K.with_(B=1, Hq=4, Hkv=1, L=1000, topk=4, seed=602)
    q, k, v, lmk = synth.make_inputs(w, "cpu")
    kp, vp, table = paginate(k, v, seed=8)
    own = (w.L - 1) // C  # every head attends its own chunk, so this entry is read
    table[0, own] = kp.shape[0] + 7
    with pytest.raises(hb.HilsError) as e:
        hb.decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), lmk.cuda(), w.L, w.topk,
                        debug_checks=True)
    assert "device-side check" in str(e.value)
    torch.cuda.synchronize()


def test_paged_full_size():
    """The full decode workload (B=16, N=524288, k=64) through a shuffled
    page pool: equal to the dense decode on every head."""
    w = W.DECODE_512K
    q, k, v, lmk = synth.make_inputs(w, "cuda")
    dense = hb.decode(q, k, v, lmk, w.topk)
    npg = w.L // C
    g = torch.Generator(device="cuda").manual_seed(11)
    perm = torch.randperm(w.B * npg, generator=g, device="cuda")
    table = perm.view(w.B, npg).to(torch.int32)
    kp = torch.empty((w.B * npg, w.Hkv, C, w.d), dtype=k.dtype, device="cuda")
    vp = torch.empty_like(kp)
    for b in range(w.B):
        kp.index_copy_(0, perm[b * npg:(b + 1) * npg], k[b].view(w.Hkv, npg, C, w.d).transpose(0, 1))
        vp.index_copy_(0, perm[b * npg:(b + 1) * npg], v[b].view(w.Hkv, npg, C, w.d).transpose(0, 1))
    del k, v
    got = hb.decode_paged(q, kp, vp, table, lmk, w.L, w.topk)
    torch.cuda.synchronize()
    for key in ("sel_idx", "out", "lse"):
        assert torch.equal(got[key], dense[key]), key

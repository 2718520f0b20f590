"""GPU parity of the HoPE pre-pass (hils_hope) against the oracle's hope().

The oracle rotates in fp64 from the same (bf16 or fp32) input values.  The
kernel forms the angle in double precision, reduces it modulo 2*pi and
evaluates sincosf in fp32, so per element the error is within a few fp32
ulps of the two inputs' magnitudes; bf16 outputs add their own rounding
(at most half an ulp, 2^-8 relative)."""
import numpy as np
import pytest
import torch

import oracle
from chunk_wise_hierarchical_landmark_b200 import binding as hb

pytestmark = pytest.mark.gpu


def check(x, n_pairs, pos0, base):
    B, H, L, d = x.shape
    ref = oracle.hope(x.reshape(B * H, L, d), np.arange(L) + pos0, n_pairs, base)
    y = x.cuda()
    hb.hils_hope(y, n_pairs, pos0, base)
    got = y.float().cpu().numpy().reshape(B * H, L, d).astype(np.float64)
    xa = x.float().numpy().reshape(B * H, L, d).astype(np.float64)
    half = d // 2
    mag = np.abs(xa[..., :half]) + np.abs(xa[..., half:])
    mag = np.concatenate([mag, mag], -1)
    tol = 2e-6 * mag + 1e-30
    if x.dtype == torch.bfloat16:
        tol = tol + 2.0 ** -8 * np.abs(ref)
    err = np.abs(got - ref)
    assert (err <= tol).all(), f"max excess {(err - tol).max():.3g}"
    # NoPE pairs are bit-for-bit untouched
    keep = [j for j in range(half) if j >= n_pairs]
    keep = keep + [j + half for j in keep]
    assert np.array_equal(got[..., keep], xa[..., keep])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("d,n_pairs", [(128, 46), (128, 64), (64, 1), (64, 17), (64, 32)])
@pytest.mark.parametrize("L,pos0", [(1, 0), (1000, 0), (333, 4_000_000 - 333)])
def test_hope_matches_oracle(dtype, d, n_pairs, L, pos0):
    g = torch.Generator().manual_seed(d * 1000 + n_pairs + L)
    x = torch.randn((2, 3, L, d), generator=g).to(dtype)
    check(x, n_pairs, pos0, 500000.0 if d == 128 else 10000.0)


def test_hope_decode_query_and_zero_pairs():
    """A decode query [B,H,d] takes one position; n_rope_pairs = 0 is a no-op."""
    g = torch.Generator().manual_seed(5)
    q = torch.randn((4, 8, 128), generator=g).to(torch.bfloat16)
    y = q.cuda()
    hb.hils_hope(y, 40, pos0=524287, base=500000.0)
    ref = oracle.hope(q.reshape(32, 1, 128), [524287], 40, 500000.0).reshape(4, 8, 128)
    assert np.abs(y.float().cpu().numpy() - ref).max() <= 2.0 ** -8 * np.abs(ref).max() + 1e-5
    z = q.cuda()
    hb.hils_hope(z, 0, pos0=7)
    assert torch.equal(z.cpu(), q)

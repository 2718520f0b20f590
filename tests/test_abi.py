"""The C-ABI library loads, exports every symbol include/hils.h declares, and
rejects bad arguments before launching anything (runs without a GPU: no call
here reaches a kernel)."""
import ctypes
import os
import re

import pytest

from chunk_wise_hierarchical_landmark_b200 import binding as hb
from chunk_wise_hierarchical_landmark_b200 import build as hbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "hils.h")


@pytest.fixture(scope="module")
def lib():
    hbuild.build()
    return hb.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hils_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), f"{n} declared in hils.h but not exported"
    assert set(hb.EXPORTS) <= set(names)


def _params(**kw):
    base = dict(B=1, Hq=4, Hkv=2, L=1024, d=128, topk=8, M=64)
    base.update(kw)
    return hb.make_params(**base)


FAKE = ctypes.c_void_p(1 << 20)       # aligned, never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p((1 << 20) + 4)


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), 2), (dict(topk=65), 2), (dict(topk=0), 1), (dict(Hq=3, Hkv=2), 1),
    (dict(M=48), 2), (dict(L=0), 1), (dict(L=(1 << 24) + 1), 2), (dict(chunk=32), 2),
])
def test_bad_params_rejected(lib, kw, status):
    p = _params(**kw)
    rc = lib.hils_select(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, None, 0, None)
    assert rc == status, hb.lib().hils_last_error()
    assert lib.hils_last_error().decode()


def test_null_and_misaligned_pointers_rejected(lib):
    p = _params()
    assert lib.hils_select(None, FAKE, FAKE, FAKE, FAKE, None, None, 0, None) == 1
    assert lib.hils_select(ctypes.byref(p), None, FAKE, FAKE, FAKE, None, None, 0, None) == 1
    assert lib.hils_select(ctypes.byref(p), MISALIGNED, FAKE, FAKE, FAKE, None, None, 0, None) == 1
    assert b"aligned" in lib.hils_last_error()
    assert lib.hils_attn_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None,
                             None, 0, None) == 1
    assert lib.hils_decode_fwd(ctypes.byref(p), FAKE, FAKE, None, FAKE, FAKE, FAKE, None, FAKE,
                               FAKE, None, 0, None) == 1


def test_debug_mode_needs_workspace(lib):
    p = _params(debug_checks=True)
    assert lib.hils_workspace_size(ctypes.byref(p), hb.HILS_OP_PREFILL) >= 4
    rc = lib.hils_attn_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None,
                           0, None)
    assert rc == 3


def test_workspace_and_capacity(lib):
    p = _params()
    assert lib.hils_workspace_size(ctypes.byref(p), hb.HILS_OP_PREFILL) == 0
    assert lib.hils_workspace_size(ctypes.byref(p), 7) == 0
    cap = lib.hils_union_capacity(ctypes.byref(p))
    assert cap == 1 * 4 * (1024 // 64) * min(16, 64 * 8 + 1 + 2)
    bad = _params(d=96)
    assert lib.hils_union_capacity(ctypes.byref(bad)) == -1


def test_status_strings(lib):
    for s in range(7):
        assert lib.hils_status_string(s)
    assert lib.hils_status_string(0) == b"ok"
    assert lib.hils_launch_count() >= 0


def test_decode_workspace_size(lib):
    p = hb.make_params(B=16, Hq=32, Hkv=8, L=524288, d=128, topk=64)
    n = lib.hils_workspace_size(ctypes.byref(p), hb.HILS_OP_DECODE)
    assert 10_000_000 < n < 100_000_000   # slab top-k lists, union, attention partials
    too_many_heads = hb.make_params(B=1, Hq=32, Hkv=2, L=4096, d=128, topk=8)
    assert lib.hils_workspace_size(ctypes.byref(too_many_heads), hb.HILS_OP_DECODE) == 0
    rc = lib.hils_decode_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                             FAKE, None, 0, None)
    assert rc == 3   # workspace too small, rejected before any launch


def test_paged_decode_rejects_bad_tables(lib):
    """hils_decode_fwd_paged: a table narrower than the pages of N, an empty
    pool or a missing table are refused before any launch."""
    p = _params(L=1000)  # 1000 tokens: 16 pages of 64

    def call(num_pages, table, max_pages):
        return lib.hils_decode_fwd_paged(ctypes.byref(p), FAKE, FAKE, FAKE, num_pages, table,
                                         max_pages, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE,
                                         1 << 20, None)
    assert call(16, FAKE, 15) == 1
    assert call(0, FAKE, 16) == 1
    assert call(16, None, 16) == 1
    assert call(16, MISALIGNED, 16) == 1


@pytest.mark.parametrize("kw", [dict(n_rope_pairs=65), dict(n_rope_pairs=-1), dict(base=1.0),
                                dict(base=float("nan")), dict(d=96), dict(L=0), dict(dtype=7),
                                dict(pos0=-1), dict(pos0=(1 << 31) - 10, L=20)])
def test_hope_rejects_bad_arguments(lib, kw):
    """hils_hope validates before any launch."""
    a = dict(dtype=hb.HILS_BF16, B=1, H=2, L=16, d=128, pos0=0, n_rope_pairs=8, base=10000.0)
    a.update(kw)
    rc = lib.hils_hope(FAKE, a["dtype"], a["B"], a["H"], a["L"], a["d"], a["pos0"],
                       a["n_rope_pairs"], a["base"], None)
    assert rc in (1, 2), lib.hils_last_error()
    assert lib.hils_hope(None, hb.HILS_BF16, 1, 1, 1, 64, 0, 1, 10000.0, None) == 1


def test_hope_split_rule_matches_the_oracle(lib):
    """hils_hope_rope_pairs (the library's HoPE split) equals the pinned
    oracle split on a grid of head sizes, bases and windows, and refuses
    arguments outside its domain."""
    import oracle
    for d in (2, 16, 64, 128):
        for base in (1.5, 10000.0, 500000.0):
            for train in (1, 6, 2 * 3.141592653589793, 4096, 65536, 1e12):
                assert lib.hils_hope_rope_pairs(d, base, float(train)) == oracle.rope_pairs(d, base, train)
                assert hb.rope_pairs_for(d, base, train) == oracle.rope_pairs(d, base, train)
    assert lib.hils_hope_rope_pairs(1, 1e4, 100.0) == -1
    assert lib.hils_hope_rope_pairs(64, 1.0, 100.0) == -1
    assert lib.hils_hope_rope_pairs(64, 1e4, float("nan")) == -1


def test_qcal_rejects_bad_arguments(lib):
    p = _params()
    assert lib.hils_qcal_workspace_size(ctypes.byref(p), 0) == 0
    assert lib.hils_qcal_workspace_size(ctypes.byref(p), 65) == 0
    assert lib.hils_qcal_workspace_size(ctypes.byref(p), 16) == 256 + 1 * 1024 * 16 * 4
    ws = lib.hils_qcal_workspace_size(ctypes.byref(p), 16)
    args = lambda D, r, wsb: (ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, D, r, FAKE, FAKE, wsb, None)
    assert lib.hils_qcal_query(*args(512, 0, ws)) == 2      # rank outside 1..64
    assert lib.hils_qcal_query(*args(512, 65, ws)) == 2
    assert lib.hils_qcal_query(*args(0, 16, ws)) == 1       # D < 1
    assert lib.hils_qcal_query(*args(512, 16, ws - 1)) == 3  # workspace too small
    assert lib.hils_qcal_query(ctypes.byref(p), FAKE, MISALIGNED, FAKE, FAKE, 512, 16, FAKE, FAKE,
                               ws, None) == 1

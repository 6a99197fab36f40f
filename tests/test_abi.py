"""The C-ABI library loads on a host without a GPU, exports every symbol the header
declares, and rejects bad host-side arguments before touching the device."""
import ctypes
import os
import re

import pytest

import mla_absorbed_latent_mtp_b200 as m
from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "mla.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()
    return m.lib()


def test_exports_match_header(lib):
    declared = _declared()
    assert set(declared) == set(m.EXPORTS)
    for name in declared:
        assert hasattr(lib, name)


def test_status_strings(lib):
    assert m.status_string(0) == "MLA_OK"
    assert m.status_string(5) == "MLA_ERR_INDEX"
    assert m.status_string(6) == "MLA_ERR_TIMEOUT"
    assert m.status_string(99) == "MLA_ERR_UNKNOWN"


def test_workspace_query_rejects_bad_sizes(lib):
    assert lib.mla_attend_workspace_bytes(0, 1, 64, 512) == 0
    assert lib.mla_attend_workspace_bytes(1, 0, 64, 512) == 0
    assert lib.mla_attend_workspace_bytes(1, 1, 32, 512) == 0
    assert lib.mla_attend_workspace_bytes(1, 1, 64, 576) == 0


P = ctypes.c_void_p
GOOD = P(1 << 20)  # aligned dummy address; never dereferenced on these paths


def test_attend_rejects_host_errors(lib):
    f = lib.mla_attend_dense
    args = dict(qt=GOOD, c=GOOD, lens=None, B=1, Q=1, H=64, R=512, L=8, s=0.0625, ws=GOOD, wsb=1 << 30, o=GOOD)

    def call(**kw):
        a = dict(args, **kw)
        return f(a["qt"], a["c"], a["lens"], a["B"], a["Q"], a["H"], a["R"], a["L"], a["s"], a["ws"], a["wsb"], a["o"],
                 None, None, None)

    assert call(qt=None) == m.MLA_ERR_ARG
    assert call(o=None) == m.MLA_ERR_ARG
    assert call(B=0) == m.MLA_ERR_ARG
    assert call(Q=0) == m.MLA_ERR_ARG
    assert call(H=32) == m.MLA_ERR_UNSUPPORTED
    assert call(R=576) == m.MLA_ERR_UNSUPPORTED
    assert call(c=P((1 << 20) + 2)) == m.MLA_ERR_UNSUPPORTED
    assert call(L=0) == m.MLA_ERR_ARG
    assert call(s=float("nan")) == m.MLA_ERR_ARG


def test_paged_and_indexed_reject_host_errors(lib):
    g = lib.mla_attend_paged
    assert g(GOOD, GOOD, None, GOOD, 1, 1, 64, 512, 64, 4, 4, 0.0625, GOOD, 1 << 30, GOOD, None, None, None) == \
        m.MLA_ERR_ARG
    assert g(GOOD, GOOD, GOOD, GOOD, 1, 1, 64, 512, 32, 4, 4, 0.0625, GOOD, 1 << 30, GOOD, None, None, None) == \
        m.MLA_ERR_UNSUPPORTED
    # positions are int32: a sequence of max_pages * 64 >= 2^31 rows, or a pool that size, is refused
    assert g(GOOD, GOOD, GOOD, GOOD, 1, 1, 64, 512, 64, 1 << 25, 4, 0.0625, GOOD, 1 << 30, GOOD, None, None, None) == \
        m.MLA_ERR_ARG
    assert g(GOOD, GOOD, GOOD, GOOD, 1, 1, 64, 512, 64, 4, 1 << 25, 0.0625, GOOD, 1 << 30, GOOD, None, None, None) == \
        m.MLA_ERR_ARG
    h = lib.mla_attend_indexed
    assert h(GOOD, GOOD, None, None, 1, 1, 64, 512, 8, 4, 0.0625, GOOD, 1 << 30, GOOD, None, None, None) == \
        m.MLA_ERR_ARG
    assert h(GOOD, GOOD, GOOD, None, 1, 1, 64, 512, 8, 0, 0.0625, GOOD, 1 << 30, GOOD, None, None, None) == \
        m.MLA_ERR_ARG


def test_projections_reject_host_errors(lib):
    for f in (lib.mla_absorb_q, lib.mla_up_proj):
        assert f(None, GOOD, GOOD, 1, 64, 256, 512, None) == m.MLA_ERR_ARG
        assert f(GOOD, GOOD, GOOD, 0, 64, 256, 512, None) == m.MLA_ERR_ARG
        assert f(GOOD, GOOD, GOOD, 1, 64, 128, 512, None) == m.MLA_ERR_UNSUPPORTED
        assert f(GOOD, P((1 << 20) + 8), GOOD, 1, 64, 256, 512, None) == m.MLA_ERR_UNSUPPORTED


def test_debug_gather_rejects_host_errors(lib):
    f = lib.mla_debug_gather
    assert f(3, GOOD, None, None, 1, 1, 512, 8, 0, 0, 0, GOOD, 1, GOOD, None, None) == m.MLA_ERR_ARG
    assert f(1, GOOD, None, None, 1, 1, 512, 8, 0, 0, 0, GOOD, 1, GOOD, None, None) == m.MLA_ERR_ARG
    assert f(1, GOOD, GOOD, None, 1, 1, 512, 8, 1 << 25, 4, 0, GOOD, 1, GOOD, None, None) == m.MLA_ERR_ARG
    assert f(0, GOOD, None, None, 1, 1, 512, 8, 0, 0, 0, GOOD, 0, GOOD, None, None) == m.MLA_OK


def test_cache_bookkeeping_and_timeout_aid_reject_host_errors(lib):
    p = ctypes.c_void_p(16)
    # null store / lengths / rows, non-positive sizes, unsupported latent width
    assert lib.mla_cache_append_dense(None, p, p, 1, 1, 512, 8, None, None) == m.MLA_ERR_ARG
    assert lib.mla_cache_append_dense(p, p, p, 0, 1, 512, 8, None, None) == m.MLA_ERR_ARG
    assert lib.mla_cache_append_dense(p, p, p, 1, 0, 512, 8, None, None) == m.MLA_ERR_ARG
    assert lib.mla_cache_append_dense(p, p, p, 1, 1, 256, 8, None, None) == m.MLA_ERR_UNSUPPORTED
    assert lib.mla_cache_truncate_dense(p, p, None, 1, 1, 512, 8, None, None) == m.MLA_ERR_ARG
    assert lib.mla_cache_append_paged(p, None, p, p, 1, 1, 512, 64, 4, 4, None, None) == m.MLA_ERR_ARG
    assert lib.mla_cache_append_paged(p, p, p, p, 1, 1, 512, 32, 4, 4, None, None) == m.MLA_ERR_UNSUPPORTED
    assert lib.mla_cache_truncate_paged(p, p, p, p, 1, 1, 512, 64, 0, 4, None, None) == m.MLA_ERR_ARG
    assert lib.mla_debug_wait_timeout(1000, None, None) == m.MLA_ERR_ARG
    assert lib.mla_debug_wait_timeout(0, p, None) == m.MLA_ERR_ARG


def test_kpool_entry_points_reject_host_errors(lib):
    """Every case below returns before any device call."""
    p, odd = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 20) + 4)
    keys = lib.mla_kpool_keys  # (cache, seq_lens, B, R, Lmax, pool, pooled, stream)
    assert keys(None, None, 1, 512, 64, 4, p, None) == m.MLA_ERR_ARG
    assert keys(p, None, 1, 512, 64, 4, None, None) == m.MLA_ERR_ARG
    assert keys(p, None, 0, 512, 64, 4, p, None) == m.MLA_ERR_ARG
    assert keys(p, None, 1, 512, 0, 4, p, None) == m.MLA_ERR_ARG
    assert keys(p, None, 1, 512, 64, 0, p, None) == m.MLA_ERR_ARG
    assert keys(p, None, 1, 256, 64, 4, p, None) == m.MLA_ERR_UNSUPPORTED
    assert keys(odd, None, 1, 512, 64, 4, p, None) == m.MLA_ERR_UNSUPPORTED
    assert keys(p, None, 1, 512, 64, 4, odd, None) == m.MLA_ERR_UNSUPPORTED
    assert keys(p, None, 65536, 512, 64, 4, p, None) == m.MLA_ERR_UNSUPPORTED  # grid rows
    assert keys(p, None, 1, 512, 3, 4, p, None) == m.MLA_OK  # no complete pool: nothing to launch

    sel = lib.mla_kpool_select  # (pooled, w_query, seq_lens, B, Q, R, Lmax, pool, topk, tail, indices, W, stream)

    def call(pooled=p, wq=p, B=1, Q=1, R=512, L=1024, pool=4, topk=16, tail=1, idx=p, W=None):
        W = topk + (pool - 1 if tail else 0) if W is None else W
        return sel(pooled, wq, None, B, Q, R, L, pool, topk, tail, idx, W, None)

    assert call(pooled=None) == m.MLA_ERR_ARG
    assert call(wq=None) == m.MLA_ERR_ARG
    assert call(idx=None) == m.MLA_ERR_ARG
    assert call(B=0) == m.MLA_ERR_ARG and call(Q=0) == m.MLA_ERR_ARG
    assert call(B=1 << 16, Q=1 << 15) == m.MLA_ERR_ARG  # B * Q query rows overflow the grid
    assert call(L=0) == m.MLA_ERR_ARG and call(pool=0) == m.MLA_ERR_ARG
    assert call(R=576) == m.MLA_ERR_UNSUPPORTED
    assert call(topk=2) == m.MLA_ERR_ARG            # fewer positions than one pool
    assert call(topk=18) == m.MLA_ERR_ARG           # not whole pools
    assert call(pool=1, topk=1025) == m.MLA_ERR_ARG  # more chosen pools than the list holds
    assert call(W=16) == m.MLA_ERR_ARG              # with a tail the width is topk + pool - 1
    assert call(tail=0, W=19) == m.MLA_ERR_ARG      # without one it is topk
    assert call(pooled=odd) == m.MLA_ERR_UNSUPPORTED
    assert call(pool=1, topk=16, L=64 * 1024) == m.MLA_ERR_UNSUPPORTED  # pooled scores exceed shared memory


def test_product_path_does_not_touch_oracle():
    """The binding and kernels never import the oracle (test infrastructure only)."""
    pkg = os.path.join(ROOT, "mla_absorbed_latent_mtp_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in text and "from oracle" not in text, fn

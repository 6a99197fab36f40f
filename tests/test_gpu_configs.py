"""Full-size workloads (the five synthetic configurations) through the whole path
(absorb -> attend -> up-project), in the launch configuration the benchmark times, checked
against the oracle on sampled (sequence, query) pairs: the absorbed fp64 form on all 64
heads (pinned to the expanded form by the oracle tests) and the expanded definition
itself on a few heads where its cost allows.  Gate: max-abs <= 2e-2, mean-abs <= 2e-3."""
import math

import numpy as np
import pytest
import torch

import mla_absorbed_latent_mtp_b200 as m
import oracle
import synth
from gpu_util import bf16_to_f64, pinned_cache
from helpers import MAX_ABS_TOL, MEAN_ABS_TOL, errors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def device():
    import __graft_entry__
    __graft_entry__.build()
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    yield
    torch.cuda.empty_cache()


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _run(wl):
    host = pinned_cache(wl)
    cache = host.cuda().view(torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    mode = {"dense": m.MODE_DENSE, "paged": m.MODE_PAGED, "indexed": m.MODE_INDEXED}[wl.mode]
    out, lse = m.mla_decode(
        _dev(wl.q), _dev(wl.w_uk), _dev(wl.w_uv), cache, torch.from_numpy(wl.seq_lens).cuda(), mode=mode,
        page_table=torch.from_numpy(wl.page_table).cuda() if wl.mode == "paged" else None,
        indices=torch.from_numpy(wl.indices).cuda() if wl.mode == "indexed" else None, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, m.status_string(int(st.item()))
    got = bf16_to_f64(out)
    assert np.all(np.isfinite(got)) and bool(torch.isfinite(lse).all())
    del cache
    if wl.mode == "paged":
        wl.pool = host.numpy().view(np.uint16)
    else:
        wl.cache = host.numpy().view(np.uint16)
    return got, lse.cpu().numpy()


def _check(wl, got, lse, pairs, expanded_heads):
    ref = oracle.reference(wl, pairs=pairs, form="absorbed")
    for (b, i), r in ref.items():
        mx, mean = errors(got[b, i], r["out"])
        assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (b, i, mx, mean)
        assert np.abs(lse[b, i] - r["lse"]).max() <= 5e-3
    if expanded_heads:
        exp = oracle.reference(wl, pairs=pairs[:1], heads=expanded_heads, form="expanded")
        for (b, i), r in exp.items():
            mx, mean = errors(got[b, i][expanded_heads], r["out"])
            assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (b, i, mx, mean)


def test_tiny_dense_decode_all_heads_expanded():
    wl = synth.make_workload("tiny_dense_decode", with_data=False)
    got, lse = _run(wl)
    _check(wl, got, lse, [(0, 0)], list(range(64)))


def test_dense_decode_full_size():
    wl = synth.make_workload("dense_decode", with_data=False)
    got, lse = _run(wl)
    _check(wl, got, lse, [(0, 0), (13, 0), (31, 0)], [0, 37])


def test_mtp_verify_full_size():
    wl = synth.make_workload("mtp_verify", with_data=False)
    got, lse = _run(wl)
    pairs = [(0, i) for i in range(6)] + [(15, 0), (15, 5)]
    _check(wl, got, lse, pairs, [5])


def test_ragged_paged_decode_full_size():
    wl = synth.make_workload("ragged_paged_decode", with_data=False)
    got, lse = _run(wl)
    lens = wl.seq_lens
    short, long_ = int(np.argmin(lens)), int(np.argmax(lens))
    _check(wl, got, lse, [(short, 0), (long_, 0), (7, 0)], [])
    exp = oracle.reference(wl, pairs=[(short, 0)], heads=[0, 63], form="expanded")
    mx, mean = errors(got[short, 0][[0, 63]], exp[(short, 0)]["out"])
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL


def test_indexed_sparse_decode_full_size():
    wl = synth.make_workload("indexed_sparse_decode", with_data=False)
    got, lse = _run(wl)
    _check(wl, got, lse, [(0, 0), (31, 0)], [0, 1, 2, 3, 60, 61, 62, 63])

"""GPU k-pool index producer against the oracle: pooled keys (fp32 against fp64), the
selection (identical lists; a difference is allowed only between pools whose fp64 scores
tie to within fp32 rounding), the causality and tail rules exactly, and the lists fed to
the index-list attention, whose -1 entries must contribute nothing."""
import math

import numpy as np
import pytest
import torch

import mla_absorbed_latent_mtp_b200 as m
import oracle
import synth
from gpu_util import bf16_to_f64, ints_to_dev, synthetic_qtilde, to_dev
from helpers import MAX_ABS_TOL, MEAN_ABS_TOL, errors, tiny_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def device():
    import __graft_entry__
    __graft_entry__.build()
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def _setup(lens, Q, pool, Lmax=None, seed=0):
    lens = np.asarray(lens, dtype=np.int32)
    B = len(lens)
    Lmax = int(lens.max()) if Lmax is None else Lmax
    cache = synth.normal_bf16((B, Lmax, 512), seed, synth.STREAM_CACHE)
    wq = synth.normal_bf16((B, Q, 512), seed, synth.STREAM_Q)
    return lens, cache, wq


def _check_lists(got, pooled_ref, wq, lens, Q, pool, topk, with_tail):
    for b in range(len(lens)):
        for i in range(Q):
            pos = int(lens[b]) - Q + i
            w = oracle.widen(wq[b, i])
            ref = oracle.kpool_select(pooled_ref[b], w, pos, pool, topk, with_tail)
            g = got[b, i]
            if np.array_equal(g, ref):
                continue
            # Several lists are correct when pools tie; whatever the GPU chose must still be a
            # valid list: whole, complete, visible pools in ascending order, then -1 up to topk,
            # then the same tail.  Only near-ties may be swapped.
            n_sel = max(pos + 1, 0) // pool
            head = [int(x) for x in g[:topk]]
            used = [x for x in head if x >= 0]
            assert head == used + [-1] * (topk - len(used)), (b, i, "padding must follow the pools")
            assert len(used) % pool == 0, (b, i)
            chosen = [used[k] // pool for k in range(0, len(used), pool)]
            for k, p in enumerate(chosen):
                assert used[k * pool:(k + 1) * pool] == list(range(p * pool, (p + 1) * pool)), (b, i, p)
            assert chosen == sorted(set(chosen)), (b, i, "pools ascending and distinct")
            assert all(0 <= p < n_sel for p in chosen), (b, i, "only complete, visible pools")
            scores = pooled_ref[b][:n_sel] @ w
            gs = set(chosen)
            rs = {int(x) // pool for x in ref[:topk] if x >= 0}
            assert len(gs) == len(rs)
            kth = min(scores[p] for p in rs)
            for p in gs ^ rs:
                assert abs(scores[p] - kth) <= 1e-5 * (1 + abs(kth)), (b, i, p)
            assert np.array_equal(g[topk:], ref[topk:])


@pytest.mark.parametrize("pool", [16, 64])
def test_pooled_keys_match_oracle(pool):
    lens, cache, _ = _setup([300, 131, 64, 5], 1, pool, seed=pool)
    pooled = m.mla_kpool_keys(to_dev(cache), pool, ints_to_dev(lens))
    torch.cuda.synchronize()
    got = pooled.cpu().numpy().astype(np.float64)
    for b, L in enumerate(lens):
        ref = oracle.kpool_pooled_keys(cache[b, :L], pool)
        n = ref.shape[0]
        assert np.all(np.abs(got[b, :n] - ref) <= 2e-6 * (1 + np.abs(ref))), float(np.abs(got[b, :n] - ref).max())


@pytest.mark.parametrize("with_tail", [True, False])
@pytest.mark.parametrize("pool,topk", [(16, 64), (64, 256), (8, 8)])
def test_selection_matches_oracle(pool, topk, with_tail):
    Q = 6
    lens, cache, wq = _setup([1000, 300, 70, 6, 1], Q, pool, seed=pool + topk)
    d_lens = ints_to_dev(lens)
    pooled = m.mla_kpool_keys(to_dev(cache), pool, d_lens)
    lists = m.mla_kpool_select(pooled, to_dev(wq), pool, topk, d_lens, with_tail, Lmax=cache.shape[1])
    torch.cuda.synchronize()
    got = lists.cpu().numpy()
    assert got.shape == (len(lens), Q, topk + (pool - 1 if with_tail else 0))
    pooled_ref = [oracle.kpool_pooled_keys(cache[b, :L], pool) for b, L in enumerate(lens)]
    _check_lists(got, pooled_ref, wq, lens, Q, pool, topk, with_tail)


def test_produced_lists_drive_the_indexed_attention():
    """Producer -> mla_attend_indexed: the -1 entries (padding and short tails) are unused."""
    Q, pool, topk = 6, 16, 128
    lens = np.array([700, 150], dtype=np.int32)
    wl = tiny_workload("dense", 2, Q, lens, H=64, D=256, R=512, seed=31)
    wq = synth.normal_bf16((2, Q, 512), 32, synth.STREAM_Q)
    d_cache, d_lens = to_dev(wl.cache), ints_to_dev(lens)
    pooled = m.mla_kpool_keys(d_cache, pool, d_lens)
    lists = m.mla_kpool_select(pooled, to_dev(wq), pool, topk, d_lens, True, Lmax=wl.cache.shape[1])
    qt = synthetic_qtilde(2, Q, seed=33)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = m.mla_attend_indexed(to_dev(qt), d_cache, lists, d_lens, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got_lists = lists.cpu().numpy()
    assert (got_lists == -1).any()  # the short sequence and the tails leave unused entries
    wl.mode, wl.indices = "indexed", got_lists
    ref = oracle.reference_latent(qt, wl)
    got = bf16_to_f64(o)
    for (b, i), r in ref.items():
        mx, mean = errors(got[b, i], r["o_latent"])
        assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (b, i, mx, mean)


def test_padding_entries_equal_a_shorter_list():
    """A list with -1 entries gives the result of the same list without them."""
    wl = tiny_workload("indexed", 2, 1, [900, 900], H=64, D=256, R=512, seed=5, K=200)
    qt = synthetic_qtilde(2, 1, seed=6)
    padded = wl.indices.copy()
    padded[:, :, 150:] = -1
    padded[1, 0, 10:40] = -1
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    o1, l1 = m.mla_attend_indexed(to_dev(qt), to_dev(wl.cache), ints_to_dev(padded), ints_to_dev(wl.seq_lens),
                                  status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    wl.indices = padded
    ref = oracle.reference_latent(qt, wl)
    got = bf16_to_f64(o1)
    for (b, i), r in ref.items():
        mx, mean = errors(got[b, i], r["o_latent"])
        assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (b, i, mx, mean)


def test_full_length_selection_sampled():
    """The indexed-decode scale: 131,072 cached rows, pools of 64, 2,048 selected rows plus
    the tail, checked against the oracle on sampled queries."""
    pool, topk, L = 64, 2048, 131072
    lens = np.array([L, L - 37], dtype=np.int32)
    cache = synth.normal_bf16((2, L, 512), 7, synth.STREAM_CACHE)
    wq = synth.normal_bf16((2, 1, 512), 8, synth.STREAM_Q)
    d_lens = ints_to_dev(lens)
    pooled = m.mla_kpool_keys(to_dev(cache), pool, d_lens)
    lists = m.mla_kpool_select(pooled, to_dev(wq), pool, topk, d_lens, True, Lmax=L)
    torch.cuda.synchronize()
    got = lists.cpu().numpy()
    pooled_ref = [oracle.kpool_pooled_keys(cache[b, :lens[b]], pool) for b in range(2)]
    _check_lists(got, pooled_ref, wq, lens, 1, pool, topk, True)

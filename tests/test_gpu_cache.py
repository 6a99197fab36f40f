"""GPU latent-cache bookkeeping around a verify step, through the C ABI, against the
oracle bit for bit ("Module 08 -- Vision, MTP, and Hybrid Serving State", section 3:
the latent cache is truncated to the accepted prefix, and the state after rollback must
equal that of a run that never generated the rejected tokens)."""
import numpy as np
import pytest
import torch

import mla_absorbed_latent_mtp_b200 as m
import oracle
import synth
from gpu_util import bf16_bits, bf16_to_f64, ints_to_dev, synthetic_qtilde, to_dev
from helpers import MAX_ABS_TOL, MEAN_ABS_TOL, errors

pytestmark = pytest.mark.gpu

R = 512
PAGE = 64


@pytest.fixture(scope="module", autouse=True)
def device():
    import __graft_entry__
    __graft_entry__.build()
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _state(mode, lens, room, seed=0):
    """Random rows below each length, zeros elsewhere, `room` free positions per sequence."""
    lens = np.asarray(lens, dtype=np.int32)
    B = len(lens)
    cap = lens + room
    rows = synth.normal_bf16((B, int(cap.max()), R), seed, synth.STREAM_CACHE)
    if mode == "dense":
        store = np.zeros((B, int(cap.max()), R), dtype=np.uint16)
        for b in range(B):
            store[b, : lens[b]] = rows[b, : lens[b]]
        return store, lens, None
    table, P = synth.page_layout(cap, seed)
    store = np.zeros((P, PAGE, R), dtype=np.uint16)
    for b in range(B):
        for j in range(int(lens[b])):
            store[table[b, j // PAGE], j % PAGE] = rows[b, j]
    return store, lens, table


def _gpu_append(mode, d_store, d_lens, d_table, drafts, status):
    if mode == "dense":
        m.mla_cache_append_dense(d_store, d_lens, to_dev(drafts), status=status)
    else:
        m.mla_cache_append_paged(d_store, d_table, d_lens, to_dev(drafts), status=status)


def _gpu_truncate(mode, d_store, d_lens, d_table, keep, q_len, status):
    if mode == "dense":
        m.mla_cache_truncate_dense(d_store, d_lens, ints_to_dev(keep), q_len, status=status)
    else:
        m.mla_cache_truncate_paged(d_store, d_table, d_lens, ints_to_dev(keep), q_len, status=status)


@pytest.mark.parametrize("mode", ["dense", "paged"])
def test_append_and_truncate_match_oracle_bitwise(mode):
    lens, q_len = [0, 1, 63, 64, 65, 130, 7], 6
    keep = np.array([0, 6, 3, 1, 5, 2, 4], dtype=np.int32)
    s0, l0, table = _state(mode, lens, q_len)
    drafts = synth.normal_bf16((len(lens), q_len, R), 1, synth.STREAM_Q)
    d_store, d_lens = to_dev(s0), ints_to_dev(l0)
    d_table = ints_to_dev(table) if table is not None else None
    st = _status()
    _gpu_append(mode, d_store, d_lens, d_table, drafts, st)
    torch.cuda.synchronize()
    s1, l1 = oracle.cache_append(mode, s0, l0, drafts, table)
    assert int(st.item()) == 0
    assert np.array_equal(d_lens.cpu().numpy(), l1)
    assert np.array_equal(bf16_bits(d_store), s1)
    _gpu_truncate(mode, d_store, d_lens, d_table, keep, q_len, st)
    torch.cuda.synchronize()
    s2, l2 = oracle.cache_truncate(mode, s1, l1, keep, q_len, table)
    assert int(st.item()) == 0
    assert np.array_equal(d_lens.cpu().numpy(), l2)
    assert np.array_equal(bf16_bits(d_store), s2)


@pytest.mark.parametrize("mode", ["dense", "paged"])
def test_rollback_leaves_the_never_generated_state(mode):
    """Append a window, reject all of it: every bit of the cache and every length is back."""
    lens, q_len = [5, 64, 200], 6
    s0, l0, table = _state(mode, lens, q_len, seed=3)
    d_store, d_lens = to_dev(s0), ints_to_dev(l0)
    d_table = ints_to_dev(table) if table is not None else None
    st = _status()
    for step in range(3):  # several verify steps in a row, each fully rejected
        drafts = synth.normal_bf16((len(lens), q_len, R), 10 + step, synth.STREAM_Q)
        _gpu_append(mode, d_store, d_lens, d_table, drafts, st)
        _gpu_truncate(mode, d_store, d_lens, d_table, np.zeros(len(lens), np.int32), q_len, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(d_lens.cpu().numpy(), l0)
    assert np.array_equal(bf16_bits(d_store), s0)


def test_overflowing_sequence_is_untouched_and_flagged():
    lens = np.array([10, 60], dtype=np.int32)  # the second has room for 4 rows only
    store = np.zeros((2, 64, R), dtype=np.uint16)
    d_store, d_lens = to_dev(store), ints_to_dev(lens)
    st = _status()
    drafts = synth.normal_bf16((2, 6, R), 2, synth.STREAM_Q)
    m.mla_cache_append_dense(d_store, d_lens, to_dev(drafts), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == m.MLA_ERR_INDEX
    assert d_lens.cpu().numpy().tolist() == [16, 60]
    got = bf16_bits(d_store)
    assert np.array_equal(got[0, 10:16], drafts[0]) and not got[1].any()


def test_unmapped_page_and_bad_keep_are_flagged():
    lens = np.array([60, 10], dtype=np.int32)
    table = np.array([[0, -1], [1, 2]], dtype=np.int32)  # sequence 0 has no second page
    pool = np.zeros((3, PAGE, R), dtype=np.uint16)
    d_pool, d_lens, d_table = to_dev(pool), ints_to_dev(lens), ints_to_dev(table)
    st = _status()
    drafts = synth.normal_bf16((2, 6, R), 4, synth.STREAM_Q)
    m.mla_cache_append_paged(d_pool, d_table, d_lens, to_dev(drafts), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == m.MLA_ERR_INDEX
    assert d_lens.cpu().numpy().tolist() == [60, 16]
    st.zero_()
    # sequence 0 keeps all 6 of its last rows (a no-op); sequence 1 asks for 7 > q_len
    m.mla_cache_truncate_paged(d_pool, d_table, d_lens, ints_to_dev([6, 7]), 6, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == m.MLA_ERR_INDEX
    assert d_lens.cpu().numpy().tolist() == [60, 16]


def test_verify_then_rollback_then_decode_matches_oracle():
    """The whole speculative step on the GPU: append the window, verify it (q_len = 6),
    keep an accepted prefix, then decode the next token on the truncated cache."""
    q_len = 1 + oracle.MTP_DRAFT_TOKENS
    prefix = np.array([70, 129], dtype=np.int32)
    B = len(prefix)
    s0, l0, _ = _state("dense", prefix, q_len + 1, seed=5)
    d_cache, d_lens = to_dev(s0), ints_to_dev(l0)
    st = _status()
    drafts = synth.normal_bf16((B, q_len, R), 6, synth.STREAM_Q)
    m.mla_cache_append_dense(d_cache, d_lens, to_dev(drafts), status=st)
    qt = synthetic_qtilde(B, q_len, seed=7)
    o, lse = m.mla_attend_dense(to_dev(qt), d_cache, d_lens, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0

    def check(cache_bits, lens, qt_bits, Q, o_dev):
        wl = synth.Workload("verify", "dense", B, Q, lens, None, None, None)
        wl.cache = cache_bits
        ref = oracle.reference_latent(qt_bits, wl)
        got = bf16_to_f64(o_dev)
        for (b, i), r in ref.items():
            mx, mean = errors(got[b, i], r["o_latent"])
            assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (b, i, mx, mean)

    s1, l1 = oracle.cache_append("dense", s0, l0, drafts)
    check(s1, l1, qt, q_len, o)
    keep = np.array([3, 0], dtype=np.int32)
    m.mla_cache_truncate_dense(d_cache, d_lens, ints_to_dev(keep), q_len, status=st)
    s2, l2 = oracle.cache_truncate("dense", s1, l1, keep, q_len)
    # next decode step: append the accepted token's successor, then attend with q_len = 1
    nxt = synth.normal_bf16((B, 1, R), 8, synth.STREAM_Q)
    m.mla_cache_append_dense(d_cache, d_lens, to_dev(nxt), status=st)
    s3, l3 = oracle.cache_append("dense", s2, l2, nxt)
    qt1 = synthetic_qtilde(B, 1, seed=9)
    o1, _ = m.mla_attend_dense(to_dev(qt1), d_cache, d_lens, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(d_lens.cpu().numpy(), l3)
    assert np.array_equal(bf16_bits(d_cache), s3)
    check(s3, l3, qt1, 1, o1)

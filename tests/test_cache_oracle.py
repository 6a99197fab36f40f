"""Pins for the oracle's latent-cache bookkeeping under speculative decoding.

"Module 08 -- Vision, MTP, and Hybrid Serving State", section 3: the MLA latent cache is
truncatable by position, and after rolling back a verify step its state must equal the
state of a run that never generated the rejected tokens.  The pins below are that
invariant, its special cases (nothing kept, everything kept), the agreement of the paged
and dense layouts, and the MTP window itself: appending the window's rows to the prefix
rebuilds the verify workload's cache bit for bit."""
import numpy as np
import pytest

import oracle
import synth

R = 16
PAGE = oracle.PAGE_TOKENS


def _state(mode, lens, q_len, seed=0):
    """A store holding random rows below each length and zeros everywhere else, with room
    for q_len more rows per sequence.  Returns (store, lens, page_table)."""
    lens = np.asarray(lens, dtype=np.int32)
    B = len(lens)
    cap = lens + q_len
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


def _draft_rows(B, q_len, seed=1):
    return synth.normal_bf16((B, q_len, R), seed, synth.STREAM_Q)


def _logical(mode, store, cap, table):
    """Rows 0..cap[b]-1 of every sequence read through the layout, zero-padded to a block."""
    B = len(cap)
    out = np.zeros((B, int(max(cap)), R), dtype=np.uint16)
    for b in range(B):
        out[b, : cap[b]] = oracle.logical_rows(mode, b, np.arange(int(cap[b])), cache=store, pool=store,
                                               page_table=table)
    return out


@pytest.mark.parametrize("mode", ["dense", "paged"])
def test_rollback_of_everything_restores_the_state(mode):
    lens, q_len = [5, 64, 63, 130], 6
    s0, l0, table = _state(mode, lens, q_len)
    s1, l1 = oracle.cache_append(mode, s0, l0, _draft_rows(len(lens), q_len), table)
    assert np.array_equal(l1, l0 + q_len)
    s2, l2 = oracle.cache_truncate(mode, s1, l1, np.zeros(len(lens), np.int32), q_len, table)
    assert np.array_equal(l2, l0)
    assert np.array_equal(s2, s0)  # every bit of the store, not just the visible rows


@pytest.mark.parametrize("mode", ["dense", "paged"])
def test_keeping_everything_is_the_identity(mode):
    lens, q_len = [0, 1, 70], 6
    s0, l0, table = _state(mode, lens, q_len)
    s1, l1 = oracle.cache_append(mode, s0, l0, _draft_rows(len(lens), q_len), table)
    s2, l2 = oracle.cache_truncate(mode, s1, l1, np.full(len(lens), q_len, np.int32), q_len, table)
    assert np.array_equal(s2, s1) and np.array_equal(l2, l1)


@pytest.mark.parametrize("mode", ["dense", "paged"])
def test_rollback_equals_never_generated(mode):
    """Appending q_len rows and keeping k of them == appending only those k rows."""
    lens, q_len = [3, 64, 127, 200, 1], 6
    keep = np.array([0, 2, 6, 5, 1], dtype=np.int32)
    s0, l0, table = _state(mode, lens, q_len)
    drafts = _draft_rows(len(lens), q_len)
    s1, l1 = oracle.cache_append(mode, s0, l0, drafts, table)
    s2, l2 = oracle.cache_truncate(mode, s1, l1, keep, q_len, table)
    # the never-generated run: ordinary one-token decode steps that append only the
    # accepted rows, sequence by sequence
    ref, ref_l = s0.copy(), l0.copy()
    for b in range(len(lens)):
        for i in range(int(keep[b])):
            if mode == "dense":
                sub, sub_l = oracle.cache_append("dense", ref[b:b + 1], ref_l[b:b + 1], drafts[b:b + 1, i:i + 1])
                ref[b] = sub[0]
            else:
                ref, sub_l = oracle.cache_append("paged", ref, ref_l[b:b + 1], drafts[b:b + 1, i:i + 1], table[b:b + 1])
            ref_l[b] = sub_l[0]
    assert np.array_equal(l2, ref_l)
    assert np.array_equal(s2, ref)


def test_paged_and_dense_agree_after_append_and_truncate():
    lens, q_len = [10, 64, 65, 191], 6
    keep = np.array([6, 0, 3, 1], dtype=np.int32)
    drafts = _draft_rows(len(lens), q_len)
    views = []
    for mode in ("dense", "paged"):
        s0, l0, table = _state(mode, lens, q_len)
        s1, l1 = oracle.cache_append(mode, s0, l0, drafts, table)
        s2, l2 = oracle.cache_truncate(mode, s1, l1, keep, q_len, table)
        cap = l0 + q_len
        views.append((_logical(mode, s1, cap, table), l1, _logical(mode, s2, cap, table), l2))
    for a, b in zip(views[0], views[1]):
        assert np.array_equal(a, b)


def test_append_rebuilds_the_verify_window_cache():
    """The MTP verify cache holds the prefix plus the q_len window rows; appending the
    window to the prefix alone reproduces it exactly, in both layouts."""
    q_len = 1 + oracle.MTP_DRAFT_TOKENS
    wl = synth.make_workload(mode="dense", B=3, Q=q_len, L=70 + q_len)
    full = wl.cache  # [B, L, 512]
    B, L = full.shape[0], full.shape[1]
    prefix = full.copy()
    prefix[:, L - q_len:] = 0
    lens = np.full(B, L - q_len, dtype=np.int32)
    s1, l1 = oracle.cache_append("dense", prefix, lens, full[:, L - q_len:])
    assert np.array_equal(s1, full) and np.array_equal(l1, wl.seq_lens)
    # and the oracle's verify result on the rebuilt cache is the same computation
    ref = oracle.reference(wl, pairs=[(0, 0), (2, q_len - 1)], heads=[0, 63], form="absorbed")
    wl.cache = s1
    again = oracle.reference(wl, pairs=[(0, 0), (2, q_len - 1)], heads=[0, 63], form="absorbed")
    assert ref.keys() == again.keys()
    for key in ref:
        assert np.array_equal(ref[key]["out"], again[key]["out"])
        assert np.array_equal(ref[key]["lse"], again[key]["lse"])


def test_truncate_rejects_nothing_it_should_keep():
    """Rows below the accepted length are never touched by a rollback."""
    lens, q_len = [40, 64], 6
    s0, l0, table = _state("paged", lens, q_len)
    s1, l1 = oracle.cache_append("paged", s0, l0, _draft_rows(2, q_len), table)
    s2, l2 = oracle.cache_truncate("paged", s1, l1, np.array([4, 2], np.int32), q_len, table)
    for b in range(2):
        kept = oracle.logical_rows("paged", b, np.arange(int(l2[b])), pool=s1, page_table=table)
        assert np.array_equal(oracle.logical_rows("paged", b, np.arange(int(l2[b])), pool=s2, page_table=table), kept)

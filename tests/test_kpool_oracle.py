"""Pins for the oracle's k-pool index producer: a hand-derived example (tests/golden/
kpool_worked_example.txt), closed forms of the per-channel softmax mixture, and brute
force on the selection rules (complete and causally visible pools only, best scores,
ties to the lower pool, tail appended, -1 padding)."""
import os

import numpy as np
import pytest

import oracle
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _golden():
    vals = {}
    with open(os.path.join(ROOT, "tests", "golden", "kpool_worked_example.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split("=")
                vals[k.strip()] = [float(x) for x in v.split()]
    return vals


def _bits(values):
    """Exact bf16 bits of small values (all representable)."""
    return synth.f64_to_bf16_bits(np.asarray(values, dtype=np.float64))


def test_worked_example():
    g = _golden()
    rows = _bits([[0.0], [1.0], [2.0], [2.0], [5.0], [5.0], [3.0]])
    pooled = oracle.kpool_pooled_keys(rows, 2)
    assert pooled.shape == (3, 1)
    assert np.allclose(pooled[:, 0], g["pool0"] + g["pool1"] + g["pool2"], rtol=0, atol=1e-15)
    for key, w, pos in (("select_w1", 1.0, 6), ("select_wm1", -1.0, 6), ("select_w0", 0.0, 6), ("select_w1_pos5", 1.0, 5)):
        got = oracle.kpool_select(pooled, np.array([w]), pos, pool=2, topk=4, with_tail=True)
        assert got.tolist() == [int(x) for x in g[key]], key


def test_pool_of_identical_rows_is_the_row():
    row = synth.normal_bf16((1, 32), 1, synth.STREAM_CACHE)
    rows = np.repeat(row, 8, axis=0)
    assert np.array_equal(oracle.kpool_pooled_keys(rows, 8)[0], oracle.widen(row[0]))


def test_pool_of_one_is_the_row():
    rows = synth.normal_bf16((5, 16), 2, synth.STREAM_CACHE)
    assert np.array_equal(oracle.kpool_pooled_keys(rows, 1), oracle.widen(rows))


def test_mixture_lies_between_mean_and_max():
    """Softmax weights grow with the value, so the mixture is at least the plain average
    (Chebyshev's sum inequality) and at most the largest member."""
    rows = synth.normal_bf16((64, 40), 3, synth.STREAM_CACHE)
    x = oracle.widen(rows).reshape(8, 8, 40)
    pooled = oracle.kpool_pooled_keys(rows, 8)
    assert np.all(pooled >= x.mean(axis=1) - 1e-12)
    assert np.all(pooled <= x.max(axis=1) + 1e-12)
    # a dominant member pulls the mixture to itself
    big = oracle.widen(rows).copy()
    rows2 = rows.copy()
    rows2[3, 0] = _bits([60.0])[0]
    assert abs(oracle.kpool_pooled_keys(rows2, 8)[0, 0] - 60.0) < 1e-12


@pytest.mark.parametrize("pos", [0, 6, 7, 63, 64, 100, 127, 128])
@pytest.mark.parametrize("with_tail", [False, True])
def test_selection_rules_by_brute_force(pos, with_tail):
    pool, topk = 8, 24
    rows = synth.normal_bf16((160, 12), pos + 1, synth.STREAM_CACHE)
    pooled = oracle.kpool_pooled_keys(rows, pool)
    w = oracle.widen(synth.normal_bf16((12,), 9, synth.STREAM_Q))
    got = oracle.kpool_select(pooled, w, pos, pool, topk, with_tail)
    assert len(got) == topk + (pool - 1 if with_tail else 0)
    head = got[:topk]
    chosen = sorted({int(j) // pool for j in head if j >= 0})
    complete = [p for p in range(len(pooled)) if (p + 1) * pool - 1 <= pos]
    # complete, visible, whole pools, ascending, then -1 padding
    assert all(p in complete for p in chosen)
    assert head[: len(chosen) * pool].tolist() == [p * pool + j for p in chosen for j in range(pool)]
    assert np.all(head[len(chosen) * pool:] == -1)
    assert len(chosen) == min(topk // pool, len(complete))
    # every chosen pool beats every other complete pool (ties to the lower index)
    s = {p: float(pooled[p] @ w) for p in complete}
    for c in chosen:
        for u in complete:
            if u not in chosen:
                assert s[c] > s[u] or (s[c] == s[u] and c < u)
    if with_tail:
        tail = got[topk:]
        start = len(complete) * pool
        expect = list(range(start, pos + 1))
        assert tail[: len(expect)].tolist() == expect and np.all(tail[len(expect):] == -1)

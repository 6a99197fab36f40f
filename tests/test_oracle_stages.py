"""Pins for the oracle's per-stage functions: the bit widening, the query absorption, the
value up-projection and the latent-space attention that the stage-level GPU tests use as
their checker.

Each function is tied to something other than itself:
* ``widen`` to a field-by-field decoding of every one of the 65,536 bfloat16 patterns;
* ``absorb_all`` and ``up_project_all`` to pure-Python loops over the definitions of
  "Module 05 -- MLA" section 3 (q~_h = (U_h^K)^T q_h; out_h = U_h^V o_h), on shapes where a
  transposed operand still type-checks (D = R) so that it shows in the values;
* ``reference_latent`` to pure-Python loops, and to the pinned expanded-form ``reference``
  through the chain absorb -> latent attention -> up-projection, once exactly (queries
  whose absorbed form is exactly representable) and once with the bf16 roundings the GPU
  stages apply between them.
The mutation tests at the end plant a plausible slip in a copy of each function and check
that the pins above catch it."""
import math

import numpy as np
import pytest

import oracle
import synth
from helpers import MAX_ABS_TOL, decode_bf16, decode_list, errors, gate, tiny_workload


# ----------------------------------------------------------------------------- widen

def test_widen_every_bit_pattern():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.widen(bits)
    for u in range(1 << 16):
        want = decode_bf16(u)
        g = float(got[u])
        if math.isnan(want):
            assert math.isnan(g), hex(u)
        else:
            assert g == want and math.copysign(1.0, g) == math.copysign(1.0, want), hex(u)


def test_widen_round_trips_representable_values():
    vals = [0.0, -0.0, 1.0, -1.0, 0.5, -3.0, 65280.0, -2.0 ** -126, 2.0 ** -133, -(2.0 ** -133) * 5,
            2.0 ** 127 * 1.9921875, math.inf, -math.inf, 1.0078125, -0.0078125]
    bits = synth.f64_to_bf16_bits(np.array(vals))
    back = oracle.widen(bits)
    for v, b in zip(vals, back):
        assert float(b) == v and math.copysign(1.0, float(b)) == math.copysign(1.0, v), v


# ----------------------------------------------------------------------------- projections

def _brute_absorb(q_bits, w_bits):
    """q~[n][h][r] = sum_d U^K[h][d][r] * q[n][h][d]  (k = U^K c, so q.k = (U^T q).c)."""
    n, H, D = q_bits.shape
    R = w_bits.shape[2]
    q = np.array(decode_list(q_bits)).reshape(n, H, D).tolist()
    w = np.array(decode_list(w_bits)).reshape(H, D, R).tolist()
    return np.array([[[sum(w[h][d][r] * q[t][h][d] for d in range(D)) for r in range(R)] for h in range(H)]
                     for t in range(n)])


def _brute_up(o_bits, w_bits):
    """out[n][h][d] = sum_r U^V[h][d][r] * o[n][h][r]."""
    n, H, R = o_bits.shape
    D = w_bits.shape[1]
    o = np.array(decode_list(o_bits)).reshape(n, H, R).tolist()
    w = np.array(decode_list(w_bits)).reshape(H, D, R).tolist()
    return np.array([[[sum(w[h][d][r] * o[t][h][r] for r in range(R)) for d in range(D)] for h in range(H)]
                     for t in range(n)])


@pytest.mark.parametrize("n,H,D,R", [(3, 2, 4, 8), (2, 3, 6, 6), (1, 2, 8, 4)])
def test_absorb_all_matches_loops(n, H, D, R):
    q = synth.normal_bf16((n, H, D), 4, synth.STREAM_Q)
    w = synth.normal_bf16((H, D, R), 4, synth.STREAM_WUK, 0.3)
    np.testing.assert_allclose(oracle.absorb_all(q, w), _brute_absorb(q, w), rtol=1e-13, atol=1e-15)
    # per head it is the single-query form used by the absorbed reference
    for t in range(n):
        for h in range(H):
            np.testing.assert_allclose(oracle.absorb_all(q, w)[t, h],
                                       oracle.absorb_query(oracle.widen(q[t, h]), oracle.widen(w[h])),
                                       rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("n,H,D,R", [(3, 2, 4, 8), (2, 3, 6, 6), (1, 2, 8, 4)])
def test_up_project_all_matches_loops(n, H, D, R):
    o = synth.normal_bf16((n, H, R), 5, synth.STREAM_OLAT, 0.2)
    w = synth.normal_bf16((H, D, R), 5, synth.STREAM_WUV, 0.3)
    np.testing.assert_allclose(oracle.up_project_all(o, w), _brute_up(o, w), rtol=1e-13, atol=1e-15)
    for t in range(n):
        for h in range(H):
            np.testing.assert_allclose(oracle.up_project_all(o, w)[t, h],
                                       oracle.up_project(oracle.widen(o[t, h]), oracle.widen(w[h])),
                                       rtol=1e-14, atol=1e-15)


# ----------------------------------------------------------------------------- latent attention

def _brute_latent(qt_bits, wl):
    """Pure-Python latent attention: visible rows, scores scale * q~.c_j, softmax, sum a_j c_j."""
    B, Q, H, R = qt_bits.shape
    out = {}
    for b in range(B):
        for i in range(Q):
            if wl.mode == "indexed":
                vis = [int(x) for x in wl.indices[b, i] if int(x) != -1]
            else:
                vis = list(range(0, int(wl.seq_lens[b]) - Q + i + 1))
            rows = []
            for j in vis:
                if wl.mode == "paged":
                    rows.append(decode_list(wl.pool[wl.page_table[b, j // 64], j % 64]))
                else:
                    rows.append(decode_list(wl.cache[b, j]))
            o_all, lse_all = [], []
            for h in range(H):
                q = decode_list(qt_bits[b, i, h])
                s = [wl.scale * sum(q[r] * c[r] for r in range(R)) for c in rows]
                if not s:
                    o_all.append([0.0] * R)
                    lse_all.append(-math.inf)
                    continue
                m = max(s)
                e = [math.exp(x - m) for x in s]
                z = sum(e)
                o_all.append([sum(e[j] / z * rows[j][r] for j in range(len(rows))) for r in range(R)])
                lse_all.append(m + math.log(z))
            out[(b, i)] = (np.array(o_all), np.array(lse_all))
    return out


@pytest.mark.parametrize("mode,B,Q,lens,K", [
    ("dense", 2, 1, [1, 5], None),
    ("dense", 2, 3, [3, 6], None),
    ("dense", 1, 3, [2], None),     # first query sees nothing
    ("paged", 2, 1, [5, 3], None),
    ("paged", 1, 3, [6], None),
    ("indexed", 2, 1, [5, 4], 3),
    ("indexed", 1, 2, [6], 3),
])
def test_reference_latent_matches_loops(mode, B, Q, lens, K):
    wl = tiny_workload(mode, B, Q, lens, H=2, D=4, R=8, seed=7, K=K)
    wl.scale = 0.37
    if mode == "indexed":
        wl.indices[0, 0, -1] = -1  # an unused entry of a fixed-width list
    qt = synth.normal_bf16((B, Q, 2, 8), 7, synth.STREAM_QTILDE)
    ref = oracle.reference_latent(qt, wl)
    bf = _brute_latent(qt, wl)
    for key, (o, lse) in bf.items():
        np.testing.assert_allclose(ref[key]["o_latent"], o, rtol=1e-12, atol=1e-14)
        fin = np.isfinite(lse)
        assert np.array_equal(np.isfinite(ref[key]["lse"]), fin)
        np.testing.assert_allclose(ref[key]["lse"][fin], lse[fin], rtol=1e-13, atol=1e-14)


def _one_hot_queries(wl, seed):
    """Queries with a single non-zero entry of 1 per (b, i, h): then q~ = W_UK^T q is a row of
    W_UK, exactly representable, so the absorbed chain has no rounding between stages."""
    B, Q, H, D = wl.q.shape
    pick = synth.uniform_int(B * Q * H, seed, synth.STREAM_Q, 0, D - 1).reshape(B, Q, H)
    q = np.zeros((B, Q, H, D), dtype=np.uint16)
    one = synth.f64_to_bf16_bits(np.array([1.0]))[0]
    for b in range(B):
        for i in range(Q):
            for h in range(H):
                q[b, i, h, pick[b, i, h]] = one
    return q


CHAIN_CASES = [
    ("dense", 2, 1, [70, 5], None),
    ("dense", 2, 6, [70, 9], None),
    ("paged", 2, 1, [130, 64], None),
    ("paged", 2, 6, [100, 7], None),
    ("indexed", 2, 1, [300, 90], 40),
    ("indexed", 1, 6, [120], 30),
]


@pytest.mark.parametrize("mode,B,Q,lens,K", CHAIN_CASES)
def test_chain_equals_expanded_reference_exactly(mode, B, Q, lens, K):
    """up_project(reference_latent(absorb(q))) == reference(form="expanded") when the
    absorbed queries are exact (one-hot q picks a row of W_UK)."""
    wl = tiny_workload(mode, B, Q, lens, H=4, D=256, R=512, seed=17, K=K)
    wl.q = _one_hot_queries(wl, 17)
    qt_exact = oracle.absorb_all(wl.q.reshape(B * Q, 4, 256), wl.w_uk)
    qt_bits = synth.f64_to_bf16_bits(qt_exact).reshape(B, Q, 4, 512)
    assert np.array_equal(oracle.widen(qt_bits), qt_exact.reshape(B, Q, 4, 512))  # no rounding happened
    lat = oracle.reference_latent(qt_bits, wl)
    ref = oracle.reference(wl, form="expanded")
    u_v = oracle.widen(wl.w_uv)
    for key, r in ref.items():
        out = np.stack([u_v[h] @ lat[key]["o_latent"][h] for h in range(4)])
        np.testing.assert_allclose(out, r["out"], rtol=1e-9, atol=1e-12)
        fin = np.isfinite(r["lse"])
        assert np.array_equal(np.isfinite(lat[key]["lse"]), fin)
        np.testing.assert_allclose(lat[key]["lse"][fin], r["lse"][fin], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode,B,Q,lens,K", CHAIN_CASES)
def test_chain_with_stage_rounding_passes_gate(mode, B, Q, lens, K):
    """The GPU path rounds q~ and o to bf16 between stages; at the full head geometry
    (64 x 256 x 512) the chain of oracle stages with those roundings stays within the parity
    gate of the expanded definition."""
    wl = tiny_workload(mode, B, Q, lens, H=64, D=256, R=512, seed=19, K=K)
    qt = synth.f64_to_bf16_bits(oracle.absorb_all(wl.q.reshape(B * Q, 64, 256), wl.w_uk)).reshape(B, Q, 64, 512)
    lat = oracle.reference_latent(qt, wl)
    o_bits = np.stack([synth.f64_to_bf16_bits(lat[(b, i)]["o_latent"]) for b in range(B) for i in range(Q)])
    out = oracle.up_project_all(o_bits, wl.w_uv).reshape(B, Q, 64, 256)
    ref = oracle.reference(wl, form="expanded")
    for (b, i), r in ref.items():
        mx, mean = errors(out[b, i], r["out"])
        assert gate(out[b, i], r["out"]), (b, i, mx, mean)
        # well inside the gate: only two bf16 roundings separate the chain from the definition
        assert mx <= MAX_ABS_TOL / 2


# ----------------------------------------------------------------------------- the pins catch planted slips

def _widen_bad_shift(bits):
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 15
    return u.view(np.float32).astype(np.float64)


def _absorb_transposed(q_bits, w_bits):
    q, u = oracle.widen(q_bits), oracle.widen(w_bits)
    return np.stack([q[:, h, :] @ u[h].T for h in range(q.shape[1])], axis=1)


def _up_transposed(o_bits, w_bits):
    o, u = oracle.widen(o_bits), oracle.widen(w_bits)
    return np.stack([o[:, h, :] @ u[h] for h in range(o.shape[1])], axis=1)


def test_planted_widen_slip_is_caught():
    bits = np.array([0x3F80, 0xC040, 0x0001, 0x7F7F], dtype=np.uint16)
    assert [float(x) for x in _widen_bad_shift(bits)] != [decode_bf16(int(u)) for u in bits]


def test_planted_transposes_are_caught():
    q = synth.normal_bf16((2, 3, 6), 4, synth.STREAM_Q)
    w = synth.normal_bf16((3, 6, 6), 4, synth.STREAM_WUK, 0.3)
    assert not np.allclose(_absorb_transposed(q, w), _brute_absorb(q, w), rtol=1e-6)
    o = synth.normal_bf16((2, 3, 6), 5, synth.STREAM_OLAT, 0.2)
    assert not np.allclose(_up_transposed(o, w), _brute_up(o, w), rtol=1e-6)


@pytest.mark.parametrize("slip", ["scale", "window", "sign"])
def test_planted_latent_slips_are_caught(slip):
    """A copy of reference_latent with a slip (scale doubled, window one row short, scores
    negated) must fail the exact chain identity against the expanded definition."""
    mode, B, Q, lens = "dense", 2, 6, [70, 9]
    wl = tiny_workload(mode, B, Q, lens, H=4, D=256, R=512, seed=17)
    wl.q = _one_hot_queries(wl, 17)
    qt_bits = synth.f64_to_bf16_bits(oracle.absorb_all(wl.q.reshape(B * Q, 4, 256), wl.w_uk)).reshape(B, Q, 4, 512)
    bad = tiny_workload(mode, B, Q, lens, H=4, D=256, R=512, seed=17)
    bad.cache = wl.cache
    if slip == "scale":
        bad.scale = 2 * wl.scale
    elif slip == "window":
        bad.seq_lens = wl.seq_lens - 1
    else:
        qt_bits = qt_bits ^ np.uint16(0x8000)  # every q~ entry negated: scores change sign
    lat = oracle.reference_latent(qt_bits, bad)
    ref = oracle.reference(wl, form="expanded")
    u_v = oracle.widen(wl.w_uv)
    worst = 0.0
    for key, r in ref.items():
        if not np.all(np.isfinite(r["lse"])) or key not in lat:
            continue
        out = np.stack([u_v[h] @ lat[key]["o_latent"][h] for h in range(4)])
        worst = max(worst, float(np.abs(out - r["out"]).max()))
    assert worst > 1e-3

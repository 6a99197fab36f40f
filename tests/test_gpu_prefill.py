"""Prefill in both forms ("Module 05 -- MLA", section 5), against the fp64 oracle.

A prefill is the oracle's definition with every token a query: q_len = L over a cache of
the same L latents, query t seeing rows 0..t.  The expanded form expands keys and values
per head (mla_expand_kv, checked element-wise against the oracle's expansion) and runs
ordinary causal attention over 256-wide heads (mla_prefill_expanded); the absorbed form is
mla_absorb_q -> mla_attend_dense (q_len = L) -> mla_up_proj.  Both must meet the parity
gate of the definition, and agree with each other."""
import math

import numpy as np
import pytest
import torch

import mla_absorbed_latent_mtp_b200 as m
import oracle
import synth
from gpu_util import bf16_to_f64, ints_to_dev, to_dev
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


# Scores are computed from bf16-rounded keys (expanded form) or absorbed queries (absorbed
# form): a score moves by at most 2^-9 * scale * sum_d |q_d k_d|, about 2^-9 * 163 / 16 = 0.02
# for unit-variance q and k over 256 dims, and the log-sum-exp by no more than its largest
# score (a query that sees one key shows exactly that error).
LSE_TOL = 2e-2


def _proj_tol(ref):
    return 2.0 ** -8 * np.abs(ref) + 1e-5


@pytest.mark.parametrize("n", [1, 5, 64, 129, 300])
def test_expand_kv_matches_oracle(n):
    c = synth.normal_bf16((n, 512), 3, synth.STREAM_CACHE)
    wk = synth.normal_bf16((64, 256, 512), 3, synth.STREAM_WUK, 1 / math.sqrt(512))
    wv = synth.normal_bf16((64, 256, 512), 3, synth.STREAM_WUV, 1 / math.sqrt(512))
    k, v = m.mla_expand_kv(to_dev(c), to_dev(wk), to_dev(wv))
    torch.cuda.synchronize()
    gk, gv = bf16_to_f64(k), bf16_to_f64(v)
    cc = oracle.widen(c)
    for h in range(0, 64, 9):
        rk, rv = oracle.expand_kv(cc, oracle.widen(wk[h]), oracle.widen(wv[h]))
        assert np.all(np.abs(gk[:, h] - rk) <= _proj_tol(rk)), (h, float(np.abs(gk[:, h] - rk).max()))
        assert np.all(np.abs(gv[:, h] - rv) <= _proj_tol(rv)), (h, float(np.abs(gv[:, h] - rv).max()))


def _prefill_workload(B, L, seed):
    # q_len = L over L rows: query t sits at position t and sees rows 0..t
    return tiny_workload("dense", B, L, [L] * B, H=64, D=256, R=512, seed=seed)


def _both_forms(wl):
    B, L = wl.B, wl.Q
    q, wk, wv, cache = to_dev(wl.q), to_dev(wl.w_uk), to_dev(wl.w_uv), to_dev(wl.cache)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    k, v = m.mla_expand_kv(cache, wk, wv)
    out_e, lse_e = m.mla_prefill_expanded(q, k, v, wl.scale, status=st)
    qt = m.mla_absorb_q(q, wk)
    o, lse_a = m.mla_attend_dense(qt, cache, ints_to_dev(wl.seq_lens), wl.scale, status=st)
    out_a = m.mla_up_proj(o, wv)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, m.status_string(int(st.item()))
    return bf16_to_f64(out_e), lse_e, bf16_to_f64(out_a), lse_a


@pytest.mark.parametrize("B,L", [(1, 1), (1, 5), (2, 64), (1, 127), (2, 129), (1, 300), (1, 1000)])
def test_prefill_both_forms_match_oracle(B, L):
    wl = _prefill_workload(B, L, seed=60 + L)
    out_e, lse_e, out_a, lse_a = _both_forms(wl)
    pairs = [(b, t) for b in range(B) for t in range(L)]
    if len(pairs) > 40:  # first rows, block edges and the last rows, plus a spread
        keep = {0, 1, 63, 64, 65, 127, 128, 129, L - 2, L - 1}
        pairs = [(b, t) for (b, t) in pairs if t in keep or t % 37 == 0]
    ref = oracle.reference(wl, pairs=pairs)
    for (b, t), r in ref.items():
        for name, got, lse in (("expanded", out_e, lse_e), ("absorbed", out_a, lse_a)):
            mx, mean = errors(got[b, t], r["out"])
            assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (name, b, t, mx, mean)
            gl = lse[b, t].cpu().numpy().astype(np.float64)
            assert np.abs(gl - r["lse"]).max() <= LSE_TOL, (name, b, t)
    # the two forms round different intermediates (k, v against q~, o): they agree to the gate
    mx, mean = errors(out_e, out_a)
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (mx, mean)


def test_prefill_expanded_rows_past_a_sequence_do_not_leak():
    """Two sequences of 100 tokens: the second's keys (the rows after the first's last
    query in the same key tile) must not reach the first; each sequence equals its own
    prefill computed alone."""
    wl = _prefill_workload(2, 100, seed=71)
    q, wk, wv, cache = to_dev(wl.q), to_dev(wl.w_uk), to_dev(wl.w_uv), to_dev(wl.cache)
    k, v = m.mla_expand_kv(cache, wk, wv)
    both, _ = m.mla_prefill_expanded(q, k, v, wl.scale)
    alone0, _ = m.mla_prefill_expanded(q[:1].contiguous(), k[:1].contiguous(), v[:1].contiguous(), wl.scale)
    alone1, _ = m.mla_prefill_expanded(q[1:].contiguous(), k[1:].contiguous(), v[1:].contiguous(), wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(both[0], alone0[0]) and torch.equal(both[1], alone1[0])

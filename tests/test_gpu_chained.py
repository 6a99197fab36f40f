"""Back-to-back steps with no synchronisation in between.

The library chains its launches (each kernel may start while the previous one in the
stream drains, and waits on the grid dependency before it reads anything an earlier
kernel wrote).  These tests run several whole steps -- absorb, attend, combine,
up-projection -- and cache appends back to back on one stream, each step on different
inputs and into different outputs, and check every step against the oracle: a kernel
that read a predecessor's output before it was complete would show up as a mismatch."""
import math

import numpy as np
import pytest
import torch

import mla_absorbed_latent_mtp_b200 as m
import oracle
import synth
from gpu_util import bf16_bits, bf16_to_f64, ints_to_dev, to_dev
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


def _assert_gate(got, ref, what):
    mx, mean = errors(got, ref)
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, f"{what}: max-abs {mx:.3e} mean-abs {mean:.3e}"


@pytest.mark.parametrize("Q", [1, 6])
def test_back_to_back_steps_match_oracle(Q):
    steps = []
    for k in range(4):
        lens = [300 + 97 * k, 1000 - 61 * k, 64 + k]
        steps.append(tiny_workload("dense", 3, Q, [L + Q for L in lens], H=64, D=256, R=512, seed=20 + k))
    # one set of weights (as in a model layer), per-step queries and caches
    w_uk, w_uv = to_dev(steps[0].w_uk), to_dev(steps[0].w_uv)
    dev = []
    for wl in steps:
        wl.w_uk, wl.w_uv = steps[0].w_uk, steps[0].w_uv
        dev.append((to_dev(wl.q), to_dev(wl.cache), ints_to_dev(wl.seq_lens)))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = m.new_workspace(3, Q)  # shared by every step, as a caller would
    outs = []
    for q, cache, lens in dev:
        qt = m.mla_absorb_q(q, w_uk)
        o, lse = m.mla_attend_dense(qt, cache, lens, workspace=ws, status=st)
        outs.append((m.mla_up_proj(o, w_uv), lse))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for k, (wl, (out, lse)) in enumerate(zip(steps, outs)):
        ref = oracle.reference(wl, form="absorbed")
        got = bf16_to_f64(out)
        for (b, i), r in ref.items():
            _assert_gate(got[b, i], r["out"], f"step {k} b={b} i={i}")


def test_append_then_attend_back_to_back():
    """A verify window appended to the cache and attended right after, three times."""
    Q, B = 6, 2
    prefix = np.array([70, 200], dtype=np.int32)
    cap = int(prefix.max()) + 3 * Q
    cache_bits = np.zeros((B, cap, 512), dtype=np.uint16)
    rows = synth.normal_bf16((B, cap, 512), 3, synth.STREAM_CACHE)
    for b in range(B):
        cache_bits[b, : prefix[b]] = rows[b, : prefix[b]]
    d_cache, d_lens = to_dev(cache_bits), ints_to_dev(prefix)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qts, windows, results = [], [], []
    for k in range(3):
        win = synth.normal_bf16((B, Q, 512), 40 + k, synth.STREAM_Q)
        qt = synth.normal_bf16((B, Q, 64, 512), 50 + k, synth.STREAM_QTILDE, math.sqrt(0.5))
        m.mla_cache_append_dense(d_cache, d_lens, to_dev(win), status=st)
        results.append(m.mla_attend_dense(to_dev(qt), d_cache, d_lens, status=st))
        qts.append(qt)
        windows.append(win)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    state, lens = cache_bits, prefix
    for k in range(3):
        state, lens = oracle.cache_append("dense", state, lens, windows[k])
        wl = synth.Workload("chain", "dense", B, Q, lens, None, None, None)
        wl.cache = state
        ref = oracle.reference_latent(qts[k], wl)
        got = bf16_to_f64(results[k][0])
        for (b, i), r in ref.items():
            _assert_gate(got[b, i], r["o_latent"], f"window {k} b={b} i={i}")
    assert np.array_equal(bf16_bits(d_cache), state) and np.array_equal(d_lens.cpu().numpy(), lens)

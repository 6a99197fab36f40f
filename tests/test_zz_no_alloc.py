"""mla_attend_dense_noalloc: the attention entry point for callers that cannot allocate
device memory (a plugin inside a host runtime that owns all device memory and passes no
workspace, or a runtime whose memory plan is fixed at start-up).  It uses scratch built
into the library instead of a caller workspace, so its results must match
mla_attend_dense, here on two calls in a row (the second call sees the scratch the first
one left behind).  This file is collected last so that a failure here does not stop the
other tests of a run that halts at the first failure."""
import numpy as np
import pytest
import torch

import mla_absorbed_latent_mtp_b200 as m
from gpu_util import bf16_to_f64, ints_to_dev, synthetic_qtilde, to_dev
from helpers import MAX_ABS_TOL, MEAN_ABS_TOL, errors, tiny_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def device():
    import __graft_entry__
    __graft_entry__.build()
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)


def _close(a, b):
    mx, mean = errors(bf16_to_f64(a), bf16_to_f64(b))
    return mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL


def _both(wl, qt_bits):
    qt = to_dev(qt_bits)
    cache = to_dev(wl.cache)
    lens = ints_to_dev(wl.seq_lens)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    o_ref, lse_ref = m.mla_attend_dense(qt, cache, lens, wl.scale, status=st)
    o_na, lse_na = m.mla_attend_dense_noalloc(qt, cache, lens, wl.scale, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return (o_ref, lse_ref), (o_na, lse_na)


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    first = tiny_workload("dense", 3, 2, [700, 129, 64], H=64, D=256, R=512, seed=31)
    second = tiny_workload("dense", 2, 1, [1000, 5], H=64, D=256, R=512, seed=32)
    for wl, seed in ((first, 1), (second, 2)):
        (o_ref, lse_ref), (o_na, lse_na) = _both(wl, synthetic_qtilde(wl.B, wl.Q, seed=seed))
        assert _close(o_na, o_ref)
        fin = torch.isfinite(lse_ref)
        assert torch.equal(fin, torch.isfinite(lse_na))
        assert float((lse_na[fin] - lse_ref[fin]).abs().max()) <= 5e-3


def test_noalloc_rejects_sizes_beyond_its_scratch():
    B, Q = 4096, 1  # needs far more than the built-in 32 MiB
    assert m.mla_attend_workspace_bytes(B, Q) > 32 << 20
    qt = torch.zeros(B, Q, 64, 512, dtype=torch.bfloat16, device="cuda")
    cache = torch.zeros(B, 4, 512, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.MLAError) as e:
        m.mla_attend_dense_noalloc(qt, cache)
    assert e.value.code == m.MLA_ERR_WORKSPACE


def test_noalloc_call_allocates_no_device_memory_and_runs_on_a_side_stream():
    """The point of the entry point: with its outputs supplied, a call takes no device memory
    (the free-memory figure of the device does not move), and on a side stream it gives the
    same result once that stream is synchronised."""
    wl = tiny_workload("dense", 2, 6, [900, 300], H=64, D=256, R=512, seed=33)
    qt = to_dev(synthetic_qtilde(2, 6, seed=3))
    cache, lens = to_dev(wl.cache), ints_to_dev(wl.seq_lens)
    o = torch.empty(2, 6, 64, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(2, 6, 64, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    m.mla_attend_dense_noalloc(qt, cache, lens, wl.scale, o_latent=o, lse=lse, status=st)  # first call: set-up
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    m.mla_attend_dense_noalloc(qt, cache, lens, wl.scale, o_latent=o, lse=lse, status=st)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    ref = o.clone()
    side = torch.cuda.Stream()
    o2 = torch.zeros_like(o)
    lse2 = torch.zeros_like(lse)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        m.mla_attend_dense_noalloc(qt, cache, lens, wl.scale, o_latent=o2, lse=lse2, status=st, stream=side)
    side.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(o2, ref)

"""Failure detection on the GPU without a GPU fault: a bounded wait that nothing
satisfies must give up, report MLA_ERR_TIMEOUT in the status word and return, leaving the
context usable for the next call."""
import time

import numpy as np
import pytest
import torch

import mla_absorbed_latent_mtp_b200 as m
import oracle
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


def test_bounded_wait_times_out_and_the_context_survives():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    m.mla_debug_wait_timeout(4_000_000, st)  # about 2 ms of SM cycles
    torch.cuda.synchronize()
    assert int(st.item()) == m.MLA_ERR_TIMEOUT
    assert time.time() - t0 < 10.0
    # the first error is kept: a second expiry does not overwrite a different code
    st.fill_(m.MLA_ERR_INDEX)
    m.mla_debug_wait_timeout(1_000_000, st)
    torch.cuda.synchronize()
    assert int(st.item()) == m.MLA_ERR_INDEX
    # and the next real call runs normally
    wl = tiny_workload("dense", 2, 1, [300, 77], H=64, D=256, R=512, seed=11)
    qt = synthetic_qtilde(2, 1, seed=12)
    st.zero_()
    o, lse = m.mla_attend_dense(to_dev(qt), to_dev(wl.cache), ints_to_dev(wl.seq_lens), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = oracle.reference_latent(qt, wl)
    got = bf16_to_f64(o)
    for (b, i), r in ref.items():
        mx, mean = errors(got[b, i], r["o_latent"])
        assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL

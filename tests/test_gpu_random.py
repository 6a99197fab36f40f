"""Seeded random sweep of attend shapes against the oracle: mode (contiguous, paged, index
list), batch, q_len, ragged lengths (including windows longer than the cache) and list
lengths, all drawn from a fixed seed so every run checks the same cases."""
import random

import numpy as np
import pytest
import torch

import mla_absorbed_latent_mtp_b200 as m
import oracle
from gpu_util import bf16_to_f64, ints_to_dev, synthetic_qtilde, to_dev
from helpers import MAX_ABS_TOL, MEAN_ABS_TOL, errors, tiny_workload

pytestmark = pytest.mark.gpu

LSE_TOL = 5e-3


@pytest.fixture(scope="module", autouse=True)
def device():
    import __graft_entry__
    __graft_entry__.build()
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def _case(seed):
    rnd = random.Random(1000 + seed)
    mode = ("dense", "paged", "indexed")[seed % 3]
    B = rnd.randint(1, 6)
    Q = rnd.choice([1, 1, 2, 6])
    if mode == "indexed":
        K = rnd.randint(1, 200)
        lens = [rnd.randint(Q + K - 1, Q + K + 600) for _ in range(B)]
        wl = tiny_workload(mode, B, Q, lens, H=64, D=256, R=512, seed=seed, K=K)
    else:
        lens = [rnd.randint(1, 700) for _ in range(B)]
        wl = tiny_workload(mode, B, Q, lens, H=64, D=256, R=512, seed=seed)
    return wl, Q


@pytest.mark.parametrize("seed", range(18))
def test_random_shapes_match_oracle(seed):
    wl, Q = _case(seed)
    qt = synthetic_qtilde(wl.B, Q, seed=seed + 500)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if wl.mode == "dense":
        o, lse = m.mla_attend_dense(to_dev(qt), to_dev(wl.cache), ints_to_dev(wl.seq_lens), status=st)
    elif wl.mode == "paged":
        o, lse = m.mla_attend_paged(to_dev(qt), to_dev(wl.pool), ints_to_dev(wl.page_table),
                                    ints_to_dev(wl.seq_lens), status=st)
    else:
        o, lse = m.mla_attend_indexed(to_dev(qt), to_dev(wl.cache), ints_to_dev(wl.indices),
                                      ints_to_dev(wl.seq_lens), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = oracle.reference_latent(qt, wl)
    got = bf16_to_f64(o)
    glse = lse.cpu().numpy().astype(np.float64)
    for (b, i), r in ref.items():
        mx, mean = errors(got[b, i], r["o_latent"])
        assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (wl.mode, b, i, mx, mean)
        fin = np.isfinite(r["lse"])
        assert np.array_equal(np.isfinite(glse[b, i]), fin)
        if fin.any():
            assert np.abs(glse[b, i][fin] - r["lse"][fin]).max() <= LSE_TOL

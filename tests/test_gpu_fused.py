"""The up-projection fused into the split-L merge (mla_attend_up_*) against the fp64 oracle's
definition (expanded keys and values), and against the unfused path (mla_attend_* then
mla_up_proj) on the same inputs: the two differ only in the order of fp32 merges, so their
outputs agree to a bf16 rounding.  Shapes cover one and several 32-row query tiles,
verify windows, windows longer than the cache, one sequence split over every CTA group,
and the paged and index-list caches."""
import numpy as np
import pytest
import torch

import mla_absorbed_latent_mtp_b200 as m
import oracle
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


def _inputs(wl):
    d = {"q": to_dev(wl.q), "w_uk": to_dev(wl.w_uk), "w_uv": to_dev(wl.w_uv), "lens": ints_to_dev(wl.seq_lens)}
    if wl.mode == "paged":
        d["pool"], d["table"] = to_dev(wl.pool), ints_to_dev(wl.page_table)
    else:
        d["cache"] = to_dev(wl.cache)
    if wl.mode == "indexed":
        d["idx"] = ints_to_dev(wl.indices)
    return d


def _fused(wl, d, qt, st, o_latent=None):
    if wl.mode == "dense":
        return m.mla_attend_up_dense(qt, d["cache"], d["w_uv"], d["lens"], wl.scale, o_latent=o_latent, status=st)
    if wl.mode == "paged":
        return m.mla_attend_up_paged(qt, d["pool"], d["table"], d["lens"], d["w_uv"], wl.scale, o_latent=o_latent,
                                     status=st)
    return m.mla_attend_up_indexed(qt, d["cache"], d["idx"], d["w_uv"], d["lens"], wl.scale, o_latent=o_latent,
                                   status=st)


def _unfused(wl, d, qt, st):
    if wl.mode == "dense":
        o, lse = m.mla_attend_dense(qt, d["cache"], d["lens"], wl.scale, status=st)
    elif wl.mode == "paged":
        o, lse = m.mla_attend_paged(qt, d["pool"], d["table"], d["lens"], wl.scale, status=st)
    else:
        o, lse = m.mla_attend_indexed(qt, d["cache"], d["idx"], d["lens"], wl.scale, status=st)
    return m.mla_up_proj(o, d["w_uv"]), o, lse


CASES = [
    ("dense", 1, [1], None),
    ("dense", 1, [300, 129, 64, 1000], None),
    ("dense", 6, [70, 6 + 65, 200], None),
    ("dense", 6, [3, 6], None),          # early queries see nothing: out = 0, lse = -inf
    ("dense", 1, [40000], None),          # one sequence split over every CTA group
    ("dense", 1, [64 + (7 * k) % 300 for k in range(70)], None),  # 70 rows: three query tiles
    ("paged", 1, [130, 64, 1, 700], None),
    ("paged", 6, [500, 71], None),
    ("indexed", 1, [900, 300], 200),
    ("indexed", 6, [400, 128], 96),
]


@pytest.mark.parametrize("mode,Q,lens,K", CASES)
def test_fused_matches_oracle_and_unfused(mode, Q, lens, K):
    B = len(lens)
    wl = tiny_workload(mode, B, Q, lens, H=64, D=256, R=512, seed=51 + B + Q, K=K)
    d = _inputs(wl)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qt = m.mla_absorb_q(d["q"], d["w_uk"])
    o_lat = torch.empty(B, Q, 64, 512, dtype=torch.bfloat16, device="cuda")
    out, lse = _fused(wl, d, qt, st, o_latent=o_lat)
    out_u, o_u, lse_u = _unfused(wl, d, qt, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, m.status_string(int(st.item()))
    got = bf16_to_f64(out)
    # against the definition
    pairs = [(b, i) for b in range(B) for i in range(Q)]
    if len(pairs) > 24:
        pairs = pairs[::len(pairs) // 24]
    ref = oracle.reference(wl, pairs=pairs)
    for (b, i), r in ref.items():
        mx, mean = errors(got[b, i], r["out"])
        assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (b, i, mx, mean)
        fin = np.isfinite(r["lse"])
        glse = lse[b, i].cpu().numpy().astype(np.float64)
        assert np.array_equal(np.isfinite(glse), fin)
        if (~fin).any():
            assert np.all(got[b, i][~fin] == 0)
    # against the unfused path: same inputs, merges in another order
    mx, mean = errors(got, bf16_to_f64(out_u))
    assert mx <= 1e-2 and mean <= 1e-4, (mx, mean)
    mx, mean = errors(bf16_to_f64(o_lat), bf16_to_f64(o_u))
    assert mx <= 4e-3 and mean <= 1e-5, (mx, mean)
    fin = torch.isfinite(lse_u)
    assert torch.equal(fin, torch.isfinite(lse))
    if fin.any():
        assert float((lse[fin] - lse_u[fin]).abs().max()) <= 1e-4


def test_fused_without_optional_outputs():
    """o_latent and lse are optional: the output is unchanged without them."""
    wl = tiny_workload("dense", 3, 1, [500, 64, 129], H=64, D=256, R=512, seed=57)
    d = _inputs(wl)
    qt = m.mla_absorb_q(d["q"], d["w_uk"])
    a, _ = m.mla_attend_up_dense(qt, d["cache"], d["w_uv"], d["lens"], wl.scale)
    b, lse = m.mla_attend_up_dense(qt, d["cache"], d["w_uv"], d["lens"], wl.scale, want_lse=False)
    torch.cuda.synchronize()
    assert lse is None and torch.equal(a, b)


def test_fused_flags_bad_page():
    wl = tiny_workload("paged", 2, 1, [130, 64], H=64, D=256, R=512, seed=58)
    wl.page_table[0, 1] = wl.pool.shape[0] + 5
    d = _inputs(wl)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qt = m.mla_absorb_q(d["q"], d["w_uk"])
    _fused(wl, d, qt, st)
    torch.cuda.synchronize()
    assert int(st.item()) == m.MLA_ERR_INDEX

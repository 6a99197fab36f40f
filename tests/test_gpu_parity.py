"""GPU parity: every kernel, called through the C ABI, against the fp64 oracle on the
same seeded inputs.  Gate for bf16 outputs with fp32 accumulation: max-abs <= 2e-2 and
mean-abs <= 2e-3; page-table and index handling is compared bit for bit."""
import math

import numpy as np
import pytest
import torch

import mla_absorbed_latent_mtp_b200 as m
import oracle
import synth
from gpu_util import bf16_bits, bf16_to_f64, ints_to_dev, synthetic_qtilde, to_dev
from helpers import MAX_ABS_TOL, MEAN_ABS_TOL, errors, tiny_workload

pytestmark = pytest.mark.gpu

LSE_TOL = 5e-3  # fp32 scores; l sums bf16-rounded probabilities (relative error <= 2^-9)


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


def _assert_gate(got, ref, what=""):
    mx, mean = errors(got, ref)
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, f"{what}: max-abs {mx:.3e} mean-abs {mean:.3e}"


# ----------------------------------------------------------------------------- projections

def _proj_tol(ref):
    # bf16 output rounding (2^-9 relative) plus fp32 accumulation slack
    return 2.0 ** -8 * np.abs(ref) + 1e-5


@pytest.mark.parametrize("n", [1, 7, 32, 96, 130, 300])
def test_absorb_q_matches_oracle(n):
    q = synth.normal_bf16((n, 64, 256), 1, synth.STREAM_Q)
    w = synth.normal_bf16((64, 256, 512), 1, synth.STREAM_WUK, 1 / math.sqrt(512))
    got = bf16_to_f64(m.mla_absorb_q(to_dev(q), to_dev(w)))
    torch.cuda.synchronize()
    ref = oracle.absorb_all(q, w)
    assert np.all(np.abs(got - ref) <= _proj_tol(ref)), float(np.abs(got - ref).max())


@pytest.mark.parametrize("n", [1, 7, 32, 96, 130, 300])
def test_up_proj_matches_oracle(n):
    o = synth.normal_bf16((n, 64, 512), 2, synth.STREAM_OLAT, 0.05)
    w = synth.normal_bf16((64, 256, 512), 2, synth.STREAM_WUV, 1 / math.sqrt(512))
    got = bf16_to_f64(m.mla_up_proj(to_dev(o), to_dev(w)))
    torch.cuda.synchronize()
    ref = oracle.up_project_all(o, w)
    assert np.all(np.abs(got - ref) <= _proj_tol(ref)), float(np.abs(got - ref).max())


# ----------------------------------------------------------------------------- attend stage

def _run_attend(wl, qt_bits, status=None, seq_lens_none=False):
    qt = to_dev(qt_bits)
    st = _status() if status is None else status
    if wl.mode == "dense":
        lens = None if seq_lens_none else ints_to_dev(wl.seq_lens)
        o, lse = m.mla_attend_dense(qt, to_dev(wl.cache), lens, wl.scale, status=st)
    elif wl.mode == "paged":
        o, lse = m.mla_attend_paged(qt, to_dev(wl.pool), ints_to_dev(wl.page_table), ints_to_dev(wl.seq_lens),
                                    wl.scale, status=st)
    else:
        o, lse = m.mla_attend_indexed(qt, to_dev(wl.cache), ints_to_dev(wl.indices), ints_to_dev(wl.seq_lens),
                                      wl.scale, status=st)
    torch.cuda.synchronize()
    return o, lse, int(st.item())


def _check_latent(wl, qt_bits, o, lse, pairs=None):
    ref = oracle.reference_latent(qt_bits, wl, pairs)
    got = bf16_to_f64(o)
    glse = lse.cpu().numpy().astype(np.float64)
    for (b, i), r in ref.items():
        _assert_gate(got[b, i], r["o_latent"], f"o_latent b={b} i={i}")
        fin = np.isfinite(r["lse"])
        assert np.array_equal(np.isfinite(glse[b, i]), fin)
        if fin.any():
            assert np.abs(glse[b, i][fin] - r["lse"][fin]).max() <= LSE_TOL
        if (~fin).any():
            assert np.all(got[b, i][~fin] == 0)


@pytest.mark.parametrize("lens", [[1], [5], [127], [128], [129], [300], [1, 129, 300], [1000, 2, 257, 64]])
def test_attend_dense_decode(lens):
    wl = tiny_workload("dense", len(lens), 1, lens, H=64, D=256, R=512, seed=len(lens) + lens[0])
    qt = synthetic_qtilde(wl.B, 1, seed=lens[-1])
    o, lse, st = _run_attend(wl, qt)
    assert st == 0
    _check_latent(wl, qt, o, lse)


def test_attend_dense_null_lengths_and_padding():
    wl = tiny_workload("dense", 3, 1, [200, 200, 200], H=64, D=256, R=512, seed=4)
    qt = synthetic_qtilde(3, 1, seed=9)
    o1, l1, st1 = _run_attend(wl, qt, seq_lens_none=True)
    o2, l2, st2 = _run_attend(wl, qt)
    assert st1 == 0 and st2 == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    _check_latent(wl, qt, o1, l1)


@pytest.mark.parametrize("prefix", [0, 1, 5, 63, 64, 65, 122, 123, 130, 1000])
def test_attend_mtp_window(prefix):
    """q_len = 1 + 5 drafts appended: query i sees rows 0..prefix+i (causal window)."""
    Q = 6
    L = prefix + Q
    wl = tiny_workload("dense", 2, Q, [L, L + 3], H=64, D=256, R=512, seed=prefix + 1)
    qt = synthetic_qtilde(2, Q, seed=prefix)
    o, lse, st = _run_attend(wl, qt)
    assert st == 0
    _check_latent(wl, qt, o, lse)


def test_attend_window_longer_than_cache():
    """Fewer rows than queries: early queries see nothing (o = 0, lse = -inf)."""
    wl = tiny_workload("dense", 2, 6, [3, 6], H=64, D=256, R=512, seed=2)
    qt = synthetic_qtilde(2, 6, seed=3)
    o, lse, st = _run_attend(wl, qt)
    assert st == 0
    assert torch.all(o[0, :3] == 0) and torch.all(torch.isneginf(lse[0, :3]))
    _check_latent(wl, qt, o, lse)


def test_attend_rows_past_end_are_ignored_even_if_nan():
    wl = tiny_workload("dense", 2, 1, [129, 200], H=64, D=256, R=512, seed=6, Lmax=320)
    qt = synthetic_qtilde(2, 1, seed=6)
    o_clean, l_clean, st = _run_attend(wl, qt)
    assert st == 0
    wl.cache[0, 129:] = 0x7FC0  # NaN
    wl.cache[1, 200:] = 0x7F80  # +Inf
    o_nan, l_nan, st = _run_attend(wl, qt)
    assert st == 0
    assert torch.equal(o_clean, o_nan) and torch.equal(l_clean, l_nan)


@pytest.mark.parametrize("lens", [[1, 64, 65, 200], [130, 6, 700]])
def test_attend_paged_matches_oracle_and_dense_bitwise(lens):
    Q = 1 if len(lens) == 4 else 6
    wl = tiny_workload("paged", len(lens), Q, lens, H=64, D=256, R=512, seed=sum(lens))
    qt = synthetic_qtilde(wl.B, Q, seed=7)
    o, lse, st = _run_attend(wl, qt)
    assert st == 0
    _check_latent(wl, qt, o, lse)
    # the same logical rows laid out contiguously give the identical result
    dense = tiny_workload("dense", len(lens), Q, lens, H=64, D=256, R=512, seed=1)
    for b, L in enumerate(lens):
        dense.cache[b, :L] = oracle.logical_rows("paged", b, np.arange(L), pool=wl.pool, page_table=wl.page_table)
    o2, l2, st2 = _run_attend(dense, qt)
    assert st2 == 0
    assert torch.equal(o, o2) and torch.equal(lse, l2)


@pytest.mark.parametrize("Q,K,L", [(1, 1, 50), (1, 100, 1000), (1, 128, 1000), (2, 300, 1000), (6, 257, 4000)])
def test_attend_indexed(Q, K, L):
    wl = tiny_workload("indexed", 2, Q, [L, L - 7], H=64, D=256, R=512, seed=K, K=K)
    qt = synthetic_qtilde(2, Q, seed=K + 1)
    o, lse, st = _run_attend(wl, qt)
    assert st == 0
    _check_latent(wl, qt, o, lse)


def test_attend_indexed_full_list_equals_dense_bitwise():
    L = 300
    idx = tiny_workload("indexed", 1, 1, [L], H=64, D=256, R=512, seed=5, K=L)
    dense = tiny_workload("dense", 1, 1, [L], H=64, D=256, R=512, seed=5)
    assert np.array_equal(idx.indices[0, 0], np.arange(L)) and np.array_equal(idx.cache, dense.cache)
    qt = synthetic_qtilde(1, 1, seed=5)
    a = _run_attend(idx, qt)
    b = _run_attend(dense, qt)
    assert a[2] == 0 and b[2] == 0
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_bad_page_id_sets_index_status():
    wl = tiny_workload("paged", 2, 1, [130, 70], H=64, D=256, R=512, seed=3)
    wl.page_table[1, 1] = wl.pool.shape[0] + 5
    qt = synthetic_qtilde(2, 1, seed=3)
    _, _, st = _run_attend(wl, qt)
    assert st == m.MLA_ERR_INDEX


def test_bad_index_sets_index_status():
    wl = tiny_workload("indexed", 1, 1, [500], H=64, D=256, R=512, seed=3, K=40)
    wl.indices[0, 0, 7] = 500  # not causally visible (query sits at 499)
    qt = synthetic_qtilde(1, 1, seed=3)
    _, _, st = _run_attend(wl, qt)
    assert st == m.MLA_ERR_INDEX


def test_length_beyond_cache_sets_index_status():
    wl = tiny_workload("dense", 1, 1, [100], H=64, D=256, R=512, seed=3)
    qt = synthetic_qtilde(1, 1, seed=3)
    st = _status()
    m.mla_attend_dense(to_dev(qt), to_dev(wl.cache), ints_to_dev(np.array([101])), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == m.MLA_ERR_INDEX


def test_small_workspace_rejected():
    """The binding refuses a short workspace before the call; the C ABI itself, handed one
    directly, returns MLA_ERR_WORKSPACE and launches nothing."""
    import ctypes
    qt = torch.zeros(1, 1, 64, 512, dtype=torch.bfloat16, device="cuda")
    cache = torch.zeros(1, 8, 512, dtype=torch.bfloat16, device="cuda")
    o = torch.empty(1, 1, 64, 512, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError, match="workspace"):
        m.mla_attend_dense(qt, cache, None, workspace=ws)
    vp = ctypes.c_void_p
    code = m.lib().mla_attend_dense(vp(qt.data_ptr()), vp(cache.data_ptr()), None, 1, 1, 64, 512, 8, 1.0 / 16,
                                    vp(ws.data_ptr()), 16, vp(o.data_ptr()), None, None,
                                    vp(torch.cuda.current_stream().cuda_stream))
    assert code == m.MLA_ERR_WORKSPACE


# ----------------------------------------------------------------------------- addressing, bit for bit

def test_debug_gather_bitwise():
    lens = [70, 200, 1]
    pw = tiny_workload("paged", 3, 1, lens, H=64, D=256, R=512, seed=11)
    req = np.array([(b, 0, j) for b, L in enumerate(lens) for j in range(L)], dtype=np.int32)
    got = bf16_bits(m.mla_debug_gather(m.MODE_PAGED, to_dev(pw.pool), ints_to_dev(req),
                                       page_table=ints_to_dev(pw.page_table), B=3))
    ref = np.stack([oracle.logical_rows("paged", b, np.array([j]), pool=pw.pool, page_table=pw.page_table)[0]
                    for b, _, j in req])
    assert np.array_equal(got, ref)

    iw = tiny_workload("indexed", 2, 2, [300, 280], H=64, D=256, R=512, seed=12, K=50)
    req = np.array([(b, i, k) for b in range(2) for i in range(2) for k in range(50)], dtype=np.int32)
    got = bf16_bits(m.mla_debug_gather(m.MODE_INDEXED, to_dev(iw.cache), ints_to_dev(req),
                                       indices=ints_to_dev(iw.indices), B=2, Q=2, Lmax=300))
    ref = np.stack([iw.cache[b, iw.indices[b, i, k]] for b, i, k in req])
    assert np.array_equal(got, ref)

    dw = tiny_workload("dense", 2, 1, [40, 40], H=64, D=256, R=512, seed=13)
    req = np.array([(b, 0, j) for b in range(2) for j in range(40)], dtype=np.int32)
    got = bf16_bits(m.mla_debug_gather(m.MODE_DENSE, to_dev(dw.cache), ints_to_dev(req), B=2, Lmax=40))
    assert np.array_equal(got, dw.cache.reshape(80, 512))

    st = _status()
    bad = np.array([(0, 0, 40)], dtype=np.int32)
    got = bf16_bits(m.mla_debug_gather(m.MODE_DENSE, to_dev(dw.cache), ints_to_dev(bad), B=2, Lmax=40, status=st))
    torch.cuda.synchronize()
    assert int(st.item()) == m.MLA_ERR_INDEX and np.all(got == 0)


# ----------------------------------------------------------------------------- whole path

def test_full_path_tiny_config_against_expanded_oracle():
    wl = synth.make_workload("tiny_dense_decode")
    st = _status()
    out, lse = m.mla_decode(to_dev(wl.q), to_dev(wl.w_uk), to_dev(wl.w_uv), to_dev(wl.cache),
                            ints_to_dev(wl.seq_lens), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = oracle.reference(wl)
    _assert_gate(bf16_to_f64(out)[0, 0], ref[(0, 0)]["out"], "tiny")
    assert np.abs(lse.cpu().numpy()[0, 0] - ref[(0, 0)]["lse"]).max() <= LSE_TOL


@pytest.mark.parametrize("mode,Q,lens,K", [
    ("dense", 6, [600, 129], None),
    ("paged", 1, [1, 400, 1111], None),
    ("indexed", 2, [3000, 900], 200),
])
def test_full_path_small_against_expanded_oracle(mode, Q, lens, K):
    wl = tiny_workload(mode, len(lens), Q, lens, H=64, D=256, R=512, seed=17, K=K)
    wl.scale = 1.0 / 16.0
    st = _status()
    cache = wl.pool if mode == "paged" else wl.cache
    out, lse = m.mla_decode(to_dev(wl.q), to_dev(wl.w_uk), to_dev(wl.w_uv), to_dev(cache), ints_to_dev(wl.seq_lens),
                            mode={"dense": 0, "paged": 1, "indexed": 2}[mode],
                            page_table=ints_to_dev(wl.page_table) if mode == "paged" else None,
                            indices=ints_to_dev(wl.indices) if mode == "indexed" else None, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = oracle.reference(wl)
    got = bf16_to_f64(out)
    for (b, i), r in ref.items():
        _assert_gate(got[b, i], r["out"], f"{mode} b={b} i={i}")


# ----------------------------------------------------------------------------- split edge cases

@pytest.mark.parametrize("mode", ["dense", "paged"])
def test_zero_length_sequence_among_others(mode):
    """A sequence with no rows has no tiles: its output is 0 and its lse -inf, and the
    other sequences' splits are unaffected."""
    lens = [300, 0, 65, 1]
    wl = tiny_workload(mode, len(lens), 1, lens, H=64, D=256, R=512, seed=41)
    qt = synthetic_qtilde(wl.B, 1, seed=42)
    o, lse, st = _run_attend(wl, qt)
    assert st == 0
    _check_latent(wl, qt, o, lse)
    assert not bool(torch.isfinite(lse[1]).any()) and not bool(o[1].any())


def test_one_long_sequence_split_over_every_group():
    """A single sequence spread over all CTA groups: about one partial per SM to merge."""
    L = 100_000
    wl = tiny_workload("dense", 1, 1, [L], H=64, D=256, R=512, seed=43)
    qt = synthetic_qtilde(1, 1, seed=44)
    o, lse, st = _run_attend(wl, qt)
    assert st == 0
    _check_latent(wl, qt, o, lse)


def test_many_short_sequences():
    """More sequences than SMs, each a single partial tile."""
    lens = [1 + (7 * b) % 64 for b in range(300)]
    wl = tiny_workload("dense", len(lens), 1, lens, H=64, D=256, R=512, seed=45)
    qt = synthetic_qtilde(wl.B, 1, seed=46)
    o, lse, st = _run_attend(wl, qt)
    assert st == 0
    pairs = [(b, 0) for b in range(0, len(lens), 37)]
    _check_latent(wl, qt, o, lse, pairs=pairs)

"""Index-list attention whose CTAs merge in a thread-block cluster.

When a list's tiles are split over C <= 8 CTAs and the clusters fit the GPU at once, the C
CTAs of a list run as one cluster: each writes its partial (O, m, l) to the workspace, and
after a cluster barrier the cluster merges the list's partials (from L2) and writes
o_latent and lse itself -- no combine kernel.  C = min(SMs // lists, tiles per list), so
the list length picks the cluster size here (two lists, K = 64 C - 13 entries: a ragged
last tile).  The merge follows the combine kernel's arithmetic step for step, so a full
index list still equals the dense path bit for bit at every cluster size."""
import numpy as np
import pytest
import torch

import mla_absorbed_latent_mtp_b200 as m
import oracle
from gpu_util import bf16_to_f64, ints_to_dev, synthetic_qtilde, to_dev
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


def _attend(wl, qt_bits):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qt = to_dev(qt_bits)
    if wl.mode == "dense":
        o, lse = m.mla_attend_dense(qt, to_dev(wl.cache), ints_to_dev(wl.seq_lens), wl.scale, status=st)
    else:
        o, lse = m.mla_attend_indexed(qt, to_dev(wl.cache), ints_to_dev(wl.indices), ints_to_dev(wl.seq_lens),
                                      wl.scale, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, m.status_string(int(st.item()))
    return o, lse


def _check(wl, qt, o, lse):
    ref = oracle.reference_latent(qt, wl)
    got = bf16_to_f64(o)
    glse = lse.cpu().numpy().astype(np.float64)
    for (b, i), r in ref.items():
        mx, mean = errors(got[b, i], r["o_latent"])
        assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (b, i, mx, mean)
        fin = np.isfinite(r["lse"])
        assert np.array_equal(np.isfinite(glse[b, i]), fin)
        if fin.any():
            assert np.abs(glse[b, i][fin] - r["lse"][fin]).max() <= LSE_TOL
        if (~fin).any():
            assert np.all(got[b, i][~fin] == 0)


@pytest.mark.parametrize("C", [1, 2, 3, 4, 7, 8])
def test_cluster_sizes_against_oracle(C):
    K = 64 * C - 13
    wl = tiny_workload("indexed", 2, 1, [3000, 2500], H=64, D=256, R=512, seed=60 + C, K=K)
    qt = synthetic_qtilde(2, 1, seed=61 + C)
    o, lse = _attend(wl, qt)
    _check(wl, qt, o, lse)


def test_verify_window_lists_against_oracle():
    """q_len = 6 lists (12 lists of 4 tiles: clusters of 4)."""
    wl = tiny_workload("indexed", 2, 6, [4000, 3100], H=64, D=256, R=512, seed=70, K=250)
    qt = synthetic_qtilde(2, 6, seed=71)
    o, lse = _attend(wl, qt)
    _check(wl, qt, o, lse)


def test_empty_segments_and_an_empty_list():
    """List 0 has 70 used entries of 256, so the CTAs of tiles 2 and 3 hold empty partials
    (weight zero) and tile 1 holds six rows; list 1 has none (o = 0, lse = -inf)."""
    wl = tiny_workload("indexed", 2, 1, [3000, 2000], H=64, D=256, R=512, seed=72, K=256)
    wl.indices[0, 0, 70:] = -1
    wl.indices[1, 0, :] = -1
    qt = synthetic_qtilde(2, 1, seed=73)
    o, lse = _attend(wl, qt)
    assert torch.all(o[1, 0] == 0) and torch.all(torch.isneginf(lse[1, 0]))
    _check(wl, qt, o, lse)


@pytest.mark.parametrize("L", [50, 150, 300, 492])
def test_full_list_equals_dense_bitwise(L):
    """One list of L entries 0..L-1 (a cluster of ceil(L / 64) CTAs, one tile each) against
    dense decode of the same L rows (one tile per CTA group, merged by the combine)."""
    idx = tiny_workload("indexed", 1, 1, [L], H=64, D=256, R=512, seed=74, K=L)
    dense = tiny_workload("dense", 1, 1, [L], H=64, D=256, R=512, seed=74)
    assert np.array_equal(idx.indices[0, 0], np.arange(L)) and np.array_equal(idx.cache, dense.cache)
    qt = synthetic_qtilde(1, 1, seed=75)
    a = _attend(idx, qt)
    b = _attend(dense, qt)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def _kernel_nodes(fn):
    """Kernel launches fn records in a CUDA graph."""
    from cuda.bindings import runtime as rt
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(g):
        fn()
    h = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
    err, _, n = rt.cudaGraphGetNodes(h, 0)
    assert err == rt.cudaError_t.cudaSuccess
    err, nodes, n = rt.cudaGraphGetNodes(h, n)
    assert err == rt.cudaError_t.cudaSuccess
    kinds = [rt.cudaGraphNodeGetType(x)[1] for x in nodes[:n]]
    return sum(k == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel for k in kinds)


def test_one_kernel_per_call_at_the_benchmark_shape():
    """32 lists of 2,048 entries (clusters of 4 on 148 SMs): the attend kernel alone; dense
    decode of the same cache: attend + combine."""
    B, K, L = 32, 2048, 8192
    qt = torch.zeros(B, 1, 64, 512, dtype=torch.bfloat16, device="cuda")
    cache = torch.zeros(B, L, 512, dtype=torch.bfloat16, device="cuda")
    idx = torch.arange(K, dtype=torch.int32, device="cuda").repeat(B, 1).view(B, 1, K).contiguous()
    lens = torch.full((B,), L, dtype=torch.int32, device="cuda")
    ws = m.new_workspace(B, 1)
    o = torch.empty(B, 1, 64, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, 1, 64, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    n_idx = _kernel_nodes(lambda: m.mla_attend_indexed(qt, cache, idx, lens, 0.0625, ws, o, lse, st))
    n_dense = _kernel_nodes(lambda: m.mla_attend_dense(qt, cache, lens, 0.0625, ws, o, lse, st))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert (n_idx, n_dense) == (1, 2)

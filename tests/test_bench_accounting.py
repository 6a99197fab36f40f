"""bench.py's accounting against the arithmetic of the method (no GPU).

"Module 05 -- MLA: Compressing Per-Token History" (sections 2-4): a cached token is one 512-wide
bf16 latent, 1,024 bytes, read once however many query rows share it; the absorbed score
and the latent value sum each take 512 multiply-adds per (head, query, visible row), so
2,048 FLOP.  A verify window's query i sees the rows j <= L - q_len + i.  The roofline is
bound by whichever of the cache bytes at the HBM peak and those FLOPs at the tensor peak
takes longer."""
import pytest

import bench
import synth

PEAKS = {"hbm_gbs": 6557.8, "bf16_tflops": 1663.7}


def _brute_pairs(lens, Q):
    return sum(1 for L in lens for i in range(Q) for j in range(int(L)) if j <= int(L) - Q + i)


def test_dense_decode_bytes_and_flops():
    wl = synth.make_workload("dense_decode", with_data=False)
    acc = bench.step_bytes(wl)
    assert acc["cache"] == 32 * 8192 * 1024
    assert acc["flops_attend"] == 32 * 8192 * 64 * 2048
    # both weight matrices (64 x 256 x 512 bf16 each), q in and out written
    assert acc["total"] - acc["cache"] == 2 * 64 * 256 * 512 * 2 + 2 * 32 * 64 * 256 * 2


@pytest.mark.parametrize("Q,L", [(6, 40), (3, 7), (1, 5)])
def test_verify_window_counts_causal_pairs_and_reads_rows_once(Q, L):
    wl = synth.make_workload(mode="dense", B=2, Q=Q, L=L, with_data=False)
    acc = bench.step_bytes(wl)
    assert acc["cache"] == 2 * L * 1024  # every row once, shared by the window's Q queries
    assert acc["flops_attend"] == _brute_pairs(wl.seq_lens, Q) * 64 * 2048


def test_mtp_verify_pair_count_closed_form():
    wl = synth.make_workload("mtp_verify", with_data=False)
    acc = bench.step_bytes(wl)
    L, Q = int(wl.seq_lens[0]), wl.Q
    assert acc["flops_attend"] == 16 * (Q * L - Q * (Q - 1) // 2) * 64 * 2048


def test_indexed_counts_list_rows():
    wl = synth.make_workload("indexed_sparse_decode", with_data=False)
    acc = bench.step_bytes(wl)
    K = wl.indices.shape[2]
    assert acc["cache"] == wl.B * wl.Q * K * 1024
    assert acc["flops_attend"] == wl.B * wl.Q * K * 64 * 2048


def test_roofline_bound_follows_the_ridge():
    ridge = PEAKS["bf16_tflops"] * 1e12 / (PEAKS["hbm_gbs"] * 1e9)  # FLOP per byte
    below = {"cache": 10**9, "flops_attend": int(0.99 * ridge * 10**9)}
    above = {"cache": 10**9, "flops_attend": int(1.01 * ridge * 10**9)}
    r = bench.attend_roofline(below, 1.0, PEAKS, "measured", None)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(1000.0) and r["frac"] == pytest.approx(1000.0 / PEAKS["hbm_gbs"])
    r = bench.attend_roofline(above, 1.0, PEAKS, "measured", 123)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["traffic"] == 123
    assert r["achieved"] == pytest.approx(above["flops_attend"] / 1e-3 / 1e12)


def test_workload_bounds_are_the_expected_ones():
    """q_len = 1 (128 FLOP/B) sits below the ridge (~254 FLOP/B), q_len = 6 above it."""
    dense = bench.step_bytes(synth.make_workload("dense_decode", with_data=False))
    mtp = bench.step_bytes(synth.make_workload("mtp_verify", with_data=False))
    assert bench.attend_roofline(dense, 0.068, PEAKS, "measured", None)["bound"] == "hbm"
    assert bench.attend_roofline(mtp, 0.58, PEAKS, "measured", None)["bound"] == "tensor"


def test_recorded_traffic_is_close_to_the_algorithmic_bytes():
    """A recorded DRAM traffic figure well above the cache bytes would mean re-reads.  Allowed
    on top of 10%: q~ (64 KiB per query row, read once) and 128 KiB of fixed per-launch reads
    (lengths, tables, tensor maps), which dominate only the tiny workload."""
    for (name, _src), traffic in bench.TRAFFIC.items():
        wl = synth.make_workload(name, with_data=False)
        cache = bench.step_bytes(wl)["cache"]
        qt = wl.B * wl.Q * 64 * 512 * 2
        assert cache <= traffic <= 1.1 * cache + qt + (1 << 17), (name, traffic, cache)


@pytest.mark.parametrize("L", [1, 5, 64, 130])
def test_prefill_flop_counts(L):
    """A prefill's causal (query, key) pairs, counted one by one; the absorbed attention does
    twice the expanded one's arithmetic per pair (512-wide latent against 256-wide heads)."""
    pairs = sum(1 for t in range(L) for j in range(L) if j <= t)
    f = bench.prefill_flops(L)
    assert f["expanded_attention"] == pairs * 64 * 2 * 2 * 256
    assert f["absorbed_attention"] == 2 * f["expanded_attention"]
    assert f["expanded"] - f["expanded_attention"] == 2 * 2 * L * 512 * 64 * 256
    assert f["absorbed"] - f["absorbed_attention"] == 2 * 2 * L * 64 * 256 * 512


@pytest.mark.parametrize("K,n_rot", [(20, 4), (20, 1), (1000, 1), (1000, 4), (3, 4), (7, 1), (1, 1)])
def test_graph_batches_time_exactly_k_steps(K, n_rot):
    """The timed loops replay graphs of G steps K / G times: G must divide K."""
    G = bench.steps_per_graph(K, n_rot)
    assert 1 <= G <= 32 and K % G == 0
    if any(K % g == 0 and g % n_rot == 0 for g in range(1, min(K, 32) + 1)):
        assert G % n_rot == 0


class _FakeRuntime:
    """Stands in for the CUDA runtime binding: a graph of the given node kinds."""

    class cudaError_t:
        cudaSuccess = 0
        cudaErrorInvalidValue = 1

    class cudaGraphNodeType:
        cudaGraphNodeTypeKernel = "kernel"
        cudaGraphNodeTypeMemcpy = "memcpy"
        cudaGraphNodeTypeEventRecord = "event"

    def __init__(self, kinds, fail=False):
        self.kinds, self.fail, self.handles = kinds, fail, []

    def cudaGraph_t(self, init_value):
        self.handles.append(init_value)
        return ("graph", init_value)

    def cudaGraphGetNodes(self, h, n):
        assert h == ("graph", 1234)
        if self.fail:
            return self.cudaError_t.cudaErrorInvalidValue, [], 0
        # a count query first (n = 0), then the nodes themselves
        return self.cudaError_t.cudaSuccess, list(range(len(self.kinds)))[:n], len(self.kinds)

    def cudaGraphNodeGetType(self, node):
        return self.cudaError_t.cudaSuccess, self.kinds[node]


class _FakeGraph:
    def raw_cuda_graph(self):
        return 1234


def _with_runtime(monkeypatch, rt):
    import sys
    import types
    pkg = types.ModuleType("cuda.bindings")
    pkg.runtime = rt
    monkeypatch.setitem(sys.modules, "cuda.bindings", pkg)
    monkeypatch.setitem(sys.modules, "cuda.bindings.runtime", rt)


def test_launch_count_counts_kernel_nodes_only(monkeypatch):
    """gpu_launches comes from the captured step graph: kernel nodes counted, copies and
    event nodes not."""
    K = _FakeRuntime.cudaGraphNodeType
    kinds = [K.cudaGraphNodeTypeKernel] * 3 + [K.cudaGraphNodeTypeMemcpy, K.cudaGraphNodeTypeEventRecord] + \
        [K.cudaGraphNodeTypeKernel] * 4
    rt = _FakeRuntime(kinds)
    _with_runtime(monkeypatch, rt)
    assert bench.graph_kernel_nodes(_FakeGraph()) == 7
    assert rt.handles == [1234]


def test_launch_count_fails_loudly(monkeypatch):
    _with_runtime(monkeypatch, _FakeRuntime([], fail=True))
    with pytest.raises(RuntimeError):
        bench.graph_kernel_nodes(_FakeGraph())

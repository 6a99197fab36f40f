"""The online softmax's rescale of O in TMEM, exercised on purpose.

The attend kernel keeps a running max per head and moves it only when a score beats it
by more than 2^8 in log2 units; when that happens after a CTA segment's first tile, the
accumulated O^T columns in TMEM are multiplied by 2^(m_old - m_new) before the next value
product.  Broad N(0,1) scores never trigger it, so these inputs plant, for every head, a
ramp of four rows in consecutive tiles whose log2-scaled scores are 20, 32, 44 and 56
(about 10 above the largest background score, then 12 above the previous step).  Every
step therefore raises the running max by more than 8, and every step that is not the first
tile of its segment runs the rescale.  The test counts those steps from the kernel's tile
partition (the same formula the kernel uses) and requires many of them, then compares
o_latent and lse with the oracle.  The heads' ramps sit at different places, so the steps
also cross segment boundaries, where the split-L combine has to weigh partials whose
maxima differ by 2^12 and more.

Score construction: head h's absorbed query is 32 on latent dims 8h..8h+7 and N(0, 1/16)
elsewhere; cache rows are N(0, 1/16) (std 0.25), so background scores have a standard
deviation of about 2 in log2 units.  A planted row for head h sets its dims 8h..8h+7 to
d / (scale * log2(e) * 8 * 32), which gives head h the log2 score d and leaves the other
heads' scores at background level."""
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

LSE_TOL = 5e-3
TAU = 8.0                      # the kernel's lazy-rescale threshold (log2 units)
RAMP = (20.0, 32.0, 44.0, 56.0)
GAMMA = 32.0


@pytest.fixture(scope="module", autouse=True)
def device():
    import __graft_entry__
    __graft_entry__.build()
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def _qtilde(B, Q, seed):
    qt = synth.f64_to_bf16_bits(synth.normal_f64(B * Q * 64 * 512, seed, synth.STREAM_QTILDE, 0.25)
                                .reshape(B, Q, 64, 512))
    g = synth.f64_to_bf16_bits(np.array([GAMMA]))[0]
    for h in range(64):
        qt[:, :, h, 8 * h:8 * h + 8] = g
    return qt


def _planted_value(d, scale):
    return synth.f64_to_bf16_bits(np.array([d / (scale * math.log2(math.e) * 8 * GAMMA)]))[0]


def _ramp_tile(h, b, n_tiles):
    """First tile (within its sequence or list) of head h's ramp."""
    return (h * 37 + b * 11) % max(n_tiles - 4, 1)


def _groups(mode, B, Q, K):
    """The kernel's CTA-group count: for index lists (all of the same length) a multiple of
    the number of lists, so that no group straddles two lists; else SMs / Q."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if mode != "indexed":
        return max(1, sms // Q)
    lists, nt = B * Q, (K + 63) // 64
    per_list = min(sms // lists, nt)
    return per_list * lists if per_list >= 1 else sms


def _interior_steps(tile_lists, G):
    """Number of ramp steps (global tile index t, previous tile t - 1 of the same sequence)
    that land in the same CTA group as t - 1: those steps run the rescale branch.
    tile_lists: per sequence of the tile list, (first global tile, [step tiles])."""
    T = tile_lists[-1][2]
    starts = [g * T // G for g in range(G + 1)]

    def group_of(t):
        lo, hi = 0, G - 1
        while lo < hi:  # largest g with starts[g] <= t
            mid = (lo + hi + 1) // 2
            if starts[mid] <= t:
                lo = mid
            else:
                hi = mid - 1
        return lo

    n = 0
    for base, steps, _ in tile_lists:
        for t in steps:
            if t - 1 >= base and group_of(t) == group_of(t - 1):
                n += 1
    return n


def _plant(wl, Q):
    """Write the ramps into the cache; return the per-sequence tile bookkeeping."""
    tiles = []
    T = 0
    if wl.mode == "indexed":
        K = wl.indices.shape[2]
        nt = (K + 63) // 64
        # the queries of a window get disjoint lists (positions i mod Q), so that a row
        # planted for one query's ramp is never part of another query's list
        for b in range(wl.B):
            for i in range(Q):
                n_res = (int(wl.seq_lens[b]) - Q) // Q + 1
                wl.indices[b, i] = i + Q * synth.sorted_sample(K, n_res, 47, synth.STREAM_INDEX_BASE + b * Q + i)
        for b in range(wl.B):
            for i in range(Q):
                steps = []
                for h in range(64):
                    a = _ramp_tile(h, b * Q + i, nt)
                    for k, d in enumerate(RAMP):
                        pos = (a + k) * 64 + (h * 7 + k * 13) % 64
                        row = int(wl.indices[b, i, min(pos, K - 1)])
                        wl.cache[b, row, 8 * h:8 * h + 8] = _planted_value(d, wl.scale)
                        if k > 0:
                            steps.append(T + a + k)
                tiles.append((T, steps, T + nt))
                T += nt
        return tiles
    for b in range(wl.B):
        L = int(wl.seq_lens[b])
        nt = (L + 63) // 64
        steps = []
        for h in range(64):
            a = _ramp_tile(h, b, (L - Q) // 64)
            for k, d in enumerate(RAMP):
                j = (a + k) * 64 + (h * 7 + k * 13) % 64
                assert j < L - Q + 1  # visible to every query of the window
                v = _planted_value(d, wl.scale)
                if wl.mode == "paged":
                    wl.pool[wl.page_table[b, j // 64], j % 64, 8 * h:8 * h + 8] = v
                else:
                    wl.cache[b, j, 8 * h:8 * h + 8] = v
                if k > 0:
                    steps.append(T + a + k)
        tiles.append((T, steps, T + nt))
        T += nt
    return tiles


def _run(wl, qt_bits):
    qt = to_dev(qt_bits)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if wl.mode == "dense":
        o, lse = m.mla_attend_dense(qt, to_dev(wl.cache), ints_to_dev(wl.seq_lens), wl.scale, status=st)
    elif wl.mode == "paged":
        o, lse = m.mla_attend_paged(qt, to_dev(wl.pool), ints_to_dev(wl.page_table), ints_to_dev(wl.seq_lens),
                                    wl.scale, status=st)
    else:
        o, lse = m.mla_attend_indexed(qt, to_dev(wl.cache), ints_to_dev(wl.indices), ints_to_dev(wl.seq_lens),
                                      wl.scale, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, m.status_string(int(st.item()))
    return bf16_to_f64(o), lse.cpu().numpy().astype(np.float64)


CASES = [
    ("dense", 1, [8192, 8192, 8192, 8192], None),
    ("dense", 6, [4096 + 6, 4000 + 6], None),
    ("dense", 1, [100000], None),  # one long sequence split over every CTA group
    ("paged", 1, [8192, 7001, 9000, 8500], None),
    ("paged", 6, [4100, 3900], None),
    ("indexed", 1, [4096] * 16, 2048),
    ("indexed", 6, [16384] * 3, 2048),
]


@pytest.mark.parametrize("mode,Q,lens,K", CASES)
def test_rescale_branch_against_oracle(mode, Q, lens, K):
    B = len(lens)
    wl = tiny_workload(mode, B, Q, lens, H=64, D=256, R=512, seed=41 + B + Q, K=K, c_std=0.25)
    tiles = _plant(wl, Q)
    qt = _qtilde(B, Q, seed=43 + B)
    # the ramps must reach the branch: steps inside a segment, after its first tile
    interior = _interior_steps(tiles, _groups(mode, B, Q, K))
    assert interior >= 32, interior
    # and the planted scores really are the margins stated above (log2 units, fp64)
    if mode == "indexed":
        pos0 = wl.indices[0, 0]
    else:
        pos0 = np.arange(int(wl.seq_lens[0]) - Q + 1)
    c0 = oracle.widen(oracle.logical_rows(mode, 0, pos0, cache=wl.cache, pool=wl.pool, page_table=wl.page_table))
    back = wl.scale * math.log2(math.e) * (c0 @ oracle.widen(qt[0, 0]).T)
    peak = np.sort(back, axis=0)[-5]  # below the four planted rows of each head
    assert np.all(RAMP[0] - peak > TAU + 1.0), float((RAMP[0] - peak).min())
    o, lse = _run(wl, qt)
    ref = oracle.reference_latent(qt, wl)
    for (b, i), r in ref.items():
        mx, mean = errors(o[b, i], r["o_latent"])
        assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (b, i, mx, mean)
        assert np.abs(lse[b, i] - r["lse"]).max() <= LSE_TOL, (b, i)

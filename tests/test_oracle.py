"""Pins for the fp64 oracle: values and facts fixed by the pages and by mathematics,
chosen so that a plausible slip in the oracle (dropped term, wrong sign or index,
transposed operand, wrong scale, shifted window) fails at least one of them."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import read_golden
from helpers import decode_list, gate, errors, tiny_workload


# ----------------------------------------------------------------------------- page facts

def test_memory_arithmetic_matches_page():
    g = read_golden("memory_arithmetic.txt")
    assert oracle.expanded_bytes_per_token() == g["expanded_bytes"]
    assert oracle.latent_bytes_per_token() == g["latent_bytes"]
    assert oracle.expanded_bytes_per_token() // oracle.latent_bytes_per_token() == g["ratio"]
    assert oracle.expanded_bytes_per_token() % oracle.latent_bytes_per_token() == 0


def test_dimensions_match_page():
    g = read_golden("dimensions.txt")
    assert oracle.LATENT_WIDTH == g["latent"]
    assert oracle.NUM_HEADS == g["heads"]
    assert oracle.HEAD_DIM == g["head_dim"]
    assert oracle.MTP_DRAFT_TOKENS == g["draft_tokens"]
    assert 1 + oracle.MTP_DRAFT_TOKENS == g["verify_q_len"]
    assert oracle.SCALE == 1.0 / 16.0  # 1/sqrt(256), exact power of two
    assert (synth.H, synth.D, synth.R) == (g["heads"], g["head_dim"], g["latent"])


# ----------------------------------------------------------------------------- brute force

def _brute_force(wl):
    """Pure-Python loops: expanded keys/values, softmax, weighted sum (tiny shapes only)."""
    f = decode_list  # bits decoded field by field, not through oracle.widen

    H, D, R = wl.q.shape[2], wl.q.shape[3], wl.w_uk.shape[2]
    out = {}
    for b in range(wl.B):
        for i in range(wl.Q):
            if wl.mode == "indexed":
                vis = [int(x) for x in wl.indices[b, i]]
            else:
                t = int(wl.seq_lens[b]) - wl.Q + i
                vis = list(range(0, t + 1))
            rows = []
            for j in vis:
                if wl.mode == "paged":
                    rows.append(f(wl.pool[wl.page_table[b, j // 64], j % 64]))
                else:
                    rows.append(f(wl.cache[b, j]))
            res = []
            for h in range(H):
                uk = [f(wl.w_uk[h, d]) for d in range(D)]
                uv = [f(wl.w_uv[h, d]) for d in range(D)]
                q = f(wl.q[b, i, h])
                ks = [[sum(uk[d][r] * c[r] for r in range(R)) for d in range(D)] for c in rows]
                vs = [[sum(uv[d][r] * c[r] for r in range(R)) for d in range(D)] for c in rows]
                s = [wl.scale * sum(q[d] * k[d] for d in range(D)) for k in ks]
                if not s:
                    res.append([0.0] * D)
                    continue
                m = max(s)
                e = [math.exp(x - m) for x in s]
                z = sum(e)
                res.append([sum(e[j] / z * vs[j][d] for j in range(len(vs))) for d in range(D)])
            out[(b, i)] = np.array(res)
    return out


@pytest.mark.parametrize("mode,B,Q,lens,K", [
    ("dense", 2, 1, [1, 5], None),
    ("dense", 2, 3, [3, 5], None),
    ("dense", 1, 2, [4], None),
    ("paged", 2, 1, [5, 3], None),
    ("paged", 1, 3, [5], None),
    ("indexed", 2, 1, [5, 4], 3),
    ("indexed", 1, 2, [5], 2),
])
def test_oracle_matches_brute_force(mode, B, Q, lens, K):
    wl = tiny_workload(mode, B, Q, lens, H=2, D=4, R=8, seed=3, K=K)
    wl.scale = 1.0 / math.sqrt(4)
    bf = _brute_force(wl)
    for form in ("expanded", "absorbed"):
        ref = oracle.reference(wl, form=form)
        for key, v in bf.items():
            np.testing.assert_allclose(ref[key]["out"], v, rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------- identity

@pytest.mark.parametrize("mode", ["dense", "paged", "indexed"])
def test_absorbed_equals_expanded(mode):
    """Module 05 section 3: absorption changes only the order of products."""
    lens = [300, 129]
    wl = tiny_workload(mode, 2, 6 if mode != "indexed" else 2, lens, H=4, D=256, R=512, seed=5, K=100)
    a = oracle.reference(wl, form="expanded")
    b = oracle.reference(wl, form="absorbed")
    for key in a:
        np.testing.assert_allclose(b[key]["out"], a[key]["out"], rtol=1e-10, atol=1e-13)
        np.testing.assert_allclose(b[key]["lse"], a[key]["lse"], rtol=1e-12)


def test_scores_identical_not_proportional():
    """Module 05 section 3: absorbed scores equal the original q.k scores, same scale."""
    wl = tiny_workload("dense", 1, 1, [40], H=3, D=256, R=512, seed=11)
    u_k = oracle.widen(wl.w_uk)
    c = oracle.widen(wl.cache[0])
    for h in range(3):
        q = oracle.widen(wl.q[0, 0, h])
        k, _ = oracle.expand_kv(c, u_k[h], u_k[h])
        s_exp = wl.scale * (k @ q)
        s_abs = wl.scale * (c @ oracle.absorb_query(q, u_k[h]))
        np.testing.assert_allclose(s_abs, s_exp, rtol=1e-11, atol=1e-13)


# ----------------------------------------------------------------------------- library routine

def test_oracle_matches_torch_sdpa_fp64():
    """Ordinary attention over expanded k/v equals torch's scaled_dot_product_attention
    in float64 (CPU), with the MTP causal window as an explicit mask."""
    B, Q, L = 2, 6, 37
    wl = tiny_workload("dense", B, Q, [L, L - 9], H=4, D=256, R=512, seed=7)
    ref = oracle.reference(wl)
    u_k = oracle.widen(wl.w_uk)
    u_v = oracle.widen(wl.w_uv)
    for b in range(B):
        Lb = int(wl.seq_lens[b])
        c = oracle.widen(wl.cache[b, :Lb])
        for h in range(4):
            k = torch.from_numpy(c @ u_k[h].T)[None, None]
            v = torch.from_numpy(c @ u_v[h].T)[None, None]
            q = torch.from_numpy(oracle.widen(wl.q[b, :, h]))[None, None]
            pos = torch.arange(Q) + (Lb - Q)
            mask = torch.arange(Lb)[None, :] <= pos[:, None]
            o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask[None, None], scale=1.0 / 16)
            for i in range(Q):
                np.testing.assert_allclose(ref[(b, i)]["out"][h], o[0, 0, i].numpy(), rtol=1e-10, atol=1e-13)


# ----------------------------------------------------------------------------- closed forms

def test_single_position_returns_value_projection():
    wl = tiny_workload("dense", 1, 1, [1], H=4, D=256, R=512, seed=2)
    ref = oracle.reference(wl)[(0, 0)]["out"]
    c = oracle.widen(wl.cache[0, 0])
    for h in range(4):
        np.testing.assert_allclose(ref[h], oracle.widen(wl.w_uv[h]) @ c, rtol=1e-12, atol=1e-14)


def test_equal_latents_return_value_projection():
    wl = tiny_workload("dense", 1, 1, [50], H=2, D=256, R=512, seed=2)
    wl.cache[0, :, :] = wl.cache[0, 7, :]
    ref = oracle.reference(wl)[(0, 0)]["out"]
    c = oracle.widen(wl.cache[0, 7])
    for h in range(2):
        np.testing.assert_allclose(ref[h], oracle.widen(wl.w_uv[h]) @ c, rtol=1e-10, atol=1e-13)


def test_zero_query_gives_uniform_average():
    wl = tiny_workload("dense", 1, 1, [33], H=2, D=256, R=512, seed=4)
    wl.q[:] = 0
    ref = oracle.reference(wl)[(0, 0)]["out"]
    cbar = oracle.widen(wl.cache[0]).mean(axis=0)
    for h in range(2):
        np.testing.assert_allclose(ref[h], oracle.widen(wl.w_uv[h]) @ cbar, rtol=1e-10, atol=1e-13)


def test_dominant_score_selects_one_position():
    """One latent aligned with q~ and scaled up: the softmax concentrates on it."""
    wl = tiny_workload("dense", 1, 1, [20], H=1, D=256, R=512, seed=9, c_std=0.01)
    u_k = oracle.widen(wl.w_uk[0])
    qt = oracle.absorb_query(oracle.widen(wl.q[0, 0, 0]), u_k)
    j = 13
    wl.cache[0, j] = synth.f64_to_bf16_bits(qt / np.linalg.norm(qt) * 64.0)
    ref = oracle.reference(wl)[(0, 0)]["out"][0]
    target = oracle.widen(wl.w_uv[0]) @ oracle.widen(wl.cache[0, j])
    np.testing.assert_allclose(ref, target, rtol=1e-6, atol=1e-8)


def test_empty_window_is_zero():
    """A cache shorter than the query window leaves early queries nothing to see."""
    wl = tiny_workload("dense", 1, 6, [3], H=2, D=256, R=512, seed=1)
    ref = oracle.reference(wl)
    for i in range(3):
        assert np.all(ref[(0, i)]["out"] == 0) and np.all(np.isneginf(ref[(0, i)]["lse"]))
    assert np.all(np.isfinite(ref[(0, 3)]["lse"]))


# ----------------------------------------------------------------------------- invariants

def test_page_table_does_not_change_result():
    lens = [130, 64, 1]
    dense = tiny_workload("dense", 3, 1, lens, H=2, D=256, R=512, seed=6)
    paged = tiny_workload("paged", 3, 1, lens, H=2, D=256, R=512, seed=6)
    # copy the dense rows into the pool through the page table
    for b, L in enumerate(lens):
        for j in range(L):
            paged.pool[paged.page_table[b, j // 64], j % 64] = dense.cache[b, j]
    paged.q, paged.w_uk, paged.w_uv = dense.q, dense.w_uk, dense.w_uv
    a = oracle.reference(dense)
    b = oracle.reference(paged)
    for key in a:
        assert np.array_equal(a[key]["out"], b[key]["out"])


def test_indexed_full_list_equals_dense():
    lens = [70]
    dense = tiny_workload("dense", 1, 1, lens, H=2, D=256, R=512, seed=8)
    idx = tiny_workload("indexed", 1, 1, lens, H=2, D=256, R=512, seed=8, K=70)
    assert np.array_equal(idx.indices[0, 0], np.arange(70))
    a = oracle.reference(dense)[(0, 0)]["out"]
    b = oracle.reference(idx)[(0, 0)]["out"]
    assert np.array_equal(a, b)


def test_indexed_equals_dense_on_gathered_cache():
    lens = [300]
    idx = tiny_workload("indexed", 1, 1, lens, H=2, D=256, R=512, seed=12, K=40)
    sub = tiny_workload("dense", 1, 1, [40], H=2, D=256, R=512, seed=12)
    sub.cache = idx.cache[:, idx.indices[0, 0]]
    sub.q, sub.w_uk, sub.w_uv = idx.q, idx.w_uk, idx.w_uv
    a = oracle.reference(idx)[(0, 0)]["out"]
    b = oracle.reference(sub)[(0, 0)]["out"]
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-15)


def test_split_lse_identity():
    """Softmax over a union of disjoint parts = LSE-weighted merge of the parts."""
    wl = tiny_workload("dense", 1, 1, [200], H=2, D=256, R=512, seed=13)
    u_k = oracle.widen(wl.w_uk[1])
    qt = oracle.absorb_query(oracle.widen(wl.q[0, 0, 1]), u_k)
    c = oracle.widen(wl.cache[0])
    o_all, _, lse_all = oracle.attend_latent(qt, c, wl.scale)
    parts = [oracle.attend_latent(qt, c[a:b], wl.scale) for a, b in [(0, 77), (77, 128), (128, 200)]]
    M = max(p[2] for p in parts)
    w = np.array([math.exp(p[2] - M) for p in parts])
    merged = sum(wi * p[0] for wi, p in zip(w, parts)) / w.sum()
    np.testing.assert_allclose(merged, o_all, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(M + math.log(w.sum()), lse_all, rtol=1e-13)


# ----------------------------------------------------------------------------- negative controls

@pytest.mark.parametrize("prefix", [0, 1, 5, 63, 64, 65])
def test_gate_rejects_planted_mistakes(prefix):
    """At small L the parity gate must reject plausible kernel bugs (planted in a copy of
    the oracle on the CPU): wrong scale, window shifted by one, last 64-row block dropped."""
    Q = 6
    L = prefix + Q
    wl = tiny_workload("dense", 2, Q, [L, L], H=64, D=256, R=512, seed=21)
    good = oracle.reference(wl)
    got = np.concatenate([good[k]["out"] for k in sorted(good)])

    bad_scale = tiny_workload("dense", 2, Q, [L, L], H=64, D=256, R=512, seed=21)
    bad_scale.scale = 1.0 / math.sqrt(512)
    ref = oracle.reference(bad_scale)
    assert not gate(np.concatenate([ref[k]["out"] for k in sorted(ref)]), got)

    # window shifted by one: each query sees one position fewer (its own row hidden)
    shifted = tiny_workload("dense", 2, Q, [L - 1, L - 1], H=64, D=256, R=512, seed=21, Lmax=L)
    shifted.cache = wl.cache
    ref = oracle.reference(shifted)
    keys = [k for k in sorted(ref) if k[1] >= 1]
    a = np.concatenate([ref[(b, i - 1)]["out"] for (b, i) in keys])
    g = np.concatenate([good[(b, i)]["out"] for (b, i) in keys])
    assert not gate(a, g)

    if L > 64:
        dropped = tiny_workload("dense", 2, Q, [L, L], H=64, D=256, R=512, seed=21)
        dropped.cache = wl.cache.copy()
        for b in range(2):
            rows = dropped.cache[b, :64].copy()
            dropped.cache[b, :64] = rows[::-1]  # scramble: content of a block moved
        dropped.cache[:, 64:] = synth.normal_bf16(dropped.cache[:, 64:].shape, 99, 2)
        ref = oracle.reference(dropped)
        assert not gate(np.concatenate([ref[k]["out"] for k in sorted(ref)]), got)


def test_gate_rejects_foreign_page():
    lens = [130, 100]
    wl = tiny_workload("paged", 2, 1, lens, H=64, D=256, R=512, seed=22)
    good = oracle.reference(wl)
    bad = tiny_workload("paged", 2, 1, lens, H=64, D=256, R=512, seed=22)
    t = bad.page_table.copy()
    t[0, 1], t[1, 0] = wl.page_table[1, 0], wl.page_table[0, 1]  # swap a page between sequences
    bad.page_table = t
    ref = oracle.reference(bad)
    assert not gate(ref[(0, 0)]["out"], good[(0, 0)]["out"]) or not gate(ref[(1, 0)]["out"], good[(1, 0)]["out"])


# ----------------------------------------------------------------------------- generator

def test_generator_deterministic_and_sliceable():
    a = synth.normal_bf16((1000,), 0, 2)
    b = synth.normal_bf16((1000,), 0, 2)
    assert np.array_equal(a, b)
    c = synth.normal_bf16((300,), 0, 2, offset=501)
    assert np.array_equal(a[501:801], c)
    assert not np.array_equal(a, synth.normal_bf16((1000,), 1, 2))
    assert not np.array_equal(a, synth.normal_bf16((1000,), 0, 3))


def test_generator_distribution():
    x = synth.normal_f64(1 << 20, 0, 2)
    assert abs(x.mean()) < 5e-3 and abs(x.std() - 1.0) < 5e-3
    # fourth moment of a standard normal is 3
    assert abs((x ** 4).mean() - 3.0) < 0.05
    w = synth.normal_f64(1 << 18, 0, 3, std=1.0 / math.sqrt(512))
    assert abs(w.std() * math.sqrt(512) - 1.0) < 1e-2
    bits = synth.normal_bf16((4096,), 0, 2)
    assert np.array_equal(bits, synth.f64_to_bf16_bits(synth.normal_f64(4096, 0, 2)))


def test_generator_integers_and_layouts():
    lens = synth.ragged_lengths(64, 1024, 131072)
    assert lens.min() >= 1024 and lens.max() <= 131072 and len(set(lens.tolist())) > 50
    p = synth.permutation(1000, 0, 6)
    assert np.array_equal(np.sort(p), np.arange(1000)) and not np.array_equal(p, np.arange(1000))
    s = synth.sorted_sample(2048, 131072, 0, 0x1000)
    assert len(np.unique(s)) == 2048 and np.all(np.diff(s) > 0) and s.min() >= 0 and s.max() < 131072
    table, P = synth.page_layout(np.array([65, 64, 1]))
    assert P == 4
    used = table[table >= 0]
    assert np.array_equal(np.sort(used), np.arange(4))
    assert table.shape == (3, 2) and table[1, 1] == -1 and table[2, 1] == -1


def test_workload_shapes():
    wl = synth.make_workload("tiny_dense_decode")
    assert wl.q.shape == (1, 1, 64, 256) and wl.cache.shape == (1, 256, 512)
    assert wl.w_uk.shape == (64, 256, 512)
    wl = synth.make_workload("mtp_verify", with_data=False)
    assert wl.Q == 6 and int(wl.seq_lens[0]) == 32774 and wl.extra["cache_shape"] == (16, 32774, 512)
    wl = synth.make_workload("indexed_sparse_decode", with_data=False)
    assert wl.indices.shape == (32, 1, 2048) and int(wl.indices.max()) <= 131071
    wl = synth.make_workload("ragged_paged_decode", with_data=False)
    P = wl.extra["cache_shape"][0]
    assert P == sum((int(L) + 63) // 64 for L in wl.seq_lens)


def test_cache_rows_regeneration_matches_full_cache():
    wl = synth.make_workload(None, mode="paged", B=3, Q=1, seq_lens=[100, 200, 64])
    pos = np.array([0, 1, 63, 64, 65, 99])
    rows = synth.cache_rows(wl, 0, pos)
    assert np.array_equal(rows, oracle.logical_rows("paged", 0, pos, pool=wl.pool, page_table=wl.page_table))
    wl = synth.make_workload(None, mode="dense", B=2, Q=1, L=50)
    assert np.array_equal(synth.cache_rows(wl, 1, np.arange(50)), wl.cache[1])

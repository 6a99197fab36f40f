"""The Python binding refuses, before any pointer reaches the C ABI, tensors whose dtype,
layout or size would let a kernel address memory outside them (the kernels see only a
pointer and the sizes passed).  CPU tensors suffice: these checks run before the device
check, and a call that passes them all still stops at the device check here."""
import pytest
import torch

import mla_absorbed_latent_mtp_b200 as m

B, Q, L = 2, 1, 130


@pytest.fixture(scope="module", autouse=True)
def built():
    import __graft_entry__
    __graft_entry__.build()  # the workspace-size query goes through the library


def bf(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def i32(*shape):
    return torch.zeros(*shape, dtype=torch.int32)


def _refused(fn, *args, match, **kw):
    with pytest.raises(ValueError, match=match):
        fn(*args, **kw)


def test_attend_dense_refusals():
    qt, cache, lens = bf(B, Q, 64, 512), bf(B, L, 512), i32(B)
    _refused(m.mla_attend_dense, qt.float(), cache, lens, match="q_tilde must be")
    _refused(m.mla_attend_dense, bf(B, Q, 64, 256), cache, lens, match="q_tilde must have shape")
    _refused(m.mla_attend_dense, qt, cache.float(), lens, match="cache must be")
    _refused(m.mla_attend_dense, qt, bf(B, L, 256), lens, match="cache must have shape")
    _refused(m.mla_attend_dense, qt, bf(1, L, 512), lens, match="cache holds 1 sequences")
    _refused(m.mla_attend_dense, qt, bf(B, 512, L).transpose(1, 2), lens, match="cache must be contiguous")
    _refused(m.mla_attend_dense, qt, cache, i32(1), match="seq_lens needs at least 2")
    _refused(m.mla_attend_dense, qt, cache, lens.long(), match="seq_lens must be")
    _refused(m.mla_attend_dense, qt, cache, lens, o_latent=bf(B, Q, 64, 256), match="o_latent must have shape")
    _refused(m.mla_attend_dense, qt, cache, lens, lse=torch.zeros(B, Q, 64, dtype=torch.float64), match="lse must be")
    _refused(m.mla_attend_dense, qt, cache, lens, status=torch.zeros(1, dtype=torch.int64), match="status must be")
    _refused(m.mla_attend_dense, qt, cache, lens, workspace=torch.zeros(16, dtype=torch.uint8),
             match="workspace needs at least")
    _refused(m.mla_attend_dense, qt, cache, lens, match="CUDA tensors")  # everything else is right


def test_attend_noalloc_refusals():
    qt, cache = bf(B, Q, 64, 512), bf(B, L, 512)
    _refused(m.mla_attend_dense_noalloc, qt, bf(1, L, 512), match="cache holds 1 sequences")
    _refused(m.mla_attend_dense_noalloc, qt, cache, i32(1), match="seq_lens needs at least")
    _refused(m.mla_attend_dense_noalloc, qt, cache, match="CUDA tensors")


def test_attend_paged_refusals():
    qt, pool, table, lens = bf(B, Q, 64, 512), bf(5, 64, 512), i32(B, 3), i32(B)
    _refused(m.mla_attend_paged, qt, bf(5, 32, 512), table, lens, match="pool must have shape")
    _refused(m.mla_attend_paged, qt, pool, i32(1, 3), lens, match="page_table has 1 rows")
    _refused(m.mla_attend_paged, qt, pool, table.long(), lens, match="page_table must be")
    _refused(m.mla_attend_paged, qt, pool, i32(3, B).t(), lens, match="page_table must be contiguous")
    _refused(m.mla_attend_paged, qt, pool, table, None, match="seq_lens is required")
    _refused(m.mla_attend_paged, qt, pool, table, lens, match="CUDA tensors")


def test_attend_indexed_refusals():
    qt, cache, idx = bf(B, Q, 64, 512), bf(B, L, 512), i32(B, Q, 16)
    _refused(m.mla_attend_indexed, qt, cache, i32(B, Q + 1, 16), match="indices must have shape")
    _refused(m.mla_attend_indexed, qt, cache, idx.long(), match="indices must be")
    _refused(m.mla_attend_indexed, qt, bf(1, L, 512), idx, match="cache holds 1 sequences")
    _refused(m.mla_attend_indexed, qt, cache, idx, match="CUDA tensors")


def test_projection_refusals():
    q, w = bf(3, 64, 256), bf(64, 256, 512)
    _refused(m.mla_absorb_q, q, bf(64, 512, 256), match="w_uk must have shape")
    _refused(m.mla_absorb_q, bf(3, 64, 512), w, match="q must be")
    _refused(m.mla_absorb_q, q.float(), w, match="q must be")
    _refused(m.mla_absorb_q, q, w, bf(3, 64, 256), match="q_tilde must have shape")
    _refused(m.mla_absorb_q, bf(3, 256, 64).transpose(1, 2), w, match="q must be contiguous")
    _refused(m.mla_absorb_q, q, w, match="CUDA tensors")
    o = bf(3, 64, 512)
    _refused(m.mla_up_proj, o, bf(64, 512, 256), match="w_uv must have shape")
    _refused(m.mla_up_proj, bf(3, 64, 256), w, match="o_latent must be")
    _refused(m.mla_up_proj, o, w, bf(3, 64, 512), match="out must have shape")
    _refused(m.mla_up_proj, o, w, match="CUDA tensors")


def test_cache_and_kpool_refusals():
    cache, lens, rows = bf(B, L, 512), i32(B), bf(B, 6, 512)
    _refused(m.mla_cache_append_dense, bf(1, L, 512), lens, rows, match="cache holds 1 sequences")
    _refused(m.mla_cache_append_dense, cache, i32(1), rows, match="seq_lens needs at least")
    _refused(m.mla_cache_append_dense, cache, lens, bf(B, 6, 256), match="rows must have shape")
    _refused(m.mla_cache_append_paged, bf(5, 64, 512), i32(1, 3), lens, rows, match="page_table has 1 rows")
    _refused(m.mla_cache_truncate_dense, cache, lens, i32(1), 6, match="keep needs at least")
    _refused(m.mla_cache_truncate_paged, bf(5, 64, 512), i32(1, 3), lens, i32(B), 6, match="page_table has 1 rows")
    _refused(m.mla_kpool_keys, cache, 64, pooled=torch.zeros(B, 1, 512), match="pooled must have shape")
    _refused(m.mla_kpool_select, torch.zeros(B, 2, 512), bf(B, 1, 512), 64, 128, Lmax=L * 4,
             match="pooled holds 2 pools")
    _refused(m.mla_kpool_select, torch.zeros(B, 2, 512), bf(B, 1, 256), 64, 128, match="w_query must have shape")
    _refused(m.mla_debug_gather, m.MODE_PAGED, bf(5, 64, 512), i32(4, 3), page_table=None, B=B,
             match="page_table is required")
    _refused(m.mla_debug_gather, m.MODE_DENSE, cache, i32(4, 2), B=B, match="req must have shape")

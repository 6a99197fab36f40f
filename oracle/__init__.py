"""fp64 CPU oracle for absorbed Multi-head Latent Attention (decode and MTP verify).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use it.  It shares no code with the CUDA library; the only
thing both sides share is the seeded input generator (package ``synth``).

What it computes is the plain definition of attention over a latent cache,
in the *expanded* (non-absorbed) form, from the page "Module 05 -- MLA:
Compressing Per-Token History" (jared-hpc.com, GLM-5.3-Flash Architecture
Mastery, Lecture-05):

* section 1: each cached token keeps one shared latent c_j (width 512); per
  head the key and value are reconstructed as k_{j,h} = U_h^K c_j and
  v_{j,h} = U_h^V c_j with U_h in R^{256 x 512} (64 heads, NoPE);
* section 3: scores are q_h . k_{j,h} at the *original* temperature
  (scale 1/sqrt(256) = 1/16), softmax over the visible positions, output
  sum_j a_j v_{j,h};
* section 4: causal masking, a query at position t sees j <= t;
* the MTP page (dimsnsums.com, GLM-5.3-Flash MTP): the target scores every
  proposed position of the draft run in one pass, so a verify step has
  q_len = 1 + 5 queries at consecutive positions.

The absorbed form (section 3's identities q~_h = (U_h^K)^T q_h and
out = U_h^V sum_j a_j c_j) is implemented separately as a cross-check.

Every computation is float64 on bfloat16 inputs widened exactly.  Matrix
products use numpy (a library primitive); there is no blocking, splitting or
reordering beyond the definitions.  Pins (tests/test_oracle.py) tie both forms
to brute force, closed forms, a library attention routine and the page's own
memory arithmetic.
"""
from __future__ import annotations

import math

import numpy as np

# Module 05, section 1 and "Current as of": latent width, heads, head dim.
LATENT_WIDTH = 512
NUM_HEADS = 64
HEAD_DIM = 256
BYTES_BF16 = 2
# Module 05, section 3 ("the one thing this algebra must never change"): the
# scale is the original q.k temperature, 1/sqrt(head_dim).
SCALE = 1.0 / math.sqrt(HEAD_DIM)
# MTP page: the serving recipe runs five speculative tokens -> q_len = 6.
MTP_DRAFT_TOKENS = 5
PAGE_TOKENS = 64


# ----------------------------------------------------------------------------- memory arithmetic

def expanded_bytes_per_token(heads: int = NUM_HEADS, head_dim: int = HEAD_DIM) -> int:
    """Module 05, section 2: a fully expanded bf16 cache stores a key and a value per head."""
    return heads * 2 * head_dim * BYTES_BF16


def latent_bytes_per_token(latent: int = LATENT_WIDTH) -> int:
    """Module 05, section 2: the cached latent is one 512-wide bf16 vector."""
    return latent * BYTES_BF16


# ----------------------------------------------------------------------------- bits

def widen(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> exact float64 values."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------- visibility

def visible_positions(L_b: int, q_len: int, i: int) -> np.ndarray:
    """Module 05 section 4 (j <= t) with the MTP window: the cache of length L_b already
    holds the q_len new rows, so query i sits at t = L_b - q_len + i and sees 0..t."""
    t = L_b - q_len + i
    return np.arange(0, max(t + 1, 0), dtype=np.int64)


def logical_rows(mode: str, b: int, positions: np.ndarray, *, cache=None, pool=None, page_table=None) -> np.ndarray:
    """Latent rows (bits) of sequence b at logical positions, materialised plainly.

    dense/indexed: cache[b, j]; paged: pool[page_table[b, j // 64], j % 64]."""
    positions = np.asarray(positions, dtype=np.int64)
    if mode == "paged":
        pages = page_table[b, positions // PAGE_TOKENS]
        if np.any(pages < 0):
            raise ValueError("position maps to an unused page-table slot")
        return pool[pages, positions % PAGE_TOKENS]
    return cache[b, positions]


# ----------------------------------------------------------------------------- expanded form

def expand_kv(c: np.ndarray, u_k: np.ndarray, u_v: np.ndarray):
    """Module 05 section 1: k_j = U^K c_j, v_j = U^V c_j for every row c_j of c.

    c: [n, R] float64; u_k, u_v: [D, R] float64 -> k, v: [n, D]."""
    return c @ u_k.T, c @ u_v.T


def attend_expanded(q_h: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """Ordinary softmax attention of one query head over expanded keys/values.

    Returns (out [D], weights [n], lse).  An empty visible set gives out = 0,
    lse = -inf (no position to attend to)."""
    n = k.shape[0]
    if n == 0:
        return np.zeros(v.shape[1]), np.zeros(0), -np.inf
    s = scale * (k @ q_h)
    m = s.max()
    e = np.exp(s - m)
    z = e.sum()
    a = e / z
    return a @ v, a, m + math.log(z)


# ----------------------------------------------------------------------------- absorbed form

def absorb_query(q_h: np.ndarray, u_k: np.ndarray) -> np.ndarray:
    """Module 05 section 3: q~_h = (U_h^K)^T q_h, computed once per query and head."""
    return u_k.T @ q_h


def attend_latent(qt_h: np.ndarray, c: np.ndarray, scale: float):
    """Module 05 section 3: scores q~_h . c_j (same scale), softmax, and the weighted sum
    kept in latent space.  Returns (o [R], weights [n], lse)."""
    n = c.shape[0]
    if n == 0:
        return np.zeros(c.shape[1]), np.zeros(0), -np.inf
    s = scale * (c @ qt_h)
    m = s.max()
    e = np.exp(s - m)
    z = e.sum()
    a = e / z
    return a @ c, a, m + math.log(z)


def up_project(o: np.ndarray, u_v: np.ndarray) -> np.ndarray:
    """Module 05 section 3: the latent-space sum is expanded once, out = U_h^V o."""
    return u_v @ o


# ----------------------------------------------------------------------------- whole problem

def _visible(wl, b: int, i: int) -> np.ndarray:
    if wl.mode == "indexed":
        lst = np.asarray(wl.indices[b, i], dtype=np.int64)
        return lst[lst != -1]  # -1 marks an unused entry of a fixed-width list
    return visible_positions(int(wl.seq_lens[b]), wl.Q, i)


def _rows(wl, b: int, positions: np.ndarray, row_source=None) -> np.ndarray:
    if row_source is not None:
        return row_source(b, positions)
    return logical_rows(wl.mode, b, positions, cache=wl.cache, pool=wl.pool, page_table=wl.page_table)


def reference(wl, pairs=None, heads=None, form: str = "expanded", row_source=None, return_latent: bool = False):
    """Attention output of workload ``wl`` (a ``synth.Workload``) in float64.

    pairs: iterable of (b, i) to compute (default: all); heads: head indices
    (default: all).  form: "expanded" (the definition) or "absorbed" (the
    identity).  row_source(b, positions) -> bits may replace the in-memory
    cache (for full-size workloads regenerated row by row).

    Returns dict (b, i) -> dict with "out" [len(heads), D] and "lse" [len(heads)],
    plus "o_latent" [len(heads), R] for the absorbed form when return_latent."""
    heads = list(range(wl.q.shape[2])) if heads is None else list(heads)
    if pairs is None:
        pairs = [(b, i) for b in range(wl.B) for i in range(wl.Q)]
    pairs = list(pairs)
    u_k_all = widen(wl.w_uk)
    u_v_all = widen(wl.w_uv)
    result = {}
    by_b = {}
    for (b, i) in pairs:
        by_b.setdefault(b, []).append(i)
    for b, qs in by_b.items():
        vis = {i: _visible(wl, b, i) for i in qs}
        if wl.mode == "indexed":
            union = np.unique(np.concatenate([vis[i] for i in qs])) if qs else np.zeros(0, np.int64)
        else:
            union = vis[max(qs, key=lambda i: len(vis[i]))]
        c_all = widen(_rows(wl, b, union, row_source)) if len(union) else np.zeros((0, u_k_all.shape[2]))
        pos_to_row = {int(p): r for r, p in enumerate(union)}
        for i in qs:
            result[(b, i)] = {"out": np.zeros((len(heads), u_v_all.shape[1])), "lse": np.zeros(len(heads))}
            if return_latent:
                result[(b, i)]["o_latent"] = np.zeros((len(heads), u_k_all.shape[2]))
        for hh, h in enumerate(heads):
            u_k, u_v = u_k_all[h], u_v_all[h]
            if form == "expanded":
                k_all, v_all = expand_kv(c_all, u_k, u_v)
            for i in qs:
                sel = np.array([pos_to_row[int(p)] for p in vis[i]], dtype=np.int64)
                q_h = widen(wl.q[b, i, h])
                if form == "expanded":
                    out, a, lse = attend_expanded(q_h, k_all[sel], v_all[sel], wl.scale)
                else:
                    o, a, lse = attend_latent(absorb_query(q_h, u_k), c_all[sel], wl.scale)
                    out = up_project(o, u_v)
                    if return_latent:
                        result[(b, i)]["o_latent"][hh] = o
                if len(a):
                    assert abs(a.sum() - 1.0) < 1e-12, "softmax weights must sum to 1"
                result[(b, i)]["out"][hh] = out
                result[(b, i)]["lse"][hh] = lse
    return result


def reference_latent(qt_bits: np.ndarray, wl, pairs=None, heads=None, row_source=None):
    """Latent-space attention for given q~ bits [B, Q, H, R] (the input of the attend stage):
    returns dict (b, i) -> {"o_latent": [len(heads), R], "lse": [len(heads)]}."""
    heads = list(range(qt_bits.shape[2])) if heads is None else list(heads)
    if pairs is None:
        pairs = [(b, i) for b in range(wl.B) for i in range(wl.Q)]
    res = {}
    for (b, i) in pairs:
        vis = _visible(wl, b, i)
        c = widen(_rows(wl, b, vis, row_source)) if len(vis) else np.zeros((0, qt_bits.shape[3]))
        o_all = np.zeros((len(heads), qt_bits.shape[3]))
        lse_all = np.zeros(len(heads))
        for hh, h in enumerate(heads):
            o, a, lse = attend_latent(widen(qt_bits[b, i, h]), c, wl.scale)
            if len(a):
                assert abs(a.sum() - 1.0) < 1e-12
            o_all[hh] = o
            lse_all[hh] = lse
        res[(b, i)] = {"o_latent": o_all, "lse": lse_all}
    return res


def absorb_all(q_bits: np.ndarray, w_uk_bits: np.ndarray) -> np.ndarray:
    """q~[n, h, :] = (U_h^K)^T q[n, h, :] for q bits [n, H, D] -> float64 [n, H, R]."""
    q = widen(q_bits)
    u = widen(w_uk_bits)
    out = np.empty((q.shape[0], q.shape[1], u.shape[2]))
    for h in range(q.shape[1]):
        out[:, h, :] = q[:, h, :] @ u[h]
    return out


def up_project_all(o_bits: np.ndarray, w_uv_bits: np.ndarray) -> np.ndarray:
    """out[n, h, :] = U_h^V o[n, h, :] for o bits [n, H, R] -> float64 [n, H, D]."""
    o = widen(o_bits)
    u = widen(w_uv_bits)
    out = np.empty((o.shape[0], o.shape[1], u.shape[1]))
    for h in range(o.shape[1]):
        out[:, h, :] = o[:, h, :] @ u[h].T
    return out


# ----------------------------------------------------------------------------- speculative-decoding cache bookkeeping
# "Module 08 -- Vision, MTP, and Hybrid Serving State" (jared-hpc.com, GLM-5.3-Flash
# Architecture Mastery, Lecture-08), section 3: the MLA latent cache is indexed by token
# position, so after a verify step it is rolled back by truncating it to the accepted
# prefix, and the state after rollback must equal the state of a run that never produced
# the rejected tokens.  The MTP page (dimsnsums.com, GLM-5.3-Flash MTP): a verify step
# appends the q_len = 1 + 5 rows it scores.  These are plain array assignments on bits.

def _slot(mode: str, b: int, j: int, page_table):
    """(array index) of logical position j of sequence b: cache[b, j] or pool[page, j % 64]."""
    if mode == "paged":
        page = int(page_table[b, j // PAGE_TOKENS])
        if page < 0:
            raise ValueError("position maps to an unused page-table slot")
        return (page, j % PAGE_TOKENS)
    return (b, j)


def cache_append(mode: str, store: np.ndarray, seq_lens: np.ndarray, rows: np.ndarray, page_table=None):
    """Append rows[b, i] (bits, [B, q_len, R]) at positions seq_lens[b] + i.

    Returns new (store, seq_lens); the inputs are not modified."""
    store = np.array(store, copy=True)
    lens = np.array(seq_lens, dtype=np.int64, copy=True)
    B, q_len = rows.shape[0], rows.shape[1]
    for b in range(B):
        for i in range(q_len):
            store[_slot(mode, b, int(lens[b]) + i, page_table)] = rows[b, i]
        lens[b] += q_len
    return store, lens.astype(np.int32)


def cache_truncate(mode: str, store: np.ndarray, seq_lens: np.ndarray, keep: np.ndarray, q_len: int,
                   page_table=None):
    """Roll back a verify window: sequence b keeps the first keep[b] of its last q_len rows.

    The new length is seq_lens[b] - q_len + keep[b]; the discarded rows are zeroed, so a
    store whose unused rows are zero ends up identical to one that never held them."""
    store = np.array(store, copy=True)
    lens = np.array(seq_lens, dtype=np.int64, copy=True)
    for b in range(len(lens)):
        new_len = int(lens[b]) - q_len + int(keep[b])
        for j in range(new_len, int(lens[b])):
            store[_slot(mode, b, j, page_table)] = 0
        lens[b] = new_len
    return store, lens.astype(np.int32)


# ----------------------------------------------------------------------------- k-pool index producer
# "GLM-5.3-Flash engine (c/glm53.c)" (colibri docs, raw.githubusercontent.com/JustVugg/colibri),
# section "Architecture notes", DSA with k-pooling: keys are grouped into pools of
# `pool` consecutive positions; the pooled key is a per-channel softmax mixture of the
# members (not their average); a pool is selectable only if it is complete and causally
# visible; the incomplete tail is appended when asked for (a row topk + pool - 1 wide);
# ties go to the lower index.  The pages give no indexer projections, so the key of a
# position is its cached latent and the indexer query is an input vector w.

def kpool_pooled_keys(rows_bits: np.ndarray, pool: int) -> np.ndarray:
    """Pooled key of every complete pool of consecutive rows ([n, R] bits -> [n // pool, R]):
    per channel d, sum_j softmax_j(x_jd) * x_jd over the pool's members j."""
    x = widen(rows_bits)
    n_pools = x.shape[0] // pool
    x = x[: n_pools * pool].reshape(n_pools, pool, x.shape[1])
    e = np.exp(x - x.max(axis=1, keepdims=True))
    return (e * x).sum(axis=1) / e.sum(axis=1)


def kpool_select(pooled: np.ndarray, w: np.ndarray, pos: int, pool: int, topk: int, with_tail: bool) -> np.ndarray:
    """Index list of the query at position `pos`: the topk // pool best complete pools that end
    at or before pos (score = pooled . w, ties to the lower pool), their positions in
    ascending order, then -1 up to topk; with_tail appends the positions of the incomplete
    pool up to pos, then -1 up to topk + pool - 1."""
    n_sel = max(pos + 1, 0) // pool
    scores = pooled[:n_sel] @ np.asarray(w, dtype=np.float64)
    order = sorted(range(n_sel), key=lambda p: (-scores[p], p))
    chosen = sorted(order[: topk // pool])
    out = [p * pool + j for p in chosen for j in range(pool)]
    out += [-1] * (topk - len(out))
    if with_tail:
        tail = list(range(n_sel * pool, pos + 1))
        out += tail + [-1] * (pool - 1 - len(tail))
    return np.asarray(out, dtype=np.int32)

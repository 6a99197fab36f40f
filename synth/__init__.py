"""Seeded synthetic inputs for absorbed-MLA latent-cache attention.

This module draws numbers and lays them out; it contains no attention
arithmetic.  Both the GPU path's tests/benchmark and the CPU oracle consume the
same bfloat16 bit patterns produced here, so neither side depends on a library
version's random-number stream.

Workloads (all dimensions from "Module 05 -- MLA: Compressing Per-Token
History", section 1: 64 heads, 256-dim NoPE heads, 512-wide latent):

* ``tiny_dense_decode``     B=1,  q_len=1, L=256
* ``dense_decode``          B=32, q_len=1, L=8192, contiguous cache [B, L, 512]
* ``mtp_verify``            B=16, q_len=6 (1 + 5 drafts), prefix 32768; the six
                            new latents are appended, so each cache holds 32774
                            rows and query i sits at position 32768 + i
* ``ragged_paged_decode``   B=64, q_len=1, lengths uniform in [1024, 131072],
                            64-token pages of one pool in a shuffled page table
* ``indexed_sparse_decode`` B=32, q_len=1, L=131072, 2048 sorted distinct
                            positions per query drawn from [0, L-1]

Distributions: q and cache ~ N(0, 1); W_UK and W_UV ~ N(0, 1/512) per head,
shape [64, 256, 512] each; seed 0; scale 1/16.  Draws are made in double,
rounded to float32 then to bfloat16 (round to nearest even).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")

H, D, R = 64, 256, 512
PAGE = 64
SCALE = 1.0 / 16.0

# one fixed stream id per tensor
STREAM_Q, STREAM_CACHE, STREAM_WUK, STREAM_WUV, STREAM_LENS, STREAM_PAGES = 1, 2, 3, 4, 5, 6
STREAM_INDEX_BASE = 0x1000
STREAM_QTILDE, STREAM_OLAT = 7, 8


def build_lib(force: bool = False) -> str:
    """Compile the generator library next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build_lib())
        i64, u64, vp = ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p
        L.synth_normal_bf16.argtypes = [vp, i64, u64, u64, ctypes.c_double, i64]
        L.synth_normal_f64.argtypes = [vp, i64, u64, u64, ctypes.c_double, i64]
        L.synth_uniform_int.argtypes = [vp, i64, u64, u64, i64, i64, i64]
        L.synth_permutation.argtypes = [vp, i64, u64, u64]
        L.synth_sorted_sample.argtypes = [vp, i64, i64, u64, u64, vp]
        L.synth_sorted_sample.restype = ctypes.c_int
        L.synth_words.argtypes = [vp, i64, u64, u64, i64]
        for f in (L.synth_normal_bf16, L.synth_normal_f64, L.synth_uniform_int, L.synth_permutation, L.synth_words):
            f.restype = None
        _lib = L
    return _lib


# ----------------------------------------------------------------------------- primitives

def normal_bf16(shape, seed: int, stream: int, std: float = 1.0, offset: int = 0) -> np.ndarray:
    """bfloat16 bits (uint16) of std * N(0,1) draws, elements offset .. offset+size-1."""
    out = np.empty(shape, dtype=np.uint16)
    lib().synth_normal_bf16(out.ctypes.data, out.size, seed, stream, std, offset)
    return out


def normal_bf16_into(ptr: int, n: int, seed: int, stream: int, std: float = 1.0, offset: int = 0) -> None:
    """Fill n uint16 slots at host address ptr (e.g. a pinned buffer)."""
    lib().synth_normal_bf16(ptr, n, seed, stream, std, offset)


def normal_f64(n: int, seed: int, stream: int, std: float = 1.0, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    lib().synth_normal_f64(out.ctypes.data, n, seed, stream, std, offset)
    return out


def uniform_int(n: int, seed: int, stream: int, lo: int, hi: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.int64)
    lib().synth_uniform_int(out.ctypes.data, n, seed, stream, lo, hi, offset)
    return out


def permutation(n: int, seed: int, stream: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    lib().synth_permutation(out.ctypes.data, n, seed, stream)
    return out


def sorted_sample(k: int, rng: int, seed: int, stream: int) -> np.ndarray:
    out = np.empty(k, dtype=np.int32)
    scratch = np.empty(max(rng, 1), dtype=np.int32)
    if lib().synth_sorted_sample(out.ctypes.data, k, rng, seed, stream, scratch.ctypes.data) != 0:
        raise ValueError("sample larger than range")
    return out


def words(n: int, seed: int, stream: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    lib().synth_words(out.ctypes.data, n, seed, stream, offset)
    return out


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round doubles to bfloat16 bits (via float32, nearest even), as the generator does."""
    f = np.ascontiguousarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------- workloads

@dataclass
class Workload:
    """One synthetic problem instance; every array holds raw bits or integers."""
    name: str
    mode: str                 # "dense" | "paged" | "indexed"
    B: int
    Q: int
    seq_lens: np.ndarray      # [B] int32, cache rows per sequence incl. appended query rows
    q: np.ndarray             # [B, Q, H, D] bf16 bits
    w_uk: np.ndarray          # [H, D, R] bf16 bits
    w_uv: np.ndarray          # [H, D, R] bf16 bits
    cache: np.ndarray | None = None       # dense/indexed: [B, Lmax, R] bf16 bits
    pool: np.ndarray | None = None        # paged: [P, PAGE, R] bf16 bits
    page_table: np.ndarray | None = None  # paged: [B, max_pages] int32, -1 = unused
    indices: np.ndarray | None = None     # indexed: [B, Q, K] int32 sorted distinct
    scale: float = SCALE
    extra: dict = field(default_factory=dict)

    @property
    def Lmax(self) -> int:
        return int(self.cache.shape[1]) if self.cache is not None else int(self.page_table.shape[1]) * PAGE


CONFIGS = {
    "tiny_dense_decode": dict(mode="dense", B=1, Q=1, L=256),
    "dense_decode": dict(mode="dense", B=32, Q=1, L=8192),
    "mtp_verify": dict(mode="dense", B=16, Q=6, L=32768 + 6),
    "ragged_paged_decode": dict(mode="paged", B=64, Q=1, Lmin=1024, Lhi=131072),
    "indexed_sparse_decode": dict(mode="indexed", B=32, Q=1, L=131072, K=2048),
}


def ragged_lengths(B: int, lo: int, hi: int, seed: int = 0) -> np.ndarray:
    return uniform_int(B, seed, STREAM_LENS, lo, hi).astype(np.int32)


def page_layout(seq_lens: np.ndarray, seed: int = 0, max_pages: int | None = None):
    """Page table over one pool holding exactly sum(ceil(L_b/64)) pages, shuffled."""
    npages = [(int(L) + PAGE - 1) // PAGE for L in seq_lens]
    P = int(sum(npages))
    perm = permutation(P, seed, STREAM_PAGES)
    mp = max_pages if max_pages is not None else max(max(npages), 1)
    table = np.full((len(seq_lens), mp), -1, dtype=np.int32)
    base = 0
    for b, n in enumerate(npages):
        table[b, :n] = perm[base:base + n]
        base += n
    return table, P


def index_lists(B: int, Q: int, K: int, seq_lens: np.ndarray, seed: int = 0) -> np.ndarray:
    """Per (b, i): K distinct sorted positions visible to query i (j <= L_b - Q + i)."""
    out = np.empty((B, Q, K), dtype=np.int32)
    for b in range(B):
        for i in range(Q):
            visible = int(seq_lens[b]) - Q + i + 1
            out[b, i] = sorted_sample(K, visible, seed, STREAM_INDEX_BASE + b * Q + i)
    return out


def make_workload(name: str | None = None, seed: int = 0, *, mode: str | None = None, B: int | None = None,
                  Q: int | None = None, L: int | None = None, seq_lens=None, K: int | None = None,
                  Lmax: int | None = None, with_data: bool = True) -> Workload:
    """Build a named workload (see CONFIGS) or a custom one from keyword sizes.

    ``seq_lens`` overrides per-sequence lengths; ``Lmax`` pads dense caches.
    With ``with_data=False`` the large cache/pool is left as None (the caller
    fills it, e.g. straight into pinned memory, with :func:`fill_cache`).
    """
    cfg = dict(CONFIGS[name]) if name is not None else {}
    mode = mode or cfg.get("mode", "dense")
    B = B if B is not None else cfg["B"]
    Q = Q if Q is not None else cfg.get("Q", 1)
    if seq_lens is not None:
        lens = np.asarray(seq_lens, dtype=np.int32).reshape(B)
    elif mode == "paged" and L is None and "Lmin" in cfg:
        lens = ragged_lengths(B, cfg["Lmin"], cfg["Lhi"], seed)
    else:
        Lc = L if L is not None else cfg["L"]
        lens = np.full(B, Lc, dtype=np.int32)
    q = normal_bf16((B, Q, H, D), seed, STREAM_Q)
    std_w = 1.0 / math.sqrt(512.0)
    w_uk = normal_bf16((H, D, R), seed, STREAM_WUK, std_w)
    w_uv = normal_bf16((H, D, R), seed, STREAM_WUV, std_w)
    wl = Workload(name or "custom", mode, B, Q, lens, q, w_uk, w_uv)
    if mode in ("dense", "indexed"):
        lm = Lmax if Lmax is not None else max(int(lens.max()), 1)
        wl.extra["cache_shape"] = (B, lm, R)
        if with_data:
            wl.cache = normal_bf16((B, lm, R), seed, STREAM_CACHE)
        if mode == "indexed":
            Kc = K if K is not None else cfg["K"]
            wl.indices = index_lists(B, Q, Kc, lens, seed)
    elif mode == "paged":
        table, P = page_layout(lens, seed)
        wl.page_table = table
        wl.extra["cache_shape"] = (P, PAGE, R)
        if with_data:
            wl.pool = normal_bf16((P, PAGE, R), seed, STREAM_CACHE)
    else:
        raise ValueError(mode)
    wl.extra["seed"] = seed
    return wl


def fill_cache(wl: Workload, ptr: int, chunk_elems: int = 1 << 26) -> None:
    """Write the workload's cache (dense/indexed) or pool (paged) bits to host address ptr."""
    n = int(np.prod(wl.extra["cache_shape"]))
    seed = wl.extra["seed"]
    for off in range(0, n, chunk_elems):
        m = min(chunk_elems, n - off)
        normal_bf16_into(ptr + 2 * off, m, seed, STREAM_CACHE, 1.0, off)


def cache_rows(wl: Workload, b: int, positions: np.ndarray) -> np.ndarray:
    """Bits of the latent rows of sequence b at the given logical positions, regenerated from
    the stream (no need for the whole cache in host memory): [len(positions), R] uint16."""
    seed = wl.extra["seed"]
    positions = np.asarray(positions, dtype=np.int64)
    out = np.empty((len(positions), R), dtype=np.uint16)
    if wl.mode == "paged":
        rows = wl.page_table[b, positions // PAGE].astype(np.int64) * PAGE + positions % PAGE
    else:
        rows = b * wl.extra["cache_shape"][1] + positions
    # group consecutive rows into runs to keep the number of calls small
    start = 0
    while start < len(rows):
        end = start + 1
        while end < len(rows) and rows[end] == rows[end - 1] + 1:
            end += 1
        n = end - start
        normal_bf16_into(out[start:end].ctypes.data, n * R, seed, STREAM_CACHE, 1.0, int(rows[start]) * R)
        start = end
    return out

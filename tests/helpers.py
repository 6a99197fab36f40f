"""Shared test utilities: the parity gate and small workload builders."""
import math

import numpy as np

import synth

# Tolerance stated for bf16 outputs with fp32 accumulation: max-abs <= 2e-2 and
# mean-abs <= 2e-3 against the unrounded fp64 oracle.
MAX_ABS_TOL = 2e-2
MEAN_ABS_TOL = 2e-3


def decode_bf16(u: int) -> float:
    """Value of one bfloat16 bit pattern, decoded field by field (IEEE 754 binary16-brain:
    1 sign bit, 8 exponent bits with bias 127, 7 fraction bits), independently of the
    oracle's array widening."""
    u = int(u) & 0xFFFF
    sign = -1.0 if u & 0x8000 else 1.0
    exp = (u >> 7) & 0xFF
    frac = u & 0x7F
    if exp == 0xFF:
        return sign * math.inf if frac == 0 else math.nan
    if exp == 0:  # zero or subnormal: frac * 2^-133
        return sign * math.ldexp(frac, -126 - 7)
    return sign * math.ldexp(128 + frac, exp - 127 - 7)


def decode_list(bits):
    """Flat list of Python floats for an array of bfloat16 bit patterns."""
    return [decode_bf16(x) for x in np.asarray(bits).ravel()]


def errors(got, ref):
    err = np.abs(np.asarray(got, dtype=np.float64) - np.asarray(ref, dtype=np.float64))
    return float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0


def gate(got, ref):
    mx, mean = errors(got, ref)
    return mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL


def tiny_workload(mode, B, Q, seq_lens, H, D, R, seed=0, K=None, page=64, Lmax=None, q_std=1.0, c_std=1.0):
    """A Workload with small head/latent dims (brute-force sized)."""
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    q = synth.normal_bf16((B, Q, H, D), seed, synth.STREAM_Q, q_std)
    std_w = 1.0 / math.sqrt(R)
    w_uk = synth.normal_bf16((H, D, R), seed, synth.STREAM_WUK, std_w)
    w_uv = synth.normal_bf16((H, D, R), seed, synth.STREAM_WUV, std_w)
    wl = synth.Workload("tiny", mode, B, Q, seq_lens, q, w_uk, w_uv)
    wl.extra["seed"] = seed
    if mode in ("dense", "indexed"):
        lm = Lmax if Lmax is not None else max(int(seq_lens.max()), 1)
        wl.cache = synth.normal_bf16((B, lm, R), seed, synth.STREAM_CACHE, c_std)
        wl.extra["cache_shape"] = wl.cache.shape
        if mode == "indexed":
            out = np.empty((B, Q, K), dtype=np.int32)
            for b in range(B):
                for i in range(Q):
                    out[b, i] = synth.sorted_sample(K, int(seq_lens[b]) - Q + i + 1, seed,
                                                    synth.STREAM_INDEX_BASE + b * Q + i)
            wl.indices = out
    else:
        npages = [(int(L) + page - 1) // page for L in seq_lens]
        P = sum(npages)
        perm = synth.permutation(P, seed, synth.STREAM_PAGES)
        table = np.full((B, max(max(npages), 1)), -1, dtype=np.int32)
        base = 0
        for b, n in enumerate(npages):
            table[b, :n] = perm[base:base + n]
            base += n
        wl.page_table = table
        wl.pool = synth.normal_bf16((P, page, R), seed, synth.STREAM_CACHE, c_std)
        wl.extra["cache_shape"] = wl.pool.shape
    return wl

"""Helpers for the GPU tests: moving generator bits to the device and back."""
import math

import numpy as np
import torch

import synth

QT_STD = math.sqrt(256.0 / 512.0)  # std of W_UK^T q when q ~ N(0,1), W_UK ~ N(0,1/512)


def to_dev(bits, dtype=torch.bfloat16):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    return t.view(dtype)


def ints_to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def bf16_to_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def bf16_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def synthetic_qtilde(B, Q, seed=0):
    """Absorbed queries drawn directly (stream of their own), with the spread W_UK^T q has."""
    return synth.normal_bf16((B, Q, 64, 512), seed, synth.STREAM_QTILDE, QT_STD)


def pinned_cache(wl):
    """The workload's cache/pool generated straight into pinned host memory (uint16 bits)."""
    shape = wl.extra["cache_shape"]
    host = torch.empty(shape, dtype=torch.int16, pin_memory=True)
    synth.fill_cache(wl, host.data_ptr())
    return host

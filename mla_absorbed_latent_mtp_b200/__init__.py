"""Python binding of the B200 absorbed-MLA latent attention library (include/mla.h).

Argument marshalling only: every step runs in the CUDA kernels of libmla_b200.so.
Tensors are torch CUDA tensors (bf16 as torch.bfloat16, int32 as torch.int32); the
functions pass their device pointers and the current CUDA stream to the C ABI and
raise MLAError on a non-zero status.  There is no CPU fallback: if the library is
not built, importing the binding's functions raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla_b200.so")

MLA_OK, MLA_ERR_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_CUDA, MLA_ERR_WORKSPACE, MLA_ERR_INDEX, MLA_ERR_TIMEOUT = range(7)
MODE_DENSE, MODE_PAGED, MODE_INDEXED = 0, 1, 2
H, D, R, PAGE = 64, 256, 512, 64
SCALE = 1.0 / 16.0

EXPORTS = ("mla_status_string", "mla_last_error_string", "mla_absorb_q", "mla_attend_dense", "mla_attend_paged", "mla_attend_indexed",
           "mla_up_proj", "mla_attend_workspace_bytes", "mla_debug_gather", "mla_attend_dense_noalloc",
           "mla_cache_append_dense", "mla_cache_append_paged", "mla_cache_truncate_dense", "mla_cache_truncate_paged",
           "mla_debug_wait_timeout", "mla_kpool_keys", "mla_kpool_select", "mla_attend_up_dense",
           "mla_attend_up_paged", "mla_attend_up_indexed", "mla_expand_kv", "mla_prefill_expanded")


class MLAError(RuntimeError):
    def __init__(self, fn, code):
        detail = f": {lib().mla_last_error_string().decode()}" if code == MLA_ERR_CUDA else ""
        super().__init__(f"{fn} failed: {status_string(code)} ({code}){detail}")
        self.code = code


_lib = None


def lib():
    """The loaded shared library (ctypes), with argument types declared."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run: python -c 'import __graft_entry__ as g; g.build()'")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    L.mla_status_string.argtypes = [ctypes.c_int32]
    L.mla_status_string.restype = ctypes.c_char_p
    L.mla_last_error_string.argtypes = []
    L.mla_last_error_string.restype = ctypes.c_char_p
    L.mla_absorb_q.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp]
    L.mla_up_proj.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp]
    L.mla_attend_dense.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, sz, vp, vp, vp, vp]
    L.mla_attend_paged.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32, vp, sz, vp, vp, vp, vp]
    L.mla_attend_indexed.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp, sz, vp, vp, vp, vp]
    L.mla_attend_workspace_bytes.argtypes = [i32, i32, i32, i32]
    L.mla_attend_workspace_bytes.restype = sz
    L.mla_debug_gather.argtypes = [i32, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, i32, vp, vp, vp]
    L.mla_attend_dense_noalloc.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, vp, vp, vp]
    L.mla_cache_append_dense.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp]
    L.mla_cache_truncate_dense.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp]
    L.mla_cache_append_paged.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp]
    L.mla_cache_truncate_paged.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp]
    L.mla_kpool_keys.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp]
    L.mla_kpool_keys.restype = ctypes.c_int32
    L.mla_kpool_select.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, i32, vp]
    L.mla_kpool_select.restype = ctypes.c_int32
    L.mla_attend_up_dense.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, i32, vp, sz, vp, vp, vp, vp, vp]
    L.mla_attend_up_paged.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32, vp, i32, vp, sz, vp, vp,
                                      vp, vp, vp]
    L.mla_attend_up_indexed.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp, i32, vp, sz, vp, vp, vp,
                                        vp, vp]
    L.mla_expand_kv.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp]
    L.mla_prefill_expanded.argtypes = [vp, vp, vp, i32, i32, i32, i32, f32, vp, vp, vp, vp]
    L.mla_debug_wait_timeout.argtypes = [ctypes.c_longlong, vp, vp]
    L.mla_debug_wait_timeout.restype = ctypes.c_int32
    for name in ("mla_absorb_q", "mla_up_proj", "mla_attend_dense", "mla_attend_paged", "mla_attend_indexed",
                 "mla_debug_gather", "mla_attend_dense_noalloc", "mla_cache_append_dense", "mla_cache_append_paged",
                 "mla_cache_truncate_dense", "mla_cache_truncate_paged", "mla_attend_up_dense", "mla_attend_up_paged",
                 "mla_attend_up_indexed", "mla_expand_kv", "mla_prefill_expanded"):
        getattr(L, name).restype = ctypes.c_int32
    _lib = L
    return L


def status_string(code: int) -> str:
    return lib().mla_status_string(code).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, code):
    if code != MLA_OK:
        raise MLAError(fn, code)


def _check_cuda(*tensors):
    dev = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensors must be on one device ({dev} and {t.device})")


def _require(t, name, dtype, shape=None, min_numel=None, optional=False):
    """Refuse, before any pointer reaches the C ABI, a tensor whose dtype, layout or size
    would let a kernel read or write outside it: the kernels address memory only from the
    pointer and the sizes passed, so a strided, narrower or smaller tensor must never get
    that far.  ``shape`` may hold None for a free dimension."""
    import torch
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    want = {"bf16": torch.bfloat16, "i32": torch.int32, "f32": torch.float32, "u8": torch.uint8}[dtype]
    if t.dtype != want:
        raise ValueError(f"{name} must be {want}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None:
        if t.dim() != len(shape) or any(w is not None and int(g) != int(w) for g, w in zip(t.shape, shape)):
            raise ValueError(f"{name} must have shape {tuple('*' if w is None else w for w in shape)}, "
                             f"got {tuple(t.shape)}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name} needs at least {min_numel} elements, got {t.numel()}")


# ----------------------------------------------------------------------------- entry points

def mla_attend_workspace_bytes(B: int, Q: int, heads: int = H, latent: int = R) -> int:
    return int(lib().mla_attend_workspace_bytes(B, Q, heads, latent))


def new_workspace(B: int, Q: int):
    """Allocate (with torch) the workspace the attend calls need."""
    import torch
    n = mla_attend_workspace_bytes(B, Q)
    return torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")


def mla_absorb_q(q, w_uk, q_tilde=None, stream=None):
    """q [n, H, D] or [B, Q, H, D] bf16, w_uk [H, D, R] bf16 -> q_tilde [..., H, R] bf16."""
    import torch
    _require(q, "q", "bf16")
    if q.dim() < 3 or tuple(q.shape[-2:]) != (H, D):
        raise ValueError(f"q must be [..., {H}, {D}], got {tuple(q.shape)}")
    _require(w_uk, "w_uk", "bf16", (H, D, R))
    n = q.numel() // (H * D)
    _require(q_tilde, "q_tilde", "bf16", tuple(q.shape[:-1]) + (R,), optional=True)
    _check_cuda(q, w_uk, q_tilde)
    if q_tilde is None:
        q_tilde = torch.empty(*q.shape[:-1], R, dtype=torch.bfloat16, device=q.device)
    _check("mla_absorb_q", lib().mla_absorb_q(_ptr(q), _ptr(w_uk), _ptr(q_tilde), n, H, D, R, _stream(stream)))
    return q_tilde


def mla_up_proj(o_latent, w_uv, out=None, stream=None):
    """o_latent [..., H, R] bf16, w_uv [H, D, R] bf16 -> out [..., H, D] bf16."""
    import torch
    _require(o_latent, "o_latent", "bf16")
    if o_latent.dim() < 3 or tuple(o_latent.shape[-2:]) != (H, R):
        raise ValueError(f"o_latent must be [..., {H}, {R}], got {tuple(o_latent.shape)}")
    _require(w_uv, "w_uv", "bf16", (H, D, R))
    n = o_latent.numel() // (H * R)
    _require(out, "out", "bf16", tuple(o_latent.shape[:-1]) + (D,), optional=True)
    _check_cuda(o_latent, w_uv, out)
    if out is None:
        out = torch.empty(*o_latent.shape[:-1], D, dtype=torch.bfloat16, device=o_latent.device)
    _check("mla_up_proj", lib().mla_up_proj(_ptr(o_latent), _ptr(w_uv), _ptr(out), n, H, D, R, _stream(stream)))
    return out


def _check_attend(q_tilde, workspace, o_latent, lse, status, seq_lens, seq_lens_required=False):
    """Common checks of the attend calls; returns (B, Q)."""
    _require(q_tilde, "q_tilde", "bf16", (None, None, H, R))
    B, Q = int(q_tilde.shape[0]), int(q_tilde.shape[1])
    _require(seq_lens, "seq_lens", "i32", min_numel=B, optional=not seq_lens_required)
    if workspace is not None:
        _require(workspace, "workspace", "u8", min_numel=mla_attend_workspace_bytes(B, Q))
    _require(o_latent, "o_latent", "bf16", (B, Q, H, R), optional=True)
    _require(lse, "lse", "f32", (B, Q, H), optional=True)
    _require(status, "status", "i32", min_numel=1, optional=True)
    return B, Q


def _attend_outputs(q_tilde, o_latent, lse, want_lse):
    import torch
    B, Q = q_tilde.shape[0], q_tilde.shape[1]
    if o_latent is None:
        o_latent = torch.empty(B, Q, H, R, dtype=torch.bfloat16, device=q_tilde.device)
    if lse is None and want_lse:
        lse = torch.empty(B, Q, H, dtype=torch.float32, device=q_tilde.device)
    return o_latent, lse


def mla_attend_dense(q_tilde, cache, seq_lens=None, scale=SCALE, workspace=None, o_latent=None, lse=None,
                     status=None, want_lse=True, stream=None):
    """q_tilde [B, Q, H, R], cache [B, Lmax, R] (bf16), seq_lens [B] int32 or None."""
    B, Q = _check_attend(q_tilde, workspace, o_latent, lse, status, seq_lens)
    _require(cache, "cache", "bf16", (None, None, R))
    if cache.shape[0] < B:
        raise ValueError(f"cache holds {cache.shape[0]} sequences, q_tilde {B}")
    _check_cuda(q_tilde, cache, seq_lens, workspace, o_latent, lse, status)
    Lmax = cache.shape[1]
    workspace = new_workspace(B, Q) if workspace is None else workspace
    o_latent, lse = _attend_outputs(q_tilde, o_latent, lse, want_lse)
    _check("mla_attend_dense", lib().mla_attend_dense(
        _ptr(q_tilde), _ptr(cache), _ptr(seq_lens), B, Q, H, R, Lmax, scale, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(o_latent), _ptr(lse), _ptr(status), _stream(stream)))
    return o_latent, lse


def mla_attend_dense_noalloc(q_tilde, cache, seq_lens=None, scale=SCALE, o_latent=None, lse=None, status=None,
                             want_lse=True, stream=None):
    """mla_attend_dense without a workspace argument: for callers that cannot allocate
    device memory, the scratch is a fixed 32 MiB array inside the library (see mla.h)."""
    B, Q = _check_attend(q_tilde, None, o_latent, lse, status, seq_lens)
    _require(cache, "cache", "bf16", (None, None, R))
    if cache.shape[0] < B:
        raise ValueError(f"cache holds {cache.shape[0]} sequences, q_tilde {B}")
    _check_cuda(q_tilde, cache, seq_lens, o_latent, lse, status)
    o_latent, lse = _attend_outputs(q_tilde, o_latent, lse, want_lse)
    _check("mla_attend_dense_noalloc", lib().mla_attend_dense_noalloc(
        _ptr(q_tilde), _ptr(cache), _ptr(seq_lens), B, Q, H, R, cache.shape[1], scale, _ptr(o_latent), _ptr(lse),
        _ptr(status), _stream(stream)))
    return o_latent, lse


def mla_attend_paged(q_tilde, pool, page_table, seq_lens, scale=SCALE, workspace=None, o_latent=None, lse=None,
                     status=None, want_lse=True, stream=None):
    """pool [P, 64, R] bf16, page_table [B, max_pages] int32, seq_lens [B] int32."""
    B, Q = _check_attend(q_tilde, workspace, o_latent, lse, status, seq_lens, seq_lens_required=True)
    _require(pool, "pool", "bf16", (None, PAGE, R))
    _require(page_table, "page_table", "i32", (None, None))
    if page_table.shape[0] < B:
        raise ValueError(f"page_table has {page_table.shape[0]} rows, q_tilde {B} sequences")
    _check_cuda(q_tilde, pool, page_table, seq_lens, workspace, o_latent, lse, status)
    workspace = new_workspace(B, Q) if workspace is None else workspace
    o_latent, lse = _attend_outputs(q_tilde, o_latent, lse, want_lse)
    _check("mla_attend_paged", lib().mla_attend_paged(
        _ptr(q_tilde), _ptr(pool), _ptr(page_table), _ptr(seq_lens), B, Q, H, R, pool.shape[1],
        page_table.shape[1], pool.shape[0], scale, _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(o_latent), _ptr(lse), _ptr(status), _stream(stream)))
    return o_latent, lse


def mla_attend_indexed(q_tilde, cache, indices, seq_lens=None, scale=SCALE, workspace=None, o_latent=None, lse=None,
                       status=None, want_lse=True, stream=None):
    """cache [B, Lmax, R] bf16, indices [B, Q, K] int32."""
    B, Q = _check_attend(q_tilde, workspace, o_latent, lse, status, seq_lens)
    _require(cache, "cache", "bf16", (None, None, R))
    if cache.shape[0] < B:
        raise ValueError(f"cache holds {cache.shape[0]} sequences, q_tilde {B}")
    _require(indices, "indices", "i32", (B, Q, None))
    _check_cuda(q_tilde, cache, indices, seq_lens, workspace, o_latent, lse, status)
    workspace = new_workspace(B, Q) if workspace is None else workspace
    o_latent, lse = _attend_outputs(q_tilde, o_latent, lse, want_lse)
    _check("mla_attend_indexed", lib().mla_attend_indexed(
        _ptr(q_tilde), _ptr(cache), _ptr(indices), _ptr(seq_lens), B, Q, H, R, cache.shape[1], indices.shape[2],
        scale, _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(o_latent), _ptr(lse),
        _ptr(status), _stream(stream)))
    return o_latent, lse


def _fused_outputs(q_tilde, w_uv, out, o_latent, lse, want_lse):
    import torch
    B, Q = q_tilde.shape[0], q_tilde.shape[1]
    _require(w_uv, "w_uv", "bf16", (H, D, R))
    _require(out, "out", "bf16", (B, Q, H, D), optional=True)
    if out is None:
        out = torch.empty(B, Q, H, D, dtype=torch.bfloat16, device=q_tilde.device)
    if lse is None and want_lse:
        lse = torch.empty(B, Q, H, dtype=torch.float32, device=q_tilde.device)
    return out, lse


def mla_attend_up_dense(q_tilde, cache, w_uv, seq_lens=None, scale=SCALE, workspace=None, out=None, o_latent=None,
                        lse=None, status=None, want_lse=True, stream=None):
    """Attention over a contiguous cache with the W_UV up-projection fused into the split-L
    merge: q_tilde [B, Q, H, R], cache [B, Lmax, R], w_uv [H, D, R] -> out [B, Q, H, D]
    (and lse); o_latent [B, Q, H, R] is written too when given."""
    B, Q = _check_attend(q_tilde, workspace, o_latent, lse, status, seq_lens)
    _require(cache, "cache", "bf16", (None, None, R))
    if cache.shape[0] < B:
        raise ValueError(f"cache holds {cache.shape[0]} sequences, q_tilde {B}")
    out, lse = _fused_outputs(q_tilde, w_uv, out, o_latent, lse, want_lse)
    _check_cuda(q_tilde, cache, w_uv, seq_lens, workspace, out, o_latent, lse, status)
    workspace = new_workspace(B, Q) if workspace is None else workspace
    _check("mla_attend_up_dense", lib().mla_attend_up_dense(
        _ptr(q_tilde), _ptr(cache), _ptr(seq_lens), B, Q, H, R, cache.shape[1], scale, _ptr(w_uv), D,
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(out), _ptr(o_latent), _ptr(lse),
        _ptr(status), _stream(stream)))
    return out, lse


def mla_attend_up_paged(q_tilde, pool, page_table, seq_lens, w_uv, scale=SCALE, workspace=None, out=None,
                        o_latent=None, lse=None, status=None, want_lse=True, stream=None):
    """Paged counterpart of mla_attend_up_dense (pool [P, 64, R], page_table [B, max_pages])."""
    B, Q = _check_attend(q_tilde, workspace, o_latent, lse, status, seq_lens, seq_lens_required=True)
    _require(pool, "pool", "bf16", (None, PAGE, R))
    _require(page_table, "page_table", "i32", (None, None))
    if page_table.shape[0] < B:
        raise ValueError(f"page_table has {page_table.shape[0]} rows, q_tilde {B} sequences")
    out, lse = _fused_outputs(q_tilde, w_uv, out, o_latent, lse, want_lse)
    _check_cuda(q_tilde, pool, page_table, seq_lens, w_uv, workspace, out, o_latent, lse, status)
    workspace = new_workspace(B, Q) if workspace is None else workspace
    _check("mla_attend_up_paged", lib().mla_attend_up_paged(
        _ptr(q_tilde), _ptr(pool), _ptr(page_table), _ptr(seq_lens), B, Q, H, R, pool.shape[1], page_table.shape[1],
        pool.shape[0], scale, _ptr(w_uv), D, _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(out),
        _ptr(o_latent), _ptr(lse), _ptr(status), _stream(stream)))
    return out, lse


def mla_attend_up_indexed(q_tilde, cache, indices, w_uv, seq_lens=None, scale=SCALE, workspace=None, out=None,
                          o_latent=None, lse=None, status=None, want_lse=True, stream=None):
    """Index-list counterpart of mla_attend_up_dense (indices [B, Q, K] int32)."""
    B, Q = _check_attend(q_tilde, workspace, o_latent, lse, status, seq_lens)
    _require(cache, "cache", "bf16", (None, None, R))
    if cache.shape[0] < B:
        raise ValueError(f"cache holds {cache.shape[0]} sequences, q_tilde {B}")
    _require(indices, "indices", "i32", (B, Q, None))
    out, lse = _fused_outputs(q_tilde, w_uv, out, o_latent, lse, want_lse)
    _check_cuda(q_tilde, cache, indices, w_uv, seq_lens, workspace, out, o_latent, lse, status)
    workspace = new_workspace(B, Q) if workspace is None else workspace
    _check("mla_attend_up_indexed", lib().mla_attend_up_indexed(
        _ptr(q_tilde), _ptr(cache), _ptr(indices), _ptr(seq_lens), B, Q, H, R, cache.shape[1], indices.shape[2],
        scale, _ptr(w_uv), D, _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(out),
        _ptr(o_latent), _ptr(lse), _ptr(status), _stream(stream)))
    return out, lse


def mla_expand_kv(c, w_uk, w_uv, k=None, v=None, stream=None):
    """Keys and values of every head from the latents: c [..., R] bf16 -> k, v [..., H, D]."""
    import torch
    _require(c, "c", "bf16")
    if c.dim() < 1 or c.shape[-1] != R:
        raise ValueError(f"c must be [..., {R}], got {tuple(c.shape)}")
    _require(w_uk, "w_uk", "bf16", (H, D, R))
    _require(w_uv, "w_uv", "bf16", (H, D, R))
    n = c.numel() // R
    shape = tuple(c.shape[:-1]) + (H, D)
    _require(k, "k", "bf16", shape, optional=True)
    _require(v, "v", "bf16", shape, optional=True)
    _check_cuda(c, w_uk, w_uv, k, v)
    k = torch.empty(shape, dtype=torch.bfloat16, device=c.device) if k is None else k
    v = torch.empty(shape, dtype=torch.bfloat16, device=c.device) if v is None else v
    _check("mla_expand_kv", lib().mla_expand_kv(_ptr(c), _ptr(w_uk), _ptr(w_uv), _ptr(k), _ptr(v), n, H, D, R,
                                                _stream(stream)))
    return k, v


def mla_prefill_expanded(q, k, v, scale=SCALE, out=None, lse=None, status=None, want_lse=True, stream=None):
    """Causal self-attention of B sequences of L tokens: q, k, v [B, L, H, D] bf16 -> out (and lse)."""
    import torch
    _require(q, "q", "bf16", (None, None, H, D))
    B, L = int(q.shape[0]), int(q.shape[1])
    _require(k, "k", "bf16", (B, L, H, D))
    _require(v, "v", "bf16", (B, L, H, D))
    _require(out, "out", "bf16", (B, L, H, D), optional=True)
    _require(lse, "lse", "f32", (B, L, H), optional=True)
    _require(status, "status", "i32", min_numel=1, optional=True)
    _check_cuda(q, k, v, out, lse, status)
    out = torch.empty(B, L, H, D, dtype=torch.bfloat16, device=q.device) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty(B, L, H, dtype=torch.float32, device=q.device)
    _check("mla_prefill_expanded", lib().mla_prefill_expanded(
        _ptr(q), _ptr(k), _ptr(v), B, L, H, D, scale, _ptr(out), _ptr(lse), _ptr(status), _stream(stream)))
    return out, lse


def mla_debug_gather(mode, src, req, page_table=None, indices=None, B=None, Q=1, Lmax=0, status=None, stream=None):
    """Rows the attend kernels would address for requests req [n, 3] int32 (b, i, k)."""
    import torch
    _require(src, "src", "bf16", (None, None, R))
    _require(req, "req", "i32", (None, 3))
    _require(page_table, "page_table", "i32", (None, None), optional=mode != MODE_PAGED)
    _require(indices, "indices", "i32", (None, None, None), optional=mode != MODE_INDEXED)
    _require(status, "status", "i32", min_numel=1, optional=True)
    _check_cuda(src, req, page_table, indices, status)
    n = req.shape[0]
    out = torch.empty(n, R, dtype=torch.bfloat16, device=src.device)
    max_pages = page_table.shape[1] if page_table is not None else 0
    num_pages = src.shape[0] if mode == MODE_PAGED else 0
    K = indices.shape[2] if indices is not None else 0
    _check("mla_debug_gather", lib().mla_debug_gather(
        mode, _ptr(src), _ptr(page_table), _ptr(indices), B, Q, R, Lmax, max_pages, num_pages, K, _ptr(req), n,
        _ptr(out), _ptr(status), _stream(stream)))
    return out


def mla_cache_append_dense(cache, seq_lens, rows, status=None, stream=None):
    """Append rows [B, Q, R] bf16 at positions seq_lens[b] + i of cache [B, Lmax, R];
    seq_lens [B] int32 advances by Q (in place)."""
    _require(rows, "rows", "bf16", (None, None, R))
    B, Q = rows.shape[0], rows.shape[1]
    _require(cache, "cache", "bf16", (None, None, R))
    if cache.shape[0] < B:
        raise ValueError(f"cache holds {cache.shape[0]} sequences, rows {B}")
    _require(seq_lens, "seq_lens", "i32", min_numel=B)
    _require(status, "status", "i32", min_numel=1, optional=True)
    _check_cuda(cache, seq_lens, rows, status)
    _check("mla_cache_append_dense", lib().mla_cache_append_dense(
        _ptr(cache), _ptr(seq_lens), _ptr(rows), B, Q, R, cache.shape[1], _ptr(status), _stream(stream)))


def mla_cache_append_paged(pool, page_table, seq_lens, rows, status=None, stream=None):
    """Append rows [B, Q, R] bf16 through page_table [B, max_pages] into pool [P, 64, R]."""
    _require(rows, "rows", "bf16", (None, None, R))
    B, Q = rows.shape[0], rows.shape[1]
    _require(pool, "pool", "bf16", (None, PAGE, R))
    _require(page_table, "page_table", "i32", (None, None))
    if page_table.shape[0] < B:
        raise ValueError(f"page_table has {page_table.shape[0]} rows, rows {B} sequences")
    _require(seq_lens, "seq_lens", "i32", min_numel=B)
    _require(status, "status", "i32", min_numel=1, optional=True)
    _check_cuda(pool, page_table, seq_lens, rows, status)
    _check("mla_cache_append_paged", lib().mla_cache_append_paged(
        _ptr(pool), _ptr(page_table), _ptr(seq_lens), _ptr(rows), B, Q, R, pool.shape[1], page_table.shape[1],
        pool.shape[0], _ptr(status), _stream(stream)))


def mla_cache_truncate_dense(cache, seq_lens, keep, q_len, status=None, stream=None):
    """Keep the first keep[b] of the last q_len rows of each sequence; zero the rest."""
    _require(seq_lens, "seq_lens", "i32", (None,))
    _require(keep, "keep", "i32", min_numel=seq_lens.shape[0])
    _require(cache, "cache", "bf16", (None, None, R))
    if cache.shape[0] < seq_lens.shape[0]:
        raise ValueError(f"cache holds {cache.shape[0]} sequences, seq_lens {seq_lens.shape[0]}")
    _require(status, "status", "i32", min_numel=1, optional=True)
    _check_cuda(cache, seq_lens, keep, status)
    _check("mla_cache_truncate_dense", lib().mla_cache_truncate_dense(
        _ptr(cache), _ptr(seq_lens), _ptr(keep), seq_lens.shape[0], q_len, R, cache.shape[1], _ptr(status),
        _stream(stream)))


def mla_cache_truncate_paged(pool, page_table, seq_lens, keep, q_len, status=None, stream=None):
    """Paged counterpart of mla_cache_truncate_dense."""
    _require(seq_lens, "seq_lens", "i32", (None,))
    _require(keep, "keep", "i32", min_numel=seq_lens.shape[0])
    _require(pool, "pool", "bf16", (None, PAGE, R))
    _require(page_table, "page_table", "i32", (None, None))
    if page_table.shape[0] < seq_lens.shape[0]:
        raise ValueError(f"page_table has {page_table.shape[0]} rows, seq_lens {seq_lens.shape[0]}")
    _require(status, "status", "i32", min_numel=1, optional=True)
    _check_cuda(pool, page_table, seq_lens, keep, status)
    _check("mla_cache_truncate_paged", lib().mla_cache_truncate_paged(
        _ptr(pool), _ptr(page_table), _ptr(seq_lens), _ptr(keep), seq_lens.shape[0], q_len, R, pool.shape[1],
        page_table.shape[1], pool.shape[0], _ptr(status), _stream(stream)))


def mla_debug_wait_timeout(limit_cycles, status, stream=None):
    """Run the pipeline's bounded wait on a barrier nothing completes (test aid)."""
    _require(status, "status", "i32", min_numel=1)
    _check_cuda(status)
    _check("mla_debug_wait_timeout", lib().mla_debug_wait_timeout(int(limit_cycles), _ptr(status), _stream(stream)))


def mla_kpool_keys(cache, pool, seq_lens=None, pooled=None, stream=None):
    """Pooled keys [B, Lmax // pool, R] fp32 of every complete pool of cache [B, Lmax, R]."""
    import torch
    _require(cache, "cache", "bf16", (None, None, R))
    B, Lmax = cache.shape[0], cache.shape[1]
    _require(seq_lens, "seq_lens", "i32", min_numel=B, optional=True)
    if pool < 1:
        raise ValueError("pool must be positive")
    _require(pooled, "pooled", "f32", (B, Lmax // pool, R), optional=True)
    _check_cuda(cache, seq_lens, pooled)
    if pooled is None:
        pooled = torch.zeros(B, Lmax // pool, R, dtype=torch.float32, device=cache.device)
    _check("mla_kpool_keys", lib().mla_kpool_keys(_ptr(cache), _ptr(seq_lens), B, R, Lmax, pool, _ptr(pooled),
                                                  _stream(stream)))
    return pooled


def mla_kpool_select(pooled, w_query, pool, topk, seq_lens=None, with_tail=True, Lmax=None, stream=None):
    """Index lists [B, Q, topk (+ pool - 1)] int32 for w_query [B, Q, R] bf16."""
    import torch
    _require(w_query, "w_query", "bf16", (None, None, R))
    B, Q = w_query.shape[0], w_query.shape[1]
    _require(pooled, "pooled", "f32", (B, None, R))
    _require(seq_lens, "seq_lens", "i32", min_numel=B, optional=True)
    if pool < 1:
        raise ValueError("pool must be positive")
    Lmax = pooled.shape[1] * pool if Lmax is None else Lmax
    if Lmax // pool > pooled.shape[1]:
        raise ValueError(f"pooled holds {pooled.shape[1]} pools per sequence, Lmax {Lmax} needs {Lmax // pool}")
    _check_cuda(pooled, w_query, seq_lens)
    W = topk + (pool - 1 if with_tail else 0)
    out = torch.empty(B, Q, W, dtype=torch.int32, device=w_query.device)
    _check("mla_kpool_select", lib().mla_kpool_select(
        _ptr(pooled), _ptr(w_query), _ptr(seq_lens), B, Q, R, Lmax, pool, topk, 1 if with_tail else 0, _ptr(out), W,
        _stream(stream)))
    return out


def mla_decode(q, w_uk, w_uv, cache, seq_lens=None, *, mode=MODE_DENSE, page_table=None, indices=None,
               scale=SCALE, workspace=None, status=None, stream=None, fused=False):
    """The whole path: absorb -> attend (dense / paged / indexed) -> up-project.  With
    fused=True the up-projection runs inside the split-L merge (mla_attend_up_*).

    q [B, Q, H, D] bf16 -> out [B, Q, H, D] bf16 (and lse [B, Q, H])."""
    qt = mla_absorb_q(q, w_uk, stream=stream)
    if fused:
        if mode == MODE_DENSE:
            return mla_attend_up_dense(qt, cache, w_uv, seq_lens, scale, workspace, status=status, stream=stream)
        if mode == MODE_PAGED:
            return mla_attend_up_paged(qt, cache, page_table, seq_lens, w_uv, scale, workspace, status=status,
                                       stream=stream)
        return mla_attend_up_indexed(qt, cache, indices, w_uv, seq_lens, scale, workspace, status=status,
                                     stream=stream)
    if mode == MODE_DENSE:
        o, lse = mla_attend_dense(qt, cache, seq_lens, scale, workspace, status=status, stream=stream)
    elif mode == MODE_PAGED:
        o, lse = mla_attend_paged(qt, cache, page_table, seq_lens, scale, workspace, status=status, stream=stream)
    else:
        o, lse = mla_attend_indexed(qt, cache, indices, seq_lens, scale, workspace, status=status, stream=stream)
    return mla_up_proj(o, w_uv, stream=stream), lse

"""Python binding of libqsa, the B200 (sm_100a) Qwen Sparse Attention library.

Thin ctypes layer over the C ABI declared in ``include/qsa.h``: every function
here has the C entry point's name, checks that its torch tensors have the
dtype, device and contiguity the ABI requires, and passes their device
pointers, the sizes and the current CUDA stream through.  All computation
happens in the library's CUDA kernels; there is no other code path.  If the
shared library has not been built, every call raises ``QSAError``.

Tensors: bf16 tensors are ``torch.bfloat16``; ``w``/``sel_score``/``lse``
are ``torch.float32``; ``sel``/``seqlens`` are ``torch.int32``; ``q_pos0`` is
``torch.int64``.  Workspaces are ``torch.uint8`` device tensors whose first
256 bytes are zero before first use (``workspace()`` makes one).
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "QSAError", "lib_path", "load", "workspace",
    "qsa_pool", "qsa_index_topk", "qsa_index_topk_workspace_size",
    "qsa_index_topk_decode", "qsa_index_topk_decode_workspace_size",
    "qsa_sparse_attn_prefill", "qsa_sparse_attn_decode",
    "qsa_sparse_attn_decode_workspace_size", "qsa_sparse_attn_decode_noalloc",
    "qsa_dense_gqa_prefill",
    "qsa_dense_gqa_decode", "qsa_dense_gqa_decode_workspace_size",
    "qsa_index_distill", "qsa_index_distill_workspace_size", "qsa_sparse_attn_backward",
    "qsa_gdn_prefill", "qsa_gdn_decode", "qsa_gdn_prefill_chunked",
    "qsa_gdn_prefill_chunked_workspace_size", "qsa_probe_l2_read",
    "qsa_check_device_status", "qsa_status_string", "qsa_version",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libqsa.so")
_lib = None

STATUS = {
    0: "QSA_OK", 1: "QSA_ERR_INVALID_ARG", 2: "QSA_ERR_UNSUPPORTED_SHAPE",
    3: "QSA_ERR_WORKSPACE", 4: "QSA_ERR_ARCH", 5: "QSA_ERR_CUDA",
    6: "QSA_ERR_TIMEOUT", 7: "QSA_ERR_DEVICE",
}


class QSAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


def lib_path() -> str:
    return _LIB_PATH


_VP, _I, _I64, _F, _SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                          ctypes.c_float, ctypes.c_size_t)
_SIGS = {
    "qsa_pool": (_I, [_VP, _I, _I64, _I, _I, _I64, _I64, _VP, _VP]),
    "qsa_index_topk_workspace_size": (_SZ, [_I, _I64, _I64, _I, _I, _I, _I]),
    "qsa_index_topk": (_I, [_VP, _VP, _VP, _VP, _I, _I64, _I64, _I, _I, _I, _I,
                            _VP, _VP, _VP, _SZ, _VP]),
    "qsa_index_topk_decode_workspace_size": (_SZ, [_I, _I64, _I, _I]),
    "qsa_index_topk_decode": (_I, [_VP, _VP, _VP, _VP, _I, _I64, _I, _I, _I, _I,
                                   _VP, _VP, _VP, _SZ, _VP]),
    "qsa_sparse_attn_prefill": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I64, _I64, _I,
                                     _I, _I, _I, _I, _F, _VP, _VP, _VP]),
    "qsa_sparse_attn_decode_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "qsa_sparse_attn_decode": (_I, [_VP, _VP, _VP, _VP, _I64, _VP, _I, _I, _I,
                                    _I, _I, _I, _F, _VP, _VP, _VP, _SZ, _VP]),
    "qsa_sparse_attn_decode_noalloc": (_I, [_VP, _VP, _VP, _VP, _I64, _VP, _I, _I, _I,
                                            _I, _I, _I, _F, _VP, _VP, _VP]),
    "qsa_dense_gqa_prefill": (_I, [_VP, _VP, _VP, _I, _I64, _I, _I, _I, _F, _VP,
                                   _VP, _VP]),
    "qsa_dense_gqa_decode_workspace_size": (_SZ, [_I, _I64, _I, _I]),
    "qsa_dense_gqa_decode": (_I, [_VP, _VP, _VP, _VP, _I64, _I, _I, _I, _I, _F,
                                  _VP, _VP, _VP, _SZ, _VP]),
    "qsa_sparse_attn_backward": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I64, _I, _I, _I, _I, _I,
                                      _F, _VP, _VP, _VP, _VP]),
    "qsa_gdn_prefill": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I64, _I, _I, _I, _VP, _VP,
                             _VP]),
    "qsa_gdn_decode": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _VP, _VP]),
    "qsa_gdn_prefill_chunked_workspace_size": (_SZ, [_I, _I64, _I, _I, _I]),
    "qsa_probe_l2_read": (_I, [_VP, _SZ, _I, _VP, _VP]),
    "qsa_gdn_prefill_chunked": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I64, _I, _I, _I, _VP,
                                     _VP, _VP, _SZ, _VP]),
    "qsa_index_distill_workspace_size": (_SZ, [_I, _I64, _I, _I]),
    "qsa_index_distill": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I64, _I, _I, _I, _I, _I,
                               _I, _F, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "qsa_index_distill_sparse_workspace_size": (_SZ, [_I, _I64, _I, _I, _I]),
    "qsa_index_distill_sparse": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I64, _I, _I, _I,
                                      _I, _I, _I, _I, _F, _VP, _VP, _VP, _VP, _VP, _VP, _SZ,
                                      _VP]),
    "qsa_check_device_status": (_I, [_VP, _VP]),
    "qsa_status_string": (ctypes.c_char_p, [_I]),
    "qsa_version": (ctypes.c_char_p, []),
}
SIZE_MAX = ctypes.c_size_t(-1).value


def load():
    """Load libqsa.so (once).  Raises QSAError if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise QSAError(-1, f"{_LIB_PATH} is not built (run __graft_entry__.build())")
    lib = ctypes.CDLL(_LIB_PATH)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, dtype, name, ndim=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")


def _call(name, *args):
    rc = getattr(load(), name)(*args)
    if rc != 0:
        raise QSAError(rc, name)


def _size(name, *args) -> int:
    n = getattr(load(), name)(*args)
    if n == SIZE_MAX:
        raise QSAError(1, name)
    return int(n)


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zeroed uint8 device buffer (the status word must start at zero)."""
    return torch.zeros(int(nbytes), dtype=torch.uint8, device=device or "cuda")


_BF, _F32, _I32, _I64T = torch.bfloat16, torch.float32, torch.int32, torch.int64


# ------------------------------------------------------------------- pool --

def qsa_pool(k_idx, k_pooled, r=4, blk_begin=0, blk_end=None, stream=None):
    """k_idx [B,T,Di] -> k_pooled [B,T//r,Di] for blocks [blk_begin, blk_end)."""
    _need(k_idx, _BF, "k_idx", 3)
    _need(k_pooled, _BF, "k_pooled", 3)
    B, T, Di = k_idx.shape
    if tuple(k_pooled.shape) != (B, T // r, Di):
        raise ValueError("k_pooled must be [B, T//r, Di]")
    blk_end = T // r if blk_end is None else blk_end
    _call("qsa_pool", _ptr(k_idx), B, T, Di, r, blk_begin, blk_end, _ptr(k_pooled),
          _stream(stream, k_idx.device))


# ---------------------------------------------------------------- indexer --

def qsa_index_topk_workspace_size(B, Tq, n_blocks, Hi, Di, r, budget) -> int:
    return _size("qsa_index_topk_workspace_size", B, Tq, n_blocks, Hi, Di, r, budget)


def qsa_index_topk(q_idx, w, k_pooled, sel, ws, r=4, budget=2048, q_pos0=None,
                   sel_score=None, stream=None):
    """q_idx [B,Tq,Hi,Di], w [B,Tq,Hi], k_pooled [B,N,Di] -> sel [B,Tq,kb]."""
    _need(q_idx, _BF, "q_idx", 4)
    _need(w, _F32, "w", 3)
    _need(k_pooled, _BF, "k_pooled", 3)
    _need(sel, _I32, "sel", 3)
    _need(sel_score, _F32, "sel_score", 3)
    _need(q_pos0, _I64T, "q_pos0", 1)
    _need(ws, torch.uint8, "ws", 1)
    B, Tq, Hi, Di = q_idx.shape
    _call("qsa_index_topk", _ptr(q_idx), _ptr(w), _ptr(k_pooled), _ptr(q_pos0), B, Tq,
          k_pooled.shape[1], Hi, Di, r, budget, _ptr(sel), _ptr(sel_score), _ptr(ws),
          ws.numel(), _stream(stream, q_idx.device))


def qsa_index_topk_decode_workspace_size(B, n_blocks, r, budget) -> int:
    return _size("qsa_index_topk_decode_workspace_size", B, n_blocks, r, budget)


def qsa_index_topk_decode(q_idx, w, k_pooled, seqlens, sel, ws, r=4, budget=2048,
                          sel_score=None, stream=None):
    """q_idx [B,Hi,Di], w [B,Hi], k_pooled [B,N,Di], seqlens [B] -> sel [B,kb]."""
    _need(q_idx, _BF, "q_idx", 3)
    _need(w, _F32, "w", 2)
    _need(k_pooled, _BF, "k_pooled", 3)
    _need(seqlens, _I32, "seqlens", 1)
    _need(sel, _I32, "sel", 2)
    _need(sel_score, _F32, "sel_score", 2)
    _need(ws, torch.uint8, "ws", 1)
    B, Hi, Di = q_idx.shape
    _call("qsa_index_topk_decode", _ptr(q_idx), _ptr(w), _ptr(k_pooled), _ptr(seqlens), B,
          k_pooled.shape[1], Hi, Di, r, budget, _ptr(sel), _ptr(sel_score), _ptr(ws),
          ws.numel(), _stream(stream, q_idx.device))


# -------------------------------------------------------------- attention --

def qsa_sparse_attn_prefill(q, k, v, sel, o, r=4, budget=2048, scale=None, q_pos0=None,
                            lse=None, stream=None):
    """q [B,Tq,Hq,D], k/v [B,Tk,Hkv,D], sel [B,Tq,kb] -> o [B,Tq,Hq,D]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, _BF, n, 4)
    _need(sel, _I32, "sel", 3)
    _need(lse, _F32, "lse", 3)
    _need(q_pos0, _I64T, "q_pos0", 1)
    B, Tq, Hq, D = q.shape
    Tk, Hkv = k.shape[1], k.shape[2]
    scale = D ** -0.5 if scale is None else scale
    _call("qsa_sparse_attn_prefill", _ptr(q), _ptr(k), _ptr(v), _ptr(sel), _ptr(q_pos0), B,
          Tq, Tk, Hq, Hkv, D, r, budget, scale, _ptr(o), _ptr(lse), _stream(stream, q.device))


def qsa_sparse_attn_decode_workspace_size(B, Hq, D, r, budget) -> int:
    return _size("qsa_sparse_attn_decode_workspace_size", B, Hq, D, r, budget)


def qsa_sparse_attn_decode(q, k_cache, v_cache, seqlens, sel, o, ws, r=4, budget=2048,
                           scale=None, lse=None, stream=None):
    """q [B,Hq,D], caches [B,L,Hkv,D], seqlens [B], sel [B,kb] -> o [B,Hq,D]."""
    _need(q, _BF, "q", 3)
    _need(k_cache, _BF, "k_cache", 4)
    _need(v_cache, _BF, "v_cache", 4)
    _need(o, _BF, "o", 3)
    _need(seqlens, _I32, "seqlens", 1)
    _need(sel, _I32, "sel", 2)
    _need(lse, _F32, "lse", 2)
    _need(ws, torch.uint8, "ws", 1)
    B, Hq, D = q.shape
    L, Hkv = k_cache.shape[1], k_cache.shape[2]
    scale = D ** -0.5 if scale is None else scale
    _call("qsa_sparse_attn_decode", _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), L,
          _ptr(sel), B, Hq, Hkv, D, r, budget, scale, _ptr(o), _ptr(lse), _ptr(ws), ws.numel(),
          _stream(stream, q.device))


def qsa_sparse_attn_decode_noalloc(q, k_cache, v_cache, seqlens, sel, o, r=4, budget=2048,
                                   scale=None, lse=None, stream=None):
    """qsa_sparse_attn_decode without a workspace, for callers that cannot
    allocate device memory where they run the step: the library keeps the
    split partials in its own fixed 8 MiB device array (shared by all calls on
    a device; concurrent calls race).  Too large a batch raises QSAError."""
    _need(q, _BF, "q", 3)
    _need(k_cache, _BF, "k_cache", 4)
    _need(v_cache, _BF, "v_cache", 4)
    _need(o, _BF, "o", 3)
    _need(seqlens, _I32, "seqlens", 1)
    _need(sel, _I32, "sel", 2)
    _need(lse, _F32, "lse", 2)
    B, Hq, D = q.shape
    L, Hkv = k_cache.shape[1], k_cache.shape[2]
    scale = D ** -0.5 if scale is None else scale
    _call("qsa_sparse_attn_decode_noalloc", _ptr(q), _ptr(k_cache), _ptr(v_cache),
          _ptr(seqlens), L, _ptr(sel), B, Hq, Hkv, D, r, budget, scale, _ptr(o), _ptr(lse),
          _stream(stream, q.device))


def qsa_dense_gqa_prefill(q, k, v, o, scale=None, lse=None, stream=None):
    """Causal dense GQA: q [B,T,Hq,D], k/v [B,T,Hkv,D] -> o [B,T,Hq,D]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, _BF, n, 4)
    _need(lse, _F32, "lse", 3)
    B, T, Hq, D = q.shape
    scale = D ** -0.5 if scale is None else scale
    _call("qsa_dense_gqa_prefill", _ptr(q), _ptr(k), _ptr(v), B, T, Hq, k.shape[2], D, scale,
          _ptr(o), _ptr(lse), _stream(stream, q.device))


def qsa_dense_gqa_decode_workspace_size(B, L_max, Hq, D) -> int:
    return _size("qsa_dense_gqa_decode_workspace_size", B, L_max, Hq, D)


def qsa_dense_gqa_decode(q, k_cache, v_cache, seqlens, o, ws, scale=None, lse=None,
                         stream=None):
    """Dense decode over all seqlens[b] cached tokens."""
    _need(q, _BF, "q", 3)
    _need(k_cache, _BF, "k_cache", 4)
    _need(v_cache, _BF, "v_cache", 4)
    _need(o, _BF, "o", 3)
    _need(seqlens, _I32, "seqlens", 1)
    _need(lse, _F32, "lse", 2)
    _need(ws, torch.uint8, "ws", 1)
    B, Hq, D = q.shape
    L, Hkv = k_cache.shape[1], k_cache.shape[2]
    scale = D ** -0.5 if scale is None else scale
    _call("qsa_dense_gqa_decode", _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), L, B,
          Hq, Hkv, D, scale, _ptr(o), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream, q.device))


# ------------------------------------------------ sparse attention backward --

def qsa_sparse_attn_backward(q, k, v, sel, d_o, dq, dk, dv, r=4, budget=2048, scale=None,
                             stream=None):
    """Gradients of the sparse prefill attention for an output gradient d_o:
    q, d_o [B,T,Hq,D], k/v [B,T,Hkv,D] bf16, sel [B,T,kb] -> dq [B,T,Hq,D],
    dk/dv [B,T,Hkv,D] fp32 (overwritten)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (d_o, "d_o")):
        _need(t, _BF, n, 4)
    _need(sel, _I32, "sel", 3)
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need(t, _F32, n, 4)
    B, T, Hq, D = q.shape
    scale = D ** -0.5 if scale is None else scale
    _call("qsa_sparse_attn_backward", _ptr(q), _ptr(k), _ptr(v), _ptr(sel), _ptr(d_o), B, T,
          Hq, k.shape[2], D, r, budget, scale, _ptr(dq), _ptr(dk), _ptr(dv),
          _stream(stream, q.device))


# ---------------------------------------------------------- measurement aid --

def qsa_probe_l2_read(buf, reps, sink, nbytes=None, stream=None):
    """Reads the first nbytes (default: all) of the device buffer `buf` `reps`
    times through L2; `sink` is a device int32 tensor the kernel may write."""
    n = buf.numel() * buf.element_size() if nbytes is None else int(nbytes)
    _call("qsa_probe_l2_read", _ptr(buf), n, int(reps), _ptr(sink), _stream(stream, buf.device))


# ------------------------------------------------------------ Gated DeltaNet --

def qsa_gdn_prefill(q, k, v, alpha, beta, o, state_out, state_in=None, stream=None):
    """Gated delta rule over a prefill: q, k [B,T,H,dk], v [B,T,H,dv] bf16,
    alpha, beta [B,T,H] fp32, state_in [B,H,dv,dk] fp32 or None ->
    o [B,T,H,dv] fp32, state_out [B,H,dv,dk] fp32."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, _BF, n, 4)
    for t, n in ((alpha, "alpha"), (beta, "beta")):
        _need(t, _F32, n, 3)
    _need(o, _F32, "o", 4)
    _need(state_out, _F32, "state_out", 4)
    _need(state_in, _F32, "state_in", 4)
    B, T, H, dk = k.shape
    _call("qsa_gdn_prefill", _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state_in),
          B, T, H, dk, v.shape[3], _ptr(o), _ptr(state_out), _stream(stream, k.device))


def qsa_gdn_prefill_chunked_workspace_size(B, T, H, dk, dv) -> int:
    return _size("qsa_gdn_prefill_chunked_workspace_size", B, T, H, dk, dv)


def qsa_gdn_prefill_chunked(q, k, v, alpha, beta, o, state_out, ws, state_in=None,
                            stream=None):
    """The same prefill in chunks of 64 tokens (chunk-parallel solves, state
    products on the tensor cores); ws: a workspace of
    qsa_gdn_prefill_chunked_workspace_size bytes."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, _BF, n, 4)
    for t, n in ((alpha, "alpha"), (beta, "beta")):
        _need(t, _F32, n, 3)
    _need(o, _F32, "o", 4)
    _need(state_out, _F32, "state_out", 4)
    _need(state_in, _F32, "state_in", 4)
    B, T, H, dk = k.shape
    _call("qsa_gdn_prefill_chunked", _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
          _ptr(state_in), B, T, H, dk, v.shape[3], _ptr(o), _ptr(state_out), _ptr(ws),
          ws.numel() * ws.element_size(), _stream(stream, k.device))


def qsa_gdn_decode(q, k, v, alpha, beta, state, o, stream=None):
    """One token per sequence: q, k [B,H,dk], v [B,H,dv] bf16, alpha, beta [B,H]
    fp32; state [B,H,dv,dk] fp32 updated in place; o [B,H,dv] fp32."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, _BF, n, 3)
    for t, n in ((alpha, "alpha"), (beta, "beta")):
        _need(t, _F32, n, 2)
    _need(state, _F32, "state", 4)
    _need(o, _F32, "o", 3)
    B, H, dk = k.shape
    _call("qsa_gdn_decode", _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state), B,
          H, dk, v.shape[2], _ptr(o), _stream(stream, k.device))


# ----------------------------------------------------- indexer distillation --

def qsa_index_distill_workspace_size(B, T, Hkv, r=4) -> int:
    return _size("qsa_index_distill_workspace_size", B, T, Hkv, r)


def qsa_index_distill(q, k, lse, q_idx, w, k_pooled, kl, dq_idx, dw, dk_pooled, ws, r=4,
                      scale=None, dk_idx=None, stream=None):
    """Stage-1 distillation loss and indexer gradients.

    q [B,T,Hq,D], k [B,T,Hkv,D] bf16, lse [B,T,Hq] fp32 (dense attention's),
    q_idx [B,T,Hi,Di] bf16, w [B,T,Hi] fp32, k_pooled [B,T//r,Di] bf16 ->
    kl [B,T], dq_idx [B,T,Hi,Di], dw [B,T,Hi], dk_pooled [B,T//r,Di] and
    optionally dk_idx [B,T,Di], all fp32.
    """
    _need(q, _BF, "q", 4)
    _need(k, _BF, "k", 4)
    _need(lse, _F32, "lse", 3)
    _need(q_idx, _BF, "q_idx", 4)
    _need(w, _F32, "w", 3)
    _need(k_pooled, _BF, "k_pooled", 3)
    _need(kl, _F32, "kl", 2)
    _need(dq_idx, _F32, "dq_idx", 4)
    _need(dw, _F32, "dw", 3)
    _need(dk_pooled, _F32, "dk_pooled", 3)
    _need(dk_idx, _F32, "dk_idx", 3)
    _need(ws, torch.uint8, "ws", 1)
    B, T, Hq, D = q.shape
    Hkv, Hi, Di = k.shape[2], q_idx.shape[2], q_idx.shape[3]
    if tuple(k_pooled.shape) != (B, T // r, Di) or tuple(dk_pooled.shape) != (B, T // r, Di):
        raise ValueError("k_pooled and dk_pooled must be [B, T//r, Di]")
    scale = D ** -0.5 if scale is None else scale
    _call("qsa_index_distill", _ptr(q), _ptr(k), _ptr(lse), _ptr(q_idx), _ptr(w),
          _ptr(k_pooled), B, T, Hq, Hkv, D, Hi, Di, r, scale, _ptr(kl), _ptr(dq_idx), _ptr(dw),
          _ptr(dk_pooled), _ptr(dk_idx), _ptr(ws), ws.numel(), _stream(stream, q.device))


def qsa_index_distill_sparse_workspace_size(B, T, Hkv, r=4, budget=2048) -> int:
    return _size("qsa_index_distill_sparse_workspace_size", B, T, Hkv, r, budget)


def qsa_index_distill_sparse(q, k, lse, sel, q_idx, w, k_pooled, kl, dq_idx, dw, dk_pooled,
                             ws, r=4, budget=2048, scale=None, dk_idx=None, stream=None):
    """Stage-2 indexer loss over the selection and the indexer gradients.

    q [B,T,Hq,D], k [B,T,Hkv,D] bf16, lse [B,T,Hq] fp32 (the sparse attention's),
    sel [B,T,budget//r] int32, q_idx [B,T,Hi,Di] bf16, w [B,T,Hi] fp32,
    k_pooled [B,T//r,Di] bf16 -> kl [B,T], dq_idx [B,T,Hi,Di], dw [B,T,Hi],
    dk_pooled [B,T//r,Di] and optionally dk_idx [B,T,Di], all fp32.
    """
    _need(q, _BF, "q", 4)
    _need(k, _BF, "k", 4)
    _need(lse, _F32, "lse", 3)
    _need(sel, torch.int32, "sel", 3)
    _need(q_idx, _BF, "q_idx", 4)
    _need(w, _F32, "w", 3)
    _need(k_pooled, _BF, "k_pooled", 3)
    _need(kl, _F32, "kl", 2)
    _need(dq_idx, _F32, "dq_idx", 4)
    _need(dw, _F32, "dw", 3)
    _need(dk_pooled, _F32, "dk_pooled", 3)
    _need(dk_idx, _F32, "dk_idx", 3)
    _need(ws, torch.uint8, "ws", 1)
    B, T, Hq, D = q.shape
    Hkv, Hi, Di = k.shape[2], q_idx.shape[2], q_idx.shape[3]
    if tuple(sel.shape) != (B, T, budget // r):
        raise ValueError("sel must be [B, T, budget//r]")
    if tuple(k_pooled.shape) != (B, T // r, Di) or tuple(dk_pooled.shape) != (B, T // r, Di):
        raise ValueError("k_pooled and dk_pooled must be [B, T//r, Di]")
    scale = D ** -0.5 if scale is None else scale
    _call("qsa_index_distill_sparse", _ptr(q), _ptr(k), _ptr(lse), _ptr(sel), _ptr(q_idx),
          _ptr(w), _ptr(k_pooled), B, T, Hq, Hkv, D, Hi, Di, r, budget, scale, _ptr(kl),
          _ptr(dq_idx), _ptr(dw), _ptr(dk_pooled), _ptr(dk_idx), _ptr(ws), ws.numel(),
          _stream(stream, q.device))


def qsa_check_device_status(ws, stream=None) -> int:
    """Synchronise, read and clear the workspace status word; returns the code."""
    _need(ws, torch.uint8, "ws", 1)
    return int(load().qsa_check_device_status(_ptr(ws), _stream(stream, ws.device)))


def qsa_status_string(code: int) -> str:
    return load().qsa_status_string(code).decode()


def qsa_version() -> str:
    return load().qsa_version().decode()

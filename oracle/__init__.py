"""QSA CPU oracle -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT PATH.

Thin numpy/ctypes wrapper around ``qsa_oracle.c``: a plain, slow, fp64
restatement of the Qwen Sparse Attention layer (micro-block mean pooling,
DSA-style lightweight MQA indexer scores, top-k block selection with the own
block forced, exact softmax attention over the expanded token set).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  It never imports the CUDA library and the CUDA
library never imports it.

Submodules (numpy, fp64), each stating its readings of the pages:
``distill`` (stage-1 indexer distillation: KL loss and indexer gradients),
``sparse_train`` (stage-2: sparse attention backward, indexer loss over the
selection) and ``gdn`` (the gated delta rule of the hybrid's GDN layers).

Sources are cited in ``qsa_oracle.c``'s header: the article
"用125亿分之6的参数，打平3970亿的旗舰模型" (section "稀疏注意力：给检索建索引，也得先学会省纸"),
the paper summary "On the Design of Qwen3.8-Next Architecture" (token-mixing
paragraph) and the AITOP100 news page (section "二、架构 / 1. 注意力机制").

Parity unpinned: the scoring form itself (the pages print no formula); it is
pinned by closed forms, invariants and reductions in ``tests/test_oracle_pins.py``.

All bf16 tensors cross this interface as ``numpy.uint16`` arrays holding the
raw bf16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libqsa_oracle.so")
_lib = None

_I64P = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile ``libqsa_oracle.so`` with gcc (OpenMP, no FP contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    vp = ctypes.c_void_p
    i64 = ctypes.c_int64
    ci = ctypes.c_int
    lib.qsa_oracle_pool.argtypes = [vp, ci, i64, ci, ci, i64, i64, vp]
    lib.qsa_oracle_index_scores_rows.argtypes = [
        vp, vp, vp, ci, i64, i64, ci, ci, ci, vp, vp, i64, i64, vp]
    lib.qsa_oracle_score_pairs.argtypes = [
        vp, vp, vp, i64, i64, ci, ci, vp, vp, i64, vp]
    lib.qsa_oracle_index_topk_rows.argtypes = [
        vp, vp, vp, ci, i64, i64, ci, ci, ci, ci, vp, vp, i64, vp, vp, vp, vp]
    lib.qsa_oracle_attn_rows.argtypes = [
        vp, vp, vp, ci, i64, i64, ci, ci, ci, ci, ci, ctypes.c_double,
        vp, vp, vp, i64, vp, vp]
    lib.qsa_oracle_float_to_bf16.argtypes = [ctypes.c_float]
    lib.qsa_oracle_float_to_bf16.restype = ctypes.c_uint16
    lib.qsa_oracle_num_threads.restype = ci
    lib.qsa_oracle_set_num_threads.argtypes = [ci]
    _lib = lib
    return lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


# ------------------------------------------------------------------ helpers --

def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 values (exact)."""
    a = np.asarray(a, dtype=np.uint16)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f32_to_bf16_bits(x) -> np.ndarray:
    """float32 values -> bf16 bit patterns, round to nearest even (oracle's rule)."""
    lib = _load()
    x = np.asarray(x, dtype=np.float32)
    flat = [lib.qsa_oracle_float_to_bf16(float(v)) for v in x.ravel()]
    return np.asarray(flat, dtype=np.uint16).reshape(x.shape)


def num_threads() -> int:
    return int(_load().qsa_oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().qsa_oracle_set_num_threads(int(n))


def _rows_pos(B: int, Tq: int, q_pos0, rows):
    """Flat rows (b*Tq + t) and their absolute positions p = q_pos0[b] + t."""
    if rows is None:
        rows = np.arange(B * Tq, dtype=np.int64)
    rows = _c(rows, np.int64)
    b = rows // Tq
    t = rows % Tq
    base = np.zeros(B, np.int64) if q_pos0 is None else _c(q_pos0, np.int64)
    return rows, _c(base[b] + t, np.int64)


# -------------------------------------------------------------------- steps --

def pool(k_idx: np.ndarray, r: int, j0: int = 0, j1: int | None = None,
         out: np.ndarray | None = None) -> np.ndarray:
    """Micro-block mean pooling.  k_idx [B, T, Di] uint16 -> Kp [B, T//r, Di] uint16."""
    k_idx = _c(k_idx, np.uint16)
    B, T, Di = k_idx.shape
    N = T // r
    j1 = N if j1 is None else j1
    kp = np.zeros((B, N, Di), np.uint16) if out is None else out
    assert kp.flags.c_contiguous and kp.dtype == np.uint16
    _check(_load().qsa_oracle_pool(_p(k_idx), B, T, Di, r, j0, j1, _p(kp)), "pool")
    return kp


def index_scores(q_idx, w, kp, r: int, q_pos0=None, rows=None, n_cols=None):
    """Dense fp64 score matrix for the given rows; -inf off the causal candidates.

    q_idx [B, Tq, Hi, Di] uint16, w [B, Tq, Hi] f32, kp [B, N, Di] uint16.
    Returns [len(rows), n_cols] float64.
    """
    q_idx = _c(q_idx, np.uint16)
    w = _c(w, np.float32)
    kp = _c(kp, np.uint16)
    B, Tq, Hi, Di = q_idx.shape
    N = kp.shape[1]
    rows, pos = _rows_pos(B, Tq, q_pos0, rows)
    n_cols = N if n_cols is None else n_cols
    out = np.empty((rows.size, n_cols), np.float64)
    _check(_load().qsa_oracle_index_scores_rows(
        _p(q_idx), _p(w), _p(kp), B, Tq, N, Hi, Di, r, _p(rows), _p(pos),
        rows.size, n_cols, _p(out)), "index_scores")
    return out


def score_pairs(q_idx, w, kp, rows, blocks) -> np.ndarray:
    """fp64 score of each (row, block) pair."""
    q_idx = _c(q_idx, np.uint16)
    w = _c(w, np.float32)
    kp = _c(kp, np.uint16)
    B, Tq, Hi, Di = q_idx.shape
    rows = _c(rows, np.int64)
    blocks = _c(blocks, np.int64)
    assert rows.shape == blocks.shape
    out = np.empty(rows.shape, np.float64)
    _check(_load().qsa_oracle_score_pairs(
        _p(q_idx), _p(w), _p(kp), Tq, kp.shape[1], Hi, Di, _p(rows),
        _p(blocks), rows.size, _p(out)), "score_pairs")
    return out


def index_topk(q_idx, w, kp, r: int, budget: int, q_pos0=None, rows=None):
    """Top-k block selection.  Returns (sel int32 [n, kb], sel_score f32 [n, kb],
    margin f64 [n], s_cut f64 [n])."""
    q_idx = _c(q_idx, np.uint16)
    w = _c(w, np.float32)
    kp = _c(kp, np.uint16)
    B, Tq, Hi, Di = q_idx.shape
    N = kp.shape[1]
    rows, pos = _rows_pos(B, Tq, q_pos0, rows)
    kb = budget // r
    sel = np.empty((rows.size, kb), np.int32)
    sel_score = np.empty((rows.size, kb), np.float32)
    margin = np.empty(rows.size, np.float64)
    s_cut = np.empty(rows.size, np.float64)
    _check(_load().qsa_oracle_index_topk_rows(
        _p(q_idx), _p(w), _p(kp), B, Tq, N, Hi, Di, r, budget, _p(rows),
        _p(pos), rows.size, _p(sel), _p(sel_score), _p(margin), _p(s_cut)),
        "index_topk")
    return sel, sel_score, margin, s_cut


def attn(q, k, v, r: int, scale: float, sel=None, q_pos0=None, rows=None,
         kb: int | None = None):
    """Sparse (sel given, [n, kb] int32 for the rows) or dense causal attention.

    q [B, Tq, Hq, D], k/v [B, Tk, Hkv, D] uint16.  Returns (o f64 [n, Hq, D],
    lse f64 [n, Hq]).
    """
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    B, Tq, Hq, D = q.shape
    Tk, Hkv = k.shape[1], k.shape[2]
    rows, pos = _rows_pos(B, Tq, q_pos0, rows)
    if sel is not None:
        sel = _c(sel, np.int32)
        assert sel.shape[0] == rows.size
        kb = sel.shape[1]
    kb = 0 if kb is None else kb
    o = np.empty((rows.size, Hq, D), np.float64)
    lse = np.empty((rows.size, Hq), np.float64)
    _check(_load().qsa_oracle_attn_rows(
        _p(q), _p(k), _p(v), B, Tq, Tk, Hq, Hkv, D, r, kb, float(scale),
        _p(sel), _p(rows), _p(pos), rows.size, _p(o), _p(lse)), "attn")
    return o, lse


def decode(q, q_idx, w, k_cache, v_cache, kp, seqlens, r: int, budget: int,
           scale: float):
    """One decode step per sequence: select at p = L_b - 1, then attend.

    q [B, Hq, D], q_idx [B, Hi, Di], w [B, Hi], caches [B, L_max, Hkv, D],
    kp [B, L_max//r, Di], seqlens [B].  Returns (sel, o, lse, margin, s_cut).
    """
    q = _c(q, np.uint16)[:, None]
    q_idx = _c(q_idx, np.uint16)[:, None]
    w = _c(w, np.float32)[:, None]
    pos0 = _c(seqlens, np.int64) - 1
    sel, _, margin, s_cut = index_topk(q_idx, w, kp, r, budget, q_pos0=pos0)
    o, lse = attn(q, k_cache, v_cache, r, scale, sel=sel, q_pos0=pos0)
    return sel, o, lse, margin, s_cut

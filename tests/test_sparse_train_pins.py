"""Pins of the stage-2 sparse-training oracle (``oracle/sparse_train.py``):
the sparse attention backward against torch autograd of fp64
scaled_dot_product_attention (causal with a full selection; an explicit
boolean mask for a random one) and against central finite differences; the
stage-2 indexer loss against the stage-1 oracle when every block is selected,
against the C oracle's sparse attention with one-hot values for its teacher,
and against finite differences for its gradients.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import distill, sparse_train


def _np_bf16(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _inputs(seed, T=32, Hq=4, Hkv=2, D=8, Hi=2, Di=4, B=1):
    rng = np.random.default_rng(seed)
    q = _np_bf16(rng.standard_normal((B, T, Hq, D)))
    k = _np_bf16(rng.standard_normal((B, T, Hkv, D)))
    v = _np_bf16(rng.standard_normal((B, T, Hkv, D)))
    qi = _np_bf16(rng.standard_normal((B, T, Hi, Di)))
    ki = _np_bf16(rng.standard_normal((B, T, Di)))
    lg = rng.standard_normal((B, T, Hi))
    w = (np.exp(lg) / np.exp(lg).sum(-1, keepdims=True)).astype(np.float32)
    return q, k, v, qi, w, ki


def _random_selection(T, r, kb, seed):
    """Own block plus up to kb - 1 random earlier blocks per row, -1 padded."""
    rng = np.random.default_rng(seed)
    sel = np.full((1, T, kb), -1, np.int32)
    for t in range(T):
        c = t // r
        others = rng.permutation(c)[: kb - 1] if c else np.zeros(0, int)
        row = np.sort(np.concatenate([others, [c]]))
        sel[0, t, : row.size] = row
    return sel


def _full_selection(T, r):
    N = -(-T // r)
    sel = np.tile(np.arange(N, dtype=np.int32), (1, T, 1))
    return sel


def _torch_ref(q, k, v, do, scale, mask=None):
    f = lambda a: torch.tensor(oracle.bf16_bits_to_f64(a), dtype=torch.float64)
    qt, kt, vt = (f(a).transpose(1, 2).requires_grad_() for a in (q, k, v))  # [B, H, T, D]
    kw = dict(scale=scale, enable_gqa=True)
    if mask is None:
        o = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True, **kw)
    else:
        o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.tensor(mask), **kw)
    o.backward(torch.tensor(do).transpose(1, 2))
    tr = lambda a: a.detach().transpose(1, 2).numpy()
    return tr(o), tr(qt.grad), tr(kt.grad), tr(vt.grad)


def test_sparse_backward_full_selection_equals_causal_sdpa_autograd():
    q, k, v, *_ = _inputs(1, T=29)
    do = np.random.default_rng(2).standard_normal(q.shape)
    got = sparse_train.sparse_attn_backward(q, k, v, _full_selection(29, 4), do, 4, 0.31)
    o, dq, dk, dv = _torch_ref(q, k, v, do, 0.31)
    for name, ref in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv)):
        assert np.allclose(got[name], ref, rtol=1e-11, atol=1e-12), name


def test_sparse_backward_random_selection_equals_masked_sdpa_autograd():
    T, r, kb = 40, 4, 3
    q, k, v, *_ = _inputs(3, T=T)
    sel = _random_selection(T, r, kb, 4)
    do = np.random.default_rng(5).standard_normal(q.shape)
    got = sparse_train.sparse_attn_backward(q, k, v, sel, do, r, 0.4)
    mask = np.zeros((T, T), bool)
    for t in range(T):
        for j in sel[0, t]:
            if j >= 0:
                for u in range(j * r, j * r + r):
                    mask[t, u] = u <= t
    o, dq, dk, dv = _torch_ref(q, k, v, do, 0.4, mask)
    for name, ref in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv)):
        assert np.allclose(got[name], ref, rtol=1e-11, atol=1e-12), name
    # the forward is the C oracle's sparse attention
    o_c, _ = oracle.attn(q, k, v, r, 0.4, sel=sel[0])
    assert np.allclose(got["o"][0], o_c, rtol=1e-12, atol=1e-13)


def test_sparse_backward_matches_central_differences():
    T, r, kb = 20, 4, 2
    q, k, v, *_ = _inputs(6, T=T, Hq=2, Hkv=1, D=4)
    sel = _random_selection(T, r, kb, 7)[0]
    qf, kf, vf = (oracle.bf16_bits_to_f64(a[0]) for a in (q, k, v))
    do = np.random.default_rng(8).standard_normal(qf.shape)
    _, dq, dk, dv = sparse_train.sparse_attn_backward_f64(qf, kf, vf, sel, do, r, 0.5)
    eps = 1e-6

    def loss():
        return np.sum(sparse_train.sparse_attn_backward_f64(qf, kf, vf, sel, do, r, 0.5)[0] * do)

    for arr, grad in ((qf, dq), (kf, dk), (vf, dv)):
        for idx in list(np.ndindex(arr.shape))[::3]:
            a0 = arr[idx]
            arr[idx] = a0 + eps
            up = loss()
            arr[idx] = a0 - eps
            dn = loss()
            arr[idx] = a0
            assert math.isclose((up - dn) / (2 * eps), grad[idx], rel_tol=1e-6, abs_tol=1e-8), idx


def test_stage2_loss_with_every_block_selected_is_stage1():
    q, k, _, qi, w, ki = _inputs(9, T=36)
    full = _full_selection(36, 4)
    s2 = sparse_train.index_distill_sparse(q, k, qi, w, ki, full, 4, 0.3)
    s1 = distill.index_distill(q, k, qi, w, ki, 4, 0.3)
    for name in s1:
        assert np.allclose(s2[name], s1[name], rtol=1e-11, atol=1e-14), name


def test_stage2_teacher_matches_c_sparse_attention_with_one_hot_values():
    T, r, kb = 48, 4, 4
    q, k, *_ = _inputs(10, T=T, D=16)
    sel = _random_selection(T, r, kb, 11)
    vv = np.zeros((1, T, 2, 16), np.float32)
    for u in range(T):
        vv[0, u, :, u // r] = 1.0
    o, _ = oracle.attn(q, k, _np_bf16(vv), r, 0.45, sel=sel[0])   # per-head block masses
    qf, kf = oracle.bf16_bits_to_f64(q[0]), oracle.bf16_bits_to_f64(k[0])
    for t in range(T):
        blocks, pi = sparse_train.sparse_teacher_block_probs(qf[t], kf, sel[0, t], r, 0.45, t)
        want_blocks = np.sort(sel[0, t][(sel[0, t] >= 0) & (sel[0, t] < t // r)])
        assert np.array_equal(blocks, want_blocks)
        if blocks.size:
            a = o[t][:, blocks].sum(axis=0)                      # sum over heads
            assert np.allclose(pi, a / a.sum(), rtol=1e-12, atol=1e-15)


def test_stage2_gradients_match_central_differences():
    T, r, kb = 36, 4, 4
    q, k, _, qi, w, ki = _inputs(12, T=T, Hq=2, Hkv=1, D=4, Hi=2, Di=3)
    sel = _random_selection(T, r, kb, 13)[0]
    qf, kf = oracle.bf16_bits_to_f64(q[0]), oracle.bf16_bits_to_f64(k[0])
    qif = oracle.bf16_bits_to_f64(qi[0])
    wf = w[0].astype(np.float64)
    kpf = oracle.bf16_bits_to_f64(ki[0]).reshape(-1, r, 3).mean(axis=1)
    _, dqi, dw, dkp = sparse_train.sparse_distill_rows_f64(qf, kf, qif, wf, kpf, sel, r, 0.5)
    loss = lambda: sparse_train.sparse_distill_rows_f64(qf, kf, qif, wf, kpf, sel, r, 0.5)[0].sum()
    eps = 1e-6
    for arr, grad in ((qif, dqi), (wf, dw), (kpf, dkp)):
        for idx in np.ndindex(arr.shape):
            a0 = arr[idx]
            arr[idx] = a0 + eps
            up = loss()
            arr[idx] = a0 - eps
            dn = loss()
            arr[idx] = a0
            assert math.isclose((up - dn) / (2 * eps), grad[idx], rel_tol=1e-6, abs_tol=1e-8), idx
    assert np.abs(dkp).max() > 0 and np.abs(dqi).max() > 0

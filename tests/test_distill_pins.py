"""Pins of the stage-1 distillation oracle (``oracle/distill.py``) against
things other than itself: a hand-derived worked example (tests/golden), the
oracle's own C attention used through one-hot values (a second, separately
pinned code path for the teacher), scipy's softmax and relative entropy,
central finite differences of the loss for every gradient, and a constructed
indexer whose distribution equals the teacher's (loss and gradients vanish).
A dropped head, a wrong block sum, a missing renormalisation, a sign slip in
the score gradient or a wrong ReLU mask fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
from scipy.special import softmax
from scipy.stats import entropy

import oracle
from oracle import distill

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _np_bf16(x):
    # truncation is fine for generating inputs (any bf16 pattern is valid)
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _inputs(seed, T=24, Hq=4, Hkv=2, D=8, Hi=2, Di=4, B=1):
    rng = np.random.default_rng(seed)
    q = _np_bf16(rng.standard_normal((B, T, Hq, D)))
    k = _np_bf16(rng.standard_normal((B, T, Hkv, D)))
    qi = _np_bf16(rng.standard_normal((B, T, Hi, Di)))
    ki = _np_bf16(rng.standard_normal((B, T, Di)))
    lg = rng.standard_normal((B, T, Hi))
    w = (np.exp(lg) / np.exp(lg).sum(-1, keepdims=True)).astype(np.float32)
    return q, k, qi, w, ki


def test_distill_golden_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "distill_12tok.json")))
    T, r = g["T"], g["r"]
    q = _np_bf16(np.full((1, T, 1, 2), g["q_value"]))
    k = _np_bf16(np.full((1, T, 1, 2), g["k_value"]))
    ki = np.zeros((1, T, 2), np.float32)
    ki[0, :r] = g["k_idx_first_block"]
    qi = _np_bf16(np.tile(np.float32(g["q_idx"]), (1, T, 1, 1)))
    w = np.full((1, T, 1), g["w"], np.float32)
    out = distill.index_distill(q, k, qi, w, _np_bf16(ki), r, 1.0)
    ex = g["expected"]
    kl = out["kl"][0]
    assert np.all(kl[:8] == 0) and np.allclose(kl[8:], ex["kl_rows_8_to_11"], rtol=1e-13)
    gg = ex["g"]
    assert np.allclose(out["dw"][0, 8:, 0], gg, rtol=1e-13) and np.all(out["dw"][0, :8] == 0)
    assert np.allclose(out["dq_idx"][0, 8:, 0], [gg, 0.0], rtol=1e-13, atol=0)
    assert np.allclose(out["dk_pooled"][0, 0], ex["dk_pooled_block0"], rtol=1e-13)
    assert np.all(out["dk_pooled"][0, 1:] == 0)
    assert np.allclose(out["dk_idx"][0, :r], [gg, 0.0], rtol=1e-13) and np.all(out["dk_idx"][0, r:] == 0)


def test_teacher_matches_c_attention_with_one_hot_values():
    """Attention with value rows e_{u // r} returns, per head, the attention mass
    on every block: the teacher's numerator, from the C oracle's attention."""
    q, k, _, _, _ = _inputs(3, T=40, Hq=4, Hkv=2, D=16)
    r, scale, T = 4, 0.37, 40
    N = T // r
    v = np.zeros((1, T, 2, 16), np.float32)
    for u in range(T):
        v[0, u, :, u // r] = 1.0
    o, _ = oracle.attn(q, k, _np_bf16(v), r, scale)        # dense causal, fp64
    qf, kf = oracle.bf16_bits_to_f64(q[0]), oracle.bf16_bits_to_f64(k[0])
    for p in range(T):
        c = p // r
        pi = distill.teacher_block_probs(qf[p], kf, r, scale, p)
        assert pi.shape == (c,)
        if c == 0:
            continue
        a = o[p, :, :c].sum(axis=0)                          # sum over heads
        assert np.allclose(pi, a / a.sum(), rtol=1e-12, atol=1e-15)
        assert math.isclose(pi.sum(), 1.0, rel_tol=1e-14)
        assert np.all(o[p, :, N:] == 0)


def test_teacher_token_level_single_head_is_softmax_over_earlier_tokens():
    """r = 1, one head: the teacher is the softmax of the row's logits over the
    tokens before it (its own token is its own block, never a candidate)."""
    q, k, _, _, _ = _inputs(5, T=17, Hq=1, Hkv=1, D=8)
    qf, kf = oracle.bf16_bits_to_f64(q[0]), oracle.bf16_bits_to_f64(k[0])
    for p in range(1, 17):
        pi = distill.teacher_block_probs(qf[p], kf, 1, 0.5, p)
        want = softmax(0.5 * (kf[:p, 0] @ qf[p, 0]))
        assert np.allclose(pi, want, rtol=1e-12, atol=1e-16)


def test_kl_is_relative_entropy_of_score_softmax():
    q, k, qi, w, ki = _inputs(7, T=48)
    r, scale = 4, 0.3
    out = distill.index_distill(q, k, qi, w, ki, r, scale)
    kp = oracle.pool(ki, r)
    s = oracle.index_scores(qi, w, kp, r)                   # C oracle, fp64, -inf off-causal
    qf, kf = oracle.bf16_bits_to_f64(q[0]), oracle.bf16_bits_to_f64(k[0])
    for p in range(48):
        c = p // r
        if c < 2:
            assert out["kl"][0, p] == 0
            assert not out["dq_idx"][0, p].any() and not out["dw"][0, p].any()
            continue
        pi = distill.teacher_block_probs(qf[p], kf, r, scale, p)
        want = entropy(pi, softmax(s[p, :c]))
        assert out["kl"][0, p] >= 0
        assert math.isclose(out["kl"][0, p], want, rel_tol=1e-10, abs_tol=1e-15)


def _loss_f64(qf, kf, qif, wf, kpf, r, scale):
    return distill.distill_rows_f64(qf, kf, qif, wf, kpf, r, scale)[0].sum()


def test_gradients_match_central_differences():
    q, k, qi, w, ki = _inputs(11, T=28, Hq=2, Hkv=1, D=4, Hi=2, Di=3)
    r, scale = 4, 0.6
    qf, kf = oracle.bf16_bits_to_f64(q[0]), oracle.bf16_bits_to_f64(k[0])
    qif = oracle.bf16_bits_to_f64(qi[0])
    wf = w[0].astype(np.float64)
    kif = oracle.bf16_bits_to_f64(ki[0])
    kpf = kif.reshape(-1, r, kif.shape[-1]).mean(axis=1)
    _, dqi, dw, dkp = distill.distill_rows_f64(qf, kf, qif, wf, kpf, r, scale)
    eps = 1e-6

    def fd(arr, idx, f):
        a0 = arr[idx]
        arr[idx] = a0 + eps
        up = f()
        arr[idx] = a0 - eps
        dn = f()
        arr[idx] = a0
        return (up - dn) / (2 * eps)

    loss = lambda: _loss_f64(qf, kf, qif, wf, kpf, r, scale)
    for idx in np.ndindex(qif.shape):
        assert math.isclose(fd(qif, idx, loss), dqi[idx], rel_tol=1e-6, abs_tol=1e-8), idx
    for idx in np.ndindex(wf.shape):
        assert math.isclose(fd(wf, idx, loss), dw[idx], rel_tol=1e-6, abs_tol=1e-8), idx
    for idx in np.ndindex(kpf.shape):
        assert math.isclose(fd(kpf, idx, loss), dkp[idx], rel_tol=1e-6, abs_tol=1e-8), idx
    # the raw indexer keys, through the mean pool (bf16 rounding as the identity)
    dk = np.repeat(dkp / r, r, axis=0)

    def loss_raw():
        kp = kif.reshape(-1, r, kif.shape[-1]).mean(axis=1)
        return _loss_f64(qf, kf, qif, wf, kp, r, scale)

    for idx in [(0, 0), (5, 2), (13, 1), (22, 0), (27, 2)]:
        assert math.isclose(fd(kif, idx, loss_raw), dk[idx], rel_tol=1e-6, abs_tol=1e-8), idx
    assert not dqi[: 2 * r].any()                   # rows with < 2 candidates


def test_indexer_equal_to_teacher_has_zero_loss_and_gradient():
    """One indexer head with w = 1 and pooled keys Kp_j = (ln pi_j + C) u for a
    unit query u: the scores are ln pi_j + C, so the student is the teacher."""
    q, k, _, _, _ = _inputs(13, T=64, Hq=2, Hkv=1, D=8)
    r, scale, p = 4, 0.5, 63
    c = p // r
    qf, kf = oracle.bf16_bits_to_f64(q[0]), oracle.bf16_bits_to_f64(k[0])
    pi = distill.teacher_block_probs(qf[p], kf, r, scale, p)
    u = np.array([0.6, 0.8, 0.0])
    kpf = np.zeros((64 // r, 3))
    kpf[:c] = (np.log(pi) + 40.0)[:, None] * u[None, :]
    qif = np.tile(u, (64, 1, 1))
    wf = np.ones((64, 1))
    kl, dqi, dw, dkp = distill.distill_rows_f64(qf, kf, qif, wf, kpf, r, scale, rows=[p])
    assert abs(kl[0]) < 1e-12
    assert np.abs(dqi).max() < 1e-10 and np.abs(dw).max() < 1e-10 and np.abs(dkp).max() < 1e-10
    kpf[0] *= 1.01                                 # any departure gives a positive loss
    assert distill.distill_rows_f64(qf, kf, qif, wf, kpf, r, scale, rows=[p])[0][0] > 1e-8


def test_batch_rows_are_independent_and_rows_subset_agrees():
    q, k, qi, w, ki = _inputs(17, T=32, B=2)
    r, scale = 4, 0.35
    full = distill.index_distill(q, k, qi, w, ki, r, scale)
    for b in range(2):
        one = distill.index_distill(q[b:b + 1], k[b:b + 1], qi[b:b + 1], w[b:b + 1],
                                    ki[b:b + 1], r, scale)
        for name in full:
            assert np.array_equal(full[name][b], one[name][0])
    rows = np.array([9, 20, 31])
    sub = distill.index_distill(q, k, qi, w, ki, r, scale, rows=rows)
    assert np.array_equal(sub["kl"], full["kl"][:, rows])
    assert np.array_equal(sub["dq_idx"], full["dq_idx"][:, rows])

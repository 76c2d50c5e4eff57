"""Gated DeltaNet (gated delta rule) token mixing, CPU oracle -- TEST INFRASTRUCTURE,
NOT PART OF THE PRODUCT PATH.

Plain numpy, fp64, the recurrence one token at a time.  Only ``tests/`` may
import it.

Sources: the article "用125亿分之6的参数，打平3970亿的旗舰模型", section on the
hybrid token mixing (three Gated DeltaNet layers for every global-attention
layer): GDN keeps a matrix state; for each new token it measures the error
between what the token carries and what the memory already returns for it, and
updates the state under two gates, a decay gate that sets how much of the old
memory survives and a write gate that sets how much of the new information is
written, so repeated content overwrites instead of piling up.  The paper
summary "On the Design of Qwen3.8-Next Architecture", token-mixing paragraph:
GDN compresses the prefix into a fixed-size recurrent state with a decay gate
and delta writes, so decoding needs no cache that grows with length.

Readings (the pages give no formula; this is the plainest statement of the
gated delta rule the text describes):
  * one state S in R^{dv x dk} per (sequence, head), S_0 given (zero by default);
  * for token t with key k_t, value v_t, query q_t, decay gate alpha_t in [0, 1]
    and write gate beta_t in [0, 1]:
        S_t = alpha_t S_{t-1} + beta_t (v_t - alpha_t S_{t-1} k_t) k_t^T
    (the error v_t - alpha_t S_{t-1} k_t is what the decayed memory still lacks
    for k_t), and the output reads the updated state: o_t = S_t q_t;
  * keys, queries and gates are taken as given (any normalisation or scaling
    is the caller's); heads are independent.
Decode is the same update for one token from a carried state.

bf16 inputs cross as ``numpy.uint16`` bit patterns or as float arrays; gates
and states are float.
"""
from __future__ import annotations

import numpy as np

from . import bf16_bits_to_f64


def _f64(a):
    a = np.asarray(a)
    return bf16_bits_to_f64(a) if a.dtype == np.uint16 else a.astype(np.float64)


def gdn_recurrent(q, k, v, alpha, beta, state0=None):
    """The gated delta rule over a whole batch, token by token.

    q, k [B, T, H, dk], v [B, T, H, dv] (uint16 bf16 bits or float),
    alpha, beta [B, T, H], state0 [B, H, dv, dk] or None (zeros).
    Returns (o [B, T, H, dv], state [B, H, dv, dk]) in float64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    alpha, beta = _f64(alpha), _f64(beta)
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dv, dk)) if state0 is None else np.array(state0, np.float64)
    o = np.zeros((B, T, H, dv))
    for b in range(B):
        for h in range(H):
            St = S[b, h]
            for t in range(T):
                a, be = alpha[b, t, h], beta[b, t, h]
                kt = k[b, t, h]
                err = v[b, t, h] - a * (St @ kt)
                St = a * St + be * np.outer(err, kt)
                o[b, t, h] = St @ q[b, t, h]
            S[b, h] = St
    return o, S


def gdn_decode_step(q, k, v, alpha, beta, state):
    """One token per sequence: q, k [B, H, dk], v [B, H, dv], alpha, beta [B, H],
    state [B, H, dv, dk].  Returns (o [B, H, dv], new state)."""
    o, S = gdn_recurrent(_f64(q)[:, None], _f64(k)[:, None], _f64(v)[:, None],
                         _f64(alpha)[:, None], _f64(beta)[:, None], state)
    return o[:, 0], S

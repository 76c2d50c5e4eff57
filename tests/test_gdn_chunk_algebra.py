"""The chunked rewrite of the gated delta rule that the chunked prefill kernel
computes, checked on the CPU in fp64 against the oracle's token-by-token
recurrence (``oracle/gdn.py``).

The rewrite ("用125亿分之6的参数，打平3970亿的旗舰模型", hybrid token-mixing
section; "On the Design of Qwen3.8-Next Architecture", token-mixing paragraph:
the gated delta rule over chunks): with gamma_t the product of the chunk's
decay gates up to t, S0 the state entering the chunk and R_tj = gamma_t /
gamma_j,
    (I + A) U = diag(beta) V - diag(beta gamma) K S0^T,  A = strict_lower(diag(beta) R o K K^T)
    U = Ut - W S0^T,  Ut = (I + A)^-1 diag(beta) V,  W = (I + A)^-1 diag(beta gamma) K
    O = diag(gamma) Q S0^T + lower(R o Q K^T) U
    S = gamma_last S0 + U^T diag(gamma_last / gamma) K
with the gate ratios taken from log prefix sums whose terms are floored at -80
(a zero gate).  This pins the derivation itself, independently of the GPU: a
ratio taken the wrong way round, P without its diagonal, or the state update
without its decay each fail here (the last test plants them).
"""
import numpy as np
import pytest

from oracle import gdn

C = 64
LOG_FLOOR = -80.0


def _inputs(seed, B, T, H, dk, dv):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    alpha = rng.uniform(0.8, 1.0, (B, T, H))
    beta = rng.uniform(0.0, 1.0, (B, T, H))
    s0 = 0.5 * rng.standard_normal((B, H, dv, dk))
    return q, k, v, alpha, beta, s0


def _chunked(q, k, v, alpha, beta, s0, slip=None):
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    S = np.array(s0, np.float64)
    for b in range(B):
        for h in range(H):
            St = S[b, h]
            for c0 in range(0, T, C):
                sl = slice(c0, min(c0 + C, T))
                K, Q, V = k[b, sl, h], q[b, sl, h], v[b, sl, h]
                a, be = alpha[b, sl, h], beta[b, sl, h]
                with np.errstate(divide="ignore"):
                    ell = np.cumsum(np.maximum(np.log(a), LOG_FLOOR))
                gam = np.exp(ell)
                R = np.exp(ell[:, None] - ell[None, :])
                if slip == "ratio":
                    R = np.exp(ell[None, :] - ell[:, None])
                n = len(a)
                A = np.tril(be[:, None] * R * (K @ K.T), -1)
                P = np.tril(R * (Q @ K.T), -1 if slip == "p_diag" else 0)
                M = np.eye(n) + A
                Ut = np.linalg.solve(M, be[:, None] * V)
                W = np.linalg.solve(M, (be * gam)[:, None] * K)
                U = Ut - W @ St.T
                o[b, sl, h] = gam[:, None] * (Q @ St.T) + P @ U
                g = np.exp(ell[-1] - ell)
                St = (1.0 if slip == "decay" else gam[-1]) * St + U.T @ (g[:, None] * K)
            S[b, h] = St
    return o, S


def _close(x, ref):
    return np.abs(x - ref).max() <= 1e-10 * max(np.abs(ref).max(), 1.0)


@pytest.mark.parametrize("B,T,H,dk,dv", [(1, 150, 2, 8, 6), (2, 64, 1, 5, 7), (1, 1, 3, 4, 4),
                                         (1, 200, 1, 16, 16)])
def test_chunk_form_equals_the_recurrence(B, T, H, dk, dv):
    """Full chunks, a partial last chunk and a single token."""
    q, k, v, a, b, s0 = _inputs(B * 1000 + T, B, T, H, dk, dv)
    o, S = _chunked(q, k, v, a, b, s0)
    o_ref, S_ref = gdn.gdn_recurrent(q, k, v, a, b, s0)
    assert _close(o, o_ref) and _close(S, S_ref)


def test_chunk_form_with_gates_at_their_ends():
    """A zero decay gate inside a chunk (the floored log leaves a factor of
    e^-80 where the recurrence has 0), decay gates of 1, write gates of 0 and 1."""
    q, k, v, a, b, s0 = _inputs(5, 1, 190, 2, 6, 5)
    a[:, 70] = 0.0
    a[:, 100:120] = 1.0
    b[:, 20:30] = 0.0
    b[:, 150] = 1.0
    o, S = _chunked(q, k, v, a, b, s0)
    o_ref, S_ref = gdn.gdn_recurrent(q, k, v, a, b, s0)
    assert _close(o, o_ref) and _close(S, S_ref)


@pytest.mark.parametrize("slip", ["ratio", "p_diag", "decay"])
def test_planted_slips_in_the_chunk_form_are_caught(slip):
    q, k, v, a, b, s0 = _inputs(9, 1, 150, 2, 8, 6)
    o, S = _chunked(q, k, v, a, b, s0, slip=slip)
    o_ref, S_ref = gdn.gdn_recurrent(q, k, v, a, b, s0)
    assert not (_close(o, o_ref) and _close(S, S_ref))

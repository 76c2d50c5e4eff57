"""Pins of the gated delta rule oracle (``oracle/gdn.py``): a hand-derived
three-token example, closed forms of the degenerate gates (no write, no decay,
full decay), the gated-linear-attention closed form that the rule reduces to
for orthonormal keys, the delta property (a full-strength write of a unit key
makes the memory return exactly its value), and the state carried from a
prefill through decode steps.  A missing decay on the error term, a transposed
outer product, or reading the state before the update fails at least one.
"""
import json
import os

import numpy as np

from oracle import gdn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(seed, B=2, T=9, H=3, dk=5, dv=4):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    alpha = rng.uniform(0.5, 1.0, (B, T, H))
    beta = rng.uniform(0.0, 1.0, (B, T, H))
    S0 = rng.standard_normal((B, H, dv, dk))
    return q, k, v, alpha, beta, S0


def test_gdn_golden_three_tokens():
    g = json.load(open(os.path.join(GOLDEN, "gdn_3step.json")))
    sh = lambda x: np.asarray(x, np.float64)[None, :, None]
    o, S = gdn.gdn_recurrent(sh(g["q"]), sh(g["k"]), sh(g["v"]), sh(g["alpha"]), sh(g["beta"]))
    assert np.array_equal(o[0, :, 0], np.asarray(g["expected_o"]))
    assert np.array_equal(S[0, 0], np.asarray(g["expected_state"]))


def test_no_write_keeps_the_decayed_initial_state():
    q, k, v, alpha, beta, S0 = _rand(1)
    o, S = gdn.gdn_recurrent(q, k, v, alpha, np.zeros_like(beta), S0)
    decay = np.cumprod(alpha, axis=1)                                  # prod_{s<=t} alpha_s
    want = decay[..., None] * np.einsum("bhvk,bthk->bthv", S0, q)
    assert np.allclose(o, want, rtol=1e-12, atol=1e-12)
    assert np.allclose(S, decay[:, -1, :, None, None] * S0, rtol=1e-12, atol=1e-12)
    o1, S1 = gdn.gdn_recurrent(q, k, v, np.ones_like(alpha), np.zeros_like(beta), S0)
    assert np.allclose(S1, S0) and np.allclose(o1, np.einsum("bhvk,bthk->bthv", S0, q))


def test_full_decay_keeps_only_the_current_write():
    q, k, v, alpha, beta, S0 = _rand(2)
    o, _ = gdn.gdn_recurrent(q, k, v, np.zeros_like(alpha), beta, S0)
    want = beta[..., None] * np.einsum("bthk,bthk->bth", k, q)[..., None] * v
    assert np.allclose(o, want, rtol=1e-12, atol=1e-12)


def test_orthonormal_keys_reduce_to_gated_linear_attention():
    """With mutually orthonormal keys nothing earlier is stored under k_t, so the
    error is v_t and o_t = sum_{i<=t} (prod_{i<s<=t} alpha_s) beta_i (k_i . q_t) v_i."""
    rng = np.random.default_rng(3)
    T, dk, dv = 6, 8, 3
    basis, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = basis[:T][None, :, None]                                       # [1, T, 1, dk]
    q = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    alpha = rng.uniform(0.3, 1.0, (1, T, 1))
    beta = rng.uniform(0.1, 1.0, (1, T, 1))
    o, _ = gdn.gdn_recurrent(q, k, v, alpha, beta)
    for t in range(T):
        want = np.zeros(dv)
        for i in range(t + 1):
            w = np.prod(alpha[0, i + 1:t + 1, 0]) * beta[0, i, 0] * (k[0, i, 0] @ q[0, t, 0])
            want += w * v[0, i, 0]
        assert np.allclose(o[0, t, 0], want, rtol=1e-12, atol=1e-12), t


def test_full_write_of_a_unit_key_returns_its_value():
    q, k, v, alpha, _, S0 = _rand(4)
    beta = np.ones_like(alpha)
    o, _ = gdn.gdn_recurrent(k, k, v, alpha, beta, S0)                 # read with q = k_t
    assert np.allclose(o, v, rtol=1e-12, atol=1e-12)


def test_state_carries_from_prefill_through_decode_steps():
    q, k, v, alpha, beta, S0 = _rand(5, T=12)
    o_all, S_all = gdn.gdn_recurrent(q, k, v, alpha, beta, S0)
    o_pre, S = gdn.gdn_recurrent(q[:, :7], k[:, :7], v[:, :7], alpha[:, :7], beta[:, :7], S0)
    assert np.allclose(o_pre, o_all[:, :7])
    for t in range(7, 12):
        o_t, S = gdn.gdn_decode_step(q[:, t], k[:, t], v[:, t], alpha[:, t], beta[:, t], S)
        assert np.allclose(o_t, o_all[:, t], rtol=1e-12, atol=1e-12)
    assert np.allclose(S, S_all, rtol=1e-12, atol=1e-12)


def test_heads_and_sequences_are_independent():
    q, k, v, alpha, beta, S0 = _rand(6)
    o, S = gdn.gdn_recurrent(q, k, v, alpha, beta, S0)
    o1, S1 = gdn.gdn_recurrent(q[1:, :, 2:], k[1:, :, 2:], v[1:, :, 2:], alpha[1:, :, 2:],
                               beta[1:, :, 2:], S0[1:, 2:])
    assert np.array_equal(o1, o[1:, :, 2:]) and np.array_equal(S1, S[1:, 2:])

"""Stage-1 indexer distillation, CPU oracle -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT PATH.

Plain numpy, fp64, one query row at a time.  Only ``tests/`` may import it.

Source: the article "用125亿分之6的参数，打平3970亿的旗舰模型", section
"稀疏注意力：给检索建索引，也得先学会省纸" -- QSA is trained in two stages; the
first, dense distillation, trains only the indexer, teaching it to imitate the
attention distribution of the full-attention model with a KL-divergence loss.
The paper summary "On the Design of Qwen3.8-Next Architecture", token-mixing
paragraph, says the same in one clause (QSA first distils the dense attention
distribution, then trains sparsely with the backbone).

The pages give no formula.  Readings (the plainest ones the rest supports):
  * Teacher.  The dense causal softmax attention of the main layer, every one of
    its Hq heads (head h reads KV group h // (Hq / Hkv)), at the given scale:
    P_h(t, u) over the tokens u <= p.  Its mass on micro-block j is summed over
    the block's r tokens and over the heads, a(t, j) = sum_h sum_i P_h(t, r*j + i),
    and L1-normalised over the indexer's candidates (the complete blocks
    j < c = floor(p / r), the same candidates the selection ranks):
    pi(t, j) = a(t, j) / sum_{j' < c} a(t, j').  The own block is forced into
    every selection and never scored, so it takes no part.
  * Student.  The indexer's scores s(t, j) = sum_h w[t,h] * max(0, q_idx[t,h,:] . Kp[j,:])
    over the same candidates, turned into a distribution by a softmax.
  * Loss.  KL(pi_t || softmax(s_t)) per row, 0 for a row with fewer than two
    candidates; the step's loss is the sum over rows.  The teacher is a
    constant (only the indexer trains in this stage).
  * Gradients of the summed loss: dL/ds(t, j) = softmax(s_t)_j - pi(t, j);
    through the ReLU with derivative 1[q_idx . Kp > 0] (0 at the kink); to the
    raw indexer keys through the mean pool, dk_idx[r*j + i] = dKp[j] / r, the
    bf16 rounding of the pooled key taken as the identity.

All bf16 tensors cross this interface as ``numpy.uint16`` bit patterns, like
the rest of the oracle; ``w`` is float32.
"""
from __future__ import annotations

import numpy as np

from . import bf16_bits_to_f64, pool


def teacher_block_probs(qf, kf, r: int, scale: float, p: int) -> np.ndarray:
    """pi(t, .) over the candidate blocks j < floor(p / r) for one query row.

    qf [Hq, D] (the row's queries), kf [T, Hkv, D] float64.  Empty when the row
    has no candidate.
    """
    c = p // r
    if c == 0:
        return np.zeros(0)
    Hq = qf.shape[0]
    G = Hq // kf.shape[1]
    a = np.zeros(c)
    for h in range(Hq):
        logits = scale * (kf[: p + 1, h // G, :] @ qf[h])
        e = np.exp(logits - logits.max())
        prob = e / e.sum()
        a += prob[: r * c].reshape(c, r).sum(axis=1)
    return a / a.sum()


def distill_rows_f64(qf, kf, qif, wf, kpf, r: int, scale: float, rows=None, pos0: int = 0):
    """The loss and the indexer gradients for one batch row, all in float64.

    qf [Tq, Hq, D], kf [Tk, Hkv, D], qif [Tq, Hi, Di], wf [Tq, Hi], kpf [N, Di];
    query t sits at position p = pos0 + t.  Returns (kl [n], dq_idx [n, Hi, Di],
    dw [n, Hi], dkp [N, Di]) for the n requested rows, dkp summed over them.
    """
    Tq = qf.shape[0]
    rows = np.arange(Tq) if rows is None else np.asarray(rows)
    Hi, Di = qif.shape[1], qif.shape[2]
    kl = np.zeros(rows.size)
    dqi = np.zeros((rows.size, Hi, Di))
    dw = np.zeros((rows.size, Hi))
    dkp = np.zeros_like(kpf)
    for n, t in enumerate(rows):
        p = pos0 + int(t)
        c = p // r
        if c < 2:
            continue
        pi = teacher_block_probs(qf[t], kf, r, scale, p)
        dots = qif[t] @ kpf[:c].T                      # [Hi, c]
        s = wf[t] @ np.maximum(dots, 0.0)              # [c]
        m = s.max()
        log_q = s - (m + np.log(np.exp(s - m).sum()))
        nz = pi > 0
        kl[n] = np.sum(pi[nz] * (np.log(pi[nz]) - log_q[nz]))
        g = np.exp(log_q) - pi                         # dL/ds over the candidates
        dw[n] = np.maximum(dots, 0.0) @ g
        gh = (wf[t][:, None] * (dots > 0)) * g[None, :]  # [Hi, c]: dL/d(dots)
        dqi[n] = gh @ kpf[:c]
        dkp[:c] += gh.T @ qif[t]
    return kl, dqi, dw, dkp


def index_distill(q, k, q_idx, w, k_idx, r: int, scale: float, rows=None):
    """Stage-1 distillation for a whole prefill batch.

    q [B, T, Hq, D], k [B, T, Hkv, D], q_idx [B, T, Hi, Di], k_idx [B, T, Di]
    uint16 (bf16 bits); w [B, T, Hi] float32.  The indexer reads the oracle's
    pooled keys (bf16).  ``rows``: query rows of every batch row (default all).
    Returns a dict of float64 arrays: ``kl`` [B, n], ``dq_idx`` [B, n, Hi, Di],
    ``dw`` [B, n, Hi], ``dk_pooled`` [B, N, Di] and ``dk_idx`` [B, T, Di]
    (the last two summed over the requested rows).
    """
    B, T = q.shape[0], q.shape[1]
    kp = pool(k_idx, r)
    out = {"kl": [], "dq_idx": [], "dw": [], "dk_pooled": [], "dk_idx": []}
    for b in range(B):
        kl, dqi, dw, dkp = distill_rows_f64(
            bf16_bits_to_f64(q[b]), bf16_bits_to_f64(k[b]), bf16_bits_to_f64(q_idx[b]),
            np.asarray(w[b], np.float64), bf16_bits_to_f64(kp[b]), r, scale, rows)
        dk = np.zeros((T, k_idx.shape[2]))
        nb = dkp.shape[0]
        dk[: nb * r] = np.repeat(dkp / r, r, axis=0)
        for name, v in zip(out, (kl, dqi, dw, dkp, dk)):
            out[name].append(v)
    return {name: np.stack(v) for name, v in out.items()}

"""Stage-2 sparse training, CPU oracle -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT PATH.

Plain numpy, fp64, one query row at a time.  Only ``tests/`` may import it.

Source: the article "用125亿分之6的参数，打平3970亿的旗舰模型", section
"稀疏注意力：给检索建索引，也得先学会省纸" -- after the dense distillation stage,
the second stage, sparse training, trains the indexer together with the backbone
so the model adapts to the sparse attention pattern.  The pages give no formula.

Readings (the plainest ones the rest supports):
  * Sparse attention backward.  The forward is the QSA attention of the
    inference path: query t at position p, head h (KV group g = h / (Hq/Hkv)),
    attends to S(t) = the tokens r*j + i <= p of its selected blocks j, with
    o = sum_u P(u) v_g(u), P = softmax_u(scale q_h . k_g(u)).  The selection is
    discrete and held fixed; the gradients are those of the exact softmax
    attention over S(t):  dv_g(u) += P(u) do_h,  dP(u) = do_h . v_g(u),
    dS(u) = P(u) (dP(u) - do_h . o_h),  dq_h = scale sum_u dS(u) k_g(u),
    dk_g(u) += scale dS(u) q_h, summed over every (row, head) that attends to u.
  * The indexer's loss in this stage: the stage-1 loss restricted to the
    selection.  The teacher is the main layer's own (sparse) attention: the
    probabilities P_h(t, u) over S(t), summed over the r tokens of each
    selected candidate block (the selected blocks other than the forced own
    block) and over the heads, L1-normalised over those blocks.  The student is
    the softmax of the indexer scores over the same blocks.  Loss per row:
    KL(teacher || student), 0 for fewer than two selected candidates.  The
    gradients to the indexer inputs follow stage 1's rules (ReLU derivative
    1[x > 0], dk_idx = dKp / r); the teacher is a constant.

All bf16 tensors cross this interface as ``numpy.uint16`` bit patterns; ``w``
is float32 and ``do`` float64 (or float32).
"""
from __future__ import annotations

import numpy as np

from . import bf16_bits_to_f64, pool


def _token_set(sel_row: np.ndarray, p: int, r: int) -> np.ndarray:
    """Ascending token indices of the selected blocks, causal (<= p)."""
    blocks = np.unique(sel_row[sel_row >= 0])
    toks = (blocks[:, None] * r + np.arange(r)[None, :]).ravel()
    return toks[toks <= p]


def sparse_attn_backward_f64(qf, kf, vf, sel, do, r: int, scale: float, pos0: int = 0):
    """Gradients of sum(o * do) for one batch row, float64.

    qf [Tq, Hq, D], kf/vf [Tk, Hkv, D], sel [Tq, kb] int, do [Tq, Hq, D].
    Returns (o [Tq, Hq, D], dq [Tq, Hq, D], dk [Tk, Hkv, D], dv [Tk, Hkv, D]).
    """
    Tq, Hq, D = qf.shape
    G = Hq // kf.shape[1]
    o = np.zeros_like(qf)
    dq = np.zeros_like(qf)
    dk = np.zeros_like(kf)
    dv = np.zeros_like(vf)
    for t in range(Tq):
        S = _token_set(np.asarray(sel[t]), pos0 + t, r)
        if S.size == 0:
            continue
        for h in range(Hq):
            g = h // G
            K, V = kf[S, g], vf[S, g]
            logits = scale * (K @ qf[t, h])
            e = np.exp(logits - logits.max())
            P = e / e.sum()
            o[t, h] = P @ V
            dP = V @ do[t, h]
            dS = P * (dP - do[t, h] @ o[t, h])
            dq[t, h] = scale * (dS @ K)
            dk[S, g] += scale * dS[:, None] * qf[t, h][None, :]
            dv[S, g] += P[:, None] * do[t, h][None, :]
    return o, dq, dk, dv


def sparse_attn_backward(q, k, v, sel, do, r: int, scale: float):
    """Whole-batch wrapper: q [B,T,Hq,D], k/v [B,T,Hkv,D] uint16 (bf16 bits),
    sel [B,T,kb] int32, do [B,T,Hq,D] float.  Returns a dict of float64
    arrays o, dq, dk, dv."""
    out = {"o": [], "dq": [], "dk": [], "dv": []}
    for b in range(q.shape[0]):
        res = sparse_attn_backward_f64(bf16_bits_to_f64(q[b]), bf16_bits_to_f64(k[b]),
                                       bf16_bits_to_f64(v[b]), sel[b],
                                       np.asarray(do[b], np.float64), r, scale)
        for name, val in zip(out, res):
            out[name].append(val)
    return {name: np.stack(v_) for name, v_ in out.items()}


def sparse_teacher_block_probs(qf, kf, sel_row, r: int, scale: float, p: int):
    """(blocks, pi) for one row: the selected candidate blocks (ascending, the
    own block excluded) and the sparse attention's mass on them, summed over
    heads and L1-normalised.  Empty when there is no selected candidate."""
    c = p // r
    S = _token_set(np.asarray(sel_row), p, r)
    blocks = np.unique(np.asarray(sel_row)[(np.asarray(sel_row) >= 0) & (np.asarray(sel_row) < c)])
    if blocks.size == 0:
        return blocks, np.zeros(0)
    Hq = qf.shape[0]
    G = Hq // kf.shape[1]
    a = np.zeros(blocks.size)
    for h in range(Hq):
        logits = scale * (kf[S, h // G] @ qf[h])
        e = np.exp(logits - logits.max())
        prob = e / e.sum()
        for n, j in enumerate(blocks):
            a[n] += prob[(S >= j * r) & (S < (j + 1) * r)].sum()
    return blocks, a / a.sum()


def sparse_distill_rows_f64(qf, kf, qif, wf, kpf, sel, r: int, scale: float, rows=None,
                            pos0: int = 0):
    """The stage-2 indexer loss and its gradients for one batch row (float64).

    Like the stage-1 rows but over each row's selected candidate blocks, with
    the sparse attention as the teacher.  Returns (kl [n], dq_idx [n, Hi, Di],
    dw [n, Hi], dkp [N, Di])."""
    Tq = qf.shape[0]
    rows = np.arange(Tq) if rows is None else np.asarray(rows)
    Hi, Di = qif.shape[1], qif.shape[2]
    kl = np.zeros(rows.size)
    dqi = np.zeros((rows.size, Hi, Di))
    dw = np.zeros((rows.size, Hi))
    dkp = np.zeros_like(kpf)
    for n, t in enumerate(rows):
        p = pos0 + int(t)
        blocks, pi = sparse_teacher_block_probs(qf[t], kf, sel[t], r, scale, p)
        if blocks.size < 2:
            continue
        dots = qif[t] @ kpf[blocks].T                  # [Hi, m]
        s = wf[t] @ np.maximum(dots, 0.0)
        m = s.max()
        log_q = s - (m + np.log(np.exp(s - m).sum()))
        nz = pi > 0
        kl[n] = np.sum(pi[nz] * (np.log(pi[nz]) - log_q[nz]))
        g = np.exp(log_q) - pi
        dw[n] = np.maximum(dots, 0.0) @ g
        gh = (wf[t][:, None] * (dots > 0)) * g[None, :]
        dqi[n] = gh @ kpf[blocks]
        dkp[blocks] += gh.T @ qif[t]
    return kl, dqi, dw, dkp


def index_distill_sparse(q, k, q_idx, w, k_idx, sel, r: int, scale: float, rows=None):
    """Whole-batch wrapper of the stage-2 indexer loss (inputs as in
    ``distill.index_distill`` plus the selection ``sel`` [B, T, kb])."""
    B, T = q.shape[0], q.shape[1]
    kp = pool(k_idx, r)
    out = {"kl": [], "dq_idx": [], "dw": [], "dk_pooled": [], "dk_idx": []}
    for b in range(B):
        kl, dqi, dw, dkp = sparse_distill_rows_f64(
            bf16_bits_to_f64(q[b]), bf16_bits_to_f64(k[b]), bf16_bits_to_f64(q_idx[b]),
            np.asarray(w[b], np.float64), bf16_bits_to_f64(kp[b]), sel[b], r, scale, rows)
        dk = np.zeros((T, k_idx.shape[2]))
        nb = dkp.shape[0]
        dk[: nb * r] = np.repeat(dkp / r, r, axis=0)
        for name, val in zip(out, (kl, dqi, dw, dkp, dk)):
            out[name].append(val)
    return {name: np.stack(v_) for name, v_ in out.items()}

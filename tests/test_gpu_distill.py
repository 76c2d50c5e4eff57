"""GPU parity of the stage-1 indexer distillation (qsa_index_distill) against
the oracle (oracle/distill.py), through the C ABI.

The teacher's normalisers come from the library's dense attention
(qsa_dense_gqa_prefill's lse), the pooled keys from qsa_pool; the oracle
recomputes everything in fp64 from the same bf16 inputs.

Tolerance, from the arithmetic: every GPU value is an fp32 computation from
exact bf16 inputs (fp32 dot products and logits, ex2.approx for the teacher's
probabilities, fp32 sums over at most T / 4 blocks), so relative errors are of
order 1e-5; values that are differences of nearly equal terms (the score
gradient softmax - teacher) get an absolute floor.  The bar is
|gpu - ref| <= 1e-3 * max(|ref|, 1e-3 * max|ref|) per tensor.  A ReLU mask
decided differently in fp32 and fp64 (a dot product within rounding of 0)
legitimately changes a gradient by that pair's whole term: for every pair
whose oracle dot product is below 1e-4 in magnitude the bound of each
gradient element that the pair feeds is widened by the size of its term
(dw needs no widening: max(0, d) is continuous at the kink).
"""
import numpy as np
import pytest
import torch

import block_sparse_long_10_b200 as qsa
import oracle
from block_sparse_long_10_b200 import synth
from oracle import distill

pytestmark = pytest.mark.gpu
DEV = "cuda"
BF = torch.bfloat16
RTOL = 1e-3
FLOOR = 1e-3
KINK = 1e-4


def _bits(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _gpu(x, w):
    B, T, N = w.B, w.T, w.T // w.r
    f32 = dict(dtype=torch.float32, device=DEV)
    o = torch.empty_like(x["q"])
    lse = torch.empty(B, T, w.Hq, **f32)
    qsa.qsa_dense_gqa_prefill(x["q"], x["k"], x["v"], o, w.scale, lse=lse)
    kp = torch.zeros(B, N, w.Di, dtype=BF, device=DEV)
    if N:
        qsa.qsa_pool(x["k_idx"], kp, w.r)
    out = {"kl": torch.full((B, T), float("nan"), **f32),
           "dq_idx": torch.full((B, T, w.Hi, w.Di), float("nan"), **f32),
           "dw": torch.full((B, T, w.Hi), float("nan"), **f32),
           "dk_pooled": torch.full((B, N, w.Di), float("nan"), **f32),
           "dk_idx": torch.full((B, T, w.Di), float("nan"), **f32)}
    ws = qsa.workspace(qsa.qsa_index_distill_workspace_size(B, T, w.Hkv, w.r))
    qsa.qsa_index_distill(x["q"], x["k"], lse, x["q_idx"], x["w"], kp, out["kl"],
                          out["dq_idx"], out["dw"], out["dk_pooled"], ws, w.r, w.scale,
                          dk_idx=out["dk_idx"])
    assert qsa.qsa_check_device_status(ws) == 0
    torch.cuda.synchronize()
    return {n: t.cpu().numpy().astype(np.float64) for n, t in out.items()}


def _kink_allowance(x, w, rows=None):
    """Extra bounds for the gradient elements fed by a near-kink (row, block, head)."""
    B, T, N, r = w.B, w.T, w.T // w.r, w.r
    kp = oracle.bf16_bits_to_f64(oracle.pool(_bits(x["k_idx"]), r))   # [B, N, Di]
    qi = oracle.bf16_bits_to_f64(_bits(x["q_idx"]))                   # [B, T, Hi, Di]
    qf = oracle.bf16_bits_to_f64(_bits(x["q"]))
    kf = oracle.bf16_bits_to_f64(_bits(x["k"]))
    wf = x["w"].cpu().numpy().astype(np.float64)
    rows = np.arange(T) if rows is None else np.asarray(rows)
    ex = {"dq_idx": np.zeros((B, rows.size, w.Hi, w.Di)), "dk_pooled": np.zeros((B, N, w.Di)),
          "dk_idx": np.zeros((B, T, w.Di))}
    n_pairs = 0
    for b in range(B):
        for n, t in enumerate(rows):
            c = int(t) // r
            if c < 2:
                continue
            d = qi[b, t] @ kp[b, :c].T                                 # [Hi, c]
            near = np.argwhere(np.abs(d) < KINK)
            if near.size == 0:
                continue
            pi = distill.teacher_block_probs(qf[b, t], kf[b], r, w.scale, int(t))
            s_ = wf[b, t] @ np.maximum(d, 0.0)
            sm = np.exp(s_ - s_.max())
            g = sm / sm.sum() - pi
            for h, j in near:
                n_pairs += 1
                term = abs(g[j] * wf[b, t, h])
                ex["dq_idx"][b, n, h] += term * np.abs(kp[b, j])
                ex["dk_pooled"][b, j] += term * np.abs(qi[b, t, h])
                ex["dk_idx"][b, j * r:(j + 1) * r] += term * np.abs(qi[b, t, h]) / r
    return ex, n_pairs


def _close(name, gpu, ref, extra=0.0):
    assert gpu.shape == ref.shape, name
    if ref.size == 0:
        return
    assert np.isfinite(gpu).all(), name
    floor = FLOOR * max(np.abs(ref).max(), 1e-30)
    bad = np.abs(gpu - ref) > RTOL * np.maximum(np.abs(ref), floor) + extra
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, np.abs(gpu - ref), 0)), bad.shape)
        raise AssertionError(f"{name}: {bad.sum()} of {bad.size} outside tolerance; worst at {i}: "
                             f"gpu {gpu[i]!r} ref {ref[i]!r}")


def _check_full(w, seed=None):
    x = synth.make_prefill(w, DEV, seed)
    got = _gpu(x, w)
    ref = distill.index_distill(_bits(x["q"]), _bits(x["k"]), _bits(x["q_idx"]),
                                x["w"].cpu().numpy(), _bits(x["k_idx"]), w.r, w.scale)
    ex, _ = _kink_allowance(x, w)
    _close("kl", got["kl"], ref["kl"])
    _close("dw", got["dw"], ref["dw"])
    for name in ("dq_idx", "dk_pooled", "dk_idx"):
        _close(name, got[name], ref[name], ex[name])
    nb = w.T // w.r
    # rows with fewer than two candidates, and the trailing partial block, are exact zeros
    early = np.arange(w.T) < 2 * w.r
    assert not got["kl"][:, early].any() and not got["dq_idx"][:, early].any()
    assert not got["dk_idx"][:, nb * w.r:].any()
    return got, ref


def test_distill_tiny_workload():
    """The 2K-token, 4-head, 2-indexer-head workload with its planted needles."""
    _check_full(synth.WORKLOADS["prefill-2k-tiny"])


def test_distill_ragged_batch_gqa():
    """Two sequences of 1001 tokens (a trailing partial block), 8 heads on 2 KV
    heads, D = 128, 4 indexer heads of 64."""
    _check_full(synth.Workload("distill-ragged", "prefill", 2, 1001, 8, 2, 128, 4, 64, 4, 512,
                               31, 4))


@pytest.mark.parametrize("T", [1, 5, 9, 13])
def test_distill_short_sequences(T):
    got, ref = _check_full(synth.Workload(f"distill-{T}", "prefill", 1, T, 4, 1, 64, 2, 32, 4,
                                          512, 7, 0))
    assert np.all(ref["kl"][:, : min(T, 8)] == 0)


def test_distill_32k_sampled_rows():
    """The 32K-token production shape (16 heads on 2 KV heads, 4 x 64 indexer):
    the row-local outputs (loss, dq_idx, dw) of sampled rows against the oracle."""
    w = synth.WORKLOADS["prefill-32k"]
    x = synth.make_prefill(w, DEV)
    got = _gpu(x, w)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([np.array([0, 7, 8, 9, 2047, 2048, w.T - 1]),
                                     rng.integers(8, w.T, 40),
                                     np.array([t for _, t, _ in x["needles"][:8]], np.int64)]))
    q, k, qi, ki = (_bits(x[n]) for n in ("q", "k", "q_idx", "k_idx"))
    kp = oracle.bf16_bits_to_f64(oracle.pool(ki, w.r))[0]
    kl, dqi, dw, _ = distill.distill_rows_f64(
        oracle.bf16_bits_to_f64(q[0]), oracle.bf16_bits_to_f64(k[0]),
        oracle.bf16_bits_to_f64(qi[0]), x["w"][0].cpu().numpy().astype(np.float64), kp,
        w.r, w.scale, rows=rows)
    ex, _ = _kink_allowance(x, w, rows)
    _close("kl", got["kl"][0, rows], kl)
    _close("dw", got["dw"][0, rows], dw)
    _close("dq_idx", got["dq_idx"][0, rows], dqi, ex["dq_idx"][0])
    assert np.isfinite(got["dk_pooled"]).all() and np.isfinite(got["dk_idx"]).all()

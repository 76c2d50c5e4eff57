"""GPU parity of the stage-2 indexer loss (qsa_index_distill_sparse) against
the oracle (oracle/sparse_train.py), through the C ABI.

The selection comes from qsa_index_topk, the teacher's normalisers from the
sparse attention (qsa_sparse_attn_prefill's lse), the pooled keys from
qsa_pool; the oracle recomputes the loss and gradients in fp64 from the same
bf16 inputs and the same selection.

Tolerance, from the arithmetic: fp32 dot products and probabilities from
exact bf16 inputs and sums over at most budget / 4 blocks (dk_pooled by fp32
atomics in varying order), so relative errors are of order 1e-5; the bar is
|gpu - ref| <= 1e-3 * max(|ref|, 1e-3 * max|ref|) per tensor.  A ReLU mask
decided differently in fp32 and fp64 (an indexer dot product within rounding
of 0) changes a gradient by that pair's whole term, so the bound of each
element such a pair feeds is widened by the size of its term.
"""
import numpy as np
import pytest
import torch

import block_sparse_long_10_b200 as qsa
import oracle
from block_sparse_long_10_b200 import synth
from oracle import sparse_train

pytestmark = pytest.mark.gpu
DEV = "cuda"
BF = torch.bfloat16
RTOL = 1e-3
FLOOR = 1e-3
KINK = 1e-4


def _bits(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _run(w, seed=None):
    x = synth.make_prefill(w, DEV, seed=seed)
    B, T, N = w.B, w.T, w.T // w.r
    f32 = dict(dtype=torch.float32, device=DEV)
    kp = torch.zeros(B, N, w.Di, dtype=BF, device=DEV)
    if N:
        qsa.qsa_pool(x["k_idx"], kp, w.r)
    sel = torch.empty(B, T, w.kb, dtype=torch.int32, device=DEV)
    wsi = qsa.workspace(qsa.qsa_index_topk_workspace_size(B, T, N, w.Hi, w.Di, w.r, w.budget))
    qsa.qsa_index_topk(x["q_idx"], x["w"], kp, sel, wsi, w.r, w.budget)
    o = torch.empty_like(x["q"])
    lse = torch.empty(B, T, w.Hq, **f32)
    qsa.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, o, w.r, w.budget, w.scale, lse=lse)
    out = {"kl": torch.full((B, T), float("nan"), **f32),
           "dq_idx": torch.full((B, T, w.Hi, w.Di), float("nan"), **f32),
           "dw": torch.full((B, T, w.Hi), float("nan"), **f32),
           "dk_pooled": torch.full((B, N, w.Di), float("nan"), **f32),
           "dk_idx": torch.full((B, T, w.Di), float("nan"), **f32)}
    ws = qsa.workspace(qsa.qsa_index_distill_sparse_workspace_size(B, T, w.Hkv, w.r, w.budget))
    qsa.qsa_index_distill_sparse(x["q"], x["k"], lse, sel, x["q_idx"], x["w"], kp, out["kl"],
                                 out["dq_idx"], out["dw"], out["dk_pooled"], ws, w.r, w.budget,
                                 w.scale, dk_idx=out["dk_idx"])
    assert qsa.qsa_check_device_status(ws) == 0
    torch.cuda.synchronize()
    gpu = {n: t.cpu().numpy().astype(np.float64) for n, t in out.items()}
    return x, sel.cpu().numpy(), gpu


def _allowance(x, w, sel):
    """Extra bounds for the gradient elements fed by a near-kink (row, block, head)."""
    B, T, N, r = w.B, w.T, w.T // w.r, w.r
    kp = oracle.bf16_bits_to_f64(oracle.pool(_bits(x["k_idx"]), r))
    qi = oracle.bf16_bits_to_f64(_bits(x["q_idx"]))
    ex = {"dq_idx": np.zeros((B, T, w.Hi, w.Di)), "dk_pooled": np.zeros((B, N, w.Di)),
          "dk_idx": np.zeros((B, T, w.Di))}
    wf = x["w"].cpu().numpy().astype(np.float64)
    for b in range(B):
        for t in range(T):
            c = t // r
            js = sel[b, t][(sel[b, t] >= 0) & (sel[b, t] < c)]
            if js.size < 2:
                continue
            d = qi[b, t] @ kp[b, js].T                      # [Hi, m]
            hh, mm = np.nonzero(np.abs(d) < KINK)
            for h, m_ in zip(hh, mm):
                j = js[m_]
                ex["dq_idx"][b, t, h] += abs(wf[b, t, h]) * np.abs(kp[b, j])
                term = abs(wf[b, t, h]) * np.abs(qi[b, t, h])
                ex["dk_pooled"][b, j] += term
                ex["dk_idx"][b, j * r:(j + 1) * r] += term / r
    return ex


def _check(name, gpu, ref, extra=None):
    assert gpu.shape == ref.shape and np.isfinite(gpu).all(), name
    floor = FLOOR * max(np.abs(ref).max(), 1e-30)
    bound = RTOL * np.maximum(np.abs(ref), floor)
    if extra is not None:
        bound = bound + extra
    bad = np.abs(gpu - ref) > bound
    assert not bad.any(), (name, int(bad.sum()), float(np.abs(gpu - ref).max()))


CASES = [
    synth.WORKLOADS["prefill-2k-tiny"],
    synth.Workload("sds-gqa-ragged", "prefill", 2, 1001, 16, 2, 128, 4, 64, 4, 256, 9, 3),
    synth.Workload("sds-hi1", "prefill", 1, 700, 8, 4, 64, 1, 64, 4, 128, 10, 2),
    synth.Workload("sds-short", "prefill", 1, 9, 4, 1, 64, 2, 32, 4, 16, 11, 0),
]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_sparse_distill_matches_oracle(w):
    x, sel, gpu = _run(w)
    ref = sparse_train.index_distill_sparse(_bits(x["q"]), _bits(x["k"]), _bits(x["q_idx"]),
                                            x["w"].cpu().numpy(), _bits(x["k_idx"]), sel, w.r,
                                            w.scale)
    ex = _allowance(x, w, sel)
    _check("kl", gpu["kl"], ref["kl"])
    _check("dw", gpu["dw"], ref["dw"])
    _check("dq_idx", gpu["dq_idx"], ref["dq_idx"], ex["dq_idx"])
    _check("dk_pooled", gpu["dk_pooled"], ref["dk_pooled"], ex["dk_pooled"])
    _check("dk_idx", gpu["dk_idx"], ref["dk_idx"], ex["dk_idx"])
    # rows with fewer than two selected candidates have no loss
    assert np.all(gpu["kl"][:, : 2 * w.r] == 0.0)

"""GPU parity of the sparse attention backward (qsa_sparse_attn_backward)
against the stage-2 oracle (oracle/sparse_train.py), through the C ABI.

Every GPU value is fp32 arithmetic on exact bf16 inputs (fp32 dot products,
softmax statistics and sums over at most the token budget; dk and dv summed
with atomics in varying order), so relative errors are of order 1e-5.  The bar:
|gpu - ref| <= 1e-3 * max(|ref|, 1e-3 * max|ref|) per tensor.
"""
import numpy as np
import pytest
import torch

import block_sparse_long_10_b200 as qsa
from block_sparse_long_10_b200 import synth
from oracle import sparse_train

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bits(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _close(name, gpu, ref):
    assert gpu.shape == ref.shape and np.isfinite(gpu).all(), name
    floor = 1e-3 * max(np.abs(ref).max(), 1e-30)
    bad = np.abs(gpu - ref) > 1e-3 * np.maximum(np.abs(ref), floor)
    assert not bad.any(), (name, int(bad.sum()), float(np.abs(gpu - ref).max()))


def _case(w, seed=11):
    x = synth.make_prefill(w, DEV)
    B, T = w.B, w.T
    kp = torch.empty(B, T // w.r, w.Di, dtype=torch.bfloat16, device=DEV)
    qsa.qsa_pool(x["k_idx"], kp, w.r)
    sel = torch.empty(B, T, w.kb, dtype=torch.int32, device=DEV)
    ws = qsa.workspace(qsa.qsa_index_topk_workspace_size(B, T, T // w.r, w.Hi, w.Di, w.r, w.budget))
    qsa.qsa_index_topk(x["q_idx"], x["w"], kp, sel, ws, w.r, w.budget)
    g = torch.Generator(device=DEV).manual_seed(seed)
    d_o = torch.empty_like(x["q"]).normal_(generator=g)
    dq = torch.full(x["q"].shape, float("nan"), device=DEV)
    dk = torch.full(x["k"].shape, float("nan"), device=DEV)
    dv = torch.full(x["v"].shape, float("nan"), device=DEV)
    qsa.qsa_sparse_attn_backward(x["q"], x["k"], x["v"], sel, d_o, dq, dk, dv, w.r, w.budget,
                                 w.scale)
    torch.cuda.synchronize()
    ref = sparse_train.sparse_attn_backward(_bits(x["q"]), _bits(x["k"]), _bits(x["v"]),
                                            sel.cpu().numpy(), d_o.float().cpu().numpy(), w.r,
                                            w.scale)
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _close(name, t.cpu().numpy().astype(np.float64), ref[name])


def test_sparse_backward_tiny_workload():
    _case(synth.WORKLOADS["prefill-2k-tiny"])


def test_sparse_backward_ragged_gqa():
    _case(synth.Workload("sbw-ragged", "prefill", 2, 777, 16, 2, 128, 4, 64, 4, 256, 5, 2))


@pytest.mark.parametrize("T", [1, 3, 9])
def test_sparse_backward_short(T):
    _case(synth.Workload(f"sbw-{T}", "prefill", 1, T, 4, 1, 64, 2, 32, 4, 64, 6, 0))

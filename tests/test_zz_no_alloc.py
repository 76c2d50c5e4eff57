"""The workspace-free decode attention (for callers that cannot allocate
device memory where they run a decode step) against the workspace version and
against the oracle.

Collected last on purpose.  Two calls in a row through the C ABI must each
match qsa_sparse_attn_decode on the same inputs, and the oracle's attention
over the same selection, within the parity tolerances, whether this file runs
alone in a fresh process or after the other tests.  The entry point splits
each selection into its own number of slices (about 512 slices per call),
so the comparison with the oracle covers that slice configuration too."""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_long_10_b200 as qsa
import oracle
from block_sparse_long_10_b200 import synth
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _close(a, b):
    d = (a.float() - b.float()).abs()
    assert d.max().item() <= parity.O_MAX_ABS and d.mean().item() <= parity.O_MEAN_ABS


def test_noalloc_decode_matches_workspace_version_twice():
    w = synth.Workload("noalloc", "decode", 32, 16384, 16, 2, 128, 4, 64, 4, 2048, 31, 4)
    seqlens = [16384 - 37 * i for i in range(w.B)]
    x = synth.make_decode(w, DEV, seqlens=seqlens)
    B, L = w.B, w.T
    kp = torch.empty(B, L // 4, w.Di, dtype=torch.bfloat16, device=DEV)
    qsa.qsa_pool(x["k_idx_cache"], kp, 4)
    sel = torch.empty(B, w.kb, dtype=torch.int32, device=DEV)
    wsi = qsa.workspace(qsa.qsa_index_topk_decode_workspace_size(B, L // 4, 4, w.budget))
    qsa.qsa_index_topk_decode(x["q_idx"], x["w"], kp, x["seqlens"], sel, wsi, 4, w.budget)
    o_ref = torch.empty_like(x["q"])
    lse_ref = torch.empty(B, w.Hq, dtype=torch.float32, device=DEV)
    wsa = qsa.workspace(qsa.qsa_sparse_attn_decode_workspace_size(B, w.Hq, w.D, 4, w.budget))
    qsa.qsa_sparse_attn_decode(x["q"], x["k_cache"], x["v_cache"], x["seqlens"], sel, o_ref,
                               wsa, 4, w.budget, w.scale, lse=lse_ref)
    # the oracle's attention of every sequence over the same selection
    pos0 = x["seqlens"].cpu().numpy().astype(np.int64) - 1
    o_or, lse_or = oracle.attn(parity.bits(x["q"])[:, None], parity.bits(x["k_cache"]),
                               parity.bits(x["v_cache"]), 4, w.scale, sel=sel.cpu().numpy(),
                               q_pos0=pos0)
    for _ in range(2):
        o = torch.full_like(x["q"], float("nan"))
        lse = torch.full((B, w.Hq), float("nan"), dtype=torch.float32, device=DEV)
        qsa.qsa_sparse_attn_decode_noalloc(x["q"], x["k_cache"], x["v_cache"], x["seqlens"],
                                           sel, o, 4, w.budget, w.scale, lse=lse)
        torch.cuda.synchronize()
        _close(o, o_ref)
        assert (lse - lse_ref).abs().max().item() <= parity.LSE_ABS
        parity.check_attention(oracle.bf16_bits_to_f64(parity.bits(o)).reshape(B, w.Hq, w.D),
                               o_or, lse.cpu().numpy(), lse_or, "noalloc vs oracle")


def test_noalloc_rejects_batches_beyond_its_scratch():
    lib = qsa.load()
    f = ctypes.c_void_p(0x10000)
    # 4096 sequences x 1 slice x 16 heads x 130 floats = 34 MB > 8 MiB
    rc = lib.qsa_sparse_attn_decode_noalloc(f, f, f, f, 4096, f, 4096, 16, 2, 128, 4, 2048,
                                            ctypes.c_float(0.1), f, None, None)
    assert rc == 3

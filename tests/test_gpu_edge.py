"""GPU edge cases against the oracle: exact score ties, sequences shorter than
one micro-block, empty input.

Ties: indexer queries and keys drawn from {-1, 0, 1} and head weights from
{0.5, 1, 2} make every score an exact small multiple of 1/8, so the fp32
scores of the CUDA path equal the oracle's fp64 scores bit for bit and the
rule "lower block index first on equal scores" decides most of the
selection.  At 16K tokens the all-zero case keeps every candidate until the
lists reach their capacity check, which exercises the cut-and-go-strict path.
The selection is compared as an exact set, not under the margin rule.
"""
import numpy as np
import pytest
import torch

import block_sparse_long_10_b200 as qsa
import oracle
from block_sparse_long_10_b200 import synth
from tests import parity
from tests.test_gpu_parity import _check_prefill, _qsa_decode, _check_decode_rows, _qsa_prefill

pytestmark = pytest.mark.gpu
DEV = "cuda"
BF = torch.bfloat16

TIES = synth.Workload("ties-16k", "prefill", 1, 16384, 4, 2, 64, 4, 64, 4, 2048, 31, 0)


def _tied_inputs(kind: str):
    w = TIES
    x = synth.make_prefill(w, DEV)
    g = torch.Generator().manual_seed(97)
    shape_q = (w.B, w.T, w.Hi, w.Di)
    if kind == "zero":
        qi = torch.zeros(shape_q)
    else:
        qi = torch.randint(-1, 2, shape_q, generator=g).float()
    ki = torch.randint(-1, 2, (w.B, w.T, w.Di), generator=g).float()
    wt = torch.tensor([0.5, 1.0, 2.0])[torch.randint(0, 3, (w.B, w.T, w.Hi), generator=g)]
    x["q_idx"] = qi.to(BF).to(DEV)
    x["k_idx"] = ki.to(BF).to(DEV)
    x["w"] = wt.to(DEV)
    return w, x


@pytest.mark.parametrize("kind", ["zero", "ternary"])
def test_exact_ties(kind):
    w, x = _tied_inputs(kind)
    kp, sel, sc, o, lse = _qsa_prefill(x, w)
    T, K = w.T, w.kb - 1
    rows = np.unique(np.concatenate([
        np.arange(0, 16), np.arange(2040, 2060), np.arange(4 * K - 8, 4 * K + 8),
        np.arange(8180, 8200), np.linspace(0, T - 1, 200).astype(np.int64),
        np.arange(T - 160, T)])).astype(np.int64)
    h_qi = parity.bits(x["q_idx"])
    h_w = x["w"].cpu().numpy()
    kp_ref = oracle.pool(parity.bits(x["k_idx"]), w.r)
    assert np.array_equal(parity.bits(kp), kp_ref)
    sel_h = sel.view(T, w.kb).cpu().numpy()[rows]
    sc_h = sc.view(T, w.kb).cpu().numpy()[rows]
    parity.check_selection_structure(sel_h, rows, w.r, w.kb)
    sel_ref, _, _, _ = oracle.index_topk(h_qi, h_w, kp_ref, w.r, w.budget, rows=rows)
    for i, t in enumerate(rows):
        g = sorted(int(v) for v in sel_h[i] if v >= 0)
        o_ = sorted(int(v) for v in sel_ref[i] if v >= 0)
        assert g == o_, (int(t), sorted(set(g) ^ set(o_))[:8])
        if kind == "zero":  # every score is 0: the lowest blocks win, then the own block
            c = int(t) // w.r
            want = list(range(c + 1)) if c <= K else list(range(K)) + [c]
            assert g == want, int(t)
    # the kept blocks' scores are exact
    own = sel_h == (rows // w.r)[:, None]
    keep = (sel_h >= 0) & ~own
    ri, ci = np.nonzero(keep)
    if ri.size:
        ref = oracle.score_pairs(h_qi, h_w, kp_ref, rows[ri], sel_h[ri, ci])
        assert np.array_equal(sc_h[ri, ci].astype(np.float64), ref)


@pytest.mark.parametrize("T", [1, 3, 4, 5, 9])
def test_shorter_than_few_blocks(T):
    """T < 4: no complete block, every token keeps its own (partial) block."""
    w = synth.Workload(f"short-{T}", "prefill", 2, T, 4, 2, 64, 2, 32, 4, 64, 40 + T, 0)
    x = synth.make_prefill(w, DEV)
    sel, _, _ = _check_prefill(w, x)
    s = sel.cpu().numpy()
    for t in range(min(T, 4)):  # no complete block before position 4
        assert (s[:, t, 0] == 0).all() and (s[:, t, 1:] == -1).all()


def test_empty_sequence():
    w = synth.Workload("empty", "prefill", 1, 0, 4, 2, 64, 2, 32, 4, 64, 50, 0)
    z = lambda *s: torch.empty(*s, dtype=BF, device=DEV)
    q, k, v = z(1, 0, 4, 64), z(1, 0, 2, 64), z(1, 0, 2, 64)
    qi, ki = z(1, 0, 2, 32), z(1, 0, 32)
    wt = torch.empty(1, 0, 2, device=DEV)
    kp = z(1, 0, 32)
    qsa.qsa_pool(ki, kp, 4)
    sel = torch.empty(1, 0, w.kb, dtype=torch.int32, device=DEV)
    ws = qsa.workspace(qsa.qsa_index_topk_workspace_size(1, 0, 0, 2, 32, 4, 64))
    qsa.qsa_index_topk(qi, wt, kp, sel, ws, 4, 64)
    o = torch.empty_like(q)
    qsa.qsa_sparse_attn_prefill(q, k, v, sel, o, 4, 64, w.scale)
    torch.cuda.synchronize()


def test_decode_caches_shorter_than_one_block():
    w = synth.Workload("dec-short", "decode", 4, 3, 16, 2, 128, 4, 64, 4, 256, 23, 0)
    x = synth.make_decode(w, DEV, seqlens=[3, 1, 2, 3])
    kp, sel, sc, o, lse, st = _qsa_decode(x, w)
    assert st == (0, 0)
    assert (sel[:, 0] == 0).all() and (sel[:, 1:] == -1).all()
    _check_decode_rows(w, x, kp, sel, sc, o, lse, range(w.B))


def test_chunked_prefill_equals_one_shot():
    """Prefill in chunks (q_pos0 = chunk start, pooling only the blocks that each
    chunk completes) gives the same pooled keys and selections, and bit-identical
    outputs, as one call over the whole sequence."""
    w = synth.Workload("chunks", "prefill", 1, 3001, 8, 2, 128, 4, 64, 4, 256, 61, 4)
    x = synth.make_prefill(w, DEV)
    kp1, sel1, sc1, o1, lse1 = _qsa_prefill(x, w)
    T, N = w.T, w.T // w.r
    kp = torch.zeros(1, N, w.Di, dtype=BF, device=DEV)
    sel = torch.empty(1, T, w.kb, dtype=torch.int32, device=DEV)
    o = torch.empty_like(x["q"])
    lse = torch.empty(1, T, w.Hq, dtype=torch.float32, device=DEV)
    bounds = [0, 1000, 2203, T]
    done = 0
    for c0, c1 in zip(bounds[:-1], bounds[1:]):
        nb = c1 // w.r
        qsa.qsa_pool(x["k_idx"], kp, w.r, blk_begin=done, blk_end=nb)
        done = nb
        pos0 = torch.tensor([c0], dtype=torch.int64, device=DEV)
        tq = c1 - c0
        selc = torch.empty(1, tq, w.kb, dtype=torch.int32, device=DEV)
        ws = qsa.workspace(qsa.qsa_index_topk_workspace_size(1, tq, nb, w.Hi, w.Di, w.r, w.budget))
        qsa.qsa_index_topk(x["q_idx"][:, c0:c1].contiguous(), x["w"][:, c0:c1].contiguous(),
                           kp[:, :nb], selc, ws, w.r, w.budget, q_pos0=pos0)
        oc = torch.empty(1, tq, w.Hq, w.D, dtype=BF, device=DEV)
        lc = torch.empty(1, tq, w.Hq, dtype=torch.float32, device=DEV)
        qsa.qsa_sparse_attn_prefill(x["q"][:, c0:c1].contiguous(), x["k"][:, :c1].contiguous(),
                                    x["v"][:, :c1].contiguous(), selc, oc, w.r, w.budget,
                                    w.scale, q_pos0=pos0, lse=lc)
        assert qsa.qsa_check_device_status(ws) == 0
        sel[:, c0:c1] = selc
        o[:, c0:c1] = oc
        lse[:, c0:c1] = lc
    torch.cuda.synchronize()
    assert torch.equal(kp, kp1)
    assert torch.equal(sel, sel1)
    assert torch.equal(o.view(torch.int16), o1.view(torch.int16))
    assert torch.equal(lse, lse1)


@pytest.mark.parametrize("mode", ["signed", "one-head-zero"])
def test_head_weights_of_any_sign(mode):
    """The selection stays exact for head weights that are not a softmax:
    N(0,1) weights (some negative) and weights with one head at zero.  The
    prefill indexer's first pass uses a linear lower bound of the score whose
    correction term is built from the negative weights; this checks that the
    bound is valid in both cases (compared under the margin rule)."""
    w = synth.Workload(f"w-{mode}", "prefill", 2, 3000, 8, 2, 128, 4, 64, 4, 512, 41, 4)
    x = synth.make_prefill(w, DEV)
    g = torch.Generator().manual_seed(43)
    wt = torch.randn(w.B, w.T, w.Hi, generator=g)
    if mode == "one-head-zero":
        wt = wt.abs()
        wt[..., 1] = 0.0
    x["w"] = wt.to(DEV)
    _check_prefill(w, x)

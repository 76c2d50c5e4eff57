"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Small cases compare every row; the full-size workloads (32K, 128K, 1M
prefill; 64 x 256K decode) compare sampled rows -- boundary rows, every needle
row and stratified rows -- run in the same launch configuration as bench.py.
Rules and tolerances are in tests/parity.py.
"""
import dataclasses

import numpy as np
import pytest
import torch

import block_sparse_long_10_b200 as qsa
import oracle
from block_sparse_long_10_b200 import synth
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda"
BF = torch.bfloat16


def _qsa_prefill(x, w, q_pos0=None, want_lse=True):
    """pool -> index_topk -> sparse attention, through the C ABI."""
    B, T = x["q"].shape[:2]
    Tk = x["k"].shape[1]
    kp = torch.empty(B, Tk // w.r, w.Di, dtype=BF, device=DEV)
    qsa.qsa_pool(x["k_idx"], kp, w.r)
    sel = torch.empty(B, T, w.kb, dtype=torch.int32, device=DEV)
    sc = torch.empty(B, T, w.kb, dtype=torch.float32, device=DEV)
    ws = qsa.workspace(qsa.qsa_index_topk_workspace_size(B, T, kp.shape[1], w.Hi, w.Di, w.r,
                                                         w.budget))
    qsa.qsa_index_topk(x["q_idx"], x["w"], kp, sel, ws, w.r, w.budget, q_pos0=q_pos0,
                       sel_score=sc)
    o = torch.empty_like(x["q"])
    lse = torch.empty(B, T, w.Hq, dtype=torch.float32, device=DEV) if want_lse else None
    qsa.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, o, w.r, w.budget, w.scale,
                                q_pos0=q_pos0, lse=lse)
    assert qsa.qsa_check_device_status(ws) == 0
    torch.cuda.synchronize()
    return kp, sel, sc, o, lse


def _host(x):
    h = {n: parity.bits(x[n]) for n in ("q", "k", "v", "q_idx", "k_idx")}
    h["w"] = x["w"].cpu().numpy()
    return h


def _check_prefill(w, x, rows=None, q_pos0=None):
    kp, sel, sc, o, lse = _qsa_prefill(x, w)
    h = _host(x)
    kp_ref = oracle.pool(h["k_idx"], w.r)
    assert np.array_equal(parity.bits(kp), kp_ref), "pooled keys differ"
    B, T = w.B, w.T
    rows = np.arange(B * T, dtype=np.int64) if rows is None else rows
    sel_h = sel.view(B * T, w.kb).cpu().numpy()[rows]
    sc_h = sc.view(B * T, w.kb).cpu().numpy()[rows]
    n, n_exact = parity.check_selection_vs_oracle(sel_h, h["q_idx"], h["w"], kp_ref, rows, w.r,
                                                  w.budget, sel_score_gpu=sc_h)
    o_ref, lse_ref = oracle.attn(h["q"], h["k"], h["v"], w.r, w.scale, sel=sel_h, rows=rows)
    o_h = oracle.bf16_bits_to_f64(parity.bits(o)).reshape(B * T, w.Hq, w.D)[rows]
    lse_h = lse.view(B * T, w.Hq).cpu().numpy()[rows]
    parity.check_attention(o_h, o_ref, lse_h, lse_ref, w.name)
    return sel, o, n_exact


SMALL = [
    synth.WORKLOADS["prefill-2k-tiny"],
    synth.Workload("ragged-b2-t1000", "prefill", 2, 1000, 8, 2, 128, 4, 64, 4, 256, 11, 4),
    synth.Workload("hi1-di64-g2-hkv4-d64", "prefill", 1, 1536, 8, 4, 64, 1, 64, 4, 128, 12, 3),
    synth.Workload("hi4-di32-g8-hkv1", "prefill", 1, 1100, 8, 1, 128, 4, 32, 4, 200, 13, 3),
    synth.Workload("g1-hkv2-d64-hi2", "prefill", 1, 700, 2, 2, 64, 2, 64, 4, 64, 14, 2),
    synth.Workload("own-block-only", "prefill", 1, 300, 4, 1, 64, 2, 32, 4, 4, 15, 0),
    synth.Workload("budget-2048-t2048", "prefill", 1, 2048, 16, 2, 128, 4, 64, 4, 2048, 16, 0),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_prefill_all_rows(w):
    x = synth.make_prefill(w, DEV)
    _check_prefill(w, x)


def test_full_budget_is_dense_attention():
    """budget covers every prefix: QSA output = dense causal GQA (oracle)."""
    w = synth.Workload("dense-eq", "prefill", 1, 1024, 8, 2, 128, 4, 64, 4, 1024, 17, 0)
    x = synth.make_prefill(w, DEV)
    _, sel, _, o, _ = _qsa_prefill(x, w)
    h = _host(x)
    o_ref, _ = oracle.attn(h["q"], h["k"], h["v"], w.r, w.scale)  # dense
    parity.check_attention(oracle.bf16_bits_to_f64(parity.bits(o)).reshape(-1, w.Hq, w.D),
                           o_ref, what="dense-eq")


@pytest.mark.parametrize("name,n_strat", [("prefill-32k", 256), ("prefill-128k", 192),
                                          ("prefill-1m", 96)])
def test_prefill_full_size_sampled(name, n_strat):
    w = synth.WORKLOADS[name]
    x = synth.make_prefill(w, DEV)
    needle_rows = [t for (_, t, _) in x["needles"]]
    rows = parity.sample_rows(w.T, w.r, w.kb, needle_rows, n_strat, seed=w.seed)
    sel, o, n_exact = _check_prefill(w, x, rows=rows)
    assert n_exact > 0.5 * rows.size
    # every planted block is selected, and its row reads the planted value
    sel_h = sel[0].cpu().numpy()
    o_h = o[0].float().cpu().numpy()
    for (_, t, j) in x["needles"]:
        assert j in sel_h[t], (t, j)
        np.testing.assert_allclose(o_h[t, :: w.G], synth.NEEDLE_VALUE, atol=2e-2)


def test_chunked_prefill_with_q_pos0():
    """A chunk of queries at positions q_pos0 + t over a longer K/V prefix."""
    w = synth.Workload("chunk", "prefill", 2, 1536, 8, 2, 128, 4, 64, 4, 256, 18, 0)
    x = synth.make_prefill(w, DEV)
    T0, Tc = 1024, 512
    xc = dict(x)
    xc["q"] = x["q"][:, T0:].contiguous()
    xc["q_idx"] = x["q_idx"][:, T0:].contiguous()
    xc["w"] = x["w"][:, T0:].contiguous()
    pos0 = torch.full((w.B,), T0, dtype=torch.int64, device=DEV)
    kp, sel, sc, o, lse = _qsa_prefill(xc, w, q_pos0=pos0)
    h = _host(x)
    hc = _host(xc)
    kp_ref = oracle.pool(h["k_idx"], w.r)
    rows = np.arange(w.B * Tc, dtype=np.int64)
    sel_h = sel.view(-1, w.kb).cpu().numpy()
    parity.check_selection_vs_oracle(sel_h, hc["q_idx"], hc["w"], kp_ref, rows, w.r, w.budget,
                                     q_pos0=np.full(w.B, T0), sel_score_gpu=sc.view(-1, w.kb).cpu().numpy())
    o_ref, lse_ref = oracle.attn(hc["q"], h["k"], h["v"], w.r, w.scale, sel=sel_h,
                                 q_pos0=np.full(w.B, T0), rows=rows)
    parity.check_attention(oracle.bf16_bits_to_f64(parity.bits(o)).reshape(-1, w.Hq, w.D), o_ref,
                           lse.view(-1, w.Hq).cpu().numpy(), lse_ref, "chunk")


def test_pool_partial_range_and_bits():
    w = synth.WORKLOADS["prefill-128k"]
    k_idx = torch.empty(2, 4096, 64, dtype=BF, device=DEV).normal_()
    kp = torch.full((2, 1024, 64), 7.0, dtype=BF, device=DEV)
    qsa.qsa_pool(k_idx, kp, 4, 100, 613)
    ref = oracle.pool(parity.bits(k_idx), 4)
    got = parity.bits(kp)
    assert np.array_equal(got[:, 100:613], ref[:, 100:613])
    assert (kp[:, :100] == 7.0).all() and (kp[:, 613:] == 7.0).all()
    del w


def test_invalid_selection_entries_are_ignored():
    """Entries < 0, beyond the query's position or far out of range read nothing."""
    w = synth.Workload("junk-sel", "prefill", 1, 512, 8, 2, 128, 4, 64, 4, 64, 19, 0)
    x = synth.make_prefill(w, DEV)
    T = w.T
    g = torch.Generator().manual_seed(5)
    sel = torch.randint(-3, T // 4 + 40, (1, T, w.kb), generator=g, dtype=torch.int32)
    sel[0, :, 0] = 2 ** 30
    sel_d = sel.to(DEV)
    o = torch.empty_like(x["q"])
    lse = torch.empty(1, T, w.Hq, dtype=torch.float32, device=DEV)
    qsa.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel_d, o, w.r, w.budget, w.scale, lse=lse)
    torch.cuda.synchronize()
    h = _host(x)
    s = sel[0].numpy().copy()
    pos = np.arange(T)
    bad = (s < 0) | (s.astype(np.int64) * 4 > pos[:, None])
    s[bad] = -1
    # the oracle's set semantics: duplicates count once per listed entry
    o_ref, lse_ref = oracle.attn(h["q"], h["k"], h["v"], w.r, w.scale, sel=s)
    parity.check_attention(oracle.bf16_bits_to_f64(parity.bits(o)).reshape(-1, w.Hq, w.D), o_ref,
                           lse.view(-1, w.Hq).cpu().numpy(), lse_ref, "junk-sel")


# -------------------------------------------------------------------- decode

def _qsa_decode(x, w):
    B, L = w.B, w.T
    kp = torch.empty(B, L // w.r, w.Di, dtype=BF, device=DEV)
    qsa.qsa_pool(x["k_idx_cache"], kp, w.r)
    sel = torch.empty(B, w.kb, dtype=torch.int32, device=DEV)
    sc = torch.empty(B, w.kb, dtype=torch.float32, device=DEV)
    ws_i = qsa.workspace(qsa.qsa_index_topk_decode_workspace_size(B, kp.shape[1], w.r, w.budget))
    qsa.qsa_index_topk_decode(x["q_idx"], x["w"], kp, x["seqlens"], sel, ws_i, w.r, w.budget,
                              sel_score=sc)
    o = torch.empty_like(x["q"])
    lse = torch.empty(B, w.Hq, dtype=torch.float32, device=DEV)
    ws_a = qsa.workspace(qsa.qsa_sparse_attn_decode_workspace_size(B, w.Hq, w.D, w.r, w.budget))
    qsa.qsa_sparse_attn_decode(x["q"], x["k_cache"], x["v_cache"], x["seqlens"], sel, o, ws_a,
                               w.r, w.budget, w.scale, lse=lse)
    st = (qsa.qsa_check_device_status(ws_i), qsa.qsa_check_device_status(ws_a))
    return kp, sel, sc, o, lse, st


def _check_decode_rows(w, x, kp, sel, sc, o, lse, seqs):
    for b in seqs:
        L = int(x["seqlens"][b])
        ki = parity.bits(x["k_idx_cache"][b:b + 1])
        kp_ref = oracle.pool(ki, w.r)
        assert np.array_equal(parity.bits(kp[b:b + 1]), kp_ref)
        qi = parity.bits(x["q_idx"][b:b + 1])[:, None]
        wt = x["w"][b:b + 1].cpu().numpy()[:, None]
        pos0 = np.array([L - 1])
        sel_h = sel[b:b + 1].cpu().numpy()
        parity.check_selection_vs_oracle(sel_h, qi, wt, kp_ref, np.array([0]), w.r, w.budget,
                                         q_pos0=pos0, sel_score_gpu=sc[b:b + 1].cpu().numpy())
        q = parity.bits(x["q"][b:b + 1])[:, None]
        k = parity.bits(x["k_cache"][b:b + 1])
        v = parity.bits(x["v_cache"][b:b + 1])
        o_ref, lse_ref = oracle.attn(q, k, v, w.r, w.scale, sel=sel_h, q_pos0=pos0)
        parity.check_attention(oracle.bf16_bits_to_f64(parity.bits(o[b:b + 1])).reshape(1, w.Hq, w.D),
                               o_ref, lse[b:b + 1].cpu().numpy(), lse_ref, f"decode b={b}")


def test_decode_small_ragged():
    w = synth.Workload("dec-small", "decode", 8, 4096, 16, 2, 128, 4, 64, 4, 512, 21, 4)
    seqlens = [4096, 4095, 4093, 2050, 2048, 2047, 17, 1]
    x = synth.make_decode(w, DEV, seqlens=seqlens)
    kp, sel, sc, o, lse, st = _qsa_decode(x, w)
    assert st == (0, 0)
    _check_decode_rows(w, x, kp, sel, sc, o, lse, range(w.B))


def test_decode_full_size_sampled():
    w = synth.WORKLOADS["decode-256k-b64"]
    x = synth.make_decode(w, DEV)
    kp, sel, sc, o, lse, st = _qsa_decode(x, w)
    assert st == (0, 0)
    sel_h = sel.cpu().numpy()
    for (b, j) in x["needles"]:
        assert j in sel_h[b], (b, j)
    o_h = o.float().cpu().numpy()
    np.testing.assert_allclose(o_h[:, :: w.G], synth.NEEDLE_VALUE, atol=2e-2)
    _check_decode_rows(w, x, kp, sel, sc, o, lse, [0, 9, 21, 42, 63])


def test_decode_bad_seqlens_recorded_not_faulted():
    w = synth.Workload("dec-bad", "decode", 4, 1024, 16, 2, 128, 4, 64, 4, 256, 22, 0)
    x = synth.make_decode(w, DEV, seqlens=[1024, 0, 2000, 5])
    kp, sel, sc, o, lse, st = _qsa_decode(x, w)
    assert st[0] == 7 and st[1] == 7
    assert torch.isfinite(o.float()).all()
    assert (o[1].float() == 0).all()


# --------------------------------------------------------------------- dense

@pytest.mark.parametrize("w", [synth.WORKLOADS["prefill-2k-tiny"],
                               synth.Workload("dense-ragged", "prefill", 2, 1000, 16, 2, 128,
                                              4, 64, 4, 2048, 23, 0),
                               synth.Workload("dense-g2-d64", "prefill", 1, 777, 8, 4, 64,
                                              4, 64, 4, 2048, 24, 0)],
                         ids=["tiny", "ragged", "g2-d64"])
def test_dense_prefill_all_rows(w):
    x = synth.make_prefill(w, DEV)
    o = torch.empty_like(x["q"])
    lse = torch.empty(w.B, w.T, w.Hq, dtype=torch.float32, device=DEV)
    qsa.qsa_dense_gqa_prefill(x["q"], x["k"], x["v"], o, w.scale, lse=lse)
    torch.cuda.synchronize()
    h = _host(x)
    o_ref, lse_ref = oracle.attn(h["q"], h["k"], h["v"], w.r, w.scale)
    parity.check_attention(oracle.bf16_bits_to_f64(parity.bits(o)).reshape(-1, w.Hq, w.D), o_ref,
                           lse.view(-1, w.Hq).cpu().numpy(), lse_ref, w.name)
    # and against torch's own attention on the GPU
    ref = torch.nn.functional.scaled_dot_product_attention(
        x["q"].transpose(1, 2), x["k"].transpose(1, 2), x["v"].transpose(1, 2),
        is_causal=True, scale=w.scale, enable_gqa=True).transpose(1, 2)
    assert (o.float() - ref.float()).abs().max().item() <= parity.O_MAX_ABS


def test_dense_prefill_32k_sampled():
    w = synth.WORKLOADS["prefill-32k"]
    x = synth.make_prefill(w, DEV)
    o = torch.empty_like(x["q"])
    qsa.qsa_dense_gqa_prefill(x["q"], x["k"], x["v"], o, w.scale)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 63, 64, 127, 128, 4095, 16384, 32766, 32767], np.int64)
    h = _host(x)
    o_ref, _ = oracle.attn(h["q"], h["k"], h["v"], w.r, w.scale, rows=rows)
    o_h = oracle.bf16_bits_to_f64(parity.bits(o)).reshape(-1, w.Hq, w.D)[rows]
    parity.check_attention(o_h, o_ref, what="dense-32k")


@pytest.mark.parametrize("full", [False, True], ids=["small-ragged", "256k-b64-sampled"])
def test_dense_decode(full):
    if full:
        w = synth.WORKLOADS["decode-256k-b64"]
        x = synth.make_decode(w, DEV)
        seqs = [0, 33, 63]
    else:
        w = synth.Workload("dd-small", "decode", 5, 3000, 8, 2, 64, 4, 64, 4, 2048, 25, 0)
        x = synth.make_decode(w, DEV, seqlens=[3000, 2999, 1234, 4, 1])
        seqs = range(w.B)
    o = torch.empty_like(x["q"])
    lse = torch.empty(w.B, w.Hq, dtype=torch.float32, device=DEV)
    ws = qsa.workspace(qsa.qsa_dense_gqa_decode_workspace_size(w.B, w.T, w.Hq, w.D))
    qsa.qsa_dense_gqa_decode(x["q"], x["k_cache"], x["v_cache"], x["seqlens"], o, ws, w.scale,
                             lse=lse)
    assert qsa.qsa_check_device_status(ws) == 0
    for b in seqs:
        L = int(x["seqlens"][b])
        q = parity.bits(x["q"][b:b + 1])[:, None]
        k = parity.bits(x["k_cache"][b:b + 1])
        v = parity.bits(x["v_cache"][b:b + 1])
        o_ref, lse_ref = oracle.attn(q, k, v, w.r, w.scale, q_pos0=np.array([L - 1]))
        parity.check_attention(oracle.bf16_bits_to_f64(parity.bits(o[b:b + 1])).reshape(1, w.Hq, w.D),
                               o_ref, lse[b:b + 1].cpu().numpy(), lse_ref, f"dense-dec b={b}")

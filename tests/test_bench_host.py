"""The benchmark's algorithmic work counts, checked on CPU against the oracle:
the per-row token-set sizes and candidate-pair counts that its rooflines divide
by are recounted from the oracle's own selections and score matrices."""
import numpy as np
import torch

import bench
import oracle
from block_sparse_long_10_b200 import synth


def _tiny(T=203, budget=64, seed=3):
    w = synth.Workload("work-tiny", "prefill", 1, T, 4, 2, 64, 2, 32, 4, budget, seed, 2)
    x = synth.make_prefill(w, "cpu")
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    return w, x, bits


def test_token_set_sizes_match_the_oracle_selection():
    w, x, bits = _tiny()
    kp = oracle.pool(bits(x["k_idx"]), w.r)
    sel, _, _, _ = oracle.index_topk(bits(x["q_idx"]), x["w"].numpy(), kp, w.r, w.budget)
    counted = np.array([sum(1 for j in row if j >= 0 for i in range(w.r) if j * w.r + i <= t)
                        for t, row in enumerate(sel)])
    assert np.array_equal(bench.sparse_tokens_per_row(w.T, w.r, w.kb), counted)


def test_candidate_pair_counts_match_the_oracle_score_matrix():
    w, x, bits = _tiny()
    kp = oracle.pool(bits(x["k_idx"]), w.r)
    s = oracle.index_scores(bits(x["q_idx"]), x["w"].numpy(), kp, w.r)
    pairs = int(np.isfinite(s).sum())
    wk = bench.prefill_work(w)
    assert wk["index_pairs"] == pairs
    assert wk["index_flops"] == pairs * 2 * w.Hi * w.Di
    assert bench.sum_candidate_keys(w.T, w.r) == pairs * w.r


def test_candidate_key_count_closed_form():
    for T in (0, 1, 3, 4, 5, 17, 100, 1001, 4096):
        for r in (1, 4):
            assert bench.sum_candidate_keys(T, r) == sum(r * (p // r) for p in range(T))


def test_decode_work_counts():
    w = synth.WORKLOADS["decode-256k-b64"]
    L = np.array([262144, 5, 4, 1])
    wk = bench.decode_work(w, L)
    c = (L - 1) // 4
    assert wk["index_bytes"] == float((c * 64 * 2).sum() + 4 * (4 * 64 * 2 + 512 * 4))
    S = np.array([4 * 511 + 4, 4 + 1, 4, 1])                 # tokens attended per sequence
    assert wk["attn_bytes"] == float((S * 2 * 128 * 4).sum() + 4 * 16 * 128 * 4)
    assert wk["dense_bytes"] == float((L * 2 * 128 * 4).sum())


def test_dominant_roofline_names_the_slowest_kernel():
    w = synth.WORKLOADS["prefill-1m"]
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops_sustained": 1400.0, "bf16_tflops": 1600.0,
             "source": "test"}
    r = bench.dominant_roofline(w, {"pool": 0.03, "index_topk": 250.0, "sparse_attn": 170.0},
                                peaks)
    assert r["kernel"] == "index_topk" and r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["achieved"] - bench.prefill_work(w)["index_flops"] / 0.25 / 1e12) < 1e-6
    r = bench.dominant_roofline(w, {"pool": 0.03, "index_topk": 100.0, "sparse_attn": 170.0},
                                peaks)
    # the sparse attention is rated against the tensor peak: its gathered bytes
    # are mostly L2 hits, so they cannot be held against the HBM peak
    assert r["kernel"] == "sparse_attn" and r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["achieved"] - bench.prefill_work(w)["attn_flops"] / 0.17 / 1e12) < 1e-6
    assert r["frac"] < 1.0

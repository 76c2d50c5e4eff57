"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle against a hand-derived worked example (fixtures
under tests/golden/), a closed form, a library routine (numpy matmul/lexsort,
torch scaled_dot_product_attention / logsumexp in fp64), an O(n^2) rank-count
brute force, or an invariant of the mathematics.  A plausible slip anywhere in
the oracle (a dropped ReLU or head weight, a wrong tie-break, a missing causal
mask, a transposed operand, a wrong summation order) fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_10_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bits(x):
    """Exact float -> bf16 bits (asserts the value is representable)."""
    x = np.asarray(x, np.float32)
    b = (x.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(oracle.bf16_bits_to_f64(b), x.astype(np.float64)), "not bf16-exact"
    return b


def _f(v):
    if isinstance(v, str):
        return {"inf": math.inf, "ln(3)": math.log(3), "ln(4)": math.log(4),
                "ln(2)": math.log(2)}[v]
    return v


def _np_bf16(x):
    # truncation is fine for *generating* inputs (any bf16 pattern is valid)
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


# ------------------------------------------------------------------ pooling --

def test_pool_golden():
    g = _load("pool_12tok.json")
    k = _bits(g["k_idx"])[None]                     # [1, 12, 2]
    kp = oracle.pool(k, g["r"])
    want = np.array([[int(h, 16) for h in row] for row in g["expected_bits"]], np.uint16)
    assert np.array_equal(kp[0], want)


def test_pool_r1_is_identity_and_partial_range():
    rng = np.random.default_rng(1)
    k = _np_bf16(rng.standard_normal((2, 16, 8)))
    assert np.array_equal(oracle.pool(k, 1), k)
    # only [j0, j1) is written
    out = np.full((2, 4, 8), 0xFFFF, np.uint16)
    oracle.pool(k, 4, 1, 3, out=out)
    full = oracle.pool(k, 4)
    assert np.array_equal(out[:, 1:3], full[:, 1:3])
    assert (out[:, 0] == 0xFFFF).all() and (out[:, 3] == 0xFFFF).all()


def test_pool_constant_block_is_exact():
    rng = np.random.default_rng(2)
    vals = _np_bf16(rng.standard_normal((1, 8, 16)))
    k = np.repeat(vals, 4, axis=1)                  # every block = 4 equal tokens
    assert np.array_equal(oracle.pool(k, 4), vals)


def test_pool_is_rounded_exact_mean():
    """The pooled key is the bf16 rounding of the exact mean (half-ulp bound),
    and equals RNE(exact mean) wherever the fp32 pair sums are exact."""
    rng = np.random.default_rng(3)
    k = _np_bf16(rng.standard_normal((1, 4096, 16)))
    kp = oracle.bf16_bits_to_f64(oracle.pool(k, 4))
    mean = oracle.bf16_bits_to_f64(k).reshape(1, 1024, 4, 16).mean(axis=2)  # exact in fp64
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(mean), 1e-30))) - 7)
    assert (np.abs(kp - mean) <= 0.5 * ulp * (1 + 1e-6) + 1e-30).all()
    rne = oracle.bf16_bits_to_f64(oracle.f32_to_bf16_bits(mean.astype(np.float32)[0, :64]))
    assert np.array_equal(kp[0, :64], rne)


# ------------------------------------------------------------------ indexer --

def _index_fixture():
    g = _load("index_tiny.json")
    q = _bits(g["q_idx"])[None, None]                # [1, 1, Hi, Di]
    w = np.asarray(g["w"], np.float32)[None, None]   # [1, 1, Hi]
    kp = _bits(g["kp"])[None]                        # [1, 8, Di]
    pos0 = np.array([g["pos"]], np.int64)
    return g, q, w, kp, pos0


def test_index_scores_golden():
    g, q, w, kp, pos0 = _index_fixture()
    s = oracle.index_scores(q, w, kp, g["r"], q_pos0=pos0)
    assert np.array_equal(s[0, :7], np.array(g["expected_scores"]))
    assert s[0, 7] == -np.inf


@pytest.mark.parametrize("case", range(5))
def test_index_topk_golden(case):
    g, q, w, kp, pos0 = _index_fixture()
    c = g["cases"][case]
    sel, sel_score, margin, s_cut = oracle.index_topk(q, w, kp, g["r"], c["budget"], q_pos0=pos0)
    assert sel[0].tolist() == c["sel"]
    assert margin[0] == _f(c["margin"])
    assert s_cut[0] == _f(c["s_cut"])
    exp_scores = g["expected_scores"]
    for j, sc in zip(sel[0], sel_score[0]):
        want = -np.inf if j < 0 else (np.inf if j == 7 else exp_scores[j])
        assert sc == np.float32(want)


def test_index_one_hot_closed_form():
    """One-hot indexer queries pick one pooled-key dim per head:
    score(j) = sum_h w_h * max(0, Kp[j, d_h])."""
    rng = np.random.default_rng(4)
    Hi, Di, N = 4, 16, 40
    d = rng.integers(0, Di, size=Hi)
    q = np.zeros((1, 1, Hi, Di), np.float32)
    q[0, 0, np.arange(Hi), d] = 1.0
    w = rng.random((1, 1, Hi)).astype(np.float32)
    kp = _np_bf16(rng.standard_normal((1, N, Di)))
    s = oracle.index_scores(_bits(q), w, kp, 4, q_pos0=np.array([4 * N - 1]))
    kpf = oracle.bf16_bits_to_f64(kp)[0]
    want = (w[0, 0].astype(np.float64) * np.maximum(kpf[:, d], 0.0)).sum(axis=1)
    np.testing.assert_allclose(s[0, : N - 1], want[: N - 1], rtol=1e-15, atol=0)


def test_index_r1_single_head_is_textbook_relu_topk():
    """r = 1, Hi = 1, w = 1 is DSA's token-level indexer: keep the top kb-1 of
    ReLU(q . k_j) over j < t (lower index first on ties) plus token t."""
    rng = np.random.default_rng(5)
    T, Di, budget = 96, 8, 12
    q = _np_bf16(rng.standard_normal((1, T, 1, Di)))
    k = _np_bf16(rng.standard_normal((1, T, Di)))
    w = np.ones((1, T, 1), np.float32)
    kp = oracle.pool(k, 1)
    sel, _, _, _ = oracle.index_topk(q, w, kp, 1, budget)
    qf = oracle.bf16_bits_to_f64(q)[0, :, 0]
    kf = oracle.bf16_bits_to_f64(k)[0]
    s = np.maximum(qf @ kf.T, 0.0)                 # library matmul
    for t in range(T):
        cand = np.arange(t)
        order = np.lexsort((cand, -s[t, :t]))      # library sort: score desc, j asc
        keep = sorted(cand[order[: budget - 1]].tolist() + [t])
        want = keep + [-1] * (budget - len(keep))
        assert sel[t].tolist() == want, t


@pytest.mark.parametrize("quantised", [False, True])
def test_selection_matches_rank_count_bruteforce(quantised):
    """Selected iff fewer than kb-1 candidates beat it, where i beats j when
    s_i > s_j or (s_i == s_j and i < j): an O(n^2) count, no sorting.  The
    quantised case has many exact ties."""
    rng = np.random.default_rng(6 + quantised)
    T, Hi, Di, r, budget = 128, 2, 8, 4, 24
    kb = budget // r
    if quantised:
        q = _bits(rng.integers(-1, 2, (1, T, Hi, Di)).astype(np.float32))
        k = _bits(rng.integers(-1, 2, (1, T, Di)).astype(np.float32))
        w = np.full((1, T, Hi), 0.5, np.float32)
    else:
        q = _np_bf16(rng.standard_normal((1, T, Hi, Di)))
        k = _np_bf16(rng.standard_normal((1, T, Di)))
        w = rng.random((1, T, Hi)).astype(np.float32)
    kp = oracle.pool(k, r)
    sel, _, _, _ = oracle.index_topk(q, w, kp, r, budget)
    s = oracle.index_scores(q, w, kp, r)
    for t in range(T):
        c = t // r
        sc = s[t, :c]
        chosen = []
        for j in range(c):
            beats = np.sum(sc > sc[j]) + np.sum(sc[:j] == sc[j])
            if beats < kb - 1:
                chosen.append(j)
        want = sorted(chosen + [c])
        want += [-1] * (kb - len(want))
        assert sel[t].tolist() == want, t


def test_index_invariants():
    rng = np.random.default_rng(8)
    T, Hi, Di, r = 64, 4, 16, 4
    q = _np_bf16(rng.standard_normal((1, T, Hi, Di)))
    k = _np_bf16(rng.standard_normal((1, T, Di)))
    w = rng.random((1, T, Hi)).astype(np.float32)
    kp = oracle.pool(k, r)
    s = oracle.index_scores(q, w, kp, r)
    # doubling the head weights doubles every score exactly
    s2 = oracle.index_scores(q, 2 * w, kp, r)
    assert np.array_equal(s2, 2 * s)
    # permuting heads together with their weights changes nothing
    perm = np.array([2, 0, 3, 1])
    sp = oracle.index_scores(q[:, :, perm], w[:, :, perm], kp, r)
    np.testing.assert_allclose(sp, s, rtol=1e-14)
    # flipping the sign of a head's query removes its positive part only
    qn = q.copy()
    qn[:, :, 0] ^= 0x8000
    sn = oracle.index_scores(qn, w, kp, r)
    dots = np.einsum("td,jd->tj", oracle.bf16_bits_to_f64(q)[0, :, 0],
                     oracle.bf16_bits_to_f64(kp)[0])
    fin = np.isfinite(s)
    delta = sn[fin] - s[fin]
    want = (w[0, :, 0:1].astype(np.float64) * (np.maximum(-dots, 0) - np.maximum(dots, 0)))[fin[0:T]]
    np.testing.assert_allclose(delta, want, atol=1e-12)
    # zero weights -> every candidate scores 0 -> lowest indices kept
    sel, _, _, _ = oracle.index_topk(q, 0 * w, kp, r, 16)
    t = T - 1
    assert sel[t].tolist() == [0, 1, 2, t // r]


@pytest.mark.parametrize("name", ["prefill-2k-tiny", "prefill-32k", "prefill-128k"])
def test_needles_are_selected_with_margin(name):
    """Every planted needle of the workload is selected by the oracle with a
    score margin above 1e-3 over the best block left out, so the GPU's selection
    must keep it exactly (the generator plants needles strong enough for the
    margin rule; this verifies that for the 2K, 32K and 128K workloads)."""
    w_ = synth.WORKLOADS[name]
    x = synth.make_prefill(w_, "cpu")
    qi, ki = synth.bf16_bits(x["q_idx"]), synth.bf16_bits(x["k_idx"])
    wt = x["w"].numpy()
    kp = oracle.pool(ki, w_.r)
    rows = np.array([t for (_, t, _) in x["needles"]], np.int64)
    assert rows.size == w_.needles
    sel, _, margin, s_cut = oracle.index_topk(qi, wt, kp, w_.r, w_.budget, rows=rows)
    for i, (_, t, j) in enumerate(x["needles"]):
        assert j in sel[i]
        sj = oracle.score_pairs(qi, wt, kp, [t], [j])[0]
        assert sj > s_cut[i] + 1e-3


# ---------------------------------------------------------------- attention --

def _attn_fixture():
    g = _load("attn_tiny.json")
    q = _bits(g["q"])[None, None]          # [1, 1, Hq=2, D=2]
    k = _bits(g["k"])[None, :, None]       # [1, 4, Hkv=1, 2]
    v = _bits(g["v"])[None, :, None]
    return g, q, k, v


@pytest.mark.parametrize("mode", ["dense", "r1", "r4_masked"])
def test_attn_golden(mode):
    g, q, k, v = _attn_fixture()
    pos0 = np.array([g["pos"]])
    scale = _f(g["scale"])
    if mode == "dense":
        o, lse = oracle.attn(q, k, v, 1, scale, q_pos0=pos0)
    elif mode == "r1":
        o, lse = oracle.attn(q, k, v, 1, scale, sel=np.array([[0, 1, -1]], np.int32), q_pos0=pos0)
    else:
        o, lse = oracle.attn(q, k, v, 4, scale, sel=np.array([[0, -1]], np.int32), q_pos0=pos0)
    np.testing.assert_allclose(o[0], np.array(g["expected_o"]), rtol=1e-14, atol=1e-13)
    np.testing.assert_allclose(lse[0], [_f(x) for x in g["expected_lse"]], rtol=1e-14)


def test_attn_empty_token_set_is_zero():
    """A selection naming no attendable token: the sum over no tokens (o = 0),
    lse = ln 0 = -inf.  Blocks past the query's position and -1 entries."""
    g, q, k, v = _attn_fixture()
    o, lse = oracle.attn(q, k, v, 4, 1.0, sel=np.array([[-1, 5]], np.int32),
                         q_pos0=np.array([1]))
    assert (o == 0).all() and np.isneginf(lse).all()


def _rand_qkv(rng, B, T, Hq, Hkv, D):
    q = _np_bf16(rng.standard_normal((B, T, Hq, D)))
    k = _np_bf16(rng.standard_normal((B, T, Hkv, D)))
    v = _np_bf16(rng.standard_normal((B, T, Hkv, D)))
    return q, k, v


def _sdpa(q, k, v, mask, scale):
    """torch SDPA in fp64; q [T,Hq,D], k/v [Tk,Hkv,D], mask [T,Tk] bool."""
    G = q.shape[1] // k.shape[1]
    qt = torch.from_numpy(oracle.bf16_bits_to_f64(q)).permute(1, 0, 2)
    kt = torch.from_numpy(oracle.bf16_bits_to_f64(k)).permute(1, 0, 2).repeat_interleave(G, 0)
    vt = torch.from_numpy(oracle.bf16_bits_to_f64(v)).permute(1, 0, 2).repeat_interleave(G, 0)
    m = torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)
    logits = (qt @ kt.transpose(1, 2)) * scale
    lse = torch.logsumexp(logits.masked_fill(~m, -math.inf), dim=-1)
    return o.permute(1, 0, 2).numpy(), lse.T.numpy()


def test_attn_dense_matches_torch_sdpa():
    rng = np.random.default_rng(9)
    B, T, Hq, Hkv, D = 2, 40, 6, 2, 16
    q, k, v = _rand_qkv(rng, B, T, Hq, Hkv, D)
    o, lse = oracle.attn(q, k, v, 4, 0.3)
    mask = np.tril(np.ones((T, T), bool))
    for b in range(B):
        ro, rl = _sdpa(q[b], k[b], v[b], mask, 0.3)
        np.testing.assert_allclose(o[b * T:(b + 1) * T], ro, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(lse[b * T:(b + 1) * T], rl, rtol=1e-12, atol=1e-12)


def test_attn_sparse_matches_masked_sdpa():
    """Expansion rule: token u is attended iff its block u // r is selected and
    u <= p.  The mask is built here from set membership; SDPA does the math."""
    rng = np.random.default_rng(10)
    T, Hq, Hkv, D, r, budget, Hi, Di = 64, 4, 1, 16, 4, 16, 2, 8
    q, k, v = _rand_qkv(rng, 1, T, Hq, Hkv, D)
    qi = _np_bf16(rng.standard_normal((1, T, Hi, Di)))
    ki = _np_bf16(rng.standard_normal((1, T, Di)))
    w = rng.random((1, T, Hi)).astype(np.float32)
    sel, _, _, _ = oracle.index_topk(qi, w, oracle.pool(ki, r), r, budget)
    o, lse = oracle.attn(q, k, v, r, 0.25, sel=sel)
    blk = np.arange(T) // r
    mask = np.stack([np.isin(blk, sel[t][sel[t] >= 0]) & (np.arange(T) <= t) for t in range(T)])
    ro, rl = _sdpa(q[0], k[0], v[0], mask, 0.25)
    np.testing.assert_allclose(o, ro, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=1e-12, atol=1e-12)


def test_full_budget_equals_dense_and_early_rows_dense():
    """With kb >= floor(p/r) + 1 every row selects its whole causal prefix, so
    QSA equals dense causal GQA; rows p < r*kb are dense in any workload."""
    rng = np.random.default_rng(11)
    T, Hq, Hkv, D, r, Hi, Di = 48, 4, 2, 8, 4, 2, 8
    q, k, v = _rand_qkv(rng, 1, T, Hq, Hkv, D)
    qi = _np_bf16(rng.standard_normal((1, T, Hi, Di)))
    ki = _np_bf16(rng.standard_normal((1, T, Di)))
    w = rng.random((1, T, Hi)).astype(np.float32)
    kp = oracle.pool(ki, r)
    od, ld = oracle.attn(q, k, v, r, 0.35)
    sel, _, _, _ = oracle.index_topk(qi, w, kp, r, T)
    os_, ls = oracle.attn(q, k, v, r, 0.35, sel=sel)
    np.testing.assert_allclose(os_, od, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(ls, ld, rtol=1e-13)
    sel, _, _, _ = oracle.index_topk(qi, w, kp, r, 16)   # kb = 4: rows < 16 dense
    os_, _ = oracle.attn(q, k, v, r, 0.35, sel=sel)
    np.testing.assert_allclose(os_[:16], od[:16], rtol=1e-13, atol=1e-14)
    assert np.abs(os_[16:] - od[16:]).max() > 1e-3


def test_gqa_head_duplication_and_value_linearity():
    rng = np.random.default_rng(12)
    T, Hq, Hkv, D = 24, 4, 2, 8
    q, k, v = _rand_qkv(rng, 1, T, Hq, Hkv, D)
    o, _ = oracle.attn(q, k, v, 4, 0.3)
    kd, vd = np.repeat(k, 2, axis=2), np.repeat(v, 2, axis=2)   # one KV head per query head
    o2, _ = oracle.attn(q, kd, vd, 4, 0.3)
    np.testing.assert_allclose(o2, o, rtol=1e-14, atol=1e-15)
    v2 = _np_bf16(2.0 * oracle.bf16_bits_to_f64(v).astype(np.float32))  # exact doubling
    o3, _ = oracle.attn(q, k, v2, 4, 0.3)
    np.testing.assert_allclose(o3, 2 * o, rtol=1e-13, atol=1e-14)


def test_decode_equals_last_prefill_row():
    rng = np.random.default_rng(13)
    B, T, Hq, Hkv, D, Hi, Di, r, budget = 3, 80, 4, 2, 16, 2, 8, 4, 16
    q, k, v = _rand_qkv(rng, B, T, Hq, Hkv, D)
    qi = _np_bf16(rng.standard_normal((B, T, Hi, Di)))
    ki = _np_bf16(rng.standard_normal((B, T, Di)))
    w = rng.random((B, T, Hi)).astype(np.float32)
    kp = oracle.pool(ki, r)
    seqlens = np.array([T, 37, 64])
    rows = np.arange(B) * T + (seqlens - 1)
    sel_p, _, _, _ = oracle.index_topk(qi, w, kp, r, budget, rows=rows)
    o_p, l_p = oracle.attn(q, k, v, r, 0.25, sel=sel_p, rows=rows)
    bi = np.arange(B)
    sel_d, o_d, l_d, _, _ = oracle.decode(q[bi, seqlens - 1], qi[bi, seqlens - 1],
                                          w[bi, seqlens - 1], k, v, kp, seqlens, r,
                                          budget, 0.25)
    assert np.array_equal(sel_d, sel_p)
    np.testing.assert_array_equal(o_d, o_p)
    np.testing.assert_array_equal(l_d, l_p)


def test_needle_row_output_is_needle_value():
    w_ = synth.WORKLOADS["prefill-2k-tiny"]
    x = synth.make_prefill(w_, "cpu")
    bits = {n: synth.bf16_bits(x[n]) for n in ("q", "k", "v", "q_idx", "k_idx")}
    kp = oracle.pool(bits["k_idx"], w_.r)
    rows = np.array([t for (_, t, _) in x["needles"]], np.int64)
    sel, _, _, _ = oracle.index_topk(bits["q_idx"], x["w"].numpy(), kp, w_.r, w_.budget, rows=rows)
    o, _ = oracle.attn(bits["q"], bits["k"], bits["v"], w_.r, w_.scale, sel=sel, rows=rows)
    heads = np.arange(w_.Hkv) * w_.G             # the head each needle key copies
    np.testing.assert_allclose(o[:, heads], synth.NEEDLE_VALUE, atol=1e-3)


# ------------------------------------------------------------ batch offsets --

def test_batched_calls_equal_per_sequence_calls():
    """A batch of sequences is the same computation as one call per sequence
    (an identity of the definition: sequences never see each other).  The two
    sequences get different indexer keys, pooled keys, K and V, so an oracle
    that read sequence 0's pooled keys (or K/V) for sequence 1 -- a dropped
    batch offset -- would fail here."""
    rng = np.random.default_rng(5)
    B, T, Hi, Di, Hq, Hkv, D, r, budget = 2, 96, 3, 16, 4, 2, 16, 4, 32
    q_idx = _np_bf16(rng.standard_normal((B, T, Hi, Di)))
    w = rng.random((B, T, Hi)).astype(np.float32)
    k_idx = _np_bf16(rng.standard_normal((B, T, Di)))
    q = _np_bf16(rng.standard_normal((B, T, Hq, D)))
    k = _np_bf16(rng.standard_normal((B, T, Hkv, D)))
    v = _np_bf16(rng.standard_normal((B, T, Hkv, D)))
    kp = oracle.pool(k_idx, r)
    assert not np.array_equal(kp[0], kp[1])
    scale = 0.25
    one = [(q_idx[b:b + 1], w[b:b + 1], kp[b:b + 1], q[b:b + 1], k[b:b + 1], v[b:b + 1])
           for b in range(B)]

    s2 = oracle.index_scores(q_idx, w, kp, r)
    s1 = np.concatenate([oracle.index_scores(qi, wi, kpi, r) for qi, wi, kpi, *_ in one])
    assert np.array_equal(s2, s1)

    rows = np.array([5, 50, 95, T + 5, T + 50, T + 95], np.int64)
    blocks = np.array([0, 7, 20, 0, 7, 20], np.int64)
    p2 = oracle.score_pairs(q_idx, w, kp, rows, blocks)
    p1 = np.concatenate([oracle.score_pairs(one[b][0], one[b][1], one[b][2], rows[3 * b:3 * b + 3] - b * T,
                                            blocks[3 * b:3 * b + 3]) for b in range(B)])
    assert np.array_equal(p2, p1)
    # pairs of sequence 1 agree with its own dense score matrix, not sequence 0's
    assert np.array_equal(p2[3:], s1[rows[3:], blocks[3:]])
    assert not np.array_equal(p2[3:], s1[rows[3:] - T, blocks[3:]])

    sel2, sc2, m2, c2 = oracle.index_topk(q_idx, w, kp, r, budget)
    parts = [oracle.index_topk(qi, wi, kpi, r, budget) for qi, wi, kpi, *_ in one]
    for a, i in ((sel2, 0), (sc2, 1), (m2, 2), (c2, 3)):
        assert np.array_equal(a, np.concatenate([p[i] for p in parts]))

    o2, l2 = oracle.attn(q, k, v, r, scale, sel=sel2)
    for b in range(B):
        o1, l1 = oracle.attn(one[b][3], one[b][4], one[b][5], r, scale, sel=parts[b][0])
        assert np.array_equal(o2[b * T:(b + 1) * T], o1)
        assert np.array_equal(l2[b * T:(b + 1) * T], l1)

"""Property tests of the oracle over random small shapes (hypothesis): the
selection equals an O(n^2) rank count with the lower-block-first tie rule and
has the stated structure; the attention output is a convex combination of the
attended values and its log-sum-exp lies between the largest logit and that
plus log |S|; decode equals the last prefill row.  Shapes, ratios, budgets and
value scales are drawn, so the fixed-shape pins are not the only witnesses."""
import math

import numpy as np
from hypothesis import given, settings, strategies as st

import oracle


def _bf16(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


@st.composite
def layer(draw):
    r = draw(st.sampled_from([1, 2, 4]))
    T = draw(st.integers(1, 40))
    Hkv = draw(st.sampled_from([1, 2]))
    G = draw(st.sampled_from([1, 2, 4]))
    D = draw(st.sampled_from([4, 8]))
    Hi = draw(st.sampled_from([1, 2, 3]))
    Di = draw(st.sampled_from([2, 4, 8]))
    kb = draw(st.integers(1, 6))
    quant = draw(st.booleans())
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    gen = (lambda s: rng.integers(-1, 2, s).astype(np.float32)) if quant else \
        (lambda s: rng.standard_normal(s) * 2)
    x = {
        "q": _bf16(gen((1, T, Hkv * G, D))), "k": _bf16(gen((1, T, Hkv, D))),
        "v": _bf16(gen((1, T, Hkv, D))), "q_idx": _bf16(gen((1, T, Hi, Di))),
        "k_idx": _bf16(gen((1, T, Di))),
        "w": (rng.random((1, T, Hi)) if not quant else np.full((1, T, Hi), 0.5)).astype(np.float32),
    }
    return x, r, kb * r


@settings(max_examples=60, deadline=None)
@given(layer())
def test_selection_is_the_rank_count_and_well_formed(case):
    x, r, budget = case
    kb = budget // r
    T = x["q"].shape[1]
    kp = oracle.pool(x["k_idx"], r)
    sel, score, _, _ = oracle.index_topk(x["q_idx"], x["w"], kp, r, budget)
    s = oracle.index_scores(x["q_idx"], x["w"], kp, r)
    for t in range(T):
        c = t // r
        sc = s[t, :c]
        chosen = [j for j in range(c)
                  if np.sum(sc > sc[j]) + np.sum(sc[:j] == sc[j]) < kb - 1]
        want = sorted(chosen + [c])
        assert sel[t].tolist() == want + [-1] * (kb - len(want))
        n = len(want)
        assert score[t, n - 1] == np.inf and np.all(score[t, n:] == -np.inf)
        for i, j in enumerate(want[:-1]):
            assert score[t, i] == np.float32(s[t, j])


@settings(max_examples=60, deadline=None)
@given(layer(), st.floats(0.05, 2.0))
def test_attention_is_a_convex_combination_with_bounded_lse(case, scale):
    x, r, budget = case
    T, Hq, D = x["q"].shape[1], x["q"].shape[2], x["q"].shape[3]
    Hkv = x["k"].shape[2]
    kp = oracle.pool(x["k_idx"], r)
    sel, _, _, _ = oracle.index_topk(x["q_idx"], x["w"], kp, r, budget)
    o, lse = oracle.attn(x["q"], x["k"], x["v"], r, scale, sel=sel)
    q = oracle.bf16_bits_to_f64(x["q"])[0]
    k = oracle.bf16_bits_to_f64(x["k"])[0]
    v = oracle.bf16_bits_to_f64(x["v"])[0]
    for t in range(T):
        toks = sorted({j * r + i for j in sel[t] if j >= 0 for i in range(r) if j * r + i <= t})
        assert toks and toks[-1] == t                      # the query sees itself
        for h in range(Hq):
            g = h // (Hq // Hkv)
            vv = v[toks, g]
            assert np.all(o[t, h] >= vv.min(axis=0) - 1e-12)
            assert np.all(o[t, h] <= vv.max(axis=0) + 1e-12)
            logits = scale * (k[toks, g] @ q[t, h])
            assert logits.max() - 1e-12 <= lse[t, h] <= logits.max() + math.log(len(toks)) + 1e-12


@settings(max_examples=40, deadline=None)
@given(layer(), st.floats(0.05, 2.0))
def test_decode_is_the_last_prefill_row(case, scale):
    x, r, budget = case
    T = x["q"].shape[1]
    kp = oracle.pool(x["k_idx"], r)
    sel_p, _, _, _ = oracle.index_topk(x["q_idx"], x["w"], kp, r, budget)
    o_p, lse_p = oracle.attn(x["q"], x["k"], x["v"], r, scale, sel=sel_p)
    sel_d, o_d, lse_d, _, _ = oracle.decode(
        x["q"][:, -1], x["q_idx"][:, -1], x["w"][:, -1], x["k"], x["v"], kp,
        np.array([T], np.int32), r, budget, scale)
    assert np.array_equal(sel_d[0], sel_p[-1])
    assert np.array_equal(o_d[0], o_p[-1]) and np.array_equal(lse_d[0], lse_p[-1])

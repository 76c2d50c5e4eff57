"""The two inequalities the prefill indexer's two-pass selection rests on,
checked in fp64 on random inputs (no GPU, no oracle arithmetic).

Score ("用125亿分之6的参数，打平3970亿的旗舰模型", section
"稀疏注意力：给检索建索引，也得先学会省纸": a lightweight MQA indexer in DSA's
form): s(t, j) = sum_h w_h max(0, q_h . Kp_j).

1. The linear lower bound of the first pass: with u = sum_h max(w_h, 0) q_h and
   c = sum_{w_h < 0} |w_h| |q_h|_1 max|Kp|,  s(t, j) >= u . Kp_j - c.
2. theta, the (kb-1)-th largest of per-group maxima of any lower bound (groups
   of distinct candidates), is at most the (kb-1)-th largest score, so every
   one of the kb-1 best candidates has s >= theta and survives the second pass.
"""
import numpy as np
import pytest


def _case(seed, Hi=4, Di=16, N=3000, signs="mixed"):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((Hi, Di))
    kp = 0.5 * rng.standard_normal((N, Di))
    w = rng.standard_normal(Hi)
    if signs == "positive":
        w = np.exp(w) / np.exp(w).sum()
    return q, kp, w


def _score(q, kp, w):
    return (np.maximum(kp @ q.T, 0.0) * w).sum(axis=1)


def _bound(q, kp, w, with_c=True):
    u = (np.maximum(w, 0.0)[:, None] * q).sum(axis=0)
    c = (np.abs(w) * (w < 0) * np.abs(q).sum(axis=1)).sum() * np.abs(kp).max()
    return kp @ u - (c if with_c else 0.0)


@pytest.mark.parametrize("seed,signs", [(1, "positive"), (2, "mixed"), (3, "mixed"), (4, "positive")])
def test_linear_bound_holds_for_every_pair(seed, signs):
    q, kp, w = _case(seed, signs=signs)
    s, lb = _score(q, kp, w), _bound(q, kp, w)
    assert (lb <= s + 1e-12).all()
    if signs == "positive":  # no negative weight: the bound is s plus the clipped part
        assert np.isclose(lb, s + (np.minimum(kp @ q.T, 0.0) * w).sum(axis=1)).all()


def test_bound_without_the_negative_weight_term_fails():
    """Folding negative weights into u without c breaks the bound somewhere."""
    q, kp, w = _case(5, signs="mixed")
    w[0] = -abs(w[0]) - 0.5
    s = _score(q, kp, w)
    u_all = (w[:, None] * q).sum(axis=0)
    assert (kp @ u_all > s + 1e-9).any()
    assert (_bound(q, kp, w) <= s + 1e-12).all()


@pytest.mark.parametrize("seed,R,signs", [(6, 1, "positive"), (7, 3, "positive"),
                                          (8, 16, "positive"), (9, 3, "mixed")])
def test_theta_from_group_maxima_keeps_every_top_candidate(seed, R, signs):
    q, kp, w = _case(seed, N=4096, signs=signs)
    s, lb = _score(q, kp, w), _bound(q, kp, w)
    K = 127
    # groups: a lane p of 128-block tiles, R consecutive tiles per group
    MB = 128
    tiles = len(s) // MB
    gm = []
    for p in range(MB):
        for g0 in range(0, tiles, R):
            idx = [kt * MB + p for kt in range(g0, min(g0 + R, tiles))]
            gm.append(lb[idx].max())
    theta = np.sort(gm)[::-1][K - 1]
    kth = np.sort(s)[::-1][K - 1]
    assert theta <= kth
    top = np.argsort(-s, kind="stable")[:K]
    assert (s[top] >= theta).all()
    if signs == "positive":  # and with weights of one sign the filter is selective
        assert (s >= theta).sum() < len(s) // 4

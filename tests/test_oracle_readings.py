"""Pins of the oracle's alternative readings (score formula, tie-break, entry
order, scatter weights), each against something other than its own formula:
invariances of the selection, a brute-force sort, an independent recursive
walk of the selection tree, and adjointness of the weighted scatter pair.
"""

import math
import os

import numpy as np
import pytest

import oracle as orc

P, L, K, N, D = 4, 3, 5, 256, 16


def _tokens(seed, n=N, d=D):
    rng = np.random.default_rng(seed)
    return orc.round_to_dtype(rng.standard_normal((n, d)), "bf16")


def _select(q, k, score="max", ties="low", p=P, l_=L, k_=K):
    mq, _ = orc.pool_head(q, p, l_, "bf16")
    mk, _ = orc.pool_head(k, p, l_, "bf16")
    scores, _, _ = orc.scores_head(mq, mk, l_, score)
    return orc.select_head(scores, p, l_, k_, ties)


def _same(a, b):
    return all((x is None and y is None) or np.array_equal(x, y) for x, y in zip(a, b))


def test_key_score_ignores_queries():
    """score='k' ranks by the key means only: any Q gives the same selection."""
    k = _tokens(1)
    sel_a, inc_a = _select(_tokens(2), k, "k")
    sel_b, inc_b = _select(np.zeros_like(k), k, "k")
    sel_c, _ = _select(10.0 * _tokens(3), k, "k")
    assert _same(sel_a, sel_b) and _same(inc_a, inc_b) and _same(sel_a, sel_c)


def test_sum_and_product_reduce_to_key_order():
    """|q|+|k| with Q = 0, and |q|^2|k|^2 with Q = K, are increasing functions of
    |k|^2, so they must select exactly what score='k' selects; with Q != K the
    readings differ on these inputs (they do depend on Q)."""
    k = _tokens(4)
    ref, _ = _select(np.zeros_like(k), k, "k")
    assert _same(_select(np.zeros_like(k), k, "sum")[0], ref)
    ref_qk, _ = _select(k, k, "k")
    assert _same(_select(k, k, "prod")[0], ref_qk)
    q = _tokens(5)
    assert not _same(_select(q, k, "sum")[0], _select(np.zeros_like(k), k, "sum")[0])


def test_sum_score_values_against_long_double():
    """The 'sum' score equals sqrt(|q|^2) + sqrt(|k|^2) to the last bit of an
    independent extended-precision computation rounded back to fp64."""
    q, k = _tokens(6), _tokens(7)
    mq, _ = orc.pool_head(q, P, L, "bf16")
    mk, _ = orc.pool_head(k, P, L, "bf16")
    s, nq, nk = orc.scores_head(mq, mk, L, "sum")
    for l in range(1, L):
        ext = np.sqrt(nq[l].astype(np.longdouble)) + np.sqrt(nk[l].astype(np.longdouble))
        assert np.max(np.abs(s[l] - ext.astype(np.float64)) / ext.astype(np.float64)) <= 2 ** -52


@pytest.mark.parametrize("score", ["max", "maxpool"])
@pytest.mark.parametrize("ties", ["low", "high"])
def test_ties_brute_force_on_equal_scores(ties, score):
    """All tokens equal: every entry of a level has the same score (under the
    max-pool reading too), so the selection is decided by the tie rule alone;
    brute force over Python sorting of (score, index) pairs."""
    x = np.tile(_tokens(8, n=1), (N, 1))
    mq, _ = orc.pool_head(x, P, L, "bf16")
    scores, _, _ = orc.scores_head(mq, mq, L, score)
    assert all(np.all(scores[l] == scores[l][0]) for l in range(1, L))
    sel, _ = orc.select_head(scores, P, L, K, ties)
    cand = list(range(len(scores[L - 1])))
    for l in range(L - 1, 0, -1):
        keyed = sorted(cand, key=lambda i: (-scores[l][i], i if ties == "low" else -i))
        want = sorted(keyed[:min(K, len(cand))])
        assert list(sel[l]) == want, (ties, l)
        cand = [c * P + j for c in want for j in range(P)]
    if ties == "high":
        assert sel[L - 1][-1] == len(scores[L - 1]) - 1


def _walk(sel, p, l_, n_top, pre):
    """Independent construction of the entry order: recursive walk of the
    selection tree (coarsest entries in index order; an expanded entry's
    children in index order), emitting an entry before (pre) or after (post)
    its subtree."""
    expanded = [set() if s is None else set(int(i) for i in s) for s in sel]
    out = []

    def visit(l, i):
        if pre:
            out.append((l, i))
        if l >= 1 and i in expanded[l]:
            for c in range(p):
                visit(l - 1, i * p + c)
        if not pre:
            out.append((l, i))

    for i in range(n_top):
        visit(l_ - 1, i)
    return out


@pytest.mark.parametrize("order", ["post", "pre"])
@pytest.mark.parametrize("p,l_,k_", [(4, 3, 5), (3, 4, 4), (2, 5, 3)])
def test_order_equals_recursive_tree_walk(order, p, l_, k_):
    n = p ** (l_ - 1) * 6
    q, k = _tokens(9, n=n), _tokens(10, n=n)
    sel, inc = _select(q, k, p=p, l_=l_, k_=k_)
    lvl, idx = orc.order_head(inc, p, l_, n, order)
    want = _walk(sel, p, l_, len(inc[l_ - 1]), pre=(order == "pre"))
    assert list(zip(lvl.tolist(), idx.tolist())) == want


@pytest.mark.parametrize("weight", ["one", "mean"])
def test_weighted_scatter_and_blocksum_are_adjoint(weight):
    """<scatter_w(rows), g> = <rows, blocksum_w(g)> in fp64 for both weightings."""
    rng = np.random.default_rng(11)
    q, k = _tokens(12), _tokens(13)
    sel, inc = _select(q, k)
    lvl, idx = orc.order_head(inc, P, L, N)
    rows = rng.standard_normal((len(lvl), D))
    g = rng.standard_normal((N, D))
    w = weight == "mean"
    lhs = np.sum(orc.scatter_head(rows, lvl, idx, P, N, weighted=w) * g)
    rhs = np.sum(rows * orc.blocksum_head(g, lvl, idx, P, weighted=w))
    assert abs(lhs - rhs) <= 1e-9 * max(1.0, abs(lhs))
    if w:   # weighted scatter of rows of ones: every token gets one 1/p^l per covering level
        ones = orc.scatter_head(np.ones((len(lvl), D)), lvl, idx, P, N, weighted=True)
        assert np.all(ones >= 1.0 / P ** (L - 1) - 1e-15)


@pytest.mark.parametrize("p,l_", [(4, 3), (3, 4), (2, 5)])
def test_maxpool_score_is_block_maximum_of_token_scores(p, l_):
    """The recursive max-pool equals, for every entry, the maximum over the
    tokens it covers of max(|q_t|^2, |k_t|^2) computed directly (a token's
    squared norm in plain fp64 against the pinned order: the same value within
    a few ulps, and the same maximiser); the returned per-side maxima
    reproduce it as their max."""
    n = p ** (l_ - 1) * 5
    q, k = _tokens(20, n=n), _tokens(21, n=n)
    mq, _ = orc.pool_head(q, p, l_, "bf16")
    mk, _ = orc.pool_head(k, p, l_, "bf16")
    scores, sq_q, sq_k = orc.scores_head(mq, mk, l_, "maxpool")
    tok = np.maximum(np.sum(q * q, axis=1), np.sum(k * k, axis=1))
    for l in range(1, l_):
        span = p ** l
        want = tok.reshape(-1, span).max(axis=1)
        assert np.max(np.abs(scores[l] - want) / want) <= 64 * 2 ** -52
        assert np.array_equal(scores[l], np.maximum(sq_q[l], sq_k[l]))


def test_maxpool_selects_the_outlier_chain():
    """One token with a much larger norm than all others: under the max-pool
    score every ancestor of it scores highest at its level and is expanded
    first, even with a budget of one entry per level; the mean-norm score
    dilutes it by p^l and need not."""
    p, l_, n = 4, 4, 4 ** 3 * 4
    q = _tokens(22, n=n)
    k = _tokens(23, n=n)
    t = 137
    q[t] *= 40.0
    sel, inc = _select(q, k, "maxpool", p=p, l_=l_, k_=1)
    for l in range(1, l_):
        assert list(sel[l]) == [t // p ** l], l
    assert t in inc[0]


def _read_score_golden():
    vals = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", "score_readings.txt")) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            key, rest = line.split(":", 1)
            vals[key.strip()] = np.array([float(t) for t in rest.split()])
    return vals


@pytest.mark.parametrize("score", ["max", "k", "sum", "prod"])
def test_hand_worked_score_readings_with_distinct_queries(score):
    """Hand-worked scores and selections (tests/golden/score_readings.txt) with
    Q != K, chosen so that each of the four pooled-entry scores expands a
    different pair: a slip such as a sum of squared norms, a missing square
    root or max() in place of the product selects another pair and fails here."""
    g = _read_score_golden()
    N, p, L_, K_, D_ = 8, 2, 2, 1, 8
    q = np.repeat(g["a"][:, None], D_, axis=1)
    k = np.repeat(g["b"][:, None], D_, axis=1)
    v = np.repeat(np.arange(N, dtype=np.float64)[:, None], D_, axis=1)
    fw = orc.forward_head(q, k, v, p, L_, K_, "bf16", score=score)
    want = g["score_sum_over_sqrt8"] * math.sqrt(8.0) if score == "sum" else g[f"score_{score}"]
    np.testing.assert_allclose(fw["scores"][1], want, rtol=1e-15, atol=0)
    assert list(fw["sel"][1]) == [int(g[f"sel_{score}"][0])]
    assert list(fw["lvl"]) == list(g[f"map_level_{score}"].astype(int))
    assert list(fw["idx"]) == list(g[f"map_index_{score}"].astype(int))
    # the four winners are pairwise distinct (the fixture separates the readings)
    assert len({int(g[f"sel_{s}"][0]) for s in ("max", "k", "sum", "prod")}) == 4

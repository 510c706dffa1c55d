"""Pins of the oracle's partition reading of the selection (inclusion="partition":
an expanded entry leaves the sub-sequence, its children take its place), each
against something other than its own formula: the covering property of a
partition, the nested reading's sets, an independent recursive walk of the
selection tree, and dense causal attention from torch when the budget
expands everything.
"""

import numpy as np
import pytest
import torch

import oracle as orc

SHAPES = [(4, 3, 5, 4 ** 2 * 16), (3, 4, 4, 3 ** 3 * 6), (2, 5, 3, 2 ** 4 * 8), (8, 2, 1, 8 * 5)]


def _tokens(seed, n, d=16):
    rng = np.random.default_rng(seed)
    return orc.round_to_dtype(rng.standard_normal((n, d)), "bf16")


def _select(q, k, p, l_, k_, inclusion):
    mq, _ = orc.pool_head(q, p, l_, "bf16")
    mk, _ = orc.pool_head(k, p, l_, "bf16")
    scores, _, _ = orc.scores_head(mq, mk, l_)
    return orc.select_head(scores, p, l_, k_, "low", inclusion)


@pytest.mark.parametrize("p,l_,k_,n", SHAPES)
def test_partition_covers_every_token_once(p, l_, k_, n):
    """The included entries tile the tokens: a weight-1 scatter of rows of ones
    gives exactly 1 everywhere, and the entry spans add up to N."""
    sel, inc = _select(_tokens(1, n), _tokens(2, n), p, l_, k_, "partition")
    lvl, idx = orc.order_head(inc, p, l_, n)
    ones = orc.scatter_head(np.ones((len(lvl), 3)), lvl, idx, p, n, weighted=False)
    assert np.array_equal(ones, np.ones((n, 3)))
    assert int(np.sum(p ** lvl)) == n
    # the nested reading covers a token once per included ancestor: more than once somewhere
    _, inc_n = _select(_tokens(1, n), _tokens(2, n), p, l_, k_, "nested")
    lvl_n, idx_n = orc.order_head(inc_n, p, l_, n)
    assert orc.scatter_head(np.ones((len(lvl_n), 1)), lvl_n, idx_n, p, n, weighted=False).max() > 1


@pytest.mark.parametrize("p,l_,k_,n", SHAPES)
def test_partition_is_nested_minus_expanded(p, l_, k_, n):
    """Level by level, the partition's entries and the expanded entries are
    disjoint and together form the nested reading's entries; the plan's sizes
    agree (S = nested S - sum of k_l)."""
    q, k = _tokens(3, n), _tokens(4, n)
    sel, inc_p = _select(q, k, p, l_, k_, "partition")
    sel_n, inc_n = _select(q, k, p, l_, k_, "nested")
    for l in range(l_):
        if l == 0:
            assert np.array_equal(inc_p[0], inc_n[0])
            continue
        assert np.array_equal(sel[l], sel_n[l])
        assert len(np.intersect1d(inc_p[l], sel[l])) == 0
        assert np.array_equal(np.union1d(inc_p[l], sel[l]), inc_n[l])
    pl_p, pl_n = orc.plan(n, p, l_, k_, "partition"), orc.plan(n, p, l_, k_)
    assert pl_p.S == pl_n.S - sum(pl_n.k) == sum(len(x) for x in inc_p)
    assert pl_p.m == pl_n.m == pl_n.c


def _leaves(sel, p, l_, n_top):
    """Independent order: recursive walk of the selection tree emitting only the
    entries that are not expanded, coarsest entries and children in index order."""
    expanded = [set() if s is None else set(int(i) for i in s) for s in sel]
    out = []

    def visit(l, i):
        if l >= 1 and i in expanded[l]:
            for c in range(p):
                visit(l - 1, i * p + c)
        else:
            out.append((l, i))

    for i in range(n_top):
        visit(l_ - 1, i)
    return out


@pytest.mark.parametrize("p,l_,k_,n", SHAPES)
def test_partition_orders_coincide_with_leaf_walk(p, l_, k_, n):
    """Under the partition the two order readings give the same sequence, the
    leaves of the selection tree from left to right."""
    sel, inc = _select(_tokens(5, n), _tokens(6, n), p, l_, k_, "partition")
    post = orc.order_head(inc, p, l_, n, "post")
    pre = orc.order_head(inc, p, l_, n, "pre")
    assert np.array_equal(post[0], pre[0]) and np.array_equal(post[1], pre[1])
    want = _leaves(sel, p, l_, n // p ** (l_ - 1))
    assert list(zip(post[0].tolist(), post[1].tolist())) == want


def test_partition_full_budget_is_dense_causal_attention():
    """With K at least every candidate count, every pooled entry is expanded, the
    sub-sequence is the token sequence, and the whole forward and backward equal
    dense causal attention on the (bf16-rounded) tokens: torch SDPA in fp64 and
    its autograd gradients."""
    p, l_, n, d = 2, 4, 64, 16
    k_ = n
    q, k, v = _tokens(7, n, d), _tokens(8, n, d), _tokens(9, n, d)
    do = np.random.default_rng(10).standard_normal((n, d))
    fw = orc.forward_head(q, k, v, p, l_, k_, "bf16", inclusion="partition")
    assert fw["plan"].S == n and np.all(fw["lvl"] == 0) and np.array_equal(fw["idx"], np.arange(n))
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq[None], tk[None], tv[None], is_causal=True)[0]
    assert np.max(np.abs(fw["o"] - ref.detach().numpy())) <= 1e-12
    ref.backward(torch.tensor(do))
    bw = orc.backward_head(fw, do, p)
    for got, t in ((bw["dq"], tq), (bw["dk"], tk), (bw["dv"], tv)):
        assert np.max(np.abs(got - t.grad.numpy())) <= 1e-11
    # the nested reading keeps every pooled entry as well: a longer sequence
    assert orc.plan(n, p, l_, k_).S == n + sum(n // p ** l for l in range(1, l_))


@pytest.mark.parametrize("weight", ["one", "mean"])
def test_partition_scatter_and_blocksum_are_adjoint(weight):
    """<scatter_w(rows), g> = <rows, blocksum_w(g)> on the partition's entries."""
    p, l_, k_, n = 4, 3, 5, 256
    rng = np.random.default_rng(11)
    _, inc = _select(_tokens(12, n), _tokens(13, n), p, l_, k_, "partition")
    lvl, idx = orc.order_head(inc, p, l_, n)
    rows = rng.standard_normal((len(lvl), 16))
    g = rng.standard_normal((n, 16))
    w = weight == "mean"
    lhs = np.sum(orc.scatter_head(rows, lvl, idx, p, n, weighted=w) * g)
    rhs = np.sum(rows * orc.blocksum_head(g, lvl, idx, p, weighted=w))
    assert abs(lhs - rhs) <= 1e-9 * max(1.0, abs(lhs))

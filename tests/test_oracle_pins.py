"""Pins of the CPU oracle against what the method description and mathematics fix.

Each test checks the oracle against something other than itself: hand-worked
values (tests/golden/), closed forms, brute force on tiny inputs, an
independent library routine (torch SDPA / autograd in fp64), or invariants
the description states. No GPU needed.
"""

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- sizes

def _read_plan_golden():
    rows = []
    with open(os.path.join(GOLDEN, "plan_sizes.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, N, p, L, K, S, bound = line.split()
            rows.append((name, int(N), int(p), int(L), int(K), int(S), int(bound)))
    return rows


@pytest.mark.parametrize("row", _read_plan_golden(), ids=lambda r: r[0])
def test_plan_matches_hand_derived_sizes(row):
    """S for each workload equals the hand derivation and obeys the size law of [LH] §1."""
    name, N, p, L, K, S, bound = row
    pl = orc.plan(N, p, L, K)
    assert pl.S == S
    assert pl.S <= N // p ** (L - 1) + (L - 1) * p * K == bound


def test_plan_edge_cases():
    assert orc.plan(64, 2, 1, 5).S == 64                      # L = 1: no selection
    assert orc.plan(64, 2, 2, 1000).S == 32 + 64             # budget >= candidates: all expanded
    assert orc.plan(48, 3, 2, 1).S == 16 + 3                 # odd p
    with pytest.raises(ValueError):
        orc.plan(100, 4, 3, 8)                               # N not a multiple of p^(L-1)


# ---------------------------------------------------------------- rounding

def _bf16_brute(x: float) -> float:
    """Nearest bf16 by enumeration of the two bracketing bf16 bit patterns; ties to even."""
    f = np.array([x], dtype=np.float64).astype(np.float32)   # only used to find the bracket
    bits = int(f.view(np.uint32)[0]) >> 16
    cands = []
    for b in (bits - 1, bits, bits + 1, bits + 2):
        b &= 0xFFFF
        val = float(np.array([b << 16], dtype=np.uint32).view(np.float32)[0])
        if math.isfinite(val):
            cands.append((abs(Fraction(val) - Fraction(x)), b & 1, val))
    cands.sort(key=lambda c: (c[0], c[1]))
    return cands[0][2]


def test_round_bf16_brute_force():
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.integers(-6, 6, 3000),
                         rng.standard_normal(200) * 1e-39])
    got = orc.round_to_dtype(xs, "bf16")
    for x, g in zip(xs, got):
        assert g == _bf16_brute(float(x)), x


def test_round_bf16_ties_and_double_rounding():
    # exact ties go to the even neighbour
    assert orc.round_to_dtype(np.array([1 + 2 ** -8]), "bf16")[0] == 1.0
    assert orc.round_to_dtype(np.array([1 + 3 * 2 ** -8]), "bf16")[0] == 1 + 2 ** -6
    # just above a tie rounds up; a detour through fp32 would first land on the tie
    x = 1 + 2 ** -8 + 2 ** -40
    assert orc.round_to_dtype(np.array([x]), "bf16")[0] == 1 + 2 ** -7
    assert orc.round_to_dtype(np.array([-x]), "bf16")[0] == -(1 + 2 ** -7)


# ---------------------------------------------------------------- pyramid

def _bf16_values(rng, shape, scale=1.0):
    return orc.round_to_dtype(rng.standard_normal(shape) * scale, "bf16")


@pytest.mark.parametrize("p,L", [(4, 3), (8, 3), (2, 5), (3, 3)])
def test_pool_is_closed_form_mean(p, L):
    """Entry (l, i) is the mean of tokens [i p^l, (i+1) p^l) ([LH] Fig. 2, step 1)."""
    rng = np.random.default_rng(p * 10 + L)
    N, D = p ** (L - 1) * 3, 16
    x = _bf16_values(rng, (N, D))
    means, stored = orc.pool_head(x, p, L, "bf16")
    for l in range(L):
        span = p ** l
        for i in range(N // span):
            for d in range(D):
                exact = math.fsum(x[i * span:(i + 1) * span, d]) / span
                assert means[l][i, d] == exact
        assert np.array_equal(stored[l], orc.round_to_dtype(means[l], "bf16") if l else x)


def test_pool_fp32_within_rounding():
    rng = np.random.default_rng(7)
    x = orc.round_to_dtype(rng.standard_normal((64, 8)) * np.exp(rng.standard_normal((64, 8)) * 6), "fp32")
    means, _ = orc.pool_head(x, 4, 4, "fp32")
    blk = x.reshape(1, 64, 8)
    exact = np.array([[math.fsum(blk[0, :, d]) / 64 for d in range(8)]])
    bound = 64 * 2.0 ** -52 * np.abs(x).sum(axis=0) / 64
    assert np.all(np.abs(means[3] - exact) <= bound)


# ---------------------------------------------------------------- score

@pytest.mark.parametrize("D", [8, 16, 64, 128])
def test_sq_norm_value(D):
    """Pinned-order squared norm equals the exact squared norm within D rounding errors."""
    rng = np.random.default_rng(D)
    m = rng.standard_normal((40, D)) * np.exp(rng.standard_normal((40, 1)))
    got = orc.sq_norm_pinned(m)
    for r in range(40):
        exact = sum(Fraction(float(v)) ** 2 for v in m[r])
        assert abs(Fraction(float(got[r])) - exact) <= exact * Fraction(2 * D, 2 ** 53)


@pytest.mark.parametrize("D", [64, 128])
def test_sq_norm_every_component_counts(D):
    """A one-hot row in every position d gives exactly m_d^2 (no dropped or doubled term)."""
    m = np.zeros((D, D))
    for d in range(D):
        m[d, d] = 1.5 + d
    assert np.array_equal(orc.sq_norm_pinned(m), (1.5 + np.arange(D)) ** 2)
    # two components in different chunks add, not overwrite
    m2 = np.zeros((1, D))
    m2[0, 3] = 2.0
    m2[0, D - 1] = 3.0
    assert orc.sq_norm_pinned(m2)[0] == 13.0


def test_sq_norm_pinned_order():
    """The rounding pattern follows the stated order (chunk sums, then the halving tree)."""
    D = 64
    m = np.zeros((1, D))
    m[0, 0] = 1.0
    m[0, 1] = 2.0 ** -27           # square 2^-54: lost against 1 inside chunk 0
    m[0, 32] = 2.0 ** -27          # chunk 4 alone holds 2^-54 ...
    m[0, 40] = 2.0 ** -27          # ... chunk 5 too; they meet only through the tree
    # chunk0 = 1 (2^-54 lost); tree stride 4: c0 = c0 + c4 = 1 (lost again); c1 = c1 + c5 = 2^-54
    # stride 2: c0 += c2 (0); c1 += c3 (0); stride 1: c0 = 1 + 2^-54 = 1 (lost)
    assert orc.sq_norm_pinned(m)[0] == 1.0
    m[0, 48] = 2.0 ** -27          # chunk 6: stride 4 pairs it with chunk 2 -> c2 = 2^-54
    # stride 2: c0 = 1 + 2^-54 = 1; c1 = 2^-54 + c3 = 2^-54; stride 1: 1 + 2^-54 = 1
    assert orc.sq_norm_pinned(m)[0] == 1.0
    m[0, 56] = 2.0 ** -27          # chunk 7 pairs with chunk 3: c3 = 2^-54; c1 + c3 = 2^-53
    # stride 1: c0 + c1 = 1 + 2^-53 (exactly halfway: ties to even -> 1)
    assert orc.sq_norm_pinned(m)[0] == 1.0
    m[0, 16] = 2.0 ** -27          # chunk 2 = 2^-54
    m[0, 24] = 2.0 ** -26          # chunk 3 = 2^-52
    # stride 4: c0 = 1, c1 = 2^-54, c2 = 2^-53, c3 = 1.25 * 2^-52
    # stride 2: c0 = 1 + 2^-53 -> 1 (tie, even); c1 = 1.5 * 2^-52
    # stride 1: 1 + 1.5 * 2^-52 -> tie between 1 + 2^-52 and 1 + 2^-51 -> even: 1 + 2^-51
    # (a left-to-right sum over all 64 components would give 1 + 2^-52)
    assert orc.sq_norm_pinned(m)[0] == 1.0 + 2.0 ** -51


def test_scores_are_max_of_query_and_key_norms():
    rng = np.random.default_rng(3)
    mq = [None, rng.standard_normal((10, 16))]
    mk = [None, rng.standard_normal((10, 16)) * 2]
    s, nq, nk = orc.scores_head(mq, mk, 2)
    assert np.array_equal(s[1], np.maximum(nq[1], nk[1]))
    assert np.all(s[1] >= nq[1]) and np.all(s[1] >= nk[1])


# ---------------------------------------------------------------- top-K descent

def _brute_topk(scores, cand, k):
    """Candidate c is kept iff fewer than k candidates beat it under (score desc, index asc)."""
    keep = []
    for c in cand:
        beat = sum(1 for d in cand if scores[d] > scores[c] or (scores[d] == scores[c] and d < c))
        if beat < k:
            keep.append(c)
    return np.array(sorted(keep), dtype=np.int64)


@pytest.mark.parametrize("seed", range(6))
def test_descent_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    p, L, K = [(2, 4, 3), (4, 3, 5), (3, 3, 2), (2, 5, 1), (4, 2, 7), (8, 3, 4)][seed]
    N = p ** (L - 1) * int(rng.integers(2, 7))
    n = [N // p ** l for l in range(L)]
    # few distinct values -> many exact ties
    scores = [None] + [rng.integers(0, 4, n[l]).astype(np.float64) for l in range(1, L)]
    sel, inc = orc.select_head(scores, p, L, K)
    cand = np.arange(n[L - 1])
    assert np.array_equal(inc[L - 1], cand)
    for l in range(L - 1, 0, -1):
        want = _brute_topk(scores[l], cand, min(K, len(cand)))
        assert np.array_equal(sel[l], want)
        cand = np.array(sorted(c * p + r for c in want for r in range(p)), dtype=np.int64)
        assert np.array_equal(inc[l - 1], cand)


def test_descent_all_equal_scores_take_lowest_indices():
    p, L, K = 4, 3, 3
    n = [64, 16, 4]
    scores = [None, np.ones(16), np.ones(4)]
    sel, inc = orc.select_head(scores, p, L, K)
    assert list(sel[2]) == [0, 1, 2]
    assert list(sel[1]) == [0, 1, 2]      # candidates 0..11, lowest three


# ---------------------------------------------------------------- order / map

def _read_tiny_golden():
    vals = {}
    with open(os.path.join(GOLDEN, "tiny_descent.txt")) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            key, rest = line.split(":", 1)
            vals[key.strip()] = np.array([float(t) for t in rest.split()])
    return vals


def test_hand_worked_descent_and_order():
    g = _read_tiny_golden()
    N, p, L, K, D = 16, 2, 3, 2, 8
    x = np.repeat(g["a"][:, None], D, axis=1)
    v = np.repeat(np.arange(N, dtype=np.float64)[:, None], D, axis=1)
    fw = orc.forward_head(x, x, v, p, L, K, "bf16")
    assert list(fw["sel"][2]) == list(g["sel2"].astype(int))
    assert list(fw["sel"][1]) == list(g["sel1"].astype(int))
    assert list(fw["lvl"]) == list(g["map_level"].astype(int))
    assert list(fw["idx"]) == list(g["map_index"].astype(int))
    for order in ("post", "pre"):
        fp = orc.forward_head(x, x, v, p, L, K, "bf16", order=order, inclusion="partition")
        assert list(fp["sel"][2]) == list(g["sel2"].astype(int))
        assert list(fp["lvl"]) == list(g["part_map_level"].astype(int)), order
        assert list(fp["idx"]) == list(g["part_map_index"].astype(int)), order
    fm = orc.forward_head(x, x, v, p, L, K, "bf16", score="maxpool")
    assert list(fm["sel"][2]) == list(g["mp_sel2"].astype(int))
    assert list(fm["sel"][1]) == list(g["mp_sel1"].astype(int))
    assert list(fm["lvl"]) == list(g["mp_map_level"].astype(int))
    assert list(fm["idx"]) == list(g["mp_map_index"].astype(int))


def _check_order_invariants(lvl, idx, p, L, N, pl):
    S = len(lvl)
    assert S == pl.S
    end = (idx + 1) * p ** lvl - 1
    key = end * (L + 1) + lvl
    assert np.all(np.diff(key) > 0)                       # strictly increasing (end, level)
    start = idx * p ** lvl
    # coarsest entries tile the sequence: every token under exactly one of them (no holes)
    cov = np.zeros(N, dtype=int)
    for j in np.nonzero(lvl == L - 1)[0]:
        cov[start[j]:end[j] + 1] += 1
    assert np.all(cov == 1)
    # every entry's included descendants come before it, its ancestors after it
    slot = {(int(a), int(b)): j for j, (a, b) in enumerate(zip(lvl, idx))}
    for j in range(S):
        l, i = int(lvl[j]), int(idx[j])
        if l < L - 1:
            parent = slot.get((l + 1, i // p))
            assert parent is not None and parent > j        # parents kept, and later
    # causal: entry positions never go backwards along the sequence
    assert np.all(np.diff(end) >= 0)


@pytest.mark.parametrize("seed", range(4))
def test_order_invariants_random(seed):
    rng = np.random.default_rng(100 + seed)
    p, L, K = [(4, 3, 5), (2, 5, 3), (8, 3, 6), (3, 4, 2)][seed]
    N = p ** (L - 1) * 5
    D = 16
    q = _bf16_values(rng, (N, D))
    k = _bf16_values(rng, (N, D))
    fw = orc.forward_head(q, k, q, p, L, K, "bf16")
    _check_order_invariants(fw["lvl"], fw["idx"], p, L, N, fw["plan"])


# ---------------------------------------------------------------- attention

def _sdpa64(q, k, v):
    t = [torch.from_numpy(a)[None, None] for a in (q, k, v)]
    return torch.nn.functional.scaled_dot_product_attention(*t, is_causal=True)[0, 0].numpy()


@pytest.mark.parametrize("S,D,block", [(300, 64, 128), (257, 128, 64), (7, 16, 1024)])
def test_attention_matches_torch_sdpa(S, D, block):
    """Eq. (1) with the causal mask, against torch's SDPA in fp64 (an independent routine)."""
    rng = np.random.default_rng(S)
    q, k, v = (rng.standard_normal((S, D)) * 2 for _ in range(3))
    o, lse = orc.attention_fwd(q, k, v, block=block)
    assert np.max(np.abs(o - _sdpa64(q, k, v))) < 1e-12
    a = torch.from_numpy(q @ k.T / math.sqrt(D))
    a = a.masked_fill(torch.triu(torch.ones(S, S, dtype=torch.bool), 1), float("-inf"))
    assert np.max(np.abs(lse - torch.logsumexp(a, dim=1).numpy())) < 1e-12


def test_attention_textbook_loop():
    rng = np.random.default_rng(5)
    S, D = 6, 8
    q, k, v = (rng.standard_normal((S, D)) for _ in range(3))
    o, _ = orc.attention_fwd(q, k, v)
    for j in range(S):
        w = [math.exp(sum(q[j, d] * k[m, d] for d in range(D)) / math.sqrt(D)) for m in range(j + 1)]
        z = sum(w)
        for d in range(D):
            assert abs(o[j, d] - sum(w[m] * v[m, d] for m in range(j + 1)) / z) < 1e-13


def test_single_level_wrapper_is_dense_causal_attention():
    """With L = 1 the sub-sequence is the whole sequence: the wrapper is Eq. (1) itself."""
    rng = np.random.default_rng(11)
    B, N, H, D = 1, 96, 2, 16
    Q, K, V = (_bf16_values(rng, (B, N, H, D)) for _ in range(3))
    O, _ = orc.forward(Q, K, V, p=4, L=1, K=8, dtype="bf16")
    for h in range(H):
        want = _sdpa64(Q[0, :, h], K[0, :, h], V[0, :, h])
        assert np.max(np.abs(O[0, :, h] - want)) < 1e-12


# ---------------------------------------------------------------- scatter family

def _random_head(seed, p=4, L=3, K=3, N=None, D=16, dtype="bf16"):
    rng = np.random.default_rng(seed)
    N = N or p ** (L - 1) * 4
    q, k, v = (_bf16_values(rng, (N, D)) for _ in range(3))
    return rng, orc.forward_head(q, k, v, p, L, K, dtype)


def test_scatter_blocksum_adjoint():
    rng, fw = _random_head(1)
    lvl, idx = fw["lvl"], fw["idx"]
    N = fw["plan"].N
    rows = rng.standard_normal((len(lvl), 16))
    g = rng.standard_normal((N, 16))
    lhs = np.sum(orc.scatter_head(rows, lvl, idx, 4, N, weighted=False) * g)
    rhs = np.sum(rows * orc.blocksum_head(g, lvl, idx, 4))
    assert abs(lhs - rhs) < 1e-10 * (1 + abs(lhs))


def test_spread_is_adjoint_of_pool_and_gather():
    rng, fw = _random_head(2)
    lvl, idx = fw["lvl"], fw["idx"]
    N = fw["plan"].N
    x = rng.standard_normal((N, 16))
    means, _ = orc.pool_head(x, 4, 3, "fp64")
    gx = orc.gather_head(means, lvl, idx)
    g = rng.standard_normal(gx.shape)
    lhs = np.sum(gx * g)
    rhs = np.sum(x * orc.spread_head(g, lvl, idx, 4, N))
    assert abs(lhs - rhs) < 1e-10 * (1 + abs(lhs))


def test_scatter_brute_force_loop():
    rng, fw = _random_head(3, p=2, L=4, K=2, N=24, D=8)
    lvl, idx = fw["lvl"], fw["idx"]
    rows = rng.standard_normal((len(lvl), 8))
    out = orc.scatter_head(rows, lvl, idx, 2, 24, weighted=False)
    for t in range(24):
        want = np.zeros(8)
        for j in range(len(lvl)):
            if idx[j] * 2 ** lvl[j] <= t < (idx[j] + 1) * 2 ** lvl[j]:
                want += rows[j]
        assert np.allclose(out[t], want, atol=1e-14)


def test_fixed_point_mode():
    """R13: the fixed-point sum equals the fp64 sum to within one count per contribution,
    and exactly when every contribution is a multiple of 2^-32."""
    rng, fw = _random_head(4)
    lvl, idx = fw["lvl"], fw["idx"]
    N = fw["plan"].N
    rows = rng.standard_normal((len(lvl), 16))
    a = orc.scatter_head(rows, lvl, idx, 4, N, weighted=True, mode="fp")
    b = orc.scatter_head(rows, lvl, idx, 4, N, weighted=True, mode="fixed")
    assert np.max(np.abs(a - b)) <= 3 * 2.0 ** -32
    rows_q = np.round(rows * 2 ** 20) / 2 ** 20
    a = orc.scatter_head(rows_q, lvl, idx, 4, N, weighted=False, mode="fp")
    b = orc.scatter_head(rows_q, lvl, idx, 4, N, weighted=False, mode="fixed")
    assert np.array_equal(a, b)


# ---------------------------------------------------------------- gradients

def _frozen_loss(x3, lvl, idx, p, L, dO):
    """Sum(O * dO) of the map-frozen path, no storage rounding (fp64)."""
    N = dO.shape[0]
    subs = []
    for x in x3:
        means, _ = orc.pool_head(x, p, L, "fp64")
        subs.append(orc.gather_head(means, lvl, idx))
    os_, _ = orc.attention_fwd(*subs)
    return float(np.sum(orc.scatter_head(os_, lvl, idx, p, N, weighted=False) * dO))


def test_gradients_finite_differences():
    """Central differences of the map-frozen fp64 function ([LH] Fig. 1: the selector takes no gradient)."""
    rng = np.random.default_rng(21)
    N, D, p, L, K = 16, 8, 2, 3, 2
    q, k, v = (rng.standard_normal((N, D)) for _ in range(3))
    dO = rng.standard_normal((N, D))
    fw = orc.forward_head(q, k, v, p, L, K, "fp64")
    bw = orc.backward_head(fw, dO, p)
    lvl, idx = fw["lvl"], fw["idx"]
    eps = 1e-6
    for which, grad in ((0, bw["dq"]), (1, bw["dk"]), (2, bw["dv"])):
        for (t, d) in [(0, 0), (3, 5), (9, 2), (15, 7), (12, 1)]:
            xs = [q.copy(), k.copy(), v.copy()]
            xs[which][t, d] += eps
            fp = _frozen_loss(xs, lvl, idx, p, L, dO)
            xs[which][t, d] -= 2 * eps
            fm = _frozen_loss(xs, lvl, idx, p, L, dO)
            fd = (fp - fm) / (2 * eps)
            assert abs(fd - grad[t, d]) < 1e-6 * max(1.0, abs(fd)), (which, t, d)


def test_gradients_match_torch_autograd():
    """The same map-frozen function written with torch ops (reshape-mean pool, index gather,
    SDPA, index_add scatter) and differentiated by autograd, in fp64."""
    rng = np.random.default_rng(22)
    N, D, p, L, K = 64, 16, 4, 3, 3
    q, k, v = (rng.standard_normal((N, D)) for _ in range(3))
    dO = rng.standard_normal((N, D))
    fw = orc.forward_head(q, k, v, p, L, K, "fp64")
    bw = orc.backward_head(fw, dO, p)
    lvl = torch.from_numpy(fw["lvl"])
    idx = torch.from_numpy(fw["idx"])
    xs = [torch.from_numpy(a).requires_grad_(True) for a in (q, k, v)]

    def sub(x):
        levels = [x] + [x.reshape(N // p ** l, p ** l, D).mean(dim=1) for l in range(1, L)]
        rows = torch.zeros(len(lvl), D, dtype=torch.float64)
        for l in range(L):
            m = lvl == l
            rows = rows.index_put((torch.nonzero(m)[:, 0],), levels[l][idx[m]])
        return rows

    qs, ks, vs = (sub(x) for x in xs)
    os_ = torch.nn.functional.scaled_dot_product_attention(qs[None, None], ks[None, None], vs[None, None],
                                                           is_causal=True)[0, 0]
    out = torch.zeros(N, D, dtype=torch.float64)
    for j in range(len(lvl)):
        span = p ** int(lvl[j])
        t0 = int(idx[j]) * span
        out = out.index_add(0, torch.arange(t0, t0 + span), os_[j].expand(span, D))
    (out * torch.from_numpy(dO)).sum().backward()
    assert np.max(np.abs(out.detach().numpy() - fw["o"])) < 1e-12
    for x, g in zip(xs, (bw["dq"], bw["dk"], bw["dv"])):
        assert np.max(np.abs(x.grad.numpy() - g)) < 1e-11

"""Lighthouse Attention hot path: plain, slow, obviously-correct fp64 oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``). Parity of the CUDA path
is judged against the functions below; they favour readability over speed.
Pure numpy, fp64 throughout, one (batch, head) pair at a time. Library
primitives used as single steps: ``@`` (matmul), ``np.lexsort``, ``np.exp``.

Sources, cited by short name in the docstrings below:

  [LH]   "Long Context Pre-Training with Lighthouse Attention" (Peng, Ghosh,
         Quesnelle; arXiv 2605.06554, HTML version): §1 Introduction (the size
         law O(LpK + N/p^{L-1})), §3 Method, §3.1 Preliminaries with Eq. (1)
         and the four stages (i)-(iv), Fig. 1 (architecture and gradient
         path), Fig. 2 (Pyramid Pool and Hierarchical Selector).
  [LHT]  "Lighthouse Attention Technique" (aibriefing summary): the three key
         points (sort then gather; hole-free causal sub-sequence).
  [AS]   "Nous Research's Lighthouse Attention Trains 1.69x Faster on
         Million-Token Contexts": section "A pyramid that scores itself".

Readings taken where the sources are silent or loose (each is restated where
it is used):

  R1  the selected set is a nested union: the coarsest level is kept whole; at
      each level l = L-1..1 the top-k_l candidates are expanded and all p
      children of each expanded entry are included one level down; parents
      stay in the sub-sequence ([LH] Fig. 2: the selector keeps parents and
      prunes the tree below unselected entries). The other reading,
      inclusion="partition": an expanded entry leaves the sub-sequence and is
      replaced by its children, so the included entries tile the tokens and
      every token is covered exactly once.
  R2  score of a pyramid entry = max(||mean_Q||^2, ||mean_K||^2) of the fp64
      means (the scorer looks at both the query and the key side: [LH] §1
      and the q/k score labels of Fig. 2);
      ranking by the squared norm equals ranking by the norm.
  R2b squared norm in a pinned fp64 order: the D components are cut into
      chunks of 8 consecutive components; each chunk is summed left to right
      from its first rounded product (no fused multiply-add); the D/8 chunk
      partials are combined by a stride-halving tree (stride D/16, ..., 1:
      c[j] = c[j] + c[j + stride]).
  R3  ties in the top-k: higher score first, then lower index first.
  R5  k_l = min(K, number of candidates at level l).
  R6  an entry's position is the last token it covers; entries ending at the
      same token are ordered finer level first (a post-order of the pyramid).
  R7  forward scatter weight is 1 (each output is added to every token its
      entry covers, [LH] §3.1 stage (iv)); the gradient of the mean-pool
      spreads an entry's gradient with weight 1/p^l (adjoint of a mean).
  R8  attention scale 1/sqrt(D) for every entry, pooled or not ([LH] Eq. (1)).
  R9  a stored pooled entry is the fp64 mean rounded to nearest-even into the
      I/O dtype; pyramid sums are formed level by level, each level's sum the
      left-to-right fp64 sum of its p children's sums, starting from the first
      child.
  R10 N must be a multiple of p^(L-1); L = 1 is legal (no selection, S = N).
  R13 fixed-point accumulation mode: each contribution w*x is quantised to an
      int64 count of 2^-32 (x * 2^32 / p^l in fp64, then round-half-even),
      summed exactly as integers, and converted back as count * 2^-32.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "Plan", "plan", "round_to_dtype", "pool_head", "sq_norm_pinned",
    "scores_head", "select_head", "order_head", "gather_head",
    "attention_fwd", "attention_bwd", "scatter_head", "blocksum_head",
    "spread_head", "forward_head", "backward_head", "forward", "backward",
    "FIXED_LSB",
]

FIXED_LSB = 2.0 ** -32  # R13: value of one count of the fixed-point accumulator


# ----------------------------------------------------------------------------
# sizes
# ----------------------------------------------------------------------------

@dataclass
class Plan:
    """Sizes of one (batch, head) problem.

    n[l]  entries at level l (n_l = N / p^l)            [LH] §3.1 stage (i)
    k[l]  entries expanded at level l (l >= 1)           R5
    m[l]  candidates at level l                          R1
    c[l]  entries of level l in the sub-sequence         R1 (m[l], or m[l] - k[l] for l >= 1 under partition)
    S     sub-sequence length = sum_l c[l]               [LH] §1 size law
    """
    N: int
    p: int
    L: int
    K: int
    n: list = field(default_factory=list)
    k: list = field(default_factory=list)
    m: list = field(default_factory=list)
    c: list = field(default_factory=list)
    S: int = 0


def plan(N: int, p: int, L: int, K: int, inclusion: str = "nested") -> Plan:
    """Sub-sequence sizes under reading R1/R5 ([LH] §1: S = O(LpK + N/p^(L-1)))."""
    if p < 2 or L < 1 or K < 1 or N < 1:
        raise ValueError("need p >= 2, L >= 1, K >= 1, N >= 1")
    if N % (p ** (L - 1)) != 0:
        raise ValueError("N must be a multiple of p^(L-1) (reading R10)")
    if inclusion not in ("nested", "partition"):
        raise ValueError(inclusion)
    n = [N // p ** l for l in range(L)]
    k = [0] * L
    m = [0] * L
    m[L - 1] = n[L - 1]
    for l in range(L - 1, 0, -1):
        k[l] = min(K, m[l])
        m[l - 1] = p * k[l]
    c = [m[l] - (k[l] if inclusion == "partition" and l >= 1 else 0) for l in range(L)]
    return Plan(N=N, p=p, L=L, K=K, n=n, k=k, m=m, c=c, S=sum(c))


# ----------------------------------------------------------------------------
# rounding into the I/O dtype
# ----------------------------------------------------------------------------

def _round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 value, ties to even.

    bfloat16: 8 significant bits, exponent range of fp32 (normal >= 2^-126,
    subnormal quantum 2^-133, largest finite (2 - 2^-7) * 2^127).
    Direct rounding from fp64 (no detour through fp32, which would round twice).
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    ax = np.abs(x)
    m, e = np.frexp(x)                      # x = m * 2^e, 0.5 <= |m| < 1
    normal = ax >= 2.0 ** -126
    # 8 significant bits: scale m to [128, 256), round half to even, scale back
    out[normal] = np.ldexp(np.rint(np.ldexp(m[normal], 8)), e[normal] - 8)
    sub = ~normal
    out[sub] = np.ldexp(np.rint(np.ldexp(x[sub], 133)), -133)
    big = np.abs(out) >= 2.0 ** 128
    out[big] = np.copysign(np.inf, x[big])
    out[np.isnan(x)] = np.nan
    return out


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round-to-nearest-even of fp64 values into ``dtype`` ("fp32" | "bf16"), returned as fp64.

    dtype "fp64" returns the values unchanged (used to differentiate the
    map-frozen path without storage rounding).
    """
    if dtype == "fp64":
        return np.array(x, dtype=np.float64)
    if dtype == "fp32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        return _round_bf16(x)
    raise ValueError(dtype)


# ----------------------------------------------------------------------------
# (i) pyramid pool                                   [LH] §3.1 stage (i), Fig. 2
# ----------------------------------------------------------------------------

def pool_head(x: np.ndarray, p: int, L: int, dtype: str):
    """Symmetric mean-pool of one head's tokens into an L-level pyramid.

    x: [N, D] fp64 holding the head's tokens (values representable in dtype).
    Level l entry i is the mean of tokens [i*p^l, (i+1)*p^l) ([LH] Fig. 2,
    step 1; [AS]: every level pools p times as many tokens as the one below).

    Returns (means, stored): lists over l = 0..L-1 of [n_l, D] fp64 arrays.
    means[l] is the fp64 mean; stored[l] is the entry kept in the I/O dtype
    (R9); level 0 is the tokens themselves.
    """
    sums = [np.array(x, dtype=np.float64)]
    for l in range(1, L):
        prev = sums[l - 1]
        s = prev[0::p].copy()               # R9: start from the first child
        for ch in range(1, p):
            s = s + prev[ch::p]             # left-to-right over the p children
        sums.append(s)
    means = [sums[l] / float(p ** l) for l in range(L)]
    stored = [means[0].copy()] + [round_to_dtype(means[l], dtype) for l in range(1, L)]
    return means, stored


# ----------------------------------------------------------------------------
# (ii-a) parameter-free l2 scorer          [LH] §1, Fig. 1, Fig. 2 (R2, R2b)
# ----------------------------------------------------------------------------

def sq_norm_pinned(m: np.ndarray) -> np.ndarray:
    """Squared l2 norm of each row of m ([n, D] fp64) in the pinned order R2b."""
    n, D = m.shape
    if D % 8 or (D // 8) & (D // 8 - 1):
        raise ValueError("D must be 8 * 2^j")
    nchunk = D // 8
    parts = []
    for ch in range(nchunk):
        acc = m[:, 8 * ch] * m[:, 8 * ch]
        for d in range(8 * ch + 1, 8 * ch + 8):
            acc = acc + m[:, d] * m[:, d]
        parts.append(acc)
    stride = nchunk // 2
    while stride >= 1:
        for j in range(stride):
            parts[j] = parts[j] + parts[j + stride]
        stride //= 2
    return parts[0]


def _score(a: np.ndarray, b: np.ndarray, score: str) -> np.ndarray:
    """One level's ranking score from the query / key squared norms a, b (fp64)."""
    if score == "max":          # max(|q|^2, |k|^2): the default reading
        return np.maximum(a, b)
    if score == "k":            # |k|^2 only
        return b.copy()
    if score == "sum":          # |q| + |k|: IEEE square roots, then their sum
        return np.sqrt(a) + np.sqrt(b)
    if score == "prod":         # |q|^2 |k|^2, ranks like |q| |k|
        return a * b
    raise ValueError(score)


def _maxpool(x: np.ndarray, p: int) -> np.ndarray:
    """Max over each run of p consecutive values (one level up the pyramid)."""
    return x.reshape(-1, p).max(axis=1)


def scores_head(means_q, means_k, L: int, score: str = "max"):
    """Score of every entry of levels 1..L-1 (R2a). Default reading: max of the
    query and key squared norms; the alternatives kept behind this switch:
    the key norm alone, the sum of the two norms, their product, and
    "maxpool" ([LH] Fig. 2 step 2, "l2 norm + max-pool", read bottom-up from
    level 0): a token scores max(|q|^2, |k|^2) of its own row, and an entry
    the largest score among its p children.

    Level 0 is never ranked (only levels >= 1 are candidates for expansion),
    so no level-0 score is returned. Returns (scores, sq_q, sq_k): lists
    indexed by level, None at level 0; under "maxpool" sq_q / sq_k hold the
    largest token norm under each entry, for queries and keys separately.
    """
    if score == "maxpool":
        if L == 1:
            return [None], [None], [None]
        p = len(means_q[0]) // len(means_q[1])
        tq, tk = sq_norm_pinned(means_q[0]), sq_norm_pinned(means_k[0])
        s = [np.maximum(tq, tk)]
        sq_q, sq_k = [tq], [tk]
        for l in range(1, L):
            s.append(_maxpool(s[l - 1], p))
            sq_q.append(_maxpool(sq_q[l - 1], p))
            sq_k.append(_maxpool(sq_k[l - 1], p))
        return [None] + s[1:], [None] + sq_q[1:], [None] + sq_k[1:]
    sq_q = [None] + [sq_norm_pinned(means_q[l]) for l in range(1, L)]
    sq_k = [None] + [sq_norm_pinned(means_k[l]) for l in range(1, L)]
    scores = [None] + [_score(sq_q[l], sq_k[l], score) for l in range(1, L)]
    return scores, sq_q, sq_k


# ----------------------------------------------------------------------------
# (ii-b) hierarchical top-K, tree descent   [LH] §3.1 stage (ii), Fig. 2 (R1, R3, R5)
# ----------------------------------------------------------------------------

def select_head(scores, p: int, L: int, K: int, ties: str = "low", inclusion: str = "nested"):
    """Top-down descent over the pyramid (parents kept, tree pruned: [LH] Fig. 2, step 3).

    Candidates at the coarsest level are all its entries. At each level
    l = L-1..1 the first k_l candidates in the order (score desc, index asc)
    are expanded (ties="high": index desc, the other tie reading R3); the p
    children of every expanded entry are the candidates one level down.
    Every candidate enters the sub-sequence (R1, nested), or every candidate
    that was not expanded (inclusion="partition").

    Returns (sel, included): sel[l] (l >= 1) is the sorted array of expanded
    indices at level l; included[l] the sorted array of level-l entries that
    enter the sub-sequence.
    """
    included = [None] * L
    sel = [None] * L
    n_top = len(scores[L - 1]) if L > 1 else None
    cand = np.arange(n_top, dtype=np.int64) if L > 1 else None
    if L > 1:
        included[L - 1] = cand.copy()
    for l in range(L - 1, 0, -1):
        k = min(K, len(cand))
        s = scores[l][cand]
        tie_key = cand if ties == "low" else -cand
        order = np.lexsort((tie_key, -s))    # primary: score desc; then index asc (R3) or desc
        chosen = np.sort(cand[order[:k]])
        sel[l] = chosen
        if inclusion == "partition":
            included[l] = np.setdiff1d(included[l], chosen)
        cand = (chosen[:, None] * p + np.arange(p)[None, :]).reshape(-1)
        included[l - 1] = cand.copy()
    return sel, included


# ----------------------------------------------------------------------------
# (ii-c) ordering: topological sort into one causal sequence   [LH] Fig. 1; [LHT] (R6)
# ----------------------------------------------------------------------------

def order_head(included, p: int, L: int, N: int, order: str = "post"):
    """Order the included entries by (last covered token asc, level asc); with
    order="pre" (the other reading, R6) by (first covered token asc, level desc).

    Returns (lvl, idx): int64 arrays of length S; slot j holds entry
    (lvl[j], idx[j]). With L = 1 every token is its own entry (S = N).
    """
    if L == 1:
        return np.zeros(N, dtype=np.int64), np.arange(N, dtype=np.int64)
    lv, ix = [], []
    for l in range(L):
        lv.append(np.full(len(included[l]), l, dtype=np.int64))
        ix.append(np.asarray(included[l], dtype=np.int64))
    lv = np.concatenate(lv)
    ix = np.concatenate(ix)
    if order == "post":
        end = (ix + 1) * (p ** lv) - 1
        perm = np.lexsort((lv, end))         # primary: end asc; then level asc
    elif order == "pre":
        start = ix * (p ** lv)
        perm = np.lexsort((-lv, start))      # primary: start asc; then level desc
    else:
        raise ValueError(order)
    return lv[perm], ix[perm]


def gather_head(stored, lvl, idx):
    """Sub-sequence rows: slot j takes stored entry (lvl[j], idx[j]) ([LH] Fig. 1, the dense gather)."""
    D = stored[0].shape[1]
    out = np.empty((len(lvl), D), dtype=np.float64)
    for l in range(len(stored)):
        m = lvl == l
        out[m] = stored[l][idx[m]]
    return out


# ----------------------------------------------------------------------------
# (iii) causal attention on the sub-sequence           [LH] Eq. (1), §3.1 stage (iii)
# ----------------------------------------------------------------------------

def attention_fwd(q: np.ndarray, k: np.ndarray, v: np.ndarray, block: int = 1024):
    """softmax(q k^T / sqrt(D) + M) v with the lower-triangular mask M.

    q, k, v: [S, D] fp64. Returns (o [S, D], lse [S]) with lse the natural
    log of each row's softmax denominator (max included). Rows are processed
    in blocks only to bound memory; each row is the textbook formula.
    """
    S, D = q.shape
    o = np.empty((S, D), dtype=np.float64)
    lse = np.empty(S, dtype=np.float64)
    for r0 in range(0, S, block):
        r1 = min(S, r0 + block)
        a = (q[r0:r1] @ k[:r1].T) / math.sqrt(D)
        cols = np.arange(r1)[None, :]
        rows = np.arange(r0, r1)[:, None]
        a[cols > rows] = -np.inf
        mx = a.max(axis=1, keepdims=True)
        e = np.exp(a - mx)
        den = e.sum(axis=1, keepdims=True)
        o[r0:r1] = (e @ v[:r1]) / den
        lse[r0:r1] = (mx + np.log(den))[:, 0]
    return o, lse


def attention_bwd(q, k, v, do, block: int = 1024):
    """Gradients of Eq. (1) w.r.t. q, k, v given the output gradient do.

    Textbook softmax calculus, row block by row block:
      P = softmax(A), A = q k^T / sqrt(D) + M
      dV = P^T dO,  dP = dO v^T,  dA = P o (dP - rowsum(P o dP)),
      dQ = dA k / sqrt(D),  dK = dA^T q / sqrt(D).
    """
    S, D = q.shape
    dq = np.zeros((S, D), dtype=np.float64)
    dk = np.zeros((S, D), dtype=np.float64)
    dv = np.zeros((S, D), dtype=np.float64)
    rs = 1.0 / math.sqrt(D)
    for r0 in range(0, S, block):
        r1 = min(S, r0 + block)
        a = (q[r0:r1] @ k[:r1].T) * rs
        cols = np.arange(r1)[None, :]
        rows = np.arange(r0, r1)[:, None]
        a[cols > rows] = -np.inf
        mx = a.max(axis=1, keepdims=True)
        e = np.exp(a - mx)
        P = e / e.sum(axis=1, keepdims=True)
        dv[:r1] += P.T @ do[r0:r1]
        dP = do[r0:r1] @ v[:r1].T
        dA = P * (dP - (P * dP).sum(axis=1, keepdims=True))
        dq[r0:r1] = (dA @ k[:r1]) * rs
        dk[:r1] += (dA.T @ q[r0:r1]) * rs
    return dq, dk, dv


# ----------------------------------------------------------------------------
# (iv) scatter back, and the adjoint steps of the backward pass
#                                 [LH] §3.1 stage (iv), Fig. 1 gradient path (R7, R13)
# ----------------------------------------------------------------------------

def _quantise(x: np.ndarray, denom: float) -> np.ndarray:
    """R13: int64 count of 2^-32 for the contribution x / denom."""
    return np.rint((x * 2.0 ** 32) / denom).astype(np.int64)


def scatter_head(rows, lvl, idx, p: int, N: int, weighted: bool, mode: str = "fp"):
    """out[t] = sum over slots j whose entry covers token t of w_j * rows[j].

    w_j = 1 for the forward output (R7) and 1/p^l for the gradient of the
    mean-pool (weighted=True). mode "fp": exact-as-fp64 sum, fine to coarse;
    mode "fixed": the R13 fixed-point sum (returned as fp64).
    rows: [S, D]; returns [N, D] fp64.
    """
    D = rows.shape[1]
    if mode == "fp":
        out = np.zeros((N, D), dtype=np.float64)
    elif mode == "fixed":
        acc = np.zeros((N, D), dtype=np.int64)
    else:
        raise ValueError(mode)
    for l in range(int(lvl.max()) + 1 if len(lvl) else 0):
        sl = np.nonzero(lvl == l)[0]
        span = p ** l
        denom = float(span) if weighted else 1.0
        for j in sl:
            t0 = int(idx[j]) * span
            if mode == "fp":
                out[t0:t0 + span] += rows[j] / denom
            else:
                acc[t0:t0 + span] += _quantise(rows[j], denom)
    if mode == "fixed":
        out = acc.astype(np.float64) * FIXED_LSB
    return out


def blocksum_head(g: np.ndarray, lvl, idx, p: int, weighted: bool = False):
    """Adjoint of the forward scatter: row j = sum of g over the tokens entry j
    covers (weight 1), divided by p^l when the scatter weights are 1/p^l (R7)."""
    out = np.empty((len(lvl), g.shape[1]), dtype=np.float64)
    for j in range(len(lvl)):
        span = p ** int(lvl[j])
        t0 = int(idx[j]) * span
        out[j] = g[t0:t0 + span].sum(axis=0)
        if weighted:
            out[j] /= span
    return out


def spread_head(g_rows, lvl, idx, p: int, N: int, mode: str = "fp"):
    """Gradient of gather + mean-pool: token t gets sum_j g_rows[j] / p^(l_j) over entries covering t."""
    return scatter_head(g_rows, lvl, idx, p, N, weighted=True, mode=mode)


# ----------------------------------------------------------------------------
# whole path, one (batch, head) pair
# ----------------------------------------------------------------------------

def forward_head(qh, kh, vh, p: int, L: int, K: int, dtype: str, mode: str = "fp", score: str = "max",
                 ties: str = "low", order: str = "post", weight: str = "one", inclusion: str = "nested"):
    """Forward pass for one head: tokens [N, D] x3 -> dict of every intermediate.

    score, ties, order, weight, inclusion select the readings R2a, R3, R6, R7,
    R1 (defaults: the library's). Keys: means_*, stored_*, scores, sq_q, sq_k, sel,
    included, lvl, idx, qs, ks, vs (sub-sequence), os, lse (attention), o
    ([N, D] output, fp64, not rounded), weight.
    """
    N, D = qh.shape
    pl = plan(N, p, L, K, inclusion)
    mq, sq_ = pool_head(qh, p, L, dtype)
    mk, sk_ = pool_head(kh, p, L, dtype)
    mv, sv_ = pool_head(vh, p, L, dtype)
    if L > 1:
        scores, nq, nk = scores_head(mq, mk, L, score)
        sel, included = select_head(scores, p, L, K, ties, inclusion)
    else:
        scores, nq, nk, sel, included = [None], [None], [None], [None], [None]
    lvl, idx = order_head(included, p, L, N, order)
    assert len(lvl) == pl.S
    qs = gather_head(sq_, lvl, idx)
    ks = gather_head(sk_, lvl, idx)
    vs = gather_head(sv_, lvl, idx)
    os_, lse = attention_fwd(qs, ks, vs)
    o = scatter_head(os_, lvl, idx, p, N, weighted=(weight == "mean"), mode=mode)
    return dict(means_q=mq, means_k=mk, means_v=mv, stored_q=sq_, stored_k=sk_,
                stored_v=sv_, scores=scores, sq_q=nq, sq_k=nk, sel=sel,
                included=included, lvl=lvl, idx=idx, qs=qs, ks=ks, vs=vs,
                os=os_, lse=lse, o=o, plan=pl, weight=weight)


def backward_head(fw: dict, doh: np.ndarray, p: int, mode: str = "fp"):
    """Backward pass for one head with the selection frozen ([LH] Fig. 1, red path).

    dO -> block sums (adjoint of the scatter) -> attention gradients ->
    spread with weight 1/p^l (adjoint of gather + mean-pool). The selector
    takes no gradient ([LH] §3.1). Returns dict with dos, dqs, dks, dvs, dq,
    dk, dv (fp64, not rounded).
    """
    N = doh.shape[0]
    lvl, idx = fw["lvl"], fw["idx"]
    dos = blocksum_head(doh, lvl, idx, p, weighted=(fw.get("weight", "one") == "mean"))
    dqs, dks, dvs = attention_bwd(fw["qs"], fw["ks"], fw["vs"], dos)
    dq = spread_head(dqs, lvl, idx, p, N, mode)
    dk = spread_head(dks, lvl, idx, p, N, mode)
    dv = spread_head(dvs, lvl, idx, p, N, mode)
    return dict(dos=dos, dqs=dqs, dks=dks, dvs=dvs, dq=dq, dk=dk, dv=dv)


def forward(Q, K_, V, p: int, L: int, K: int, dtype: str, mode: str = "fp", heads=None, **readings):
    """Whole-tensor forward. Q, K_, V: [B, N, H, D] fp64. Returns (O [B,N,H,D], per-head dicts).

    ``heads`` optionally restricts the work to a list of (b, h) pairs (the
    other rows of O stay NaN).
    """
    B, N, H, D = Q.shape
    O = np.full((B, N, H, D), np.nan)
    per = {}
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in pairs:
        fw = forward_head(Q[b, :, h, :], K_[b, :, h, :], V[b, :, h, :], p, L, K, dtype, mode, **readings)
        O[b, :, h, :] = fw["o"]
        per[(b, h)] = fw
    return O, per


def backward(per: dict, dO, p: int, mode: str = "fp"):
    """Whole-tensor backward over the heads in ``per``. Returns (dQ, dK, dV) [B,N,H,D] fp64."""
    B, N, H, D = dO.shape
    dQ = np.full((B, N, H, D), np.nan)
    dK = np.full_like(dQ, np.nan)
    dV = np.full_like(dQ, np.nan)
    for (b, h), fw in per.items():
        bw = backward_head(fw, dO[b, :, h, :], p, mode)
        dQ[b, :, h, :] = bw["dq"]
        dK[b, :, h, :] = bw["dk"]
        dV[b, :, h, :] = bw["dv"]
    return dQ, dK, dV

"""Sequence-sharded (context-parallel) Lighthouse hot path: plain fp64 oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages train at 1M-token context across 32 Blackwell GPUs with context
parallelism and ring attention ("Nous Research's Lighthouse Attention Trains
1.69x Faster on Million-Token Contexts", key points; "Lighthouse Attention
Technique": beyond 100K context a 530M model no longer fits one GPU and is
scaled with context parallelism). They do not spell out how the selection is
distributed. The plainest reading, taken here:

  * R ranks; rank r holds the contiguous token shard [r n, (r+1) n), n = N / R,
    with n a multiple of p^(L-1), so no pyramid entry straddles two shards and
    every rank pools and scores its own entries ("Long Context Pre-Training
    with Lighthouse Attention", §3.1 stages (i)-(ii), Fig. 2 steps 1-2: the
    pooling and the l2 scores are local to each entry's tokens).
  * The top-K descent runs level by level over the global candidate set: at
    level l each rank takes the top-k_l of its OWN candidates (by score desc,
    then the tie rule on the global index), all ranks exchange those lists
    (an all-gather of (score, global index) pairs), and every rank cuts the
    same global top-k_l from their union. The global top-k_l holds at most
    k_l entries of any one rank, so it is contained in that union: the cut
    equals the single-process one. Children of the cut entries become the
    next level's candidates on the rank that owns them (Fig. 2 step 3).
  * Entries are ordered by position (Fig. 1): a rank's entries all end inside
    its own shard, so its included entries form one contiguous segment of the
    global sub-sequence, after the segments of all lower ranks.
  * Causal attention over the sub-sequence (Eq. (1)): rank r's queries need
    the keys and values of every earlier segment, so ranks all-gather the
    sub-sequence K and V; each rank evaluates the same textbook attention as
    the single-process oracle for its own rows (its queries placed at their
    global rows, other rows zero, so every row it keeps sees exactly the
    arithmetic of the single-process call).
  * Scatter back (stage (iv)), block sums and the spread stay on the rank that
    owns the tokens. In the backward pass every rank forms the contribution
    of its own query rows to the gradients of all keys and values; the
    contributions are summed over ranks in rank order and each rank keeps its
    own segment (a reduce-scatter).

``comm`` is any object with ``rank``, ``world`` and ``all_gather(obj) -> list``
(one entry per rank, in rank order); the tests supply one over
torch.distributed (gloo) and one that runs the ranks in a single process.
"""

from __future__ import annotations

import numpy as np

from . import lighthouse as lh_oracle

__all__ = ["shard_sizes", "forward_shard", "backward_shard", "LocalComm", "run_local"]


def shard_sizes(N: int, p: int, L: int, world: int) -> int:
    """Tokens per rank; the shard must be a whole number of coarsest blocks."""
    if N % world:
        raise ValueError("N must split evenly over the ranks")
    n = N // world
    if n % (p ** (L - 1)):
        raise ValueError("each shard must be a multiple of p^(L-1) tokens")
    return n


def _local_topk(cand: np.ndarray, score: np.ndarray, k: int, ties: str):
    """First k candidates by (score desc, index asc) (ties="high": index desc)."""
    tie_key = cand if ties == "low" else -cand
    order = np.lexsort((tie_key, -score))
    top = order[:k]
    return score[top], cand[top]


def forward_shard(comm, qh, kh, vh, p: int, L: int, K: int, dtype: str, mode: str = "fp",
                  score: str = "max", ties: str = "low", order: str = "post", weight: str = "one",
                  inclusion: str = "nested") -> dict:
    """Forward pass of one head on rank ``comm.rank``'s shard.

    qh, kh, vh: [n, D] fp64, the shard's tokens (values representable in dtype).
    Returns a dict with the global selection ``sel`` (identical on every rank),
    the rank's segment of the gather map (``lvl``, ``idx`` with global entry
    indices), ``seg`` = (first slot, length) of that segment, the segment's
    attention output ``os`` and ``lse``, and the shard's output ``o`` [n, D].
    """
    r, R = comm.rank, comm.world
    n, D = qh.shape
    N = n * R
    shard_sizes(N, p, L, R)
    mq, sq_ = lh_oracle.pool_head(qh, p, L, dtype)
    mk, sk_ = lh_oracle.pool_head(kh, p, L, dtype)
    mv, sv_ = lh_oracle.pool_head(vh, p, L, dtype)
    base = [r * (n // p ** l) for l in range(L)]           # global index of the shard's first entry per level

    sel = [None] * L
    included = [None] * L
    if L > 1:
        scores, _, _ = lh_oracle.scores_head(mq, mk, L, score)
        cand = np.arange(n // p ** (L - 1), dtype=np.int64) + base[L - 1]      # global indices
        included[L - 1] = cand.copy()
        for l in range(L - 1, 0, -1):
            m_l = sum(comm.all_gather(len(cand)))                               # candidates over all ranks
            k = min(K, m_l)
            s_loc, c_loc = _local_topk(cand, scores[l][cand - base[l]], k, ties)
            pairs = comm.all_gather((s_loc, c_loc))
            s_all = np.concatenate([a for a, _ in pairs])
            c_all = np.concatenate([b for _, b in pairs])
            _, c_cut = _local_topk(c_all, s_all, k, ties)                       # the same cut on every rank
            sel[l] = np.sort(c_cut)
            mine = sel[l][(sel[l] >= base[l]) & (sel[l] < base[l] + n // p ** l)]
            if inclusion == "partition":
                included[l] = np.setdiff1d(included[l], mine)
            cand = (mine[:, None] * p + np.arange(p)[None, :]).reshape(-1)
            included[l - 1] = cand.copy()
    # own included entries, ordered by position (global indices)
    lvl, idx = lh_oracle.order_head(included, p, L, n, order)
    if L == 1:
        idx = idx + base[0]
    S_r = len(lvl)
    sizes = comm.all_gather(S_r)
    s0 = sum(sizes[:r])
    S = sum(sizes)
    loc_idx = idx - np.array([base[l] for l in lvl], dtype=np.int64)
    qs = lh_oracle.gather_head(sq_, lvl, loc_idx)
    ks = lh_oracle.gather_head(sk_, lvl, loc_idx)
    vs = lh_oracle.gather_head(sv_, lvl, loc_idx)
    # all-gather of the sub-sequence keys and values; own queries at their global rows
    K_all = np.concatenate(comm.all_gather(ks), axis=0)
    V_all = np.concatenate(comm.all_gather(vs), axis=0)
    Q_pad = np.zeros((S, D))
    Q_pad[s0:s0 + S_r] = qs
    o_all, lse_all = lh_oracle.attention_fwd(Q_pad, K_all, V_all)
    os_ = o_all[s0:s0 + S_r]
    lse = lse_all[s0:s0 + S_r]
    o = lh_oracle.scatter_head(os_, lvl, loc_idx, p, n, weighted=(weight == "mean"), mode=mode)
    return dict(sel=sel, lvl=lvl, idx=idx, loc_idx=loc_idx, seg=(s0, S_r), S=S, qs=qs, ks=ks, vs=vs,
                K_all=K_all, V_all=V_all, os=os_, lse=lse, o=o, weight=weight, n=n)


def backward_shard(comm, fw: dict, doh: np.ndarray, p: int, mode: str = "fp") -> dict:
    """Backward pass of one head on the rank's shard (selection frozen).

    doh: [n, D] upstream gradient of the shard's tokens. Returns the shard's
    dq, dk, dv [n, D] and the segment's dqs, dks, dvs.
    """
    s0, S_r = fw["seg"]
    S, D = fw["S"], doh.shape[1]
    lvl, loc_idx, n = fw["lvl"], fw["loc_idx"], fw["n"]
    dos = lh_oracle.blocksum_head(doh, lvl, loc_idx, p, weighted=(fw.get("weight", "one") == "mean"))
    Q_pad = np.zeros((S, D))
    Q_pad[s0:s0 + S_r] = fw["qs"]
    dO_pad = np.zeros((S, D))
    dO_pad[s0:s0 + S_r] = dos
    # rows other than the rank's own carry a zero output gradient, so the call
    # returns the own rows' dQ and their contribution to every key's dK, dV
    dq_all, dk_part, dv_part = lh_oracle.attention_bwd(Q_pad, fw["K_all"], fw["V_all"], dO_pad)
    dqs = dq_all[s0:s0 + S_r]
    dks = sum(comm.all_gather(dk_part))[s0:s0 + S_r]      # reduce over ranks in rank order
    dvs = sum(comm.all_gather(dv_part))[s0:s0 + S_r]
    dq = lh_oracle.spread_head(dqs, lvl, loc_idx, p, n, mode)
    dk = lh_oracle.spread_head(dks, lvl, loc_idx, p, n, mode)
    dv = lh_oracle.spread_head(dvs, lvl, loc_idx, p, n, mode)
    return dict(dos=dos, dqs=dqs, dks=dks, dvs=dvs, dq=dq, dk=dk, dv=dv)


class LocalComm:
    """One rank of a job whose ranks run as threads of one process: every
    all_gather waits until all ranks have contributed, then hands each rank
    the list of contributions in rank order."""

    def __init__(self, rank: int, world: int, state: dict):
        self.rank, self.world, self._st = rank, world, state

    def all_gather(self, obj):
        st = self._st
        st["slots"][self.rank] = obj
        st["barrier"].wait()
        out = list(st["slots"])
        st["barrier"].wait()              # nobody overwrites a slot before everyone has read
        return out


def run_local(world: int, fn):
    """Run ``fn(comm)`` for every rank, one thread per rank, in one process;
    returns the ranks' results in rank order (a rank's exception is re-raised)."""
    import threading

    state = {"slots": [None] * world, "barrier": threading.Barrier(world, timeout=600)}
    results, errors = [None] * world, [None] * world

    def body(r):
        try:
            results[r] = fn(LocalComm(r, world, state))
        except BaseException as e:            # noqa: BLE001 - re-raised below
            errors[r] = e
            state["barrier"].abort()

    threads = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    for e in errors:
        if e is not None and not isinstance(e, threading.BrokenBarrierError):
            raise e
    if any(e is not None for e in errors):
        raise RuntimeError("a rank's collective was broken")
    return results

"""Sequence-sharded (context-parallel) Lighthouse step: per-rank buffers and
the order of liblh calls and collectives.

The pages reach 1M-token context on 32 B200s with context parallelism ("Nous
Research's Lighthouse Attention Trains 1.69x Faster on Million-Token
Contexts"; "Lighthouse Attention Technique": past 100K tokens the model is
scaled with context parallelism). Rank r holds tokens [r n, (r+1) n) of every
sequence (n a multiple of p^(L-1)). Every step of the path is a liblh kernel
(include/lh.h, the lh_cp_* entry points); the collectives between them are
NCCL over NVLink through torch.distributed:

  forward   lh_cp_pool -> all-gather(sq_loc) -> lh_cp_assemble_sq ->
            lh_score_topk (the same selection on every rank) -> lh_cp_segment ->
            lh_cp_gather -> all-reduce(ks), all-reduce(vs) -> lh_cp_attn_fwd ->
            lh_cp_scatter
  backward  lh_cp_scatter_bwd -> lh_cp_attn_bwd -> all-reduce(dks), all-reduce(dvs)
            -> lh_cp_spread

The all-gather carries 16 bytes per pyramid entry (two fp64 norms); the
all-reduces carry the sub-sequence's keys and values (fp16) and their
gradients (fp32). Remote rows arrive in this GPU's own memory before any
kernel reads them; no kernel reads another GPU's memory.

``ShardRank`` holds one rank's buffers and runs the kernels between two
collectives; ``run_distributed`` drives one rank with torch.distributed
collectives; ``run_emulated`` drives all ranks of a job in one process on one
GPU (the collectives become sums and stacks of the ranks' tensors), which is
how the kernels of this path are checked where only one GPU is available.
"""

from __future__ import annotations

import torch

from . import lh

__all__ = ["ShardRank", "run_distributed", "run_emulated"]


class ShardRank:
    """Buffers and per-rank steps of rank ``rank`` of ``world``.

    ``cfg`` describes the whole sequence (N = world * n); the token tensors
    passed to the steps are the shard's, [B, n, H, D] bf16.
    """

    def __init__(self, cfg, world: int, rank: int, device):
        self.cfg, self.world, self.rank, self.device = cfg, world, rank, device
        self.cp = cp = lh.cp_plan(cfg, world, rank)
        pl = cp.glob
        B, H, D = cfg.B, cfg.H, cfg.D
        S, E, El = pl.S, pl.E, cp.E_loc
        f16, f32, i32, f64 = torch.float16, torch.float32, torch.int32, torch.float64
        z = lambda *shape, dtype: torch.empty(*shape, dtype=dtype, device=device)
        self.S = S
        self.pyr_q, self.pyr_k, self.pyr_v = (z(B, H, El, D, dtype=torch.bfloat16) for _ in range(3))
        self.sq_loc = z(2, B, H, El, dtype=f64)
        self.sq = z(2, B, H, E, dtype=f64)
        self.sel = z(B, H, cfg.L - 1, cfg.K, dtype=i32)
        self.map = z(B, H, S, dtype=i32)
        self.slot = z(B, H, E, dtype=i32)
        self.slot_loc = z(B, H, El, dtype=i32)
        self.seg = z(B, H, 2, dtype=i32)
        # per-head operand magnitudes [4][B][H]: rows 0-2 max-reduced over the ranks
        self.scale = torch.zeros(4, B, H, dtype=i32, device=device)
        self.ws = z(max(pl.ws_bytes, 16), dtype=torch.uint8)
        self.qs, self.ks, self.vs = (z(B, H, S, D, dtype=f16) for _ in range(3))
        self.os = z(B, H, S, D, dtype=f32)
        self.lse = z(B, H, S, dtype=f32)
        self.dos = z(B, H, S, D, dtype=f16)
        self.delta = z(B, H, S, dtype=f32)
        self.dqs, self.dks, self.dvs = (z(B, H, S, D, dtype=f32) for _ in range(3))

    def gathered_shape(self):
        return (self.world,) + tuple(self.sq_loc.shape)

    # ---- forward
    def pool(self, q, k, v, stream=None):
        lh.cp_pool(self.cfg, self.world, self.rank, q, k, v, self.pyr_q, self.pyr_k, self.pyr_v, self.sq_loc,
                   self.scale, stream)

    def select_gather(self, sq_gathered, q, k, v, stream=None):
        c, W, r = self.cfg, self.world, self.rank
        lh.cp_assemble_sq(c, W, sq_gathered, self.sq, stream)
        lh.score_topk(c, self.sq, self.sel, self.map, self.slot, self.ws, stream=stream)
        lh.cp_segment(c, W, r, self.map, self.slot, self.slot_loc, self.seg, stream)
        lh.cp_gather(c, W, r, q, k, v, self.pyr_q, self.pyr_k, self.pyr_v, self.map, self.seg, self.scale, self.qs,
                     self.ks, self.vs, stream)

    def attend_scatter(self, o, stream=None):
        c, W, r = self.cfg, self.world, self.rank
        lh.cp_attn_fwd(c, W, r, self.seg, self.qs, self.ks, self.vs, self.scale, self.os, self.lse, stream)
        lh.cp_scatter(c, W, r, self.os, self.slot_loc, o, stream)

    # ---- backward
    def attend_bwd(self, do, stream=None):
        c, W, r = self.cfg, self.world, self.rank
        lh.cp_scatter_bwd(c, W, r, do, self.os, self.slot_loc, self.seg, self.dos, self.delta, self.scale, stream)
        lh.cp_attn_bwd(c, W, r, self.seg, self.qs, self.ks, self.vs, self.dos, self.lse, self.delta, self.scale,
                       self.dqs, self.dks, self.dvs, stream)

    def spread(self, dq, dk, dv, stream=None):
        lh.cp_spread(self.cfg, self.world, self.rank, self.dqs, self.dks, self.dvs, self.slot_loc, dq, dk, dv,
                     stream)


def run_distributed(rank_obj, q, k, v, o, do=None, dq=None, dk=None, dv=None, group=None):
    """One forward (and, with ``do``, backward) step of this rank, with the
    collectives of the default (or given) torch.distributed process group."""
    import torch.distributed as dist

    st = rank_obj
    st.pool(q, k, v)
    shape = st.gathered_shape()
    flat = torch.empty(shape[0] * st.sq_loc.numel(), dtype=st.sq_loc.dtype, device=st.device)
    dist.all_gather_into_tensor(flat, st.sq_loc.reshape(-1), group=group)    # rank-major concatenation
    # the operands' largest magnitudes over all shards (fp32 bit patterns of
    # non-negative values order like the values)
    dist.all_reduce(st.scale[:3], op=dist.ReduceOp.MAX, group=group)
    st.select_gather(flat.view(shape), q, k, v)
    dist.all_reduce(st.ks, group=group)
    dist.all_reduce(st.vs, group=group)
    st.attend_scatter(o)
    if do is None:
        return
    st.attend_bwd(do)
    dist.all_reduce(st.dks, group=group)
    dist.all_reduce(st.dvs, group=group)
    st.spread(dq, dk, dv)


def run_emulated(ranks, qs, ks, vs, os_, dos=None, dqs=None, dks=None, dvs=None):
    """All ranks of one job in this process on one device: each step runs for
    every rank, and each collective is formed from all ranks' tensors (an
    all-gather stacks them in rank order; an all-reduce adds them, in rank
    order, and hands every rank the sum). Argument lists are per rank."""
    for st, q, k, v in zip(ranks, qs, ks, vs):
        st.pool(q, k, v)
    gathered = torch.stack([st.sq_loc for st in ranks])
    amax = torch.stack([st.scale[:3] for st in ranks]).amax(dim=0)          # all-reduce (max)
    for st in ranks:
        st.scale[:3].copy_(amax)
    for st, q, k, v in zip(ranks, qs, ks, vs):
        st.select_gather(gathered, q, k, v)

    def all_reduce(name):
        tot = getattr(ranks[0], name).clone()
        for st in ranks[1:]:
            tot += getattr(st, name)
        for st in ranks:
            getattr(st, name).copy_(tot)

    all_reduce("ks")
    all_reduce("vs")
    for st, o in zip(ranks, os_):
        st.attend_scatter(o)
    if dos is None:
        return
    for st, do in zip(ranks, dos):
        st.attend_bwd(do)
    all_reduce("dks")
    all_reduce("dvs")
    for st, dq, dk, dv in zip(ranks, dqs, dks, dvs):
        st.spread(dq, dk, dv)

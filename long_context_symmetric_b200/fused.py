"""The Lighthouse path fused with the projections next to it, chunk by chunk
through L2.

"Long Context Pre-Training with Lighthouse Attention", Fig. 1: the Q, K, V
projections feed the pyramid pool, and the scatter-back feeds the output
projection. Run one after the other over a whole 512K-token sequence, each
of these steps streams its tensors through HBM: the projections write Q, K, V
(6.4 GB at H16 D128 bf16) and the pool reads them back; the scatter writes O
(2.1 GB) and the output projection reads it back. Here the sequence is cut
into chunks of whole coarsest blocks small enough to stay in the 126 MB L2:

  qkv_project_pool   chunk i: Q, K, V = X W_q, X W_k, X W_v (cuBLAS through
                     torch.matmul, the three at once on three streams), then
                     lh_pool_range on another stream while the projections of
                     chunk i+1 run, reading chunk i from L2;
  scatter_project    chunk i: lh_scatter_range on a second stream, then
                     Y = O W_o (on two streams in turn), reading chunk i of O
                     from L2 while chunk i+1 is being scattered.

The projections are plain library GEMMs (they are the model's, not the path's);
every step of the path stays a liblh kernel. The pool and scatter results
are bit-identical to lh_pool and lh_scatter over the whole sequence. A 512K
sequence is 128 chunks of several launches each, too many for the host to
issue at GPU speed, so ``Graphed`` captures a chunk loop once as a CUDA graph
and replays it.
"""

from __future__ import annotations

import torch

from . import lh

__all__ = ["chunk_tokens", "qkv_project_pool", "scatter_project", "Graphed"]


def chunk_tokens(cfg, target: int = 8192) -> int:
    """Chunk length: a multiple of p^(L-1) close to `target` tokens (at least one block)."""
    P = cfg.p ** (cfg.L - 1)
    c = max(P, (target // P) * P)
    while cfg.N % c:
        c -= P
    return c


def _streams(n, given):
    return list(given) if given is not None else [torch.cuda.Stream() for _ in range(n)]


def qkv_project_pool(cfg, ws, x, w_q, w_k, w_v, q, k, v, chunk=None, side=None, gemm_streams=None):
    """q, k, v [B, N, H, D] = x [B, N, d_model] @ w_* [d_model, H*D], and the
    pyramid / norms of ws (lh.Workspace) by lh_pool_range, chunk by chunk.
    A chunk's three projections run at once (the current stream and two of
    `gemm_streams`), so that together they fill the GPU; the pool of chunk i
    runs on `side` once all three have written it."""
    B, N = cfg.B, cfg.N
    HD = cfg.H * cfg.D
    c = chunk or chunk_tokens(cfg)
    main = torch.cuda.current_stream()
    side = side or torch.cuda.Stream()
    gs = [main] + _streams(2, gemm_streams)
    for st in gs[1:] + [side]:
        st.wait_stream(main)
    for t0 in range(0, N, c):
        for (w, out), st in zip(((w_q, q), (w_k, k), (w_v, v)), gs):
            with torch.cuda.stream(st):
                for b in range(B):
                    torch.matmul(x[b, t0:t0 + c], w, out=out[b, t0:t0 + c].view(c, HD))
            ev = torch.cuda.Event()
            ev.record(st)
            side.wait_event(ev)
        lh.pool_range(cfg, t0, c, q, k, v, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.sq, ws.scale, stream=side)
    for st in gs[1:] + [side]:
        main.wait_stream(st)


def scatter_project(cfg, ws, w_o, o, y, chunk=None, side=None, gemm_streams=None):
    """o [B, N, H, D] = scatter of ws.os by lh_scatter_range, and
    y [B, N, d_out] = o @ w_o [H*D, d_out], chunk by chunk: chunk i's GEMM reads
    the rows the scatter of chunk i has just written. Consecutive chunks' GEMMs
    alternate between the current stream and one of `gemm_streams`, so that one
    chunk's GEMM fills the tail of the previous one."""
    B, N = cfg.B, cfg.N
    HD = cfg.H * cfg.D
    c = chunk or chunk_tokens(cfg)
    main = torch.cuda.current_stream()
    side = side or torch.cuda.Stream()
    gs = [main] + _streams(1, gemm_streams)
    for st in gs[1:] + [side]:
        st.wait_stream(main)
    done = []
    for i, t0 in enumerate(range(0, N, c)):
        if i >= 2:
            side.wait_event(done[i - 2])       # at most two chunks of O ahead of the GEMMs (L2-resident)
        lh.scatter_range(cfg, t0, c, ws.os, ws.slot, o, stream=side)
        ev = torch.cuda.Event()
        ev.record(side)
        st = gs[i % 2]
        st.wait_event(ev)
        with torch.cuda.stream(st):
            for b in range(B):
                torch.matmul(o[b, t0:t0 + c].view(c, HD), w_o, out=y[b, t0:t0 + c])
        d = torch.cuda.Event()
        d.record(st)
        done.append(d)
    for st in gs[1:] + [side]:
        main.wait_stream(st)


class Graphed:
    """A stream-ordered function (such as a chunk loop above) captured once as a
    CUDA graph and replayed by calling the object: the host issues one graph
    launch instead of several hundred kernel launches. The function runs once
    un-captured first (library handles, device-symbol lookups and kernel
    attributes are set up outside the capture). It must read and write the same
    tensors on every call."""

    def __init__(self, fn):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            fn()

    def __call__(self):
        self.graph.replay()

"""Fusion with the neighbouring projections, chunk by chunk through L2
(long_context_symmetric_b200.fused): the pool of each projected chunk and the
scatter feeding each output-projection chunk equal the whole-sequence
lh_pool / lh_scatter bit for bit, and the projections equal the same GEMMs
run on the unfused tensors."""

import pytest
import torch

from lhtest import Case, compare_head, run_gpu
from long_context_symmetric_b200 import fused, lh, synth

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


@pytest.mark.parametrize("B,H,N,D,p,L,K,chunk", [
    (1, 4, 16384, 128, 4, 3, 64, 2048),
    (2, 3, 8192, 64, 8, 3, 16, 1024),
    (1, 2, 4096, 128, 2, 5, 32, 1 << 12),          # one chunk
    (1, 2, 8192, 128, 8, 4, 64, 2048),             # 4 coarsest blocks a chunk: the per-token scatter walk
])
def test_chunked_projection_pool_and_scatter(B, H, N, D, p, L, K, chunk):
    g = torch.Generator(device=DEV).manual_seed(9)
    dm = H * D
    x = torch.randn(B, N, dm, generator=g, device=DEV).to(torch.bfloat16)
    w = [(torch.randn(dm, dm, generator=g, device=DEV) / dm ** 0.5).to(torch.bfloat16) for _ in range(4)]
    cfg = lh.make_config(B, H, N, D, p, L, K, "bf16")
    ws = lh.Workspace(cfg, DEV, backward=False)
    q, k, v = (torch.empty(B, N, H, D, dtype=torch.bfloat16, device=DEV) for _ in range(3))
    fused.qkv_project_pool(cfg, ws, x, w[0], w[1], w[2], q, k, v, chunk=chunk)
    # the unfused reference: the same GEMMs, then the whole-sequence pool
    qr, kr, vr = (torch.empty_like(q) for _ in range(3))
    for t0 in range(0, N, chunk):
        for b in range(B):
            for wt, out in ((w[0], qr), (w[1], kr), (w[2], vr)):
                torch.matmul(x[b, t0:t0 + chunk], wt, out=out[b, t0:t0 + chunk].view(chunk, dm))
    ref = lh.Workspace(cfg, DEV, backward=False)
    lh.pool(cfg, qr, kr, vr, ref.pyr_q, ref.pyr_k, ref.pyr_v, ref.sq, ref.scale)
    torch.cuda.synchronize()
    assert torch.equal(q, qr) and torch.equal(k, kr) and torch.equal(v, vr)
    for a, b_ in ((ws.pyr_q, ref.pyr_q), (ws.pyr_k, ref.pyr_k), (ws.pyr_v, ref.pyr_v), (ws.sq, ref.sq)):
        assert torch.equal(a, b_)
    # rest of the forward, then the chunked scatter + output projection
    lh.score_topk(cfg, ws.sq, ws.sel, ws.map, ws.slot, ws.ws)
    lh.gather(cfg, q, k, v, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.map, ws.scale, ws.qs, ws.ks, ws.vs)
    lh.attn_fwd(cfg, ws.qs, ws.ks, ws.vs, ws.scale, ws.os, ws.lse)
    o = torch.empty_like(q)
    y = torch.empty(B, N, dm, dtype=torch.bfloat16, device=DEV)
    fused.scatter_project(cfg, ws, w[3], o, y, chunk=chunk)
    o_ref = torch.empty_like(q)
    lh.scatter(cfg, ws.os, ws.slot, o_ref)
    y_ref = torch.empty_like(y)
    for t0 in range(0, N, chunk):
        for b in range(B):
            torch.matmul(o_ref[b, t0:t0 + chunk].view(chunk, dm), w[3], out=y_ref[b, t0:t0 + chunk])
    torch.cuda.synchronize()
    assert lh.get_device_error() == (0, 0)
    assert torch.equal(o, o_ref)
    assert torch.equal(y, y_ref)


def test_graphed_chunk_loop_replays_the_same_results():
    """The chunk loops captured as CUDA graphs (fused.Graphed) give the same
    pyramid, norms and output as the un-captured loops."""
    B, H, N, D, p, L, K, chunk = 1, 2, 8192, 128, 4, 3, 32, 1024
    g = torch.Generator(device=DEV).manual_seed(3)
    dm = H * D
    x = torch.randn(B, N, dm, generator=g, device=DEV).to(torch.bfloat16)
    w = [(torch.randn(dm, dm, generator=g, device=DEV) / dm ** 0.5).to(torch.bfloat16) for _ in range(4)]
    cfg = lh.make_config(B, H, N, D, p, L, K, "bf16")
    ws, ref = lh.Workspace(cfg, DEV, backward=False), lh.Workspace(cfg, DEV, backward=False)
    q, k, v, o = (torch.empty(B, N, H, D, dtype=torch.bfloat16, device=DEV) for _ in range(4))
    y = torch.empty(B, N, dm, dtype=torch.bfloat16, device=DEV)
    fused.qkv_project_pool(cfg, ref, x, w[0], w[1], w[2], q, k, v, chunk=chunk)
    lh.score_topk(cfg, ref.sq, ref.sel, ref.map, ref.slot, ref.ws)
    lh.gather(cfg, q, k, v, ref.pyr_q, ref.pyr_k, ref.pyr_v, ref.map, ref.scale, ref.qs, ref.ks, ref.vs)
    lh.attn_fwd(cfg, ref.qs, ref.ks, ref.vs, ref.scale, ref.os, ref.lse)
    fused.scatter_project(cfg, ref, w[3], o, y, chunk=chunk)
    torch.cuda.synchronize()
    y_ref = y.clone()
    gq = fused.Graphed(lambda: fused.qkv_project_pool(cfg, ws, x, w[0], w[1], w[2], q, k, v, chunk=chunk))
    ws.os.copy_(ref.os)
    ws.slot.copy_(ref.slot)
    go = fused.Graphed(lambda: fused.scatter_project(cfg, ws, w[3], o, y, chunk=chunk))
    for _ in range(2):
        ws.sq.zero_()
        y.zero_()
        gq()
        go()
        torch.cuda.synchronize()
        assert torch.equal(ws.sq, ref.sq) and torch.equal(ws.pyr_k, ref.pyr_k)
        assert torch.equal(y, y_ref)
    assert lh.get_device_error() == (0, 0)


def test_ranges_reject_unaligned_tokens():
    cfg = lh.make_config(1, 2, 4096, 128, 4, 3, 16, "bf16")
    t = torch.empty(1 << 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(lh.LHError):
        lh.pool_range(cfg, 8, 16, t, t, t, t, t, t, t, t)          # t0 not a multiple of 16
    with pytest.raises(lh.LHError):
        lh.scatter_range(cfg, 0, 4112, t, t, t)                # past N

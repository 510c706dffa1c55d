"""Allocation-free top-K descent: lh_score_topk_noalloc against lh_score_topk.

Some callers cannot give liblh a device workspace: a fixed memory arena that
may not grow, or a hot path that may not call cudaMalloc because it can
synchronise the device. For them, the descent can keep its scratch in a fixed
device array inside the library. Its outputs must equal the workspace
version's bit for bit, on every call. The array keeps the previous call's
contents, so two calls in a row are checked.

Collected last on purpose (file name), so a run that stops at the first
failure has already run every other test.
"""

import ctypes

import pytest
import torch

from long_context_symmetric_b200 import lh, synth

pytestmark = pytest.mark.gpu


def _noalloc(cfg, sq, sel, map_, slot):
    f = lh.lib().lh_score_topk_noalloc
    f.argtypes = [ctypes.POINTER(lh.Config)] + [ctypes.c_void_p] * 5
    f.restype = ctypes.c_int
    return f(ctypes.byref(cfg), sq.data_ptr(), sel.data_ptr(), map_.data_ptr(), slot.data_ptr(),
             torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("name,N,H,p,L,K", [
    ("bf16_small", 8192, 4, 4, 3, 256),
    ("ties", 16384, 2, 4, 5, 64),
])
def test_noalloc_matches_workspace_version(name, N, H, p, L, K):
    w = synth.Workload(name, 1, H, N, 128, "bf16", p, L, K,
                       "codebook" if name == "ties" else "iid", "fp", False, 11)
    q, k, v = (x.cuda() for x in synth.make_inputs(w))
    cfg = lh.make_config(1, H, N, 128, p, L, K, "bf16")
    ws = lh.Workspace(cfg, q.device, backward=False)
    lh.pool(cfg, q, k, v, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.sq, ws.scale)
    lh.score_topk(cfg, ws.sq, ws.sel, ws.map, ws.slot, ws.ws)
    torch.cuda.synchronize()
    for call in range(2):
        sel = torch.full_like(ws.sel, -7)
        map_ = torch.full_like(ws.map, -7)
        slot = torch.full_like(ws.slot, -7)
        assert _noalloc(cfg, ws.sq, sel, map_, slot) == 0, f"call {call}"
        torch.cuda.synchronize()
        assert lh.get_device_error()[0] == 0
        assert torch.equal(sel, ws.sel), f"sel, call {call}"
        assert torch.equal(map_, ws.map), f"map, call {call}"
        assert torch.equal(slot, ws.slot), f"slot, call {call}"


def test_noalloc_rejects_oversized_problems():
    # 5 * S * B * H int32 beyond the fixed 8 MiB array: refused before any launch
    cfg = lh.make_config(4, 16, 524288, 128, 8, 4, 1024, "bf16")
    t = torch.empty(16, dtype=torch.int32, device="cuda")
    sq = torch.empty(16, dtype=torch.float64, device="cuda")
    assert _noalloc(cfg, sq, t, t, t) == 6   # LH_ERR_WORKSPACE

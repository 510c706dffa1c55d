"""Debug build with device-side bounds checks (liblh_debug.so, -DLH_DEBUG_BOUNDS).

The memory kernels index the sub-sequence rows and the pyramid with values
they read from the gather map and the slot table. In the debug build each such
index is checked against the buffer it addresses before use; a bad one is
reported through the device error word (LH_ERR_DEVICE, 301 for a map entry in
the gather, 303 for a slot in the block sums) and its access is skipped. On
good data the debug build gives the release build's results bit for bit; on a
corrupted index (chosen so that even an unchecked access would stay inside the
buffers) it reports the site.
"""

import ctypes

import pytest
import torch

from lhtest import Case, run_gpu
from long_context_symmetric_b200 import build, lh, synth

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
LH_ERR_DEVICE = 9


@pytest.fixture(scope="module")
def debug_lib():
    path = build.build(debug_bounds=True)
    l = ctypes.CDLL(path)
    for name, (args, res) in lh._SIGS.items():
        f = getattr(l, name)
        f.argtypes = args
        f.restype = res
    return l


class _using:
    """Route the lh wrappers to another loaded copy of the library."""

    def __init__(self, l):
        self.l = l

    def __enter__(self):
        self.saved = lh.lib()
        lh._lib = self.l

    def __exit__(self, *exc):
        lh._lib = self.saved


def _inputs(case):
    w = case.workload()
    q, k, v = synth.make_inputs(w, device="cpu")
    do = synth.make_dout(w, device="cpu")
    return [x.to(DEV) for x in (q, k, v, do)]


def test_debug_build_matches_release_bit_for_bit(debug_lib):
    case = Case("debug", 1, 2, 4096, 128, "bf16", 4, 3, 32)
    q, k, v, do = _inputs(case)
    rel = run_gpu(case, q, k, v, do)
    with _using(debug_lib):
        dbg = run_gpu(case, q, k, v, do)          # asserts no device error
    for name in ("o", "dq", "dk", "dv"):
        assert torch.equal(rel[name], dbg[name]), name
    for name in ("map", "slot", "qs", "os", "dos"):
        assert torch.equal(getattr(rel["ws"], name), getattr(dbg["ws"], name)), name


def test_debug_build_reports_bad_indices(debug_lib):
    case = Case("debug_bad", 1, 2, 4096, 128, "bf16", 4, 3, 32)
    q, k, v, do = _inputs(case)
    cfg = case.cfg()
    pl = lh.plan(cfg)
    with _using(debug_lib):
        ws = lh.Workspace(cfg, q.device, backward=True)
        lh.pool(cfg, q, k, v, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.sq, ws.scale)
        lh.score_topk(cfg, ws.sq, ws.sel, ws.map, ws.slot, ws.ws)
        torch.cuda.synchronize()
        assert lh.get_device_error() == (0, 0)
        # a level-1 map entry pointing one past its level: the pyramid row there is
        # the first of level 2, so even an unchecked read stays inside the buffer
        m = ws.map[0, 0]
        j = int(((m >> 28) == 1).nonzero()[0])
        m[j] = (1 << 28) | pl.n[1]
        lh.gather(cfg, q, k, v, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.map, ws.scale, ws.qs, ws.ks, ws.vs)
        torch.cuda.synchronize()
        assert lh.get_device_error() == (LH_ERR_DEVICE, 301)
        # a coarsest entry's slot past the sub-sequence: only the block sums run on it
        o = torch.empty_like(q)
        lh.score_topk(cfg, ws.sq, ws.sel, ws.map, ws.slot, ws.ws)
        lh.gather(cfg, q, k, v, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.map, ws.scale, ws.qs, ws.ks, ws.vs)
        lh.attn_fwd(cfg, ws.qs, ws.ks, ws.vs, ws.scale, ws.os, ws.lse)
        lh.scatter(cfg, ws.os, ws.slot, o)
        torch.cuda.synchronize()
        assert lh.get_device_error() == (0, 0)
        e = int(ws.slot[0, 0, pl.lvl_off[2]])
        ws.slot[0, 0, pl.lvl_off[2]] = 2 * (pl.S + 5) + (e & 1)
        lh.scatter_bwd(cfg, do, ws.os, ws.slot, ws.dos, ws.delta, ws.scale)
        torch.cuda.synchronize()
        assert lh.get_device_error() == (LH_ERR_DEVICE, 303)
        assert lh.get_device_error() == (0, 0)

"""Device-side range checks of the fp16 attention operands report a status.

For bf16 I/O the sub-sequence, the block sums of dO and dS enter the tensor
cores as fp16, whose largest finite value is 65504. A value beyond it is not
stored silently as infinity: the kernel records LH_ERR_DEVICE in the device
error word with a detail naming the site (102: gathered token or entry,
100: block sum of dO, 101: dS, seen as a non-finite dQ or dK), and the host
reads it with lh_get_device_error. These are statuses, not faults: every
kernel runs to completion on such data and the context stays usable, which
the last check of each test confirms with a clean run.
"""

import pytest
import torch

from lhtest import Case, compare_head, run_gpu
from long_context_symmetric_b200 import lh, synth

pytestmark = pytest.mark.gpu

LH_ERR_DEVICE = 9
DEV = "cuda:0"


def _case():
    return Case("range", 1, 1, 1024, 128, "bf16", 4, 3, 8)


def _inputs(case):
    w = case.workload()
    q, k, v = synth.make_inputs(w, device="cpu")
    do = synth.make_dout(w, device="cpu")
    return q, k, v, do


def _forward(case, q, k, v, through_gather=False):
    cfg = case.cfg()
    ws = lh.Workspace(cfg, q.device, backward=True)
    o = torch.empty_like(q)
    lh.pool(cfg, q, k, v, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.sq)
    lh.score_topk(cfg, ws.sq, ws.sel, ws.map, ws.slot, ws.ws)
    lh.gather(cfg, q, k, v, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.map, ws.qs, ws.ks, ws.vs)
    if through_gather:
        return cfg, ws, o
    lh.attn_fwd(cfg, ws.qs, ws.ks, ws.vs, ws.os, ws.lse)
    lh.scatter(cfg, ws.os, ws.slot, o)
    return cfg, ws, o


def _backward(cfg, ws, q, do):
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    lh.scatter_bwd(cfg, do, ws.os, ws.slot, ws.dos, ws.delta)
    lh.attn_bwd(cfg, ws.qs, ws.ks, ws.vs, ws.dos, ws.lse, ws.delta, ws.dqs, ws.dks, ws.dvs)
    lh.spread(cfg, ws.dqs, ws.dks, ws.dvs, ws.slot, dq, dk, dv)


def _clean_run_after():
    case = _case()
    q, k, v, do = (x.to(DEV) for x in _inputs(case))
    res = run_gpu(case, q, k, v, do)
    compare_head(case, res, q, k, v, do, 0, 0)


def test_gathered_value_beyond_fp16_reports_102():
    """A token of magnitude 1e5 (a legal bf16 value): its ancestors' norms make
    it selected at every level, so it enters the sub-sequence as itself; its
    fp16 copy would overflow, and the gather reports detail 102."""
    case = _case()
    q, k, v, do = _inputs(case)
    q[0, 100, 0, :] = 1.0e5
    assert float(q[0, 100, 0, 0]) > 65504
    q, k, v = (x.to(DEV) for x in (q, k, v))
    assert lh.get_device_error() == (0, 0)
    cfg, ws, _ = _forward(case, q, k, v, through_gather=True)
    torch.cuda.synchronize()
    m = ws.map[0, 0].cpu()
    assert int(((m >> 28) == 0).logical_and((m & 0x0FFFFFFF) == 100).sum()) == 1   # token 100 is gathered
    assert lh.get_device_error() == (LH_ERR_DEVICE, 102)
    assert lh.get_device_error() == (0, 0)
    _clean_run_after()


def test_block_sum_beyond_fp16_reports_100():
    """dO of 30000 on every token of one coarsest block (16 tokens): that
    entry's block sum is about 4.8e5, beyond fp16; the block-sum pass reports
    detail 100."""
    case = _case()
    q, k, v, do = _inputs(case)
    do[0, 32:48, 0, :] = 30000.0
    q, k, v, do = (x.to(DEV) for x in (q, k, v, do))
    assert lh.get_device_error() == (0, 0)
    cfg, ws, _ = _forward(case, q, k, v)
    torch.cuda.synchronize()
    assert lh.get_device_error() == (0, 0)          # the forward is clean
    _backward(cfg, ws, q, do)
    torch.cuda.synchronize()
    assert lh.get_device_error() == (LH_ERR_DEVICE, 100)
    assert lh.get_device_error() == (0, 0)
    _clean_run_after()


def test_ds_beyond_fp16_reports_101():
    """dO of 50000 on one token (its block sums stay below 65504) with V scaled
    by 64: dP = dO V^T reaches about 1e7 on the rows of the entries covering that
    token, dS = P (dP - delta) leaves the fp16 range, the dQ and dK accumulators
    become non-finite, and the epilogues report detail 101."""
    case = _case()
    q, k, v, do = _inputs(case)
    do[0, 40, 0, :] = 50000.0
    v = (v.float() * 64.0).to(v.dtype)
    q, k, v, do = (x.to(DEV) for x in (q, k, v, do))
    assert lh.get_device_error() == (0, 0)
    cfg, ws, _ = _forward(case, q, k, v)
    torch.cuda.synchronize()
    assert lh.get_device_error() == (0, 0)
    lh.scatter_bwd(cfg, do, ws.os, ws.slot, ws.dos, ws.delta)
    torch.cuda.synchronize()
    assert lh.get_device_error() == (0, 0)          # block sums are in range
    assert float(ws.dos.float().abs().max()) < 65504
    _backward(cfg, ws, q, do)
    torch.cuda.synchronize()
    assert lh.get_device_error() == (LH_ERR_DEVICE, 101)
    assert lh.get_device_error() == (0, 0)
    _clean_run_after()

"""Operand range of the fp16 attention path (bf16 I/O).

The sub-sequence, the block sums of dO and dS enter the tensor cores as fp16
(largest finite value 65504, smallest normal 2^-14), while bf16 reaches 3e38
and 1e-38. Each head's operands enter as x * 2^-e, with a power-of-two
exponent e per head and operand chosen from the head's largest magnitude
(lh_pool, lh_scatter_bwd), and the kernels take the powers of two out of their
results. So:
  - legal bf16 data far outside fp16's range (magnitudes around 1e5 and 1e-5,
    block sums of dO near 1e6) matches the fp64 oracle, and a problem scaled by
    powers of two gives the unscaled problem's output scaled by the same power,
    bit for bit;
  - only non-finite data is reported, as LH_ERR_DEVICE with a detail naming
    the site (102: gathered row, 100: block sum of dO, 101: non-finite dQ or
    dK), and the context stays usable (each test ends with a clean run).
"""

import numpy as np
import pytest
import torch

from lhtest import ATOL, Case, compare_head, excess_error, run_gpu, to64
import oracle as orc
from long_context_symmetric_b200 import lh

pytestmark = pytest.mark.gpu

LH_ERR_DEVICE = 9
DEV = "cuda:0"


def _case(**readings):
    return Case("range", 1, 2, 4096, 128, "bf16", 4, 3, 32, **readings)


def _inputs(case):
    w = case.workload()
    from long_context_symmetric_b200 import synth
    q, k, v = synth.make_inputs(w, device="cpu")
    do = synth.make_dout(w, device="cpu")
    return q, k, v, do


def _scaled(x, power):
    return (x.float() * 2.0 ** power).to(torch.bfloat16)


def _clean_run_after():
    case = _case()
    q, k, v, do = (x.to(DEV) for x in _inputs(case))
    res = run_gpu(case, q, k, v, do)
    compare_head(case, res, q, k, v, do, 0, 0)


def test_magnitudes_beyond_fp16_match_scaled_problem_and_oracle():
    """q * 2^17 (~1e5, beyond fp16), k * 2^-17 (~1e-5, below fp16's normals),
    v * 2^17 and dO * 2^-10: the attention logits are those of the unscaled
    problem, and under the product score (|q|^2 |k|^2, unchanged by the
    scaling) so is the selection. The output equals the unscaled problem's
    times 2^17 bit for bit, the gradients agree with the unscaled ones to fp16
    rounding, and all match the fp64 oracle of the scaled inputs within the
    stated tolerance once divided by their power of two."""
    case = _case(score="prod")
    q, k, v, do = _inputs(case)
    pq, pk, pv, pdo = 17, -17, 17, -10
    qs, ks, vs, dos = _scaled(q, pq), _scaled(k, pk), _scaled(v, pv), _scaled(do, pdo)
    assert float(qs.float().abs().max()) > 65504 and float(ks.float().abs().max()) < 2.0 ** -14
    base = run_gpu(case, *(x.to(DEV) for x in (q, k, v, do)))
    big = run_gpu(case, *(x.to(DEV) for x in (qs, ks, vs, dos)))
    ws = big["ws"]
    # the head's exponents are in use: q, k, v far outside [4, 256)
    assert int(ws.scale[0, 0, 0]) != int(base["ws"].scale[0, 0, 0])
    ds = pdo + pv                                       # dP and dS carry 2^(pdo + pv)
    powers = {"o": pv, "dq": ds + pk, "dk": ds + pq, "dv": pdo}
    # forward: the same fp16 operands (q, k, v each brought back by its exponent),
    # so O is the unscaled O times 2^17 bit for bit; the backward's dO block sums
    # land in [4, 8) rather than at their unscaled size, so the gradients agree
    # to fp16 rounding (and with the oracle, below)
    assert torch.equal(big["o"].float() * 2.0 ** -pv, base["o"].float())
    for name in ("dq", "dk", "dv"):
        a, b_ = big[name].float() * 2.0 ** -powers[name], base[name].float()
        assert float((a - b_).abs().max()) <= 2.0 ** -8 * float(b_.abs().max()), name
    assert torch.equal(big["ws"].sel, base["ws"].sel) and torch.equal(big["ws"].map, base["ws"].map)
    qd, kd, vd, dd = (x.to(DEV) for x in (qs, ks, vs, dos))
    for h in range(case.H):
        qh, kh, vh = (to64(x[0, :, h, :]) for x in (qd, kd, vd))
        fw = orc.forward_head(qh, kh, vh, case.p, case.L, case.K, "bf16", score="prod")
        bw = orc.backward_head(fw, to64(dd[0, :, h, :]), case.p)
        refs = {"o": fw["o"], "dq": bw["dq"], "dk": bw["dk"], "dv": bw["dv"]}
        for name, pw in powers.items():
            e = excess_error(to64(big[name][0, :, h, :]) * 2.0 ** -pw, refs[name] * 2.0 ** -pw, "bf16")
            assert e <= ATOL["bf16"], (name, e)


def test_block_sums_beyond_fp16_match_oracle():
    """dO * 2^14 (about 1.6e4 per element): the block sums of pooled entries reach
    about 1e6, far beyond fp16. The block-sum pass records each head's largest
    magnitude, redoes the heads with their exponents, and the gradients (2^14
    times the unscaled ones) agree with the unscaled problem's to fp16 rounding
    and with the fp64 oracle within the stated tolerance once divided by 2^14."""
    case = _case()
    q, k, v, do = _inputs(case)
    big_do = _scaled(do, 14)
    base = run_gpu(case, *(x.to(DEV) for x in (q, k, v, do)))
    q, k, v, big_do = (x.to(DEV) for x in (q, k, v, big_do))
    res = run_gpu(case, q, k, v, big_do)
    for h in range(case.H):
        assert float(res["ws"].scale[3, 0, h].view(torch.float32)) > 65504
    for name in ("dq", "dk", "dv"):
        a, b_ = res[name].float() * 2.0 ** -14, base[name].float()
        assert float((a - b_).abs().max()) <= 2.0 ** -8 * float(b_.abs().max()), name
    for h in range(case.H):
        qh, kh, vh = (to64(x[0, :, h, :]) for x in (q, k, v))
        fw = orc.forward_head(qh, kh, vh, case.p, case.L, case.K, "bf16")
        bw = orc.backward_head(fw, to64(big_do[0, :, h, :]), case.p)
        for name in ("dq", "dk", "dv"):
            e = excess_error(to64(res[name][0, :, h, :]) * 2.0 ** -14, bw[name] * 2.0 ** -14, "bf16")
            assert e <= ATOL["bf16"], (name, e)


def test_non_finite_gathered_value_reports_102():
    """An infinite token (a legal bf16 value): its ancestors' norms make it
    selected at every level, so it enters the sub-sequence as itself, and the
    gather reports detail 102."""
    case = _case()
    q, k, v, do = _inputs(case)
    q[0, 100, 0, :] = float("inf")
    q, k, v = (x.to(DEV) for x in (q, k, v))
    cfg = case.cfg()
    ws = lh.Workspace(cfg, q.device, backward=True)
    assert lh.get_device_error() == (0, 0)
    lh.pool(cfg, q, k, v, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.sq, ws.scale)
    lh.score_topk(cfg, ws.sq, ws.sel, ws.map, ws.slot, ws.ws)
    lh.gather(cfg, q, k, v, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.map, ws.scale, ws.qs, ws.ks, ws.vs)
    torch.cuda.synchronize()
    m = ws.map[0, 0].cpu()
    assert int(((m >> 28) == 0).logical_and((m & 0x0FFFFFFF) == 100).sum()) == 1   # token 100 is gathered
    assert lh.get_device_error() == (LH_ERR_DEVICE, 102)
    assert lh.get_device_error() == (0, 0)
    _clean_run_after()


def test_non_finite_block_sum_reports_100():
    case = _case()
    q, k, v, do = _inputs(case)
    do[0, 40, 1, 3] = float("inf")
    q, k, v, do = (x.to(DEV) for x in (q, k, v, do))
    cfg = case.cfg()
    ws = lh.Workspace(cfg, q.device, backward=True)
    o = torch.empty_like(q)
    lh.forward(cfg, q, k, v, o, ws)
    torch.cuda.synchronize()
    assert lh.get_device_error() == (0, 0)
    lh.scatter_bwd(cfg, do, ws.os, ws.slot, ws.dos, ws.delta, ws.scale)
    torch.cuda.synchronize()
    assert lh.get_device_error() == (LH_ERR_DEVICE, 100)
    assert lh.get_device_error() == (0, 0)
    _clean_run_after()


def test_non_finite_gradient_reports_101():
    """An infinite key: the forward reports it at the gather (102, read and
    cleared here); the backward's dQ and dK come out non-finite and the
    attention backward reports detail 101."""
    case = _case()
    q, k, v, do = _inputs(case)
    k[0, 7, 0, :] = float("inf")
    q, k, v, do = (x.to(DEV) for x in (q, k, v, do))
    cfg = case.cfg()
    ws = lh.Workspace(cfg, q.device, backward=True)
    o = torch.empty_like(q)
    lh.forward(cfg, q, k, v, o, ws)
    torch.cuda.synchronize()
    assert lh.get_device_error() == (LH_ERR_DEVICE, 102)
    lh.scatter_bwd(cfg, do, ws.os, ws.slot, ws.dos, ws.delta, ws.scale)
    torch.cuda.synchronize()
    st, detail = lh.get_device_error()          # the block sums meet NaN outputs: 100 may come first
    assert st in (0, LH_ERR_DEVICE)
    lh.attn_bwd(cfg, ws.qs, ws.ks, ws.vs, ws.dos, ws.lse, ws.delta, ws.scale, ws.dqs, ws.dks, ws.dvs)
    torch.cuda.synchronize()
    assert lh.get_device_error() == (LH_ERR_DEVICE, 101)
    assert lh.get_device_error() == (0, 0)
    _clean_run_after()

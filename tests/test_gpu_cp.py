"""Sequence-sharded (context-parallel) path on one GPU, ranks emulated.

Every rank's steps are the lh_cp_* kernels; the ranks of one job run one
after another in this process and the collectives are formed from all ranks'
tensors (cp.run_emulated), so no kernel ever waits on another rank. Checked
against the single-GPU path on the same whole-sequence inputs, and against
the fp64 oracle:
  - selection, gather map and slot table: bit-exact (every rank runs the same
    descent on the assembled norms);
  - each rank's segment is the run of slots whose entries lie in its shard;
  - O and dQ: bit-exact (each query row sees the same key tiles in the same
    order as on one GPU);
  - dK, dV: the key gradients are summed over ranks, so they agree with the
    single-GPU result to fp32 rounding and with the oracle within the stated
    tolerance.
"""

import numpy as np
import pytest
import torch

from lhtest import ATOL, Case, excess_error, run_gpu, to64
import oracle as orc
from long_context_symmetric_b200 import cp, lh, synth

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)

CASES = [
    (Case("cp_w2", 1, 2, 8192, 128, "bf16", 4, 3, 64), 2),
    (Case("cp_w4", 1, 2, 8192, 128, "bf16", 4, 3, 64), 4),
    (Case("cp_w4_d64_b2", 2, 3, 8192, 64, "bf16", 4, 4, 40, recipe="token_scale"), 4),
    (Case("cp_w8_ties", 1, 2, 16384, 128, "bf16", 4, 4, 100, recipe="codebook", accum="fixed"), 8),
    (Case("cp_w2_pre_partition", 1, 2, 8192, 128, "bf16", 4, 3, 64, order="pre", inclusion="partition",
          weight="mean"), 2),
    (Case("cp_w4_p8_l4", 1, 2, 32768, 128, "bf16", 8, 4, 256, recipe="outliers"), 4),
]


def _shard(x, world, r):
    n = x.shape[1] // world
    return x[:, r * n:(r + 1) * n].contiguous()


@pytest.mark.parametrize("case,world", CASES, ids=[c.name for c, _ in CASES])
def test_sharded_path_matches_single_gpu_and_oracle(case, world):
    w = case.workload()
    q, k, v = (x.to(DEV) for x in synth.make_inputs(w))
    do = synth.make_dout(w).to(DEV)
    ref = run_gpu(case, q, k, v, do)                      # the single-GPU path
    cfg = case.cfg()
    ranks = [cp.ShardRank(cfg, world, r, DEV) for r in range(world)]
    sh = lambda x: [_shard(x, world, r) for r in range(world)]
    qs_, ks_, vs_, dos_ = sh(q), sh(k), sh(v), sh(do)
    outs = [torch.empty_like(x) for x in qs_]
    dqs, dks, dvs = ([torch.empty_like(x) for x in qs_] for _ in range(3))
    cp.run_emulated(ranks, qs_, ks_, vs_, outs, dos_, dqs, dks, dvs)
    torch.cuda.synchronize()
    assert lh.get_device_error() == (0, 0)
    ws = ref["ws"]
    S = ws.map.shape[-1]
    starts = np.zeros((case.B, case.H), dtype=np.int64)
    for r, st in enumerate(ranks):
        assert torch.equal(st.sel, ws.sel) and torch.equal(st.map, ws.map) and torch.equal(st.slot, ws.slot)
        seg = st.seg.cpu().numpy()
        assert np.array_equal(seg[..., 0], starts)          # segments follow each other in rank order
        m = st.map.cpu().numpy().astype(np.int64)
        lvl, idx = m >> 28, m & 0x0FFFFFFF
        first = idx * case.p ** lvl                          # first token each entry covers
        n = case.N // world
        for b in range(case.B):
            for h in range(case.H):
                mine = (first[b, h] >= r * n) & (first[b, h] < (r + 1) * n)
                s0, cnt = seg[b, h]
                assert mine.sum() == cnt and np.all(mine[s0:s0 + cnt])
        starts += seg[..., 1]
    assert np.all(starts == S)
    o = torch.cat(outs, dim=1)
    dq, dk, dv = (torch.cat(x, dim=1) for x in (dqs, dks, dvs))
    assert torch.equal(o, ref["o"])
    assert torch.equal(dq, ref["dq"])
    for name, got in (("dk", dk), ("dv", dv)):
        # the key gradients' fp32 sums are grouped by rank: one bf16 ulp apart,
        # or more where the ranks' parts cancel, by at most fp32 rounding of the parts
        r32 = ref[name].float()
        diff = (got.float() - r32).abs()
        ulp = r32.abs() * 2 ** -7 + 2 ** -16 * r32.abs().max()
        print(name, "max |sharded - single GPU|", float(diff.max()), "of max", float(r32.abs().max()))
        assert bool((diff <= ulp).all()), name
    # against the fp64 oracle on the first and last heads
    for (b, h) in [(0, 0), (case.B - 1, case.H - 1)]:
        qh, kh, vh = (to64(x[b, :, h, :]) for x in (q, k, v))
        fw = orc.forward_head(qh, kh, vh, case.p, case.L, case.K, case.dtype, case.accum, **case.readings)
        bw = orc.backward_head(fw, to64(do[b, :, h, :]), case.p, case.accum)
        assert excess_error(to64(o[b, :, h, :]), fw["o"], case.dtype) <= ATOL[case.dtype]
        for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
            e = excess_error(to64(got[b, :, h, :]), bw[name], case.dtype)
            assert e <= ATOL[case.dtype], (name, e)


def test_sharded_path_full_size_512k_four_ranks():
    """The 512K workload (B1 H16 N524288 D128, p8 L4 K1024) split over 4
    emulated ranks of 131,072 tokens: selection and map equal the single-GPU
    path's, O and dQ bit for bit, dK and dV to the ranks' regrouped fp32 sums
    (the single-GPU path itself is held to the oracle at this size by
    test_gpu_parity.py)."""
    w = synth.WORKLOADS["ctx512k"]
    case = Case("cp_ctx512k_w4", w.B, w.H, w.N, w.D, w.dtype, w.p, w.L, w.K, w.recipe, w.mode, w.seed)
    world = 4
    q, k, v = synth.make_inputs(w, device=DEV)
    do = synth.make_dout(w, device=DEV)
    ref = run_gpu(case, q, k, v, do)
    cfg = case.cfg()
    ranks = [cp.ShardRank(cfg, world, r, DEV) for r in range(world)]
    sh = lambda x: [_shard(x, world, r) for r in range(world)]
    qs_, ks_, vs_, dos_ = sh(q), sh(k), sh(v), sh(do)
    outs = [torch.empty_like(x) for x in qs_]
    dqs, dks, dvs = ([torch.empty_like(x) for x in qs_] for _ in range(3))
    cp.run_emulated(ranks, qs_, ks_, vs_, outs, dos_, dqs, dks, dvs)
    torch.cuda.synchronize()
    assert lh.get_device_error() == (0, 0)
    ws = ref["ws"]
    for st in ranks:
        assert torch.equal(st.map, ws.map) and torch.equal(st.slot, ws.slot)
    o = torch.cat(outs, dim=1)
    assert torch.equal(o, ref["o"])
    assert torch.equal(torch.cat(dqs, dim=1), ref["dq"])
    for name, parts in (("dk", dks), ("dv", dvs)):
        got, r32 = torch.cat(parts, dim=1).float(), ref[name].float()
        diff = (got - r32).abs()
        assert bool((diff <= r32.abs() * 2 ** -7 + 2 ** -16 * r32.abs().max()).all()), name
        print(name, "max |sharded - single GPU|", float(diff.max()), "of max", float(r32.abs().max()))
    del ranks, outs, dqs, dks, dvs

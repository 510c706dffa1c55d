"""GPU parity: every stage of the CUDA path against the fp64 CPU oracle.

Bit-exact: pyramid, squared norms, top-K selection, gather map, slot table,
gathered sub-sequence, fixed-point scatter/spread given equal inputs, and
run-to-run repeats. Within tolerance (1e-5 fp32 / 2e-2 bf16 beyond the final
storage rounding): attention output, lse, O, dQ, dK, dV.
"""

import numpy as np
import pytest
import torch

import oracle as orc
from long_context_symmetric_b200 import lh, synth
from lhtest import ATOL, Case, case_of, compare_head, excess_error, run_gpu, to64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

SMALL = [
    case_of(synth.WORKLOADS["tiny_fp32"]),
    Case("l1_dense_bf16", 1, 2, 300, 64, "bf16", 4, 1, 8),                     # L = 1: plain causal SDPA, ragged S
    Case("odd_p3_fp32", 1, 2, 333, 64, "fp32", 3, 3, 5),                        # non power-of-two p
    Case("odd_p3_fixed", 1, 2, 333, 128, "bf16", 3, 3, 5, accum="fixed"),
    Case("full_budget", 1, 2, 256, 128, "bf16", 2, 4, 4096),                    # every candidate expanded
    Case("ties_small", 1, 2, 4096, 128, "bf16", 4, 5, 64, recipe="codebook", accum="fixed"),
    Case("d64_l4", 1, 2, 16384, 64, "bf16", 4, 4, 128),
    Case("odd_heads", 2, 3, 2048, 128, "bf16", 4, 3, 37, recipe="token_scale"),
    Case("chunked_topk", 1, 1, 131072, 64, "bf16", 2, 2, 300),                  # 65536 candidates: chunked sort
]

# the alternative readings of the open points (score formula, tie-break, entry
# order, scatter weights), each against the oracle run with the same reading
READINGS = [
    Case("score_k", 1, 2, 4096, 128, "bf16", 4, 4, 40, score="k"),
    Case("score_sum", 1, 2, 4096, 128, "bf16", 4, 4, 40, score="sum"),
    Case("score_prod", 1, 2, 4096, 128, "bf16", 4, 4, 40, score="prod"),
    Case("ties_high", 1, 2, 4096, 128, "bf16", 4, 5, 64, recipe="codebook", accum="fixed", ties="high"),
    Case("ties_high_chunked", 1, 1, 65536, 64, "bf16", 2, 2, 200, recipe="codebook", ties="high"),
    Case("order_pre", 1, 2, 4096, 128, "bf16", 4, 4, 40, order="pre"),
    Case("weight_mean", 1, 2, 4096, 128, "bf16", 4, 4, 40, weight="mean"),
    Case("weight_mean_p3_fixed", 1, 2, 333, 128, "bf16", 3, 3, 5, accum="fixed", weight="mean"),
    Case("all_alternatives", 2, 3, 2048, 64, "bf16", 4, 3, 37, recipe="token_scale", score="sum",
         ties="high", order="pre", weight="mean"),
    Case("partition", 1, 2, 4096, 128, "bf16", 4, 4, 40, inclusion="partition"),
    Case("partition_p3_fixed_mean", 1, 2, 333, 128, "bf16", 3, 3, 5, accum="fixed", weight="mean",
         inclusion="partition"),
    Case("partition_chunked", 1, 1, 65536, 64, "bf16", 2, 2, 200, recipe="codebook", inclusion="partition"),
    Case("partition_full_budget", 1, 2, 2048, 64, "bf16", 2, 3, 1024, inclusion="partition"),
    Case("partition_fp32", 1, 2, 1024, 64, "fp32", 4, 3, 32, inclusion="partition"),
    Case("all_alternatives_partition", 2, 3, 2048, 64, "bf16", 4, 3, 37, recipe="token_scale", score="sum",
         ties="high", order="pre", weight="mean", inclusion="partition"),
    Case("score_maxpool", 1, 2, 4096, 128, "bf16", 4, 4, 40, score="maxpool"),
    Case("score_maxpool_p3_fp32", 1, 2, 333, 64, "fp32", 3, 3, 5, score="maxpool"),
    Case("score_maxpool_chunked_ties", 1, 1, 65536, 64, "bf16", 2, 2, 200, recipe="codebook", score="maxpool"),
    Case("score_maxpool_partition", 1, 2, 4096, 128, "bf16", 8, 3, 20, recipe="token_scale", score="maxpool",
         inclusion="partition", weight="mean"),
]


def _inputs(case, device=DEV):
    w = case.workload()
    q, k, v = synth.make_inputs(w, device="cpu")
    do = synth.make_dout(w, device="cpu")
    return [x.to(device) for x in (q, k, v, do)]


@pytest.mark.parametrize("case", SMALL, ids=repr)
def test_small_cases_all_heads(case):
    q, k, v, do = _inputs(case)
    res = run_gpu(case, q, k, v, do)
    for b in range(case.B):
        for h in range(case.H):
            compare_head(case, res, q, k, v, do, b, h)


@pytest.mark.parametrize("case", READINGS, ids=repr)
def test_alternative_readings_all_heads(case):
    q, k, v, do = _inputs(case)
    res = run_gpu(case, q, k, v, do)
    for b in range(case.B):
        for h in range(case.H):
            compare_head(case, res, q, k, v, do, b, h)


def test_bf16_8k_workload_all_heads():
    case = case_of(synth.WORKLOADS["bf16_8k"])
    q, k, v, do = _inputs(case)
    res = run_gpu(case, q, k, v, do)
    worst = {}
    for b in range(case.B):
        for h in range(case.H):
            e = compare_head(case, res, q, k, v, do, b, h)
            for key, val in e.items():
                worst[key] = max(worst.get(key, -1.0), val)
    print("bf16_8k worst errors:", worst)


@pytest.mark.parametrize("accum", ["fp", "fixed"])
def test_scatter_and_spread_given_oracle_rows(accum):
    """Scatter/spread alone, fed the same fp32 rows as the oracle: fixed-point mode is bit-exact."""
    case = Case("scatter_only", 1, 2, 4096, 128, "bf16", 4, 4, 40, accum=accum)
    q, k, v, do = _inputs(case)
    res = run_gpu(case, q, k, v)
    ws = res["ws"]
    cfg = case.cfg()
    rng = np.random.default_rng(5)
    rows = rng.standard_normal(tuple(ws.os.shape)).astype(np.float32)
    rows_t = torch.from_numpy(rows).to(DEV)
    o = torch.empty_like(q)
    lh.scatter(cfg, rows_t, ws.slot, o)
    g3 = [torch.from_numpy(rng.standard_normal(tuple(ws.os.shape)).astype(np.float32)).to(DEV)
          for _ in range(3)]
    d3 = [torch.empty_like(q) for _ in range(3)]
    lh.spread(cfg, *g3, ws.slot, *d3)
    torch.cuda.synchronize()
    mode = "fixed" if accum == "fixed" else "fp"
    for h in range(case.H):
        m = ws.map[0, h].cpu().numpy().astype(np.int64)
        lvl, idx = m >> 28, m & 0x0FFFFFFF
        ref = orc.scatter_head(rows[0, h].astype(np.float64), lvl, idx, case.p, case.N, False, mode)
        got = to64(o[0, :, h, :])
        refs = [orc.spread_head(g.cpu().numpy()[0, h].astype(np.float64), lvl, idx, case.p, case.N, mode)
                for g in g3]
        if accum == "fixed":
            assert np.array_equal(got, orc.round_to_dtype(ref, "bf16"))
            for d, r in zip(d3, refs):
                assert np.array_equal(to64(d[0, :, h, :]), orc.round_to_dtype(r, "bf16"))
        else:
            assert excess_error(got, ref, "bf16") <= 1e-5
            for d, r in zip(d3, refs):
                assert excess_error(to64(d[0, :, h, :]), r, "bf16") <= 1e-5


def test_repeat_runs_bit_exact():
    """Three runs of the whole path (fixed-point mode) give identical bits."""
    case = Case("repeat", 1, 4, 32768, 128, "bf16", 4, 5, 128, recipe="codebook", accum="fixed")
    q, k, v, do = _inputs(case)
    outs = []
    for _ in range(3):
        r = run_gpu(case, q, k, v, do)
        outs.append([r[n].clone() for n in ("o", "dq", "dk", "dv")])
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            assert torch.equal(a, b)


def test_ties131k_three_runs_bit_exact():
    """The tie/determinism workload at full size (B1 H8 N131072 D128, p4 L5 K512,
    codebook inputs with many exactly tied scores, fixed-point accumulation):
    three runs of the whole forward and backward give identical bits."""
    w = synth.WORKLOADS["ties131k"]
    case = case_of(w)
    assert case.accum == "fixed"
    q, k, v = synth.make_inputs(w, device=DEV)
    do = synth.make_dout(w, device=DEV)
    outs = []
    for _ in range(3):
        r = run_gpu(case, q, k, v, do)
        ws = r["ws"]
        outs.append([r[n].clone() for n in ("o", "dq", "dk", "dv")] + [ws.sel.clone(), ws.map.clone()])
        del r, ws
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            assert torch.equal(a, b)


def test_autograd_wrapper_matches_stagewise():
    case = Case("autograd", 1, 2, 4096, 64, "bf16", 4, 3, 32)
    q, k, v, do = _inputs(case)
    res = run_gpu(case, q, k, v, do)
    qg, kg, vg = (x.clone().requires_grad_(True) for x in (q, k, v))
    o = lh.lighthouse_attention(qg, kg, vg, case.p, case.L, case.K)
    o.backward(do)
    assert torch.equal(o, res["o"])
    assert torch.equal(qg.grad, res["dq"]) and torch.equal(kg.grad, res["dk"]) and torch.equal(vg.grad, res["dv"])


def test_full_size_partition_sampled_heads():
    """The 512K workload under the partition reading (S = 22,528), in the launch
    configuration the bench uses: the first and last heads against the oracle."""
    w = synth.WORKLOADS["ctx512k"]
    case = Case("ctx512k_partition", w.B, w.H, w.N, w.D, w.dtype, w.p, w.L, w.K, w.recipe, w.mode, w.seed,
                inclusion="partition")
    q, k, v = synth.make_inputs(w, device=DEV)
    do = synth.make_dout(w, device=DEV)
    res = run_gpu(case, q, k, v, do)
    assert lh.plan(case.cfg()).S == 22528
    for (b, h) in [(0, 0), (w.B - 1, w.H - 1)]:
        compare_head(case, res, q, k, v, do, b, h)


def test_full_size_alternative_readings_sampled_heads():
    """The 98K workload (D = 64, 4 levels) with every alternative reading at once,
    at full size: the first and last heads against the oracle."""
    w = synth.WORKLOADS["ctx98k"]
    case = Case("ctx98k_alternatives", w.B, w.H, w.N, w.D, w.dtype, w.p, w.L, w.K, w.recipe, w.mode, w.seed,
                score="sum", ties="high", order="pre", weight="mean")
    q, k, v = synth.make_inputs(w, device=DEV)      # the same inputs as the default-reading run
    do = synth.make_dout(w, device=DEV)
    res = run_gpu(case, q, k, v, do)
    for (b, h) in [(0, 0), (w.B - 1, w.H - 1)]:
        compare_head(case, res, q, k, v, do, b, h)


@pytest.mark.parametrize("name", ["ctx98k", "ties131k", "ctx512k"])
def test_full_size_workloads_sampled_heads(name):
    """Full-size workloads in the launch configuration the bench uses; the oracle
    recomputes two whole heads (first and last) and every stage is compared."""
    w = synth.WORKLOADS[name]
    case = case_of(w)
    q, k, v = synth.make_inputs(w, device=DEV)
    do = synth.make_dout(w, device=DEV)
    res = run_gpu(case, q, k, v, do)
    for (b, h) in [(0, 0), (w.B - 1, w.H - 1)]:
        e = compare_head(case, res, q, k, v, do, b, h)
        print(name, (b, h), e)

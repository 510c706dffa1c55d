"""Benchmark of the Lighthouse Attention hot path (forward + backward) on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lh|reference] [--workload NAME]

One step = the whole hot path over one batch of synthetic input: pool+score,
top-K descent, gather, causal attention, scatter (forward) and block sums,
attention backward, spread (backward), each a liblh kernel called through the
C ABI. Default workload: ctx512k (B1 H16 N524288 D128 bf16, p8 L4 K1024,
sub-sequence S = 25600). Prints one JSON line on rank 0.

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch of
the same workload (the (b, h) problems are independent; no collective on the
data path), so per-GPU work is fixed ("scaling": "weak"); the time is the max
over ranks. `--impl reference` times the CPU oracle on the host cores instead.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_symmetric_b200 import dist as lhdist  # noqa: E402
from long_context_symmetric_b200 import lh, synth  # noqa: E402

METRIC = "Lighthouse attn fwd+bwd tokens/s at 512K on 1 B200; % HBM / tensor roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(w):
    return (f"{w.name}: B{w.B} H{w.H} N{w.N} D{w.D} {w.dtype} p{w.p} L{w.L} K{w.K}, "
            f"recipe {w.recipe}, accumulation {w.mode}")


# DRAM bytes per call of the attention stages at the 512K workload: ncu's
# dram__bytes_read.sum + dram__bytes_write.sum of each kernel on the 2-head case
# of the same workload (--heads 2), times 8 (the heads are independent problems,
# so traffic grows in proportion). Only the kernels as they are now; set back to
# None when one of them changes.
DRAM_TRAFFIC = {
    "ctx512k": {
        "attn_bwd": 8 * (52.938240e6 + 9.091328e6 + 52.884992e6 + 3.098624e6),   # dK/dV + dQ kernels
        "attn_fwd": 8 * (39.404288e6 + 0.345600e6),
    },
}


def stage_work(w, pl):
    """Algorithmic bytes (memory stages) or FLOPs (attention) per launch of each stage."""
    e = 2 if w.dtype == "bf16" else 4
    B, H, N, D, S, E = w.B, w.H, w.N, w.D, pl.S, pl.E
    tok = B * N * H * D * e
    sub = B * H * S * D
    if w.L == 1:
        # no pyramid: pool does nothing, select writes the identity map
        return {
            "pool": ("bytes", 0),
            "select": ("bytes", B * H * N * 4),
            "gather": ("bytes", 6 * sub * e + B * H * S * 4),
            "attn_fwd": ("flops", 2.0 * B * H * S * S * D),
            "scatter": ("bytes", tok + sub * 4),
            "scatter_bwd": ("bytes", tok + sub * 4 + sub * (2 if w.dtype == "bf16" else 4) + B * H * S * 4),
            "attn_bwd": ("flops", 5.0 * B * H * S * S * D),
            "spread": ("bytes", 3 * tok + 3 * sub * 4),
        }
    return {
        "pool": ("bytes", 3 * tok + 3 * B * H * E * D * e + 2 * B * H * E * 8),
        "select": ("bytes", 2 * B * H * E * 8 + B * H * (S + E + (w.L - 1) * w.K) * 4),
        "gather": ("bytes", 6 * sub * e + B * H * S * 4),
        "attn_fwd": ("flops", 2.0 * B * H * S * S * D),
        "scatter": ("bytes", tok + sub * 4 + B * H * E * 4),
        "scatter_bwd": ("bytes", tok + sub * 4 + sub * (2 if w.dtype == "bf16" else 4) + B * H * S * 4),
        "attn_bwd": ("flops", 5.0 * B * H * S * S * D),
        "spread": ("bytes", 3 * tok + 3 * sub * 4 + B * H * E * 4),
    }


# GEMMs the tensor-core kernels issue per (query tile, key tile) pair of 128 x 128
# (diagonal tiles included): forward S = Q K^T, then O += P_hi V and O += P_lo V;
# backward dK/dV kernel S^T, dP^T, dV, dK and dQ kernel S, dP, dQ += dS_hi K,
# dQ += dS_lo K. The algorithmic counts are 2 (forward) and 5 (backward).
EXEC_GEMMS = {"attn_fwd": 3, "attn_bwd": 8}


def executed_flops(w, pl, stage):
    """MMA FLOPs the bf16 tensor-core attention kernels execute per launch."""
    T = (pl.S + 127) // 128
    return w.B * w.H * (T * (T + 1) // 2) * EXEC_GEMMS[stage] * 2.0 * 128 * 128 * w.D


def sdpa_context(q, k, v, do, iters=2):
    """torch's own causal scaled_dot_product_attention, forward + backward, on the
    full token sequence of the same inputs (a library baseline, timed with CUDA
    events): median ms per step and the backend that ran."""
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel
    qt, kt, vt, dot = (x.transpose(1, 2) for x in (q, k, v, do))     # [B, H, N, D] views
    last = "no backend"
    for backend in (SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION, SDPBackend.EFFICIENT_ATTENTION):
        try:
            with sdpa_kernel(backends=[backend]):
                def step():
                    qq, kq, vq = (t.detach().requires_grad_(True) for t in (qt, kt, vt))
                    o = F.scaled_dot_product_attention(qq, kq, vq, is_causal=True)
                    o.backward(dot)
                step()
                torch.cuda.synchronize()
                times = []
                for _ in range(iters):
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record()
                    step()
                    b.record()
                    torch.cuda.synchronize()
                    times.append(a.elapsed_time(b))
                return {"ms_per_step": statistics.median(times), "backend": backend.name, "iters": iters}
        except RuntimeError as e:        # backend not available for this shape or GPU
            last = str(e).splitlines()[0][:200]
    return {"unavailable": last}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_sample(w, heads=1, seed=None):
    """Time the CPU oracle (forward + backward) on `heads` heads of the workload."""
    import numpy as np  # noqa: F401

    import oracle as orc
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    q, k, v = synth.make_inputs(w, device="cpu", seed=seed, B=1, H=heads)
    do = synth.make_dout(w, device="cpu", seed=seed, B=1, H=heads)
    Q, K, V, dO = (x.to(torch.float64).numpy() for x in (q, k, v, do))
    t0 = time.perf_counter()
    for h in range(heads):
        fw = orc.forward_head(Q[0, :, h], K[0, :, h], V[0, :, h], w.p, w.L, w.K, w.dtype, w.mode)
        orc.backward_head(fw, dO[0, :, h], w.p, w.mode)
    dt = time.perf_counter() - t0
    # heads are independent problems of equal size: the whole job is B*H head-problems
    tok_s = (w.B * w.N) / (dt / heads * w.B * w.H)
    return tok_s, dt, cores


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    # warm-up steps: the same oracle calls on a short sequence of the same shape
    # parameters (imports, allocator and thread pools warm; a few seconds in all)
    import dataclasses
    w_warm = dataclasses.replace(w, N=max(w.p ** (w.L - 1), min(w.N, 16384)))
    for _ in range(args.warmup):
        cpu_sample(w_warm, heads=1, seed=w.seed + 1)
    times = []
    cores = 1
    for i in range(args.steps):
        _, dt, cores = cpu_sample(w, heads=1, seed=w.seed + 2 + i)
        times.append(dt)
    per_head = sum(times) / len(times)
    value = (w.B * w.N) / (per_head * w.B * w.H)
    import oracle as orc
    S = orc.plan(w.N, w.p, w.L, w.K).S
    sample = (f"one (b,h) head per step (N={w.N} tokens, whole pyramid, selection, S={S} "
              f"sub-sequence, attention fwd+bwd, scatter/spread) of {w.B * w.H} heads; "
              f"ms_per_step is that step's time; tokens/s = the job's tokens over {w.B * w.H} such steps; "
              f"warm-up steps on N={w_warm.N}")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_head * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(w), "l2": "n/a (host)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def measure_fusion(cfg, w, ws, dev, iters=3):
    """The path's two ends with the model's projections next to them (x W_q,
    x W_k, x W_v before the pool; O W_o after the scatter; d_model = H * D,
    random weights): run one after the other over the whole sequence, and
    chunk by chunk through L2 (long_context_symmetric_b200.fused). Device ms
    per call, CUDA events, median of `iters` after one warm-up."""
    from long_context_symmetric_b200 import fused
    g = torch.Generator(device=dev).manual_seed(11)
    B, N, dm = w.B, w.N, w.H * w.D
    x = torch.randn(B, N, dm, generator=g, device=dev).to(torch.bfloat16)
    wt = [(torch.randn(dm, dm, generator=g, device=dev) / dm ** 0.5).to(torch.bfloat16) for _ in range(4)]
    q, k, v, o = (torch.empty(B, N, w.H, w.D, dtype=torch.bfloat16, device=dev) for _ in range(4))
    y = torch.empty(B, N, dm, dtype=torch.bfloat16, device=dev)

    def qkv_unfused():
        for b in range(B):
            for wi, out in zip(wt[:3], (q, k, v)):
                torch.matmul(x[b], wi, out=out[b].view(N, dm))
        lh.pool(cfg, q, k, v, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.sq, ws.scale)

    qkv_chunked = fused.Graphed(lambda: fused.qkv_project_pool(cfg, ws, x, wt[0], wt[1], wt[2], q, k, v))

    def out_unfused():
        lh.scatter(cfg, ws.os, ws.slot, o)
        for b in range(B):
            torch.matmul(o[b].view(N, dm), wt[3], out=y[b])

    out_chunked = fused.Graphed(lambda: fused.scatter_project(cfg, ws, wt[3], o, y))

    def timeit(fn):
        fn()
        torch.cuda.synchronize(dev)
        ts = []
        for _ in range(iters):
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b_.record()
            torch.cuda.synchronize(dev)
            ts.append(a.elapsed_time(b_))
        return round(statistics.median(ts), 4)

    res = {"d_model": dm, "chunk_tokens": fused.chunk_tokens(cfg),
           "qkv_projection_plus_pool_ms": {"unfused": timeit(qkv_unfused), "chunked_l2": timeit(qkv_chunked)},
           "scatter_plus_out_projection_ms": {"unfused": timeit(out_unfused), "chunked_l2": timeit(out_chunked)},
           "projections": "cuBLAS bf16 GEMMs through torch.matmul (the model's, outside the path)",
           "chunked_runs_as": "one CUDA graph per chunk loop (captured once, replayed)"}
    st, detail = lh.get_device_error()
    if st != 0:
        raise RuntimeError(f"device error {st} ({detail}) in the fusion timing")
    return res


def run_e2e(cfg, w, ws, q, k, v, do, results, stream, dev, world, steps):
    """End to end through the public calls (lh_forward, lh_backward): every step
    copies its inputs Q, K, V, dO from pinned host memory to the device and its
    results O, dQ, dK, dV back into pinned host memory. Inputs of step i+1 go up
    on one copy stream and results of step i come down on another while the next
    step computes; each of the two device buffer sets is reused only after its
    copies are done. `results`: the device-timed run's O, dQ, dK, dV, which the
    last step's host copies must equal."""
    hin = [x.cpu().pin_memory() for x in (q, k, v, do)]
    hout = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(4)]
    din = [[torch.empty_like(q) for _ in range(4)] for _ in range(2)]
    dout_ = [[torch.empty_like(q) for _ in range(4)] for _ in range(2)]
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]
    h2d = sum(x.numel() * x.element_size() for x in hin)
    d2h = sum(x.numel() * x.element_size() for x in hout)

    def copy_in(i):
        bi = i & 1
        if used[bi]:
            up.wait_event(ev_comp[bi])        # step i-2 is done reading these inputs
        with torch.cuda.stream(up):
            for dst, src in zip(din[bi], hin):
                dst.copy_(src, non_blocking=True)
        ev_in[bi].record(up)

    def compute(i):
        bi = i & 1
        q_, k_, v_, do_ = din[bi]
        o_, dq_, dk_, dv_ = dout_[bi]
        stream.wait_event(ev_in[bi])
        if used[bi]:
            stream.wait_event(ev_out[bi])     # results of step i-2 are on the host
        lh.forward(cfg, q_, k_, v_, o_, ws, stream)
        lh.backward(cfg, do_, dq_, dk_, dv_, ws, stream)
        ev_comp[bi].record(stream)
        down.wait_event(ev_comp[bi])
        with torch.cuda.stream(down):
            for dst, src in zip(hout, dout_[bi]):
                dst.copy_(src, non_blocking=True)
        ev_out[bi].record(down)
        used[bi] = True

    def run(n):
        copy_in(0)
        for i in range(n):
            if i + 1 < n:
                copy_in(i + 1)
            compute(i)

    run(2)
    torch.cuda.synchronize(dev)
    lhdist.barrier()
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(up)
    run(steps)
    b_.record(down)
    torch.cuda.synchronize(dev)
    e2e_ms = lhdist.max_over_ranks(a.elapsed_time(b_) / steps, dev)
    ok = all(torch.equal(hx.to(dev), dx) for hx, dx in zip(hout, results))
    return {"value": lhdist.job_throughput(w.B * w.N, world, e2e_ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": steps,
            "result": "O, dQ, dK, dV copied to pinned host memory every step",
            "matches_device_run": ok}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="lh", choices=["lh", "reference"])
    ap.add_argument("--workload", default="ctx512k", choices=list(synth.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sdpa-context", action="store_true",
                    help="skip the timing of torch's scaled_dot_product_attention (causal, fwd+bwd) on the full "
                         "token sequence of the same inputs (context for the speed-up over dense attention)")
    ap.add_argument("--no-fixed-mode", action="store_true",
                    help="skip the timing of the same step in fixed-point accumulation mode")
    ap.add_argument("--no-fusion", action="store_true",
                    help="skip the timing of the projections fused with pool / scatter chunk by chunk")
    ap.add_argument("--heads", type=int, default=None,
                    help="smaller case of the same recipe (fewer heads), e.g. for an ncu capture")
    ap.add_argument("--tokens", type=int, default=None, help="smaller case of the same recipe (fewer tokens)")
    args = ap.parse_args()
    w = synth.WORKLOADS[args.workload]
    if args.heads or args.tokens:
        import dataclasses
        w = dataclasses.replace(w, H=args.heads or w.H, N=args.tokens or w.N)

    if args.impl == "reference":
        run_reference(args, w)
        return

    info = lhdist.rank_info()
    world, rank, local = info.world, info.rank, info.local
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lhdist.init("nccl", dev, timeout_s=120)

    cfg = lh.make_config(w.B, w.H, w.N, w.D, w.p, w.L, w.K, w.dtype, w.mode)
    ws = lh.Workspace(cfg, dev, backward=True)
    pl = ws.plan
    seed = lhdist.replica_seed(w.seed, rank)       # each rank: its own batch of the workload
    q, k, v = synth.make_inputs(w, device=dev, seed=seed)
    do = synth.make_dout(w, device=dev, seed=seed)
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    stream = torch.cuda.current_stream(dev)
    stages = ["pool", "select", "gather", "attn_fwd", "scatter", "scatter_bwd", "attn_bwd", "spread"]
    fwd_stages = stages[:5]

    def step(c, ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        mark(0)
        lh.pool(c, q, k, v, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.sq, ws.scale, stream)
        mark(1)
        lh.score_topk(c, ws.sq, ws.sel, ws.map, ws.slot, ws.ws, stream=stream)
        mark(2)
        lh.gather(c, q, k, v, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.map, ws.scale, ws.qs, ws.ks, ws.vs, stream)
        mark(3)
        lh.attn_fwd(c, ws.qs, ws.ks, ws.vs, ws.scale, ws.os, ws.lse, stream)
        mark(4)
        lh.scatter(c, ws.os, ws.slot, o, stream)
        mark(5)
        lh.scatter_bwd(c, do, ws.os, ws.slot, ws.dos, ws.delta, ws.scale, stream)
        mark(6)
        lh.attn_bwd(c, ws.qs, ws.ks, ws.vs, ws.dos, ws.lse, ws.delta, ws.scale, ws.dqs, ws.dks, ws.dvs, stream)
        mark(7)
        lh.spread(c, ws.dqs, ws.dks, ws.dvs, ws.slot, dq, dk, dv, stream)
        mark(8)

    def timed(c, steps, sample_clocks=False):
        """`steps` steps of config c after a barrier and a synchronize: total and
        per-stage device ms (CUDA events on the launching stream), launches, clocks."""
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(steps)]
        sampler = ClockSampler(local) if sample_clocks else None
        lhdist.barrier()
        torch.cuda.synchronize(dev)
        if sampler:
            sampler.start()
            time.sleep(0.3)
        launches0 = lh.launch_count()
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(steps):
            step(c, evs[i])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        launches = lh.launch_count() - launches0
        clocks = sampler.stop() if sampler else None
        lhdist.barrier()
        ms_total = lhdist.max_over_ranks(t_start.elapsed_time(t_end), dev)
        per = {s: sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(steps)) / steps
               for j, s in enumerate(stages)}
        st, detail = lh.get_device_error(stream)
        if st != 0:
            raise RuntimeError(f"device error {st} ({detail}) in a timed region")
        return ms_total / steps, per, launches, clocks

    for _ in range(max(args.warmup, 0)):
        step(cfg)
    torch.cuda.synchronize(dev)
    st, detail = lh.get_device_error(stream)
    if st != 0:
        raise RuntimeError(f"device error {st} ({detail}) during warm-up")

    ms_step, stage_ms, launches, clocks = timed(cfg, args.steps, sample_clocks=True)
    # forward alone: the device time of its five stages inside the same steps
    fwd_ms = lhdist.max_over_ranks(sum(stage_ms[s] for s in fwd_stages), dev)

    # The same step in fixed-point accumulation mode (the pages' deterministic
    # int-atomic scatter-back is their slower variant): only the scatter and the
    # spread change arithmetic, every other stage is the same kernel.
    fixed = None
    if not args.no_fixed_mode and w.mode == "fp":
        cfg_fx = lh.make_config(w.B, w.H, w.N, w.D, w.p, w.L, w.K, w.dtype, "fixed")
        for _ in range(2):
            step(cfg_fx)
        fx_step, fx_stage, _, _ = timed(cfg_fx, args.steps)
        fixed = {"ms_per_step": round(fx_step, 4),
                 "scatter_ms": round(fx_stage["scatter"], 4), "spread_ms": round(fx_stage["spread"], 4),
                 "int_vs_fp": {"scatter": round(fx_stage["scatter"] / stage_ms["scatter"], 3),
                               "spread": round(fx_stage["spread"] / stage_ms["spread"], 3),
                               "scatter_plus_spread": round((fx_stage["scatter"] + fx_stage["spread"]) /
                                                            (stage_ms["scatter"] + stage_ms["spread"]), 3),
                               "step": round(fx_step / ms_step, 3)},
                 "pages": "int-atomic scatter-back 1.2-2x slower than fp-atomic (Lighthouse Attention Technique, "
                          "throughput paragraph)"}
        for _ in range(2):
            step(cfg)                 # leave the default mode's results in place
        torch.cuda.synchronize(dev)

    # End to end through the public calls (lh_forward, lh_backward): every step
    # copies its inputs Q, K, V, dO from pinned host memory to the device and its
    # results O, dQ, dK, dV back into pinned host memory. Inputs of step i+1 go up
    # on one copy stream and results of step i come down on another while the next
    # step computes; each of the two device buffer sets is reused only after its
    # copies are done.
    e2e = None
    if args.e2e_steps > 0:
        e2e = run_e2e(cfg, w, ws, q, k, v, do, (o, dq, dk, dv), stream, dev, world, args.e2e_steps)
        torch.cuda.empty_cache()

    peaks, peak_kind = load_peaks()
    # the tensor-core denominator: the burst cuBLAS figure for a short timed
    # region (the 512K Lighthouse step: ~15 ms steps, well under a second in
    # all); the sustained, power-capped figure once the region runs for seconds
    # (dense attention at full N: seconds per step)
    tc_peak_key = "bf16_tflops" if ms_step * args.steps < 1000.0 else "bf16_tflops_sustained"
    work = stage_work(w, pl)
    frac = {}
    for s in stages:
        kind, amount = work[s]
        if amount == 0:
            continue                  # a stage with nothing to do for this shape
        sec = stage_ms[s] / 1e3
        if kind == "bytes":
            ach = amount / sec / 1e9
            frac[s] = {"ms": round(stage_ms[s], 4), "achieved": round(ach, 1), "unit": "GB/s",
                       "frac": round(ach / peaks["hbm_gbs"], 4), "bound": "hbm"}
        else:
            ach = amount / sec / 1e12
            frac[s] = {"ms": round(stage_ms[s], 4), "achieved": round(ach, 2), "unit": "TFLOP/s",
                       "frac": round(ach / peaks[tc_peak_key], 4), "bound": "tensor"}
            if w.dtype == "bf16":
                ex = executed_flops(w, pl, s) / sec / 1e12
                frac[s].update(executed=round(ex, 2), executed_frac=round(ex / peaks[tc_peak_key], 4),
                               executed_gemms_per_tile_pair=EXEC_GEMMS[s])
    dom = max(frac, key=lambda s: stage_ms[s])
    kind, amount = work[dom]
    full_size = (w.B, w.H, w.N) == (synth.WORKLOADS[w.name].B, synth.WORKLOADS[w.name].H,
                                    synth.WORKLOADS[w.name].N)
    roofline = {
        "kernel": dom, "bound": frac[dom]["bound"], "achieved": frac[dom]["achieved"],
        "peak": peaks["hbm_gbs"] if kind == "bytes" else peaks[tc_peak_key],
        "unit": frac[dom]["unit"], "frac": frac[dom]["frac"],
        "traffic": DRAM_TRAFFIC.get(w.name, {}).get(dom) if full_size else None,
        "traffic_unit": "bytes per call",
        "peak_source": f"{peak_kind} ({'hbm_gbs' if kind == 'bytes' else tc_peak_key})",
    }

    context = None
    if not args.no_sdpa_context and rank == 0 and world == 1:
        context = sdpa_context(q, k, v, do)
        if "ms_per_step" in context:
            context["lighthouse_speedup_fwd_bwd"] = round(context["ms_per_step"] / ms_step, 2)
            context["pages"] = "17.3x fwd+bwd and 21x fwd over standard attention at 512K on one B200 (zubnet)"

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tok_s, dt, cores = cpu_sample(w, heads=1)
        cpu_baseline = {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                        "sample": f"oracle fwd+bwd of head (0,0) of {workload_desc(w)}; {dt:.1f} s; "
                                  f"tokens/s scaled to all {w.B * w.H} heads"}

    fusion = None
    if not args.no_fusion and rank == 0 and world == 1 and w.dtype == "bf16" and w.L > 1:
        fusion = measure_fusion(cfg, w, ws, dev)

    value = lhdist.job_throughput(w.B * w.N, world, ms_step / 1e3)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": workload_desc(w), "S": pl.S,
                   "l2": "inputs larger than L2 (Q, K, V, dO: %.1f GB per step), no flush"
                         % (4 * w.B * w.N * w.H * w.D * (2 if w.dtype == "bf16" else 4) / 1e9),
                   "parallelism": f"dp{world} (independent batches per GPU)"},
        "fwd": {"value": lhdist.job_throughput(w.B * w.N, world, fwd_ms / 1e3), "unit": "tokens/s",
                "ms": round(fwd_ms, 4), "stages": fwd_stages},
        "roofline": roofline, "stages": frac, "cpu_baseline": cpu_baseline, "e2e": e2e,
        "gpu_launches": launches, "clocks": clocks,
    }
    if fixed is not None:
        line["fixed_mode"] = fixed
    if context is not None:
        line["context_sdpa"] = context
    if fusion is not None:
        line["fusion"] = fusion
    if rank == 0:
        print(json.dumps(line), flush=True)
    lhdist.shutdown()


if __name__ == "__main__":
    main()

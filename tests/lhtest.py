"""Helpers shared by the GPU parity tests: run the CUDA path stage by stage
through the C ABI and compare each stage with the CPU oracle."""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle as orc
from long_context_symmetric_b200 import lh, synth

# Tolerances on outputs and gradients against the fp64 oracle: 1e-5 (fp32) and
# 2e-2 (bf16) max-abs, applied to the error beyond the final rounding of the
# result into its storage dtype (that rounding alone is up to half an ulp:
# 0.031 for a bf16 value in [8, 16)).
ATOL = {"fp32": 1e-5, "bf16": 2e-2}


def half_ulp(ref: np.ndarray, dtype: str) -> np.ndarray:
    bits = {"fp32": 24, "bf16": 8}[dtype]
    a = np.abs(ref)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - bits), 0.0)


def excess_error(gpu: np.ndarray, ref: np.ndarray, dtype: str) -> float:
    """max over elements of |gpu - ref| - half_ulp_dtype(ref)."""
    return float(np.max(np.abs(gpu - ref) - half_ulp(ref, dtype))) if gpu.size else 0.0


def error_report(gpu: np.ndarray, ref: np.ndarray, dtype: str, atol: float) -> dict:
    """Raw max-abs error, the error beyond the final rounding, and how many
    elements exceed the plain max-abs bound (those lean on the half-ulp allowance
    of the storage rounding)."""
    if not gpu.size:
        return dict(raw=0.0, excess=0.0, over_plain=0, n=0)
    d = np.abs(gpu - ref)
    return dict(raw=float(d.max()), excess=float(np.max(d - half_ulp(ref, dtype))),
                over_plain=int(np.count_nonzero(d > atol)), n=int(d.size))


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def scale_exp(amax_bits: int) -> int:
    """The power-of-two exponent e the library applies to a head's fp16
    operands (x * 2^-e), from the head's largest magnitude (fp32 bit pattern):
    0 while that magnitude is in [4, 256), else the exponent that brings it
    into [4, 8) (clamped to +-60)."""
    E = (int(amax_bits) >> 23) & 0xFF
    if E in (0, 255):
        return 0
    ex = E - 127
    if 2 <= ex < 8:
        return 0
    return max(-60, min(60, ex - 2))


def f32_bits(x: float) -> int:
    return int(np.array([x], dtype=np.float32).view(np.uint32)[0])


def struct_f32(bits: int) -> float:
    return float(np.array([bits & 0xFFFFFFFF], dtype=np.uint32).view(np.float32)[0])


class Case:
    def __init__(self, name, B, H, N, D, dtype, p, L, K, recipe="iid", accum="fp", seed=7, **readings):
        self.name, self.B, self.H, self.N, self.D = name, B, H, N, D
        self.dtype, self.p, self.L, self.K = dtype, p, L, K
        self.recipe, self.accum, self.seed = recipe, accum, seed
        # score / ties / order / weight readings (absent: the library's defaults)
        self.readings = readings

    def workload(self):
        return synth.Workload(self.name, self.B, self.H, self.N, self.D, self.dtype, self.p, self.L,
                              self.K, self.recipe, self.accum, True, self.seed)

    def cfg(self):
        return lh.make_config(self.B, self.H, self.N, self.D, self.p, self.L, self.K, self.dtype,
                              self.accum, **self.readings)

    def __repr__(self):
        return self.name


def case_of(w: synth.Workload) -> Case:
    return Case(w.name, w.B, w.H, w.N, w.D, w.dtype, w.p, w.L, w.K, w.recipe, w.mode, w.seed)


def run_gpu(case: Case, q, k, v, do=None, stream=None):
    """Whole path, stage by stage, through the C ABI. Returns the workspace and outputs."""
    cfg = case.cfg()
    ws = lh.Workspace(cfg, q.device, backward=do is not None)
    o = torch.empty_like(q)
    lh.pool(cfg, q, k, v, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.sq, ws.scale, stream)
    lh.score_topk(cfg, ws.sq, ws.sel, ws.map, ws.slot, ws.ws, stream=stream)
    lh.gather(cfg, q, k, v, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.map, ws.scale, ws.qs, ws.ks, ws.vs, stream)
    lh.attn_fwd(cfg, ws.qs, ws.ks, ws.vs, ws.scale, ws.os, ws.lse, stream)
    lh.scatter(cfg, ws.os, ws.slot, o, stream)
    out = dict(ws=ws, o=o)
    if do is not None:
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
        lh.scatter_bwd(cfg, do, ws.os, ws.slot, ws.dos, ws.delta, ws.scale, stream)
        lh.attn_bwd(cfg, ws.qs, ws.ks, ws.vs, ws.dos, ws.lse, ws.delta, ws.scale, ws.dqs, ws.dks, ws.dvs, stream)
        lh.spread(cfg, ws.dqs, ws.dks, ws.dvs, ws.slot, dq, dk, dv, stream)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    st, detail = lh.get_device_error()
    assert st == 0, f"device error {st} detail {detail}"
    return out


def expected_slot_table(fw, case: Case, pl) -> np.ndarray:
    """Slot table implied by the oracle's selection and order: 2 * slot + expanded
    for the entries in the sub-sequence; under the partition reading an expanded
    entry is not in it and holds 2 * (slot of the entry that starts at its first
    token) + 1 (the entries tile the tokens, so exactly one starts there)."""
    E = pl.E
    p = case.p
    tab = np.full(max(E, 1), -1, dtype=np.int64)
    slot_of = {(int(l), int(i)): j for j, (l, i) in enumerate(zip(fw["lvl"], fw["idx"]))}
    part = case.readings.get("inclusion", "nested") == "partition"
    starts = {int(i) * p ** int(l): j for j, (l, i) in enumerate(zip(fw["lvl"], fw["idx"]))} if part else {}
    for l in range(1, case.L):
        sel = set(int(x) for x in fw["sel"][l]) if fw["sel"][l] is not None else set()
        for i in fw["included"][l]:
            j = slot_of[(l, int(i))]
            tab[pl.lvl_off[l] + int(i)] = 2 * j + (1 if int(i) in sel else 0)
        if part:
            for i in sel:
                tab[pl.lvl_off[l] + i] = 2 * starts[i * p ** l] + 1
    return tab[:E]


def compare_head(case: Case, res, q, k, v, do, b: int, h: int, check_bwd=True):
    """Run the oracle on head (b, h) and compare every stage of the GPU run."""
    dt = case.dtype
    pl = lh.plan(case.cfg())
    ws = res["ws"]
    qh, kh, vh = (to64(x[b, :, h, :]) for x in (q, k, v))
    fw = orc.forward_head(qh, kh, vh, case.p, case.L, case.K, dt, case.accum, **case.readings)
    assert fw["plan"].S == pl.S
    # (i) pyramid and squared norms: bit-exact
    for l in range(1, case.L):
        o0, n = pl.lvl_off[l], pl.n[l]
        for name, gpu_t, ref in (("q", ws.pyr_q, fw["stored_q"]), ("k", ws.pyr_k, fw["stored_k"]),
                                 ("v", ws.pyr_v, fw["stored_v"])):
            got = to64(gpu_t[b, h, o0:o0 + n])
            assert np.array_equal(got, ref[l]), f"pyramid {name} level {l}"
        assert np.array_equal(ws.sq[0, b, h, o0:o0 + n].cpu().numpy(), fw["sq_q"][l]), f"sq_q level {l}"
        assert np.array_equal(ws.sq[1, b, h, o0:o0 + n].cpu().numpy(), fw["sq_k"][l]), f"sq_k level {l}"
    # (ii) selection, order, slot table: bit-exact
    for l in range(1, case.L):
        kl = pl.k[l]
        got = ws.sel[b, h, l - 1].cpu().numpy()
        assert np.array_equal(got[:kl], fw["sel"][l]), f"sel level {l}"
        assert np.all(got[kl:] == -1)
    m = ws.map[b, h].cpu().numpy().astype(np.int64)
    assert np.array_equal(m >> 28, fw["lvl"]) and np.array_equal(m & 0x0FFFFFFF, fw["idx"]), "map"
    if case.L > 1:
        assert np.array_equal(ws.slot[b, h].cpu().numpy().astype(np.int64),
                              expected_slot_table(fw, case, pl)), "slot table"
    # the head's largest magnitudes (bf16 I/O): exactly the largest |x| of its tokens
    ex = [0, 0, 0, 0]
    if dt == "bf16":
        for t, x in enumerate((qh, kh, vh)):
            bits = int(ws.scale[t, b, h].item()) & 0xFFFFFFFF
            assert bits == f32_bits(np.max(np.abs(x))), f"scale row {t}"
            ex[t] = scale_exp(bits)
    # gather: bit-exact (bf16 I/O: the stored entries times 2^-e in fp16, nearest-even)
    for t, (name, gpu_t, ref) in enumerate((("qs", ws.qs, fw["qs"]), ("ks", ws.ks, fw["ks"]), ("vs", ws.vs, fw["vs"]))):
        want = (ref * 2.0 ** -ex[t]).astype(np.float16).astype(np.float64) if dt == "bf16" else ref
        assert np.array_equal(to64(gpu_t[b, h]), want), name
    # (iii) attention
    atol = ATOL[dt]
    err_os = float(np.max(np.abs(to64(ws.os[b, h]) - fw["os"])))
    err_lse = float(np.max(np.abs(to64(ws.lse[b, h]) - fw["lse"])))
    assert err_os <= atol, f"os err {err_os}"
    assert err_lse <= atol, f"lse err {err_lse}"
    # (iv) scatter
    rep = {"o": error_report(to64(res["o"][b, :, h, :]), fw["o"], dt, atol)}
    err_o = rep["o"]["excess"]
    assert err_o <= atol, f"o err {rep['o']}"
    errs = dict(os=err_os, lse=err_lse, o=err_o)
    if do is None or not check_bwd:
        print(f"{case.name} ({b},{h}) errors:", errs, "o:", rep["o"])
        return errs
    bw = orc.backward_head(fw, to64(do[b, :, h, :]), case.p, case.accum)
    # dos: the fp16 block sums (an intermediate); its bound scales with the
    # largest block sum, since a block sum of p^l token gradients is stored with
    # fp16's relative precision
    edo = scale_exp(int(ws.scale[3, b, h].item()) & 0xFFFFFFFF) if dt == "bf16" else 0
    if dt == "bf16":
        assert (int(ws.scale[3, b, h].item()) & 0xFFFFFFFF) == f32_bits(np.max(np.abs(bw["dos"]))) or \
            abs(struct_f32(int(ws.scale[3, b, h].item())) / np.max(np.abs(bw["dos"])) - 1) < 1e-5, "scale row 3"
    err_dos = excess_error(to64(ws.dos[b, h]) * 2.0 ** edo, bw["dos"], dt)
    assert err_dos <= atol * max(1.0, float(np.max(np.abs(bw["dos"])))) , f"dos err {err_dos}"
    for name in ("dq", "dk", "dv"):
        rep[name] = error_report(to64(res[name][b, :, h, :]), bw[name], dt, atol)
        errs[name] = rep[name]["excess"]
        assert errs[name] <= atol, f"{name} err {rep[name]}"
    print(f"{case.name} ({b},{h}) raw max-abs / beyond rounding / elements over the plain bound:",
          {k: (round(v["raw"], 6), round(v["excess"], 6), v["over_plain"]) for k, v in rep.items()})
    return errs

"""Thin ctypes binding over liblh (include/lh.h).

Argument marshalling only: every step of the hot path runs in liblh's CUDA
kernels. Tensors are torch tensors on a CUDA device (PyTorch supplies device
memory and streams); each wrapper passes their data pointers and the current
stream to the C entry point of the same name and raises LHError on a non-zero
status. The library is loaded on first use; if it is missing the call raises
(there is no fallback implementation).
"""

from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblh.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "lh.h")

LH_BF16, LH_FP32 = 0, 1
LH_ACC_FP32, LH_ACC_FIXED64 = 0, 1
MAX_LEVELS = 8
MAX_K = 4096

c_int, c_void_p, c_size_t = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t


class LHError(RuntimeError):
    def __init__(self, status: int, name: str):
        super().__init__(f"{name}: {status_string(status)} (status {status})")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("B", c_int), ("H", c_int), ("N", c_int), ("D", c_int), ("p", c_int),
                ("L", c_int), ("K", c_int), ("dtype", c_int), ("accum", c_int),
                ("score", c_int), ("ties", c_int), ("order", c_int), ("weight", c_int),
                ("inclusion", c_int)]


SCORES = {"max": 0, "k": 1, "sum": 2, "prod": 3, "maxpool": 4}
TIES = {"low": 0, "high": 1}
ORDERS = {"post": 0, "pre": 1}
WEIGHTS = {"one": 0, "mean": 1}
INCLUSIONS = {"nested": 0, "partition": 1}


class Plan(ctypes.Structure):
    _fields_ = [("S", c_int), ("E", c_int), ("n", c_int * MAX_LEVELS), ("k", c_int * MAX_LEVELS),
                ("c", c_int * MAX_LEVELS), ("lvl_off", c_int * MAX_LEVELS), ("ws_bytes", c_size_t)]


class CPPlan(ctypes.Structure):
    _fields_ = [("world", c_int), ("rank", c_int), ("n_loc", c_int), ("E_loc", c_int),
                ("lvl_off_loc", c_int * MAX_LEVELS), ("glob", Plan)]


class Buffers(ctypes.Structure):
    _fields_ = [("pyr_q", c_void_p), ("pyr_k", c_void_p), ("pyr_v", c_void_p), ("sq", c_void_p),
                ("sel", c_void_p), ("map", c_void_p), ("slot", c_void_p), ("qs", c_void_p),
                ("ks", c_void_p), ("vs", c_void_p), ("os", c_void_p), ("lse", c_void_p),
                ("ws", c_void_p), ("ws_bytes", c_size_t), ("dos", c_void_p), ("delta", c_void_p),
                ("dqs", c_void_p), ("dks", c_void_p), ("dvs", c_void_p), ("scale", c_void_p)]


_lib = None

_SIGS = {
    "lh_version": ([], c_int),
    "lh_status_string": ([c_int], ctypes.c_char_p),
    "lh_plan": ([ctypes.POINTER(Config), ctypes.POINTER(Plan)], c_int),
    "lh_pool": ([ctypes.POINTER(Config)] + [c_void_p] * 9, c_int),
    "lh_score_topk": ([ctypes.POINTER(Config), c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                       c_size_t, c_void_p], c_int),
    "lh_gather": ([ctypes.POINTER(Config)] + [c_void_p] * 12, c_int),
    "lh_attn_fwd": ([ctypes.POINTER(Config)] + [c_void_p] * 7, c_int),
    "lh_scatter": ([ctypes.POINTER(Config)] + [c_void_p] * 4, c_int),
    "lh_scatter_bwd": ([ctypes.POINTER(Config)] + [c_void_p] * 7, c_int),
    "lh_attn_bwd": ([ctypes.POINTER(Config)] + [c_void_p] * 11, c_int),
    "lh_spread": ([ctypes.POINTER(Config)] + [c_void_p] * 8, c_int),
    "lh_forward": ([ctypes.POINTER(Config)] + [c_void_p] * 4 + [ctypes.POINTER(Buffers), c_void_p], c_int),
    "lh_backward": ([ctypes.POINTER(Config)] + [c_void_p] * 4 + [ctypes.POINTER(Buffers), c_void_p], c_int),
    "lh_get_device_error": ([c_void_p, ctypes.POINTER(c_int)], c_int),
    "lh_launch_count": ([], ctypes.c_ulonglong),
    "lh_selftest_timeout": ([ctypes.c_longlong, c_void_p, c_void_p], c_int),
    "lh_score_topk_noalloc": ([ctypes.POINTER(Config)] + [c_void_p] * 5, c_int),
    "lh_selftest_exp2": ([c_void_p, c_void_p, c_void_p, c_int, c_void_p], c_int),
    "lh_pool_range": ([ctypes.POINTER(Config), c_int, c_int] + [c_void_p] * 9, c_int),
    "lh_scatter_range": ([ctypes.POINTER(Config), c_int, c_int] + [c_void_p] * 4, c_int),
    "lh_cp_plan": ([ctypes.POINTER(Config), c_int, c_int, ctypes.POINTER(CPPlan)], c_int),
    "lh_cp_pool": ([ctypes.POINTER(Config), c_int, c_int] + [c_void_p] * 9, c_int),
    "lh_cp_assemble_sq": ([ctypes.POINTER(Config), c_int] + [c_void_p] * 3, c_int),
    "lh_cp_segment": ([ctypes.POINTER(Config), c_int, c_int] + [c_void_p] * 5, c_int),
    "lh_cp_gather": ([ctypes.POINTER(Config), c_int, c_int] + [c_void_p] * 13, c_int),
    "lh_cp_attn_fwd": ([ctypes.POINTER(Config), c_int, c_int] + [c_void_p] * 8, c_int),
    "lh_cp_scatter": ([ctypes.POINTER(Config), c_int, c_int] + [c_void_p] * 4, c_int),
    "lh_cp_scatter_bwd": ([ctypes.POINTER(Config), c_int, c_int] + [c_void_p] * 8, c_int),
    "lh_cp_attn_bwd": ([ctypes.POINTER(Config), c_int, c_int] + [c_void_p] * 12, c_int),
    "lh_cp_spread": ([ctypes.POINTER(Config), c_int, c_int] + [c_void_p] * 8, c_int),
}


def lib():
    """Load liblh.so (once) and declare the entry points' signatures."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"liblh.so not found at {LIB_PATH}; build it with "
                               "`python -m long_context_symmetric_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(l, name)
            f.argtypes = args
            f.restype = res
        _lib = l
    return _lib


def header_functions() -> list[str]:
    """Names of the entry points declared in include/lh.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\w[\w\s\*]*?\b(lh_\w+)\s*\(", text, flags=re.M)))


def status_string(s: int) -> str:
    return lib().lh_status_string(s).decode()


def _check(status: int, name: str):
    if status != 0:
        raise LHError(status, name)


def _p(t):
    """Data pointer of a tensor (or None / int passthrough)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_config(B, H, N, D, p, L, K, dtype="bf16", accum="fp", score="max", ties="low", order="post",
                weight="one", inclusion="nested") -> Config:
    """Problem sizes, element type, accumulation mode and the readings of the
    open points (defaults: the library's reading)."""
    return Config(B, H, N, D, p, L, K, {"bf16": LH_BF16, "fp32": LH_FP32}[dtype],
                  {"fp": LH_ACC_FP32, "fixed": LH_ACC_FIXED64}[accum], SCORES[score], TIES[ties],
                  ORDERS[order], WEIGHTS[weight], INCLUSIONS[inclusion])


def plan(cfg: Config) -> Plan:
    out = Plan()
    _check(lib().lh_plan(ctypes.byref(cfg), ctypes.byref(out)), "lh_plan")
    return out


def pool(cfg, q, k, v, pyr_q, pyr_k, pyr_v, sq, scale, stream=None):
    _check(lib().lh_pool(ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(pyr_q), _p(pyr_k), _p(pyr_v),
                         _p(sq), _p(scale), _stream(stream)), "lh_pool")


def score_topk(cfg, sq, sel, map_, slot, ws, ws_bytes=None, stream=None):
    nbytes = ws_bytes if ws_bytes is not None else (ws.numel() * ws.element_size() if ws is not None else 0)
    _check(lib().lh_score_topk(ctypes.byref(cfg), _p(sq), _p(sel), _p(map_), _p(slot), _p(ws),
                               nbytes, _stream(stream)), "lh_score_topk")


def score_topk_noalloc(cfg, sq, sel, map_, slot, stream=None):
    """lh_score_topk with the descent's scratch in liblh's fixed device array (no workspace)."""
    _check(lib().lh_score_topk_noalloc(ctypes.byref(cfg), _p(sq), _p(sel), _p(map_), _p(slot),
                                       _stream(stream)), "lh_score_topk_noalloc")


def gather(cfg, q, k, v, pyr_q, pyr_k, pyr_v, map_, scale, qs, ks, vs, stream=None):
    _check(lib().lh_gather(ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(pyr_q), _p(pyr_k), _p(pyr_v),
                           _p(map_), _p(scale), _p(qs), _p(ks), _p(vs), _stream(stream)), "lh_gather")


def attn_fwd(cfg, qs, ks, vs, scale, os_, lse, stream=None):
    _check(lib().lh_attn_fwd(ctypes.byref(cfg), _p(qs), _p(ks), _p(vs), _p(scale), _p(os_), _p(lse),
                             _stream(stream)), "lh_attn_fwd")


def scatter(cfg, os_, slot, o, stream=None):
    _check(lib().lh_scatter(ctypes.byref(cfg), _p(os_), _p(slot), _p(o), _stream(stream)), "lh_scatter")


def scatter_bwd(cfg, dout, os_, slot, dos, delta, scale, stream=None):
    _check(lib().lh_scatter_bwd(ctypes.byref(cfg), _p(dout), _p(os_), _p(slot), _p(dos), _p(delta), _p(scale),
                                _stream(stream)), "lh_scatter_bwd")


def attn_bwd(cfg, qs, ks, vs, dos, lse, delta, scale, dqs, dks, dvs, stream=None):
    _check(lib().lh_attn_bwd(ctypes.byref(cfg), _p(qs), _p(ks), _p(vs), _p(dos), _p(lse), _p(delta),
                             _p(scale), _p(dqs), _p(dks), _p(dvs), _stream(stream)), "lh_attn_bwd")


def spread(cfg, dqs, dks, dvs, slot, dq, dk, dv, stream=None):
    _check(lib().lh_spread(ctypes.byref(cfg), _p(dqs), _p(dks), _p(dvs), _p(slot), _p(dq), _p(dk),
                           _p(dv), _stream(stream)), "lh_spread")


def get_device_error(stream=None):
    detail = c_int(0)
    st = lib().lh_get_device_error(_stream(stream), ctypes.byref(detail))
    return st, detail.value


def launch_count() -> int:
    return int(lib().lh_launch_count())


def selftest_timeout(limit_cycles: int, gave_up: torch.Tensor, stream=None):
    """One warp waits, with the kernels' bounded wait, on an mbarrier nothing
    arrives on; after `limit_cycles` SM cycles it gives up and records
    LH_ERR_TIMEOUT (detail 900). `gave_up`: a device int32 tensor, set to 1."""
    _check(lib().lh_selftest_timeout(int(limit_cycles), _p(gave_up), _stream(stream)), "lh_selftest_timeout")


def selftest_exp2(x: torch.Tensor, y_fma: torch.Tensor, y_sfu: torch.Tensor, stream=None):
    """2^x of a device float32 tensor by the attention kernels' FMA-pipe
    polynomial (y_fma) and by the special-function unit's ex2.approx (y_sfu)."""
    _check(lib().lh_selftest_exp2(_p(x), _p(y_fma), _p(y_sfu), x.numel(), _stream(stream)), "lh_selftest_exp2")


def pool_range(cfg, t0, nt, q, k, v, pyr_q, pyr_k, pyr_v, sq, scale, stream=None):
    _check(lib().lh_pool_range(ctypes.byref(cfg), t0, nt, _p(q), _p(k), _p(v), _p(pyr_q), _p(pyr_k), _p(pyr_v),
                               _p(sq), _p(scale), _stream(stream)), "lh_pool_range")


def scatter_range(cfg, t0, nt, os_, slot, o, stream=None):
    _check(lib().lh_scatter_range(ctypes.byref(cfg), t0, nt, _p(os_), _p(slot), _p(o), _stream(stream)),
           "lh_scatter_range")


# ---------------------------------------------------------------------------
# sequence-sharded (context-parallel) path: the per-rank calls
# ---------------------------------------------------------------------------

def cp_plan(cfg, world: int, rank: int) -> CPPlan:
    out = CPPlan()
    _check(lib().lh_cp_plan(ctypes.byref(cfg), world, rank, ctypes.byref(out)), "lh_cp_plan")
    return out


def cp_pool(cfg, world, rank, q, k, v, pyr_q, pyr_k, pyr_v, sq_loc, scale, stream=None):
    _check(lib().lh_cp_pool(ctypes.byref(cfg), world, rank, _p(q), _p(k), _p(v), _p(pyr_q), _p(pyr_k),
                            _p(pyr_v), _p(sq_loc), _p(scale), _stream(stream)), "lh_cp_pool")


def cp_assemble_sq(cfg, world, sq_gathered, sq, stream=None):
    _check(lib().lh_cp_assemble_sq(ctypes.byref(cfg), world, _p(sq_gathered), _p(sq), _stream(stream)),
           "lh_cp_assemble_sq")


def cp_segment(cfg, world, rank, map_, slot, slot_loc, seg, stream=None):
    _check(lib().lh_cp_segment(ctypes.byref(cfg), world, rank, _p(map_), _p(slot), _p(slot_loc), _p(seg),
                               _stream(stream)), "lh_cp_segment")


def cp_gather(cfg, world, rank, q, k, v, pyr_q, pyr_k, pyr_v, map_, seg, scale, qs, ks, vs, stream=None):
    _check(lib().lh_cp_gather(ctypes.byref(cfg), world, rank, _p(q), _p(k), _p(v), _p(pyr_q), _p(pyr_k),
                              _p(pyr_v), _p(map_), _p(seg), _p(scale), _p(qs), _p(ks), _p(vs), _stream(stream)),
           "lh_cp_gather")


def cp_attn_fwd(cfg, world, rank, seg, qs, ks, vs, scale, os_, lse, stream=None):
    _check(lib().lh_cp_attn_fwd(ctypes.byref(cfg), world, rank, _p(seg), _p(qs), _p(ks), _p(vs), _p(scale),
                                _p(os_), _p(lse), _stream(stream)), "lh_cp_attn_fwd")


def cp_scatter(cfg, world, rank, os_, slot_loc, o, stream=None):
    _check(lib().lh_cp_scatter(ctypes.byref(cfg), world, rank, _p(os_), _p(slot_loc), _p(o), _stream(stream)),
           "lh_cp_scatter")


def cp_scatter_bwd(cfg, world, rank, dout, os_, slot_loc, seg, dos, delta, scale, stream=None):
    _check(lib().lh_cp_scatter_bwd(ctypes.byref(cfg), world, rank, _p(dout), _p(os_), _p(slot_loc), _p(seg),
                                   _p(dos), _p(delta), _p(scale), _stream(stream)), "lh_cp_scatter_bwd")


def cp_attn_bwd(cfg, world, rank, seg, qs, ks, vs, dos, lse, delta, scale, dqs, dks, dvs, stream=None):
    _check(lib().lh_cp_attn_bwd(ctypes.byref(cfg), world, rank, _p(seg), _p(qs), _p(ks), _p(vs), _p(dos),
                                _p(lse), _p(delta), _p(scale), _p(dqs), _p(dks), _p(dvs), _stream(stream)),
           "lh_cp_attn_bwd")


def cp_spread(cfg, world, rank, dqs, dks, dvs, slot_loc, dq, dk, dv, stream=None):
    _check(lib().lh_cp_spread(ctypes.byref(cfg), world, rank, _p(dqs), _p(dks), _p(dvs), _p(slot_loc), _p(dq),
                              _p(dk), _p(dv), _stream(stream)), "lh_cp_spread")


# ---------------------------------------------------------------------------
# buffers of one forward + backward (PyTorch allocates; liblh never does)
# ---------------------------------------------------------------------------

class Workspace:
    """Every intermediate buffer of one forward+backward, sized by lh_plan."""

    def __init__(self, cfg: Config, device, backward: bool = True):
        self.cfg = cfg
        self.plan = pl = plan(cfg)
        B, H, D = cfg.B, cfg.H, cfg.D
        S, E = pl.S, pl.E
        dt = torch.bfloat16 if cfg.dtype == LH_BF16 else torch.float32
        L, K = cfg.L, cfg.K
        f32, i32 = torch.float32, torch.int32
        z = lambda *s, dtype=dt: torch.empty(*s, dtype=dtype, device=device)
        e1 = max(E, 1)
        self.pyr_q, self.pyr_k, self.pyr_v = (z(B, H, e1, D) for _ in range(3))
        self.sq = z(2, B, H, e1, dtype=torch.float64)
        self.sel = z(B, H, max(L - 1, 1), K, dtype=i32)
        self.map = z(B, H, S, dtype=i32)
        self.slot = z(B, H, e1, dtype=i32)
        # attention operand type of the sub-sequence: fp16 for bf16 I/O
        bop = torch.float16 if cfg.dtype == LH_BF16 else dt
        self.qs, self.ks, self.vs = (z(B, H, S, D, dtype=bop) for _ in range(3))
        self.os = z(B, H, S, D, dtype=f32)
        self.lse = z(B, H, S, dtype=f32)
        self.ws = z(max(pl.ws_bytes, 16), dtype=torch.uint8)
        # per-head operand magnitudes [4][B][H] (uint32 bit patterns, held as int32)
        self.scale = torch.zeros(4, B, H, dtype=torch.int32, device=device)
        if backward:
            self.dos = z(B, H, S, D, dtype=bop)
            self.delta = z(B, H, S, dtype=f32)
            self.dqs, self.dks, self.dvs = (z(B, H, S, D, dtype=f32) for _ in range(3))
        else:
            self.dos = self.delta = self.dqs = self.dks = self.dvs = None
        self.c = Buffers(
            _p(self.pyr_q), _p(self.pyr_k), _p(self.pyr_v), _p(self.sq), _p(self.sel), _p(self.map),
            _p(self.slot), _p(self.qs), _p(self.ks), _p(self.vs), _p(self.os), _p(self.lse),
            _p(self.ws), self.ws.numel(), _p(self.dos), _p(self.delta), _p(self.dqs), _p(self.dks),
            _p(self.dvs), _p(self.scale))


def forward(cfg, q, k, v, o, ws: Workspace, stream=None):
    _check(lib().lh_forward(ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(o), ctypes.byref(ws.c),
                            _stream(stream)), "lh_forward")


def backward(cfg, dout, dq, dk, dv, ws: Workspace, stream=None):
    _check(lib().lh_backward(ctypes.byref(cfg), _p(dout), _p(dq), _p(dk), _p(dv), ctypes.byref(ws.c),
                             _stream(stream)), "lh_backward")


class LighthouseAttention(torch.autograd.Function):
    """Autograd wrapper: o = lighthouse(q, k, v) with q, k, v [B, N, H, D] on a CUDA device.

    The selection is frozen in the forward pass and takes no gradient.
    """

    @staticmethod
    def forward(ctx, q, k, v, p: int, L: int, K: int, accum: str = "fp"):
        B, N, H, D = q.shape
        dtype = {torch.bfloat16: "bf16", torch.float32: "fp32"}[q.dtype]
        cfg = make_config(B, H, N, D, p, L, K, dtype, accum)
        ws = Workspace(cfg, q.device, backward=True)
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o = torch.empty_like(q)
        forward(cfg, q, k, v, o, ws)
        ctx.cfg, ctx.ws = cfg, ws
        return o

    @staticmethod
    def backward(ctx, do):
        do = do.contiguous()
        dq, dk, dv = (torch.empty_like(do) for _ in range(3))
        backward(ctx.cfg, do, dq, dk, dv, ctx.ws)
        return dq, dk, dv, None, None, None, None


def lighthouse_attention(q, k, v, p: int, L: int, K: int, accum: str = "fp"):
    return LighthouseAttention.apply(q, k, v, p, L, K, accum)

"""C ABI checks that need no GPU: the library loads, exports every entry point
the header declares, sizes agree with the oracle, and bad arguments are
rejected with the documented status before anything is launched."""

import ctypes

import pytest

import oracle as orc
from long_context_symmetric_b200 import lh, synth

LH_ERR_NULL, LH_ERR_SHAPE, LH_ERR_ALIGN, LH_ERR_DTYPE, LH_ERR_MODE, LH_ERR_WORKSPACE = 1, 2, 3, 4, 5, 6


def test_library_exports_every_declared_symbol():
    names = lh.header_functions()
    assert len(names) >= 15
    lib = lh.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert lib.lh_version() >= 100
    assert lh.status_string(0) == "ok"


@pytest.mark.parametrize("inclusion", ["nested", "partition"])
@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_plan_agrees_with_oracle(name, inclusion):
    w = synth.WORKLOADS[name]
    pl = lh.plan(lh.make_config(w.B, w.H, w.N, w.D, w.p, w.L, w.K, w.dtype, w.mode, inclusion=inclusion))
    ref = orc.plan(w.N, w.p, w.L, w.K, inclusion)
    assert pl.S == ref.S
    assert list(pl.n)[:w.L] == ref.n
    assert list(pl.c)[:w.L] == ref.c
    assert list(pl.k)[1:w.L] == ref.k[1:]
    assert pl.E == sum(ref.n[1:])
    # the descent's workspace: 5 int32 per candidate of any level; none without a pyramid
    assert pl.ws_bytes == (w.B * w.H * 5 * sum(ref.m) * 4 if w.L > 1 else 0)


@pytest.mark.parametrize("N,p,L,K", [(64, 2, 1, 5), (48, 3, 2, 1), (243, 3, 5, 2), (4096, 8, 3, 4096),
                                     (1 << 20, 16, 3, 100)])
def test_plan_edge_sizes(N, p, L, K):
    pl = lh.plan(lh.make_config(1, 1, N, 64, p, L, K))
    assert pl.S == orc.plan(N, p, L, K).S


@pytest.mark.parametrize("bad", [
    dict(D=96), dict(D=0), dict(p=1), dict(L=0), dict(L=9), dict(K=0), dict(K=4097),
    dict(N=1000), dict(B=0), dict(H=0), dict(N=1 << 28),
])
def test_plan_rejects_bad_shapes(bad):
    kw = dict(B=1, H=2, N=4096, D=64, p=4, L=3, K=16)
    kw.update(bad)
    cfg = lh.make_config(**kw)
    assert lh.lib().lh_plan(ctypes.byref(cfg), ctypes.byref(lh.Plan())) == LH_ERR_SHAPE


def test_plan_rejects_bad_enums():
    cfg = lh.make_config(1, 2, 4096, 64, 4, 3, 16)
    cfg.dtype = 7
    assert lh.lib().lh_plan(ctypes.byref(cfg), ctypes.byref(lh.Plan())) == LH_ERR_DTYPE
    cfg = lh.make_config(1, 2, 4096, 64, 4, 3, 16)
    cfg.accum = 3
    assert lh.lib().lh_plan(ctypes.byref(cfg), ctypes.byref(lh.Plan())) == LH_ERR_MODE
    for field in ("score", "ties", "order", "weight", "inclusion"):
        cfg = lh.make_config(1, 2, 4096, 64, 4, 3, 16)
        setattr(cfg, field, 9)
        assert lh.lib().lh_plan(ctypes.byref(cfg), ctypes.byref(lh.Plan())) == LH_ERR_MODE, field


def test_entry_points_validate_before_launch():
    """Null, misaligned and short-workspace arguments return a status without any CUDA call."""
    lib = lh.lib()
    cfg = lh.make_config(1, 2, 4096, 64, 4, 3, 16)
    r = ctypes.byref(cfg)
    a = 1 << 20        # a fake, aligned address: never dereferenced on these paths
    m = a + 8          # misaligned
    assert lib.lh_pool(r, None, a, a, a, a, a, a, a, None) == LH_ERR_NULL
    assert lib.lh_pool(r, m, a, a, a, a, a, a, a, None) == LH_ERR_ALIGN
    assert lib.lh_pool(r, a, a, a, a, a, a, a, None, None) == LH_ERR_NULL         # no scale buffer
    assert lib.lh_score_topk(r, a, a, a, a, a, 16, None) == LH_ERR_WORKSPACE
    assert lib.lh_gather(r, a, a, a, a, a, a, None, a, a, a, a, None) == LH_ERR_NULL
    assert lib.lh_gather(r, a, a, a, a, a, a, a, None, a, a, a, None) == LH_ERR_NULL  # no scale buffer
    assert lib.lh_attn_fwd(r, a, a, a, a, m, a, None) == LH_ERR_ALIGN
    assert lib.lh_attn_fwd(r, a, a, a, None, a, a, None) == LH_ERR_NULL
    assert lib.lh_scatter(r, a, None, a, None) == LH_ERR_NULL
    assert lib.lh_scatter_bwd(r, a, a, a, a, None, a, None) == LH_ERR_NULL
    assert lib.lh_scatter_bwd(r, a, a, a, a, a, None, None) == LH_ERR_NULL
    assert lib.lh_attn_bwd(r, a, a, a, a, a, a, a, a, a, None, None) == LH_ERR_NULL
    assert lib.lh_attn_bwd(r, a, a, a, a, a, a, None, a, a, a, None) == LH_ERR_NULL
    assert lib.lh_spread(r, a, a, a, a, a, a, m, None) == LH_ERR_ALIGN
    assert lib.lh_forward(r, a, a, a, a, None, None) == LH_ERR_NULL
    bufs = lh.Buffers()
    assert lib.lh_forward(r, a, a, a, a, ctypes.byref(bufs), None) == LH_ERR_NULL
    bad = lh.make_config(1, 2, 4096, 96, 4, 3, 16)
    assert lib.lh_pool(ctypes.byref(bad), a, a, a, a, a, a, a, a, None) == LH_ERR_SHAPE


def test_single_level_needs_no_pyramid_or_workspace():
    """With L = 1 the pool needs no pyramid or norm buffers (it only records the
    operands' magnitudes into the scale buffer): validation passes them as
    NULL and stops only at the missing scale buffer, before any launch."""
    lib = lh.lib()
    cfg = lh.make_config(1, 2, 4096, 64, 4, 1, 16)
    a = 1 << 20
    before = lh.launch_count()
    assert lib.lh_pool(ctypes.byref(cfg), a, a, a, None, None, None, None, None, None) == LH_ERR_NULL
    assert lh.launch_count() == before


def test_sharded_entry_points_validate_before_launch():
    """The sequence-sharded calls refuse bad rank geometry and non-bf16
    attention before anything is launched (no device needed)."""
    ptr = 1 << 20                                        # any 16-byte aligned address: nothing is touched
    f = lh.lib()
    cfg = lh.make_config(1, 2, 8192, 128, 4, 3, 64)
    assert f.lh_cp_segment(ctypes.byref(cfg), 3, 0, ptr, ptr, ptr, ptr, None) == LH_ERR_SHAPE   # 8192 / 3
    assert f.lh_cp_segment(ctypes.byref(cfg), 4, 4, ptr, ptr, ptr, ptr, None) == LH_ERR_SHAPE   # rank 4 of 4
    assert f.lh_cp_segment(ctypes.byref(cfg), 0, 0, ptr, ptr, ptr, ptr, None) == LH_ERR_SHAPE   # no ranks
    assert f.lh_cp_segment(ctypes.byref(cfg), 1024, 0, ptr, ptr, ptr, ptr, None) == LH_ERR_SHAPE  # 8 tokens
    assert f.lh_cp_segment(ctypes.byref(cfg), 2, 0, None, ptr, ptr, ptr, None) == LH_ERR_NULL
    assert f.lh_cp_segment(ctypes.byref(cfg), 2, 0, ptr + 4, ptr, ptr, ptr, None) == LH_ERR_ALIGN
    c32 = lh.make_config(1, 2, 8192, 128, 4, 3, 64, "fp32")
    assert f.lh_cp_attn_fwd(ctypes.byref(c32), 2, 0, *([ptr] * 7), None) == LH_ERR_DTYPE
    assert f.lh_cp_attn_bwd(ctypes.byref(c32), 2, 0, *([ptr] * 11), None) == LH_ERR_DTYPE
    c1 = lh.make_config(1, 2, 8192, 128, 4, 1, 64)
    assert f.lh_cp_plan(ctypes.byref(c1), 2, 0, ctypes.byref(lh.CPPlan())) == LH_ERR_SHAPE    # L = 1
    pl = lh.cp_plan(cfg, 4, 3)
    assert (pl.n_loc, pl.E_loc, pl.glob.S) == (2048, 512 + 128, lh.plan(cfg).S)
    assert list(pl.lvl_off_loc)[1:3] == [0, 512]

"""Pool of bf16 rows whose exponents stress the pool's exact summation.

The pool sums a level-1 entry's p bf16 values per component in fp32 when that
chain is exact (every value normal with exponent field at most 250, fields
differing by at most 16 - log2 p) and in fp64 otherwise; either way the
result must be the fp64 left-to-right chain of the mean-pool ("Long Context
Pre-Training with Lighthouse Attention", §3.1 stage (i), Fig. 2 step 1). These
inputs put entries on both sides of every bound: spreads of exactly the
limit and one more, fields 1, 250, 251 and 254, exact zeros of both signs and
subnormals, mixed with ordinary values. The pyramid and the squared norms
must equal the fp64 oracle bit for bit, for the whole-sequence pool and for a
pool run as token ranges.
"""

import numpy as np
import pytest
import torch

import oracle as orc
from long_context_symmetric_b200 import lh

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _bf16_from_fields(sign, field, mant):
    bits = (sign.astype(np.int64) << 15) | (field.astype(np.int64) << 7) | mant.astype(np.int64)
    return torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16)


def _stress_rows(rng, n_tok, hd, p):
    """[n_tok, hd] bf16 tokens: each level-1 entry (p consecutive tokens) gets
    one exponent pattern per component, drawn from a set of cases."""
    limit = 16 - int(np.log2(p))
    n_ent = n_tok // p
    field = np.empty((n_ent, p, hd), dtype=np.int64)
    case = rng.integers(0, 9, size=(n_ent, 1, hd))
    base = rng.integers(20, 200, size=(n_ent, 1, hd))
    off = rng.integers(0, limit + 1, size=(n_ent, p, hd))
    field[:] = base + off                                       # ordinary: spread <= limit
    # spread exactly the limit, and one more
    for c, spread in ((1, limit), (2, limit + 1)):
        m = np.broadcast_to(case == c, field.shape)
        f = base + rng.integers(0, spread + 1, size=(n_ent, p, hd))
        f[:, 0, :] = base[:, 0, :]
        f[:, 1, :] = base[:, 0, :] + spread
        field = np.where(m, f, field)
    # the smallest and the largest fields
    for c, lo, hi in ((3, 1, 1 + limit), (4, 250 - limit, 250), (5, 251 - limit, 251), (6, 240, 254)):
        m = np.broadcast_to(case == c, field.shape)
        field = np.where(m, rng.integers(lo, hi + 1, size=field.shape), field)
    mant = rng.integers(0, 128, size=field.shape)
    sign = rng.integers(0, 2, size=field.shape)
    # exact zeros of either sign, and subnormals, mixed into ordinary entries
    zero = np.broadcast_to(case == 7, field.shape) & (rng.random(field.shape) < 0.3)
    field = np.where(zero, 0, field)
    mant = np.where(zero, 0, mant)
    sub = np.broadcast_to(case == 8, field.shape) & (rng.random(field.shape) < 0.3)
    field = np.where(sub, 0, field)
    mant = np.where(sub, rng.integers(1, 128, size=field.shape), mant)
    return _bf16_from_fields(sign.reshape(n_tok, hd), field.reshape(n_tok, hd), mant.reshape(n_tok, hd))


def _inputs(B, H, N, D, p, seed):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(3):
        t = torch.empty(B, N, H, D, dtype=torch.bfloat16)
        for b in range(B):
            for h in range(H):
                t[b, :, h, :] = _stress_rows(rng, N, D, p)
        out.append(t)
    return out


def _check_against_oracle(cfg, ws, q, k, v, p, L, dtype="bf16", score="max"):
    pl = lh.plan(cfg)
    B, H = q.shape[0], q.shape[2]
    for b in range(B):
        for h in range(H):
            means = {}
            for name, x, pyr in (("q", q, ws.pyr_q), ("k", k, ws.pyr_k), ("v", v, ws.pyr_v)):
                xm = x[b, :, h, :].float().double().numpy()
                m, stored = orc.pool_head(xm, p, L, dtype)
                means[name] = m
                for l in range(1, L):
                    o0, n = pl.lvl_off[l], pl.n[l]
                    got = pyr[b, h, o0:o0 + n].float().double().cpu().numpy()
                    assert np.array_equal(got, stored[l]), (name, b, h, l)
            _, sq_q, sq_k = orc.scores_head(means["q"], means["k"], L, score)
            for row, ref in ((0, sq_q), (1, sq_k)):
                for l in range(1, L):
                    o0, n = pl.lvl_off[l], pl.n[l]
                    got = ws.sq[row, b, h, o0:o0 + n].cpu().numpy()
                    assert np.array_equal(got, ref[l]), ("sq", row, b, h, l)


# H = 2: the block-parallel kernel (coarsest blocks of 512, 64, 64, 16, 16 and
# 8 tokens) and, where its level sums do not fit in shared memory (blocks of
# 4096 tokens), the shared-memory ring kernel; H = 16 with enough blocks: the
# ring kernel (8 warps per CTA at D = 128, 4 at D = 64)
@pytest.mark.parametrize("p,L,N,H,D", [(8, 4, 4096, 2, 128), (4, 4, 2048, 2, 128), (2, 7, 1024, 2, 128),
                                       (4, 3, 2048, 2, 128), (2, 5, 1024, 2, 128), (8, 2, 1024, 2, 128),
                                       (8, 5, 8192, 2, 128), (4, 4, 16384, 16, 128), (8, 4, 4096, 2, 64),
                                       (4, 4, 16384, 16, 64)])
def test_pool_exact_at_exponent_bounds(p, L, N, H, D):
    B = 1
    q, k, v = _inputs(B, H, N, D, p, seed=100 + p + L)
    cfg = lh.make_config(B, H, N, D, p, L, 16, "bf16")
    ws = lh.Workspace(cfg, DEV, backward=False)
    qd, kd, vd = (x.to(DEV) for x in (q, k, v))
    lh.pool(cfg, qd, kd, vd, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.sq, ws.scale)
    torch.cuda.synchronize()
    assert lh.get_device_error() == (0, 0)
    _check_against_oracle(cfg, ws, q, k, v, p, L)
    # the same pyramid from token ranges of one and of several coarsest blocks
    P = p ** (L - 1)
    ws2 = lh.Workspace(cfg, DEV, backward=False)
    t0 = 0
    for nt in (P, 3 * P, N):
        nt = min(nt, N - t0)
        if nt <= 0:
            break
        lh.pool_range(cfg, t0, nt, qd, kd, vd, ws2.pyr_q, ws2.pyr_k, ws2.pyr_v, ws2.sq, ws2.scale)
        t0 += nt
    torch.cuda.synchronize()
    for a, b_ in ((ws.pyr_q, ws2.pyr_q), (ws.pyr_k, ws2.pyr_k), (ws.pyr_v, ws2.pyr_v), (ws.sq, ws2.sq),
                  (ws.scale[:3], ws2.scale[:3])):
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                           b_.view(torch.int16) if b_.dtype == torch.bfloat16 else b_)


@pytest.mark.parametrize("p,L,N,H,dtype,score", [(8, 4, 4096, 2, "bf16", "maxpool"), (4, 4, 16384, 16, "bf16", "maxpool"),
                                                 (8, 4, 4096, 2, "fp32", "max"), (4, 4, 16384, 16, "fp32", "max")])
def test_pool_exponent_bounds_other_paths(p, L, N, H, dtype, score):
    """The same inputs through the paths that keep the fp64 chain throughout:
    the max-pool score reading (token norms pooled by max) and fp32 I/O."""
    B, D = 1, 128
    q, k, v = _inputs(B, H, N, D, p, seed=200 + p + L)
    if dtype == "fp32":
        q, k, v = (x.float() for x in (q, k, v))
    cfg = lh.make_config(B, H, N, D, p, L, 16, dtype, score=score)
    ws = lh.Workspace(cfg, DEV, backward=False)
    qd, kd, vd = (x.to(DEV) for x in (q, k, v))
    lh.pool(cfg, qd, kd, vd, ws.pyr_q, ws.pyr_k, ws.pyr_v, ws.sq, ws.scale)
    torch.cuda.synchronize()
    assert lh.get_device_error() == (0, 0)
    _check_against_oracle(cfg, ws, q, k, v, p, L, dtype, score)

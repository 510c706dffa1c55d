"""The FMA-pipe 2^x of the attention softmax against fp64 and against ex2.approx.

A 2^x for the FMA pipe (range reduction to [-1/2, 1/2], a degree-5 polynomial
with minimax relative error there found by the Remez exchange, and the
exponent added in the bit pattern), built to take part of each softmax
tile's exponentials off the special-function unit. Its maximum relative error
must stay within that of the ex2.approx.ftz.f32 it would stand in for (the PTX
ISA states about 2^-22 for ex2.approx.f32); it is checked here against 2^x in
fp64 over the range the softmax uses, with the special-function result
measured beside it. (Measured inside the attention kernels it did not pay off;
they keep ex2.)
"""

import numpy as np
import pytest
import torch

from long_context_symmetric_b200 import lh

pytestmark = pytest.mark.gpu


def test_exp2_polynomial_matches_ex2_error_bound():
    rng = np.random.default_rng(0)
    xs = np.concatenate([
        np.linspace(-124.0, 20.0, 1_000_001),
        rng.uniform(-30.0, 8.0, 1_000_000),
        np.arange(-124, 21, dtype=np.float64),                       # integers: f = 0
        np.arange(-124, 21, dtype=np.float64) + 0.5,                 # rounding ties of n
        np.nextafter(np.arange(-124, 21, dtype=np.float64) + 0.5, 0.0),
    ]).astype(np.float32)
    x = torch.from_numpy(xs).cuda()
    y_fma, y_sfu = torch.empty_like(x), torch.empty_like(x)
    lh.selftest_exp2(x, y_fma, y_sfu)
    torch.cuda.synchronize()
    ref = np.exp2(xs.astype(np.float64))
    rel_fma = np.abs(y_fma.cpu().numpy().astype(np.float64) / ref - 1)
    rel_sfu = np.abs(y_sfu.cpu().numpy().astype(np.float64) / ref - 1)
    # ex2.approx.ftz flushes results below 2^-126; compare both where it does not
    normal = ref >= 2.0 ** -125
    print("max relative error: polynomial 2^%.2f, ex2.approx 2^%.2f" %
          (np.log2(rel_fma[normal].max()), np.log2(rel_sfu[normal].max())))
    assert rel_fma[normal].max() <= 2.0 ** -22
    assert rel_fma[normal].max() <= max(rel_sfu[normal].max(), 2.0 ** -22)


def test_exp2_polynomial_clamps_below_range():
    x = torch.tensor([-125.0, -126.0, -1000.0, float("-inf"), -3.0e38], device="cuda")
    y_fma, y_sfu = torch.empty_like(x), torch.empty_like(x)
    lh.selftest_exp2(x, y_fma, y_sfu)
    torch.cuda.synchronize()
    got = y_fma.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got / 2.0 ** -125 - 1) <= 2.0 ** -22)      # 2^-125 to the polynomial's accuracy

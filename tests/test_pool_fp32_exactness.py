"""The bound behind the pool's fp32 level-1 sums, checked on the host.

The pool sums a level-1 entry's p bf16 values in fp32 when every value is
normal with exponent field at most 250 and the fields differ by at most
16 - log2(p); it then claims the fp32 chain ((x0 + x1) + x2) + ... equals the
fp64 chain of the mean-pool ("Long Context Pre-Training with Lighthouse
Attention", §3.1 stage (i), Fig. 2 step 1) bit for bit. Here: random entries
inside the bound give equal chains (numpy's float32 and float64 additions are
IEEE round-to-nearest-even), and entries just outside it can differ, so the
bound is not vacuous.
"""

import numpy as np
import pytest


def _bf16_values(sign, field, mant):
    bits = ((sign.astype(np.uint32) << 31) | (field.astype(np.uint32) << 23) | (mant.astype(np.uint32) << 16))
    return bits.view(np.float32)


def _chains(x):
    """Left-to-right fp32 and fp64 chains over axis 1."""
    s32 = x[:, 0].astype(np.float32)
    s64 = x[:, 0].astype(np.float64)
    for u in range(1, x.shape[1]):
        s32 = (s32 + x[:, u].astype(np.float32)).astype(np.float32)
        s64 = s64 + x[:, u].astype(np.float64)
    return s32, s64


@pytest.mark.parametrize("p", [2, 4, 8])
def test_inside_the_bound_fp32_chain_is_the_fp64_chain(p):
    rng = np.random.default_rng(p)
    limit = 16 - int(np.log2(p))
    n = 200_000
    base = rng.integers(1, 251 - limit, size=(n, 1))
    field = base + rng.integers(0, limit + 1, size=(n, p))
    field = np.minimum(field, 250)
    # put the extremes of the allowed spread into half of the entries
    field[: n // 2, 0] = base[: n // 2, 0]
    field[: n // 2, 1] = np.minimum(base[: n // 2, 0] + limit, 250)
    x = _bf16_values(rng.integers(0, 2, size=(n, p)), field, rng.integers(0, 128, size=(n, p)))
    assert np.all(np.isfinite(x))
    s32, s64 = _chains(x)
    assert np.array_equal(s32.astype(np.float64), s64)


@pytest.mark.parametrize("p", [2, 4, 8])
def test_random_entries_just_outside_the_bound_can_differ(p):
    rng = np.random.default_rng(100 + p)
    limit = 16 - int(np.log2(p))
    n = 200_000
    base = rng.integers(1, 200, size=(n, 1))
    field = base + rng.integers(0, limit + 4, size=(n, p))
    field[:, 0] = base[:, 0]
    field[:, 1] = base[:, 0] + limit + 3
    x = _bf16_values(rng.integers(0, 2, size=(n, p)), field, rng.integers(0, 128, size=(n, p)))
    s32, s64 = _chains(x)
    assert not np.array_equal(s32.astype(np.float64), s64)


def test_worked_example_outside_the_bound():
    """Seven values (2 - 2^-7) 2^13 and one (1 + 2^-7) 2^-1 (fields 140 and 126,
    spread 14 > 13): the exact sum needs bits from 2^16 down to 2^-8, 25 of them,
    so the fp32 chain rounds and the fp64 chain does not."""
    big = np.float32((2 - 2.0 ** -7) * 2.0 ** 13)
    small = np.float32((1 + 2.0 ** -7) * 2.0 ** -1)
    x = np.array([[big] * 7 + [small]], dtype=np.float32)
    s32, s64 = _chains(x)
    assert s64[0] == 7 * float(big) + float(small)
    assert float(s32[0]) != s64[0]

"""Pins of the oracle's global amax (max |x| over the fp32 values of x; the
article's sec. 7.2 example passes x.abs().max() as act_amax): a library
special case (numpy's float64 reduction), closed forms, and invariants that a
dropped abs, a wrong start value, a skipped element or a mishandled sign of
zero would break."""
import numpy as np
import pytest

import oracle


def _values(rng, n, dtype):
    v = rng.standard_normal(n) * np.exp(rng.uniform(-8, 8, n))
    return v.astype(dtype).astype(np.float32)


@pytest.mark.parametrize("dtype", [np.float32, np.float16])
@pytest.mark.parametrize("n", [1, 2, 7, 16, 17, 1000, 4099])
def test_matches_numpy_reduction(dtype, n):
    rng = np.random.default_rng(n)
    x = _values(rng, n, dtype)
    ref = np.float32(np.max(np.abs(x.astype(np.float64))))
    assert oracle.act_amax(x).view(np.uint32) == ref.view(np.uint32)


def test_closed_forms():
    assert oracle.act_amax(np.arange(-50, 31, dtype=np.float32)) == 50.0      # negative end wins
    assert oracle.act_amax(np.arange(-30, 51, dtype=np.float32)) == 50.0      # positive end wins
    assert oracle.act_amax(np.linspace(-0.25, 0.125, 7, dtype=np.float32)) == np.float32(0.25)
    assert oracle.act_amax(np.array([], np.float32)) == 0.0                     # empty
    z = oracle.act_amax(np.array([-0.0, -0.0, 0.0], np.float32))
    assert z.view(np.uint32) == 0                                                # +0, not -0
    tiny = np.array([-1e-45, 7e-46], np.float32)                                 # subnormals
    assert oracle.act_amax(tiny) == np.float32(1e-45)
    assert oracle.act_amax(np.array([1.0, -np.inf, 3.0], np.float32)) == np.inf
    assert oracle.act_amax(np.array([-7.5], np.float32)) == 7.5                  # single negative element


def test_invariants():
    rng = np.random.default_rng(7)
    for n in (3, 64, 513):
        x = _values(rng, n, np.float32)
        m = oracle.act_amax(x)
        assert oracle.act_amax(-x) == m                                          # sign symmetry
        assert oracle.act_amax(rng.permutation(x)) == m                          # order free
        assert oracle.act_amax(x * np.float32(0.5)) == m * np.float32(0.5)       # power-of-two covariance
        assert np.all(np.abs(x) <= m) and np.any(np.abs(x) == m)                 # bound, attained
        k = int(rng.integers(1, n)) if n > 1 else 1
        assert max(oracle.act_amax(x[:k]), oracle.act_amax(x[k:])) == m          # splits
        y = x.copy()
        y[-1] = np.float32(-2.0) * m                                             # the last element counts
        assert oracle.act_amax(y) == np.float32(2.0) * m
        y = x.copy()
        y[0] = np.float32(-2.0) * m                                              # so does the first
        assert oracle.act_amax(y) == np.float32(2.0) * m

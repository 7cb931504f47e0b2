"""Pins of the oracle's standalone fake-quant at the article's other block
sizes (sec. 7.1: 16, 32, 64, 128 or 256 elements per block; sec. 7.3: numel
a multiple of it).  A block's scale comes from the maximum over all of its
elements, and every element is then quantised on its own, which the
composition pin checks against the 16-element oracle; sec. 9.3's property
that finer blocks lose less (err(16) <= err(64) <= err(256), with 1.2x
slack) is checked on seeded data; sign symmetry, power-of-two covariance and
the argument rules close it."""
import numpy as np
import pytest

import oracle

SIZES = [16, 32, 64, 128, 256]


def _data(seed, n):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(n).astype(np.float32)
    x[rng.integers(0, n, n // 97)] *= 12.0  # sparse outliers
    return x


def test_block_16_is_the_standard_call():
    x = _data(1, 4096)
    amax = float(np.abs(x).max())
    assert np.array_equal(oracle.fp4_fake_quant_bs(x, amax, 16).view(np.uint32),
                          oracle.fp4_fake_quant(x, amax).view(np.uint32))


@pytest.mark.parametrize("B", [32, 64, 128, 256])
def test_block_scale_comes_from_the_whole_block(B):
    """Plant the block's largest magnitude M in sub-block j; every other
    element's output equals the 16-element oracle's output for its own
    sub-block with M planted at one position (the same scale, element-wise
    quantisation)."""
    rng = np.random.default_rng(B)
    for trial in range(20):
        x = _data(100 * B + trial, B)
        amax = float(np.abs(x).max()) * 1.5
        j = int(rng.integers(0, B // 16))
        p = 16 * j + int(rng.integers(0, 16))
        M = np.float32(np.abs(x).max() * np.float32(1.25))
        x[p] = -M if trial % 2 else M
        got = oracle.fp4_fake_quant_bs(x, amax, B)
        for i in range(B // 16):
            sub = x[16 * i:16 * i + 16].copy()
            q = p - 16 * i if i == j else int(rng.integers(0, 16))
            sub[q] = M
            ref = oracle.fp4_fake_quant(sub, amax)
            keep = np.arange(16) != q
            assert np.array_equal(got[16 * i:16 * i + 16][keep].view(np.uint32), ref[keep].view(np.uint32)), (B, i)
        assert got[p] == oracle.fp4_fake_quant(x[16 * j:16 * j + 16], amax)[p - 16 * j]


def test_finer_blocks_lose_less():
    x = _data(7, 1 << 16)
    amax = float(np.abs(x).max())
    err = {B: float(np.mean((oracle.fp4_fake_quant_bs(x, amax, B).astype(np.float64) - x) ** 2)) for B in SIZES}
    assert err[16] <= 1.2 * err[64] and err[64] <= 1.2 * err[256]
    assert err[16] < err[32] < err[64] < err[128] < err[256]  # strictly, on this data


@pytest.mark.parametrize("B", SIZES)
def test_block_size_invariants(B):
    x = _data(11 + B, 8 * B)
    amax = float(np.abs(x).max())
    y = oracle.fp4_fake_quant_bs(x, amax, B)
    assert np.array_equal(oracle.fp4_fake_quant_bs(-x, amax, B), -y)                       # sign symmetry
    assert np.array_equal(oracle.fp4_fake_quant_bs(x * np.float32(4), amax * 4, B), y * np.float32(4))  # 2^k scaling
    assert np.all(np.abs(y) <= max(amax * 1.0001, 6.0))


def test_block_size_rules():
    x = np.ones(96, np.float32)
    with pytest.raises(ValueError):
        oracle.fp4_fake_quant_bs(x, 1.0, 48)       # not one of the article's sizes
    with pytest.raises(ValueError):
        oracle.fp4_fake_quant_bs(x, 1.0, 64)       # 96 is not a multiple of 64
    assert oracle.fp4_fake_quant_bs(x, 1.0, 32).shape == (96,)

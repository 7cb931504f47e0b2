"""Pins for the oracle's NVFP4 fake-quantiser (article sec. 6.2-6.4).

Pinned by hand-derived worked examples (tests/golden/fq_worked_examples.txt)
and by properties the definition implies: sign symmetry, exact power-of-two
covariance, zero blocks, the act_amax = 0 fallback, monotonicity inside a
block, grid points reproduced exactly, zero-filled short blocks, and the
bound on the relative error of the block maximum.
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fq_worked_examples.txt")
GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float32)


def _load_golden():
    cases, cur = [], {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = line.split(":", 1)
            key = key.strip()
            if key == "name":
                if cur:
                    cases.append(cur)
                cur = {"name": val.strip()}
            elif key == "amax":
                cur["amax"] = np.float32(val.strip())
            else:
                cur[key] = np.array([np.float32(t) for t in val.split()], dtype=np.float32)
    if cur:
        cases.append(cur)
    return cases


CASES = _load_golden()


def test_golden_file_parsed():
    assert len(CASES) >= 8
    for c in CASES:
        assert c["in"].size == 16 and c["out"].size == 16, c["name"]


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_worked_examples(case):
    got = oracle.fq_block(case["in"], case["amax"])
    # compare bit patterns so that -0 and +0 are distinguished
    assert np.array_equal(got.view(np.uint32), case["out"].view(np.uint32)), (got, case["out"])


def test_reciprocal_448_in_golden_is_binary32():
    # the clamp_448 example relies on RN(1/448) written out in the fixture
    assert np.float32(1) / np.float32(448) == np.float32("0.002232142956927418708801269531")


def _rand_blocks(n, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, 16)).astype(np.float32) * np.float32(scale)
    x[rng.random((n, 16)) < 0.001] *= 20
    return x


def test_sign_symmetry():
    x = _rand_blocks(2000, 10)
    amax = float(np.abs(x).max())
    a = oracle.fp4_fake_quant(x, amax)
    b = oracle.fp4_fake_quant(-x, amax)
    assert np.array_equal(a.view(np.uint32) ^ np.uint32(0x80000000), b.view(np.uint32))


@pytest.mark.parametrize("k", [-6, -3, 1, 5, 12])
def test_power_of_two_covariance(k):
    # fq(2^k x, 2^k amax) == 2^k fq(x, amax) as long as no scale sits near the
    # 1e-5 fallback threshold (blocks are drawn with comfortable magnitudes)
    x = _rand_blocks(2000, 11, scale=4.0)
    amax = np.float32(np.abs(x).max())
    f = np.float32(2.0 ** k)
    a = oracle.fp4_fake_quant(x, amax)
    b = oracle.fp4_fake_quant(x * f, amax * f)
    assert np.array_equal(a * f, b)


def test_zero_block_gives_zero():
    z = np.zeros(16, np.float32)
    for amax in [0.0, 1.0, 1e-30, 1e30]:
        assert np.array_equal(oracle.fq_block(z, amax).view(np.uint32), np.zeros(16, np.uint32))


def test_amax_zero_uses_unit_scale():
    # g = 0 -> r = inf or nan -> clamped to 448 -> scale 0 -> fallback 1.0, so the
    # block is rounded on the bare E2M1 grid
    x = _rand_blocks(500, 12, scale=2.0)
    got = oracle.fp4_fake_quant(x, 0.0)
    assert np.array_equal(got, oracle.e2m1(x))


def test_monotone_within_block():
    x = _rand_blocks(3000, 13)
    amax = float(np.abs(x).max())
    q = oracle.fp4_fake_quant(x, amax).reshape(-1, 16)
    ax, aq = np.abs(x), np.abs(q)
    for r in range(0, q.shape[0], 7):
        order = np.argsort(ax[r], kind="stable")
        assert np.all(np.diff(aq[r][order]) >= 0)


def test_grid_points_reproduced():
    # with amax = 2688 (g = 1) and block maximum 6 * 2^j, the scale is 2^j and
    # every value q * 2^j with q on the E2M1 grid comes back unchanged
    rng = np.random.default_rng(14)
    for j in range(-8, 9):
        q = rng.choice(np.concatenate([GRID, -GRID]), size=(50, 16)).astype(np.float32)
        q[:, 0] = 6.0
        x = q * np.float32(2.0 ** j)
        got = oracle.fp4_fake_quant(x, 2688.0)
        assert np.array_equal(got, x), j


def test_short_block_equals_zero_filled():
    rng = np.random.default_rng(15)
    for n in range(1, 16):
        v = rng.standard_normal(n).astype(np.float32)
        full = np.zeros(16, np.float32)
        full[:n] = v
        assert np.array_equal(oracle.fq_block(v, 3.0), oracle.fq_block(full, 3.0)[:n])


def test_block_max_relative_error_bounded():
    # the block maximum is represented to within the E4M3 scale rounding
    # (2^-4 relative) and the E2M1 rounding near 6 (at most 1/12 relative
    # before saturation); together well under 20 %
    x = _rand_blocks(4000, 16)
    amax = float(np.abs(x).max())
    q = oracle.fp4_fake_quant(x, amax).reshape(-1, 16)
    bm = np.abs(x).max(axis=1)
    qm = np.abs(q).max(axis=1)
    keep = bm > amax * 1e-3
    assert np.all(np.abs(qm[keep] - bm[keep]) <= 0.2 * bm[keep])


def test_values_are_grid_times_scale():
    # each output is q * s for one per-block scale s and q on the E2M1 grid
    x = _rand_blocks(1000, 17)
    amax = float(np.abs(x).max())
    q = oracle.fp4_fake_quant(x, amax).reshape(-1, 16).astype(np.float64)
    for r in range(q.shape[0]):
        nz = np.abs(q[r][q[r] != 0])
        if nz.size == 0:
            continue
        s = nz.min()
        ratios = nz / s
        # all ratios are quotients of grid magnitudes
        allowed = {a / b for a in GRID[1:] for b in GRID[1:]}
        assert all(any(abs(t - a) < 1e-6 for a in allowed) for t in ratios)


def test_standalone_requires_multiple_of_16():
    with pytest.raises(ValueError):
        oracle.fp4_fake_quant(np.zeros(17, np.float32), 1.0)


def test_standalone_is_blockwise():
    x = _rand_blocks(64, 18).ravel()
    amax = float(np.abs(x).max())
    got = oracle.fp4_fake_quant(x, amax)
    for b in range(0, x.size, 16):
        assert np.array_equal(got[b:b + 16], oracle.fq_block(x[b:b + 16], amax))

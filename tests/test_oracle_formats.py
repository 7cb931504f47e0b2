"""Pins for the oracle's scalar formats (E2M1, E4M3, BF16, FP16 rounding).

E2M1 is pinned by the eight magnitudes and the seven decision boundaries of
the Model-Optimizer "Conv3D Implicit GEMM CUDA kernel" article, sec. 6.1, with
ties resolved to the even code, and by an independent nearest-point search.
E4M3, BF16 and FP16 are pinned by library conversions (torch float8_e4m3fn,
torch bfloat16, numpy float16), which are special cases the oracle must
reproduce exactly.
"""
import numpy as np
import pytest
import torch

import oracle

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float32)


def test_e2m1_grid_roundtrip():
    # every representable magnitude and its negative maps to itself (sec. 6.1)
    vals = np.concatenate([GRID, -GRID])
    assert np.array_equal(oracle.e2m1(vals), vals)


def test_e2m1_boundaries_ties_to_even():
    # boundaries listed in sec. 6.1; at the boundary the even code wins
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for b, expect in ties.items():
        b32 = np.float32(b)
        below = np.nextafter(b32, np.float32(0))
        above = np.nextafter(b32, np.float32(10))
        lo = GRID[GRID < b].max()
        hi = GRID[GRID > b].min()
        assert oracle.e2m1([b32])[0] == expect, b
        assert oracle.e2m1([below])[0] == lo, b
        assert oracle.e2m1([above])[0] == hi, b
        assert oracle.e2m1([-b32])[0] == -expect, b


def test_e2m1_saturates():
    big = np.array([6.0, 6.5, 7.0, 1e6, np.inf], dtype=np.float32)
    assert np.array_equal(oracle.e2m1(big), np.full(5, 6.0, np.float32))
    assert np.array_equal(oracle.e2m1(-big), np.full(5, -6.0, np.float32))


def test_e2m1_matches_nearest_point_search():
    # independent formulation: argmin |a - g| over the grid, ties -> even index
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.uniform(0, 7, 4000), np.arange(0, 7, 0.125)]).astype(np.float32)
    d = np.abs(a[:, None].astype(np.float64) - GRID[None, :].astype(np.float64))
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    idx = np.array([np.flatnonzero(row)[0] if row.sum() == 1 else [i for i in np.flatnonzero(row) if i % 2 == 0][0]
                    for row in cand])
    expect = np.where(a >= 6, 6.0, GRID[idx]).astype(np.float32)
    assert np.array_equal(oracle.e2m1(a), expect)


def _e4m3_torch(v):
    return torch.from_numpy(np.asarray(v, np.float32)).to(torch.float8_e4m3fn).to(torch.float32).numpy()


def test_e4m3_all_codes_roundtrip():
    codes = torch.arange(0, 127, dtype=torch.uint8)
    vals = codes.view(torch.float8_e4m3fn).to(torch.float32).numpy()
    assert vals.max() == 448.0
    assert np.array_equal(oracle.e4m3(vals), vals)


def test_e4m3_matches_torch_dense_and_midpoints():
    codes = torch.arange(0, 127, dtype=torch.uint8)
    vals = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    nb = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    rng = np.random.default_rng(1)
    dense = np.concatenate([rng.uniform(0, 448, 20000), np.exp(rng.uniform(np.log(1e-5), np.log(448), 20000))])
    v = np.concatenate([nb, dense.astype(np.float32), [0.0, 448.0]]).astype(np.float32)
    assert np.array_equal(oracle.e4m3(v), _e4m3_torch(v))


def test_e4m3_saturates_at_448():
    assert np.array_equal(oracle.e4m3([448.0, 460.0, 1e30, np.inf]), np.full(4, 448.0, np.float32))


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000)]).astype(np.float32)
    # exact ties: bf16 value + half an ulp (bit 15 set, lower bits clear)
    base = rng.standard_normal(2000).astype(np.float32)
    u = (base.view(np.uint32) & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    v = np.concatenate([v, u.view(np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(oracle.bf16_round(v), ref)
    bits = oracle.round_to_dtype_bits(v, "bfloat16")
    assert np.array_equal(bits, (ref.view(np.uint32) >> 16).astype(np.uint16))


def test_f16_bits_match_numpy():
    rng = np.random.default_rng(3)
    v = (rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 4, 20000)).astype(np.float32)
    bits = oracle.round_to_dtype_bits(v, "float16")
    assert np.array_equal(bits, v.astype(np.float16).view(np.uint16))


def test_fp32_bits_identity():
    v = np.array([1.5, -0.0, 3e-40], dtype=np.float32)
    assert np.array_equal(oracle.round_to_dtype_bits(v, "float32"), v.view(np.uint32))

"""Pins for the oracle's exact NVFP4 operands (the true-FP4 product).

The variant keeps the quantiser of the article (Model-Optimizer "Conv3D
Implicit GEMM CUDA kernel", sec. 6.1-6.3: E2M1 codes, E4M3 block scale of
bmax / (6 g) with g = amax / (6 * 448), blocks of 16) and of its weight path
(sec. 7.2: weights quantised along the reduction axis), and takes the
operand value sign * q * s8 * g exactly instead of the BF16 rounding of the
binary32 q * scale.  What pins it:

- against the separately pinned fake-quantiser: where no block falls back,
  every exact value is within the two binary32 roundings of the fake-quant
  value (a wrong code, a wrong scale step or a dropped global scale is off by
  far more), with the same signs and zeros;
- closed form: values on the grid q * s8 * g (g a power of two) are fixed;
- the fallback: a block whose scale falls below 1e-5 contributes zero (the
  reading this variant takes, since 1.0 is no E4M3 scale times g);
- brute force for the convolution: numpy im2col, each row and each weight
  row quantised block by block with the exact block function, and a float64
  matmul;
- power-of-two covariance of the whole convolution in x and in w.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle


def _im2col(x, k, s, plo, phi, d):
    """Explicit im2col: rows (n, od, oh, ow), columns (c, kd, kh, kw)."""
    N, C, D, H, W = x.shape
    xp = np.pad(x, ((0, 0), (0, 0), (plo[0], phi[0]), (plo[1], phi[1]), (plo[2], phi[2])))
    OD = (xp.shape[2] - d[0] * (k[0] - 1) - 1) // s[0] + 1
    OH = (xp.shape[3] - d[1] * (k[1] - 1) - 1) // s[1] + 1
    OW = (xp.shape[4] - d[2] * (k[2] - 1) - 1) // s[2] + 1
    cols = np.empty((N, OD, OH, OW, C, k[0], k[1], k[2]), dtype=np.float32)
    for kd, kh, kw in itertools.product(range(k[0]), range(k[1]), range(k[2])):
        sl = xp[:, :,
                kd * d[0]: kd * d[0] + s[0] * (OD - 1) + 1: s[0],
                kh * d[1]: kh * d[1] + s[1] * (OH - 1) + 1: s[1],
                kw * d[2]: kw * d[2] + s[2] * (OW - 1) + 1: s[2]]
        cols[..., kd, kh, kw] = sl.transpose(0, 2, 3, 4, 1)
    return cols.reshape(N * OD * OH * OW, -1), (N, OD, OH, OW)


def _rows_exact(A, amax):
    """Each row in blocks of 16 (a short last block zero-filled) through the
    exact block function."""
    out = np.zeros(A.shape, np.float64)
    for r in range(A.shape[0]):
        for j in range(0, A.shape[1], 16):
            n = min(16, A.shape[1] - j)
            blk = np.zeros(16, np.float32)
            blk[:n] = A[r, j:j + n]
            out[r, j:j + n] = oracle.nvfp4_block_exact(blk, amax)[:n]
    return out


@pytest.mark.parametrize("scale", [1.0, 3.0, 1e-3, 250.0])
@pytest.mark.parametrize("amax_div", [1.0, 50.0])
def test_within_two_binary32_roundings_of_the_fake_quant(scale, amax_div):
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(4096, generator=g) * scale).numpy()
    amax = float(np.abs(x).max()) / amax_div
    e = oracle.nvfp4_exact(x, amax)
    f = oracle.fp4_fake_quant(x, amax).astype(np.float64)
    # fake-quant = RN32(q * RN32(s8 * g)); exact = q * s8 * g
    assert np.array_equal(e == 0, f == 0)
    assert np.array_equal(np.signbit(e[e != 0]), np.signbit(f[f != 0]))
    nz = e != 0
    rel = np.abs(e[nz] - f[nz]) / np.abs(e[nz])
    assert rel.max() <= 2.0 ** -22
    # enough nonzero values for the comparison to mean something
    assert nz.sum() > 1000


def test_grid_values_are_fixed():
    # g = amax / 2688 a power of two; a block whose maximum is 6 * s8 * g has
    # ratio s8, so every value q * s8 * g of it is returned unchanged (s8 * g
    # stays above the 1e-5 fallback threshold)
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for g in (1.0, 2.0 ** -4):
        amax = 2688.0 * g
        for s8 in [2.0 ** -9, 0.875, 1.0, 13.0, 240.0, 448.0]:
            blk = np.array([6.0] + mags + [-m for m in mags[1:]], np.float64)[:16] * s8 * g
            assert blk.size == 16
            e = oracle.nvfp4_block_exact(blk.astype(np.float32), amax)
            np.testing.assert_array_equal(e, blk)


def test_fallback_blocks_contribute_zero():
    x = np.linspace(-3.0, 3.0, 32).astype(np.float32)
    # amax far below the block maxima: the ratio clamps to 448 and the scale
    # 448 * amax / 2688 is below 1e-5, so the article falls back to 1.0; the
    # fake-quant then keeps E2M1(|v|), the exact operand is zero
    for amax in (1e-6, 0.0):
        e = oracle.nvfp4_exact(x, amax)
        f = oracle.fp4_fake_quant(x, amax)
        assert np.all(e == 0.0)
        assert np.any(f != 0.0)
    # tiny blocks next to large ones: E4M3 code 0 gives scale 0 < 1e-5
    blk = np.zeros(16, np.float32)
    blk[3] = 1e-9
    assert np.all(oracle.nvfp4_block_exact(blk, 1000.0) == 0.0)


def test_short_block_acts_as_zero_filled():
    g = torch.Generator().manual_seed(9)
    v = torch.randn(16, generator=g).numpy()
    amax = 2.5
    for n in (1, 5, 15):
        padded = v.copy()
        padded[n:] = 0.0
        np.testing.assert_array_equal(oracle.nvfp4_block_exact(v[:n], amax), oracle.nvfp4_block_exact(padded, amax)[:n])


def test_rejects_ragged_numel():
    with pytest.raises(ValueError):
        oracle.nvfp4_exact(np.ones(20, np.float32), 1.0)


CASES = [
    # x_shape, cout, kernel, stride, pad_lo, pad_hi, dil
    ((1, 3, 4, 6, 7), 5, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1)),   # K = 81: short last block
    ((2, 4, 5, 7, 6), 3, (3, 3, 3), (1, 2, 2), (1, 1, 1), (1, 1, 1), (1, 1, 1)),
    ((1, 2, 6, 9, 9), 4, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 2, 2)),
    ((1, 16, 3, 5, 5), 6, (1, 1, 1), (1, 1, 1), (0, 0, 0), (0, 0, 0), (1, 1, 1)),  # K = 16
]


@pytest.mark.parametrize("case", CASES)
def test_conv_matches_im2col_with_exact_operands(case):
    xs, cout, k, s, plo, phi, d = case
    g = torch.Generator().manual_seed(21)
    x = (torch.randn(xs, generator=g) * 2).numpy()
    w = (torch.randn((cout, xs[1]) + k, generator=g) * 0.1).numpy()
    b = torch.randn(cout, generator=g).numpy()
    amax, wamax = float(np.abs(x).max()), float(np.abs(w).max())
    A, (N, OD, OH, OW) = _im2col(x, k, s, plo, phi, d)
    Aq = _rows_exact(A, amax)
    Wq = _rows_exact(w.reshape(cout, -1), wamax)
    ref = (Aq @ Wq.T + b.astype(np.float64)).reshape(N, OD, OH, OW, cout).transpose(0, 4, 1, 2, 3)
    got = oracle.conv3d_nvfp4(x, w, b, s, plo, phi, d, act_amax=amax, w_amax=wamax)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    # row subsets agree with the full output
    M = N * OD * OH * OW
    ml = np.array([0, M - 1, M // 2], np.int64)
    rows = oracle.conv3d_nvfp4(x, w, b, s, plo, phi, d, act_amax=amax, w_amax=wamax, m_list=ml)
    full = got.transpose(0, 2, 3, 4, 1).reshape(M, cout)
    np.testing.assert_array_equal(rows, full[ml])


def test_conv_power_of_two_covariance():
    xs, cout, k, s, plo, phi, d = CASES[0]
    g = torch.Generator().manual_seed(23)
    x = torch.randn(xs, generator=g).numpy()
    w = (torch.randn((cout, xs[1]) + k, generator=g) * 0.2).numpy()
    amax, wamax = float(np.abs(x).max()), float(np.abs(w).max())
    base = oracle.conv3d_nvfp4(x, w, None, s, plo, phi, d, act_amax=amax, w_amax=wamax)
    sx = oracle.conv3d_nvfp4(x * 8, w, None, s, plo, phi, d, act_amax=amax * 8, w_amax=wamax)
    sw = oracle.conv3d_nvfp4(x, w / 4, None, s, plo, phi, d, act_amax=amax, w_amax=wamax / 4)
    np.testing.assert_array_equal(sx, base * 8)
    np.testing.assert_array_equal(sw, base / 4)


def test_conv_differs_from_bf16_weights():
    # the weights are quantised too: the result is not the fake-quant
    # convolution over BF16 weights, yet close to it
    xs, cout, k, s, plo, phi, d = CASES[1]
    g = torch.Generator().manual_seed(29)
    x = torch.randn(xs, generator=g).numpy()
    w = (torch.randn((cout, xs[1]) + k, generator=g) * 0.2).numpy()
    amax, wamax = float(np.abs(x).max()), float(np.abs(w).max())
    a = oracle.conv3d_nvfp4(x, w, None, s, plo, phi, d, act_amax=amax, w_amax=wamax)
    b = oracle.conv3d(x, w, None, s, plo, phi, d, quant_act=True, act_amax=amax)
    assert not np.array_equal(a, b)
    assert np.abs(a - b).max() < 0.25 * np.abs(b).max()

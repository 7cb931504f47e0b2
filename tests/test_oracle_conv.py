"""Pins for the oracle's convolution (article sec. 5.1, 6.3, 7.1).

- Library special case: with quant off and BF16-exact operands, the oracle
  equals torch.nn.functional.conv3d in float64 on the CPU (asymmetric padding
  applied with F.pad first, as sec. 7.1 describes), across strides,
  dilations, paddings and kernel shapes 1x1x1, 1x3x3, 3x3x3, 5x5x5.
- BF16 operand rounding: with non-BF16-exact operands the oracle equals the
  float64 conv of the BF16-rounded tensors (torch's bfloat16 cast).
- Brute force: an explicit im2col matrix built with numpy slicing in the
  article's (c, kd, kh, kw) column order, each row fake-quantised in blocks of
  16, then a float64 matmul; equal to the oracle with quant on and off.
- Closed forms: a delta kernel reproduces the shifted input (zero in the
  padding), a hand-computed 1-D example, linearity in w and x.
- Output extents equal torch's.
"""
import itertools

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def _bf16_exact(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16).to(torch.float32).numpy()


def _torch_conv64(x, w, bias, stride, pad_lo, pad_hi, dil):
    xt = torch.from_numpy(np.asarray(x, np.float64))
    # F.pad takes (w_lo, w_hi, h_lo, h_hi, d_lo, d_hi)
    xt = F.pad(xt, (pad_lo[2], pad_hi[2], pad_lo[1], pad_hi[1], pad_lo[0], pad_hi[0]))
    wt = torch.from_numpy(np.asarray(w, np.float64))
    bt = None if bias is None else torch.from_numpy(np.asarray(bias, np.float64))
    return F.conv3d(xt, wt, bt, stride=tuple(stride), padding=0, dilation=tuple(dil)).numpy()


CASES = [
    # x_shape, cout, kernel, stride, pad_lo, pad_hi, dil
    ((1, 3, 4, 6, 7), 5, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1)),
    ((2, 4, 5, 7, 6), 3, (3, 3, 3), (1, 2, 2), (1, 1, 1), (1, 1, 1), (1, 1, 1)),
    ((1, 2, 6, 9, 9), 4, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 2, 2)),
    ((1, 5, 3, 5, 5), 2, (1, 1, 1), (1, 1, 1), (0, 0, 0), (0, 0, 0), (1, 1, 1)),
    ((1, 3, 3, 6, 6), 4, (1, 3, 3), (1, 1, 1), (0, 1, 1), (0, 1, 1), (1, 1, 1)),
    ((1, 2, 6, 7, 8), 3, (5, 5, 5), (1, 1, 1), (2, 2, 2), (2, 2, 2), (1, 1, 1)),
    ((1, 3, 5, 8, 8), 2, (3, 3, 3), (2, 3, 1), (0, 1, 2), (1, 0, 0), (2, 1, 3)),
    ((1, 7, 3, 3, 3), 2, (3, 3, 3), (1, 1, 1), (0, 0, 0), (0, 0, 0), (1, 1, 1)),  # 1x1x1 output
]


@pytest.mark.parametrize("case", CASES)
def test_quant_off_matches_torch_conv3d_float64(case):
    xs, cout, k, s, plo, phi, d = case
    x = _bf16_exact(xs, 1)
    w = _bf16_exact((cout, xs[1]) + k, 2)
    b = np.random.default_rng(3).standard_normal(cout).astype(np.float32)
    got = oracle.conv3d(x, w, b, s, plo, phi, d, quant_act=False)
    ref = _torch_conv64(x, w, b, s, plo, phi, d)
    assert got.shape == ref.shape
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_operands_are_rounded_to_bf16():
    xs, cout, k = (1, 3, 4, 5, 6), 4, (3, 3, 3)
    g = torch.Generator().manual_seed(5)
    x = torch.randn(xs, generator=g).numpy()
    w = torch.randn((cout, 3) + k, generator=g).numpy()
    got = oracle.conv3d(x, w, None, (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1), quant_act=False)
    xb = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    wb = torch.from_numpy(w).to(torch.bfloat16).to(torch.float32).numpy()
    ref = _torch_conv64(xb, wb, None, (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    # and differs from the unrounded float64 conv
    raw = _torch_conv64(x, w, None, (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1))
    assert np.abs(got - raw).max() > 1e-4


def _im2col_numpy(x, k, s, plo, phi, d):
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


@pytest.mark.parametrize("quant", [False, True])
@pytest.mark.parametrize("case", CASES[:7])
def test_matches_explicit_im2col_bruteforce(case, quant):
    xs, cout, k, s, plo, phi, d = case
    g = torch.Generator().manual_seed(7)
    x = torch.randn(xs, generator=g).numpy()
    w = torch.randn((cout, xs[1]) + k, generator=g).numpy()
    b = torch.randn(cout, generator=g).numpy()
    amax = float(np.abs(x).max())
    A, (N, OD, OH, OW) = _im2col_numpy(x, k, s, plo, phi, d)
    Kdim = A.shape[1]
    if quant:
        Aq = np.empty_like(A)
        for r in range(A.shape[0]):
            for j in range(0, Kdim, 16):
                Aq[r, j:j + 16] = oracle.fq_block(A[r, j:j + 16], amax)
        A = Aq
    A = oracle.bf16_round(A).astype(np.float64)
    Wm = oracle.bf16_round(w.reshape(cout, -1)).astype(np.float64)
    ref = A @ Wm.T + b.astype(np.float64)[None, :]
    ref = ref.reshape(N, OD, OH, OW, cout).transpose(0, 4, 1, 2, 3)
    got = oracle.conv3d(x, w, b, s, plo, phi, d, quant_act=quant, act_amax=amax)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-11)


def test_quant_on_differs_from_quant_off():
    xs, k = (1, 4, 3, 6, 6), (3, 3, 3)
    x = _bf16_exact(xs, 8)
    w = _bf16_exact((3, 4) + k, 9)
    a = oracle.conv3d(x, w, None, (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1), quant_act=False)
    q = oracle.conv3d(x, w, None, (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1), quant_act=True,
                      act_amax=float(np.abs(x).max()))
    rel = np.abs(a - q).max() / np.abs(a).max()
    assert 1e-3 < rel < 0.5


@pytest.mark.parametrize("tap", [(0, 0, 0), (1, 1, 1), (2, 0, 1), (0, 2, 2)])
def test_delta_kernel_shifts_input(tap):
    xs = (1, 2, 4, 5, 6)
    x = _bf16_exact(xs, 10)
    w = np.zeros((2, 2, 3, 3, 3), np.float32)
    w[0, 1][tap] = 1.0     # output channel 0 reads input channel 1 at the tap
    w[1, 0][tap] = 1.0
    plo = (2, 1, 1)
    phi = (0, 1, 1)
    y = oracle.conv3d(x, w, None, (1, 1, 1), plo, phi, (1, 1, 1), quant_act=False)
    xp = np.pad(x, ((0, 0), (0, 0), (plo[0], phi[0]), (plo[1], phi[1]), (plo[2], phi[2])))
    D, H, W = xs[2:]
    kd, kh, kw = tap
    shifted = xp[:, :, kd:kd + D, kh:kh + H, kw:kw + W]
    assert np.array_equal(y[:, 0], shifted[:, 1])
    assert np.array_equal(y[:, 1], shifted[:, 0])


def test_hand_computed_1d():
    # x = [1, 2, 3] along W, w = [1, 1, 1], pad 1 -> [0+1+2, 1+2+3, 2+3+0]
    x = np.array([1, 2, 3], np.float32).reshape(1, 1, 1, 1, 3)
    w = np.ones((1, 1, 1, 1, 3), np.float32)
    y = oracle.conv3d(x, w, np.array([0.5], np.float32), (1, 1, 1), (0, 0, 1), (0, 0, 1), (1, 1, 1))
    assert np.array_equal(y.ravel(), np.array([3.5, 6.5, 5.5]))
    # stride 2 along W keeps outputs 0 and 2
    y2 = oracle.conv3d(x, w, None, (1, 1, 2), (0, 0, 1), (0, 0, 1), (1, 1, 1))
    assert np.array_equal(y2.ravel(), np.array([3.0, 5.0]))
    # dilation 2 with pad 2: taps at -2, 0, +2
    y3 = oracle.conv3d(x, w, None, (1, 1, 1), (0, 0, 2), (0, 0, 2), (1, 1, 2))
    assert np.array_equal(y3.ravel(), np.array([1 + 3, 2.0, 1 + 3]))


def test_linearity_in_w_and_x():
    xs, k = (1, 3, 3, 5, 5), (3, 3, 3)
    # small integers keep every value and sum exact in bf16 and float64
    rng = np.random.default_rng(11)
    x1 = rng.integers(-4, 5, xs).astype(np.float32)
    x2 = rng.integers(-4, 5, xs).astype(np.float32)
    w1 = rng.integers(-3, 4, (2, 3) + k).astype(np.float32)
    w2 = rng.integers(-3, 4, (2, 3) + k).astype(np.float32)
    args = ((1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1))
    c = lambda x, w: oracle.conv3d(x, w, None, *args)  # noqa: E731
    assert np.array_equal(c(x1, w1 + w2), c(x1, w1) + c(x1, w2))
    assert np.array_equal(c(x1 + x2, w1), c(x1, w1) + c(x2, w1))
    # with quant on, linearity in w still holds exactly (A does not depend on w)
    amax = float(np.abs(x1).max())
    cq = lambda w: oracle.conv3d(x1, w, None, *args, quant_act=True, act_amax=amax)  # noqa: E731
    np.testing.assert_allclose(cq(w1 + w2), cq(w1) + cq(w2), rtol=0, atol=1e-9)


def test_row_subset_matches_full():
    xs, k = (2, 3, 3, 5, 6), (3, 3, 3)
    g = torch.Generator().manual_seed(12)
    x = torch.randn(xs, generator=g).numpy()
    w = torch.randn((4, 3) + k, generator=g).numpy()
    amax = float(np.abs(x).max())
    full = oracle.conv3d(x, w, None, (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1), True, amax)
    N, Co, OD, OH, OW = full.shape
    flat = full.transpose(0, 2, 3, 4, 1).reshape(-1, Co)
    ms = np.array([0, 5, 17, flat.shape[0] - 1, 33])
    sub = oracle.conv3d(x, w, None, (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1), True, amax, m_list=ms)
    assert np.array_equal(sub, flat[ms])
    # thread count does not change any value
    one = oracle.conv3d(x, w, None, (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1), True, amax, nthreads=1)
    assert np.array_equal(one, full)


@pytest.mark.parametrize("case", CASES)
def test_out_dims_match_torch(case):
    xs, cout, k, s, plo, phi, d = case
    dims = oracle.out_dims(xs[2:], k, s, plo, phi, d)
    ref = _torch_conv64(np.zeros(xs, np.float32), np.zeros((cout, xs[1]) + k, np.float32), None, s, plo, phi, d)
    assert dims == ref.shape[2:]


def test_rejects_bad_arguments():
    x = np.zeros((1, 1, 3, 3, 3), np.float32)
    w = np.zeros((1, 1, 3, 3, 3), np.float32)
    with pytest.raises(ValueError):
        oracle.conv3d(x, w, None, (0, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1))
    with pytest.raises(ValueError):
        oracle.conv3d(x, w, None, (1, 1, 1), (-1, 1, 1), (1, 1, 1), (1, 1, 1))


# the fused quantiser's other formats: NVFP4 with the article's other block
# sizes (sec. 7.1) and MXFP4 (the CANN aclnnFlatQuantV2 page); a short last
# block of a row acts as zero-filled
FORMATS = [("nvfp4", 32, 0.0), ("nvfp4", 64, 0.0), ("nvfp4", 128, 0.0), ("nvfp4", 256, 0.0),
           ("mxfp4", 32, 0.0), ("mxfp4", 32, 6.0)]


@pytest.mark.parametrize("fmt", FORMATS, ids=[f"{f}{b}_{d:g}" for f, b, d in FORMATS])
@pytest.mark.parametrize("case", CASES[:5])
def test_block_formats_match_im2col_with_standalone_quantisers(case, fmt):
    """conv3d with an explicit format equals numpy im2col, each row quantised
    by the standalone (separately pinned) block quantiser in blocks of the
    format's size, and an fp64 matmul over BF16 operands."""
    qf, bs, dst = fmt
    xs, cout, k, s, plo, phi, d = case
    g = torch.Generator().manual_seed(17)
    x = (torch.randn(xs, generator=g) * 3).numpy()
    w = torch.randn((cout, xs[1]) + k, generator=g).numpy()
    amax = float(np.abs(x).max())
    A, (N, OD, OH, OW) = _im2col_numpy(x, k, s, plo, phi, d)
    Kdim = A.shape[1]
    Aq = np.empty_like(A, dtype=np.float32)
    for r in range(A.shape[0]):
        for j in range(0, Kdim, bs):
            blk = np.zeros(bs, np.float32)
            n = min(bs, Kdim - j)
            blk[:n] = A[r, j:j + n]
            q = (oracle.fp4_fake_quant_bs(blk, amax, bs) if qf == "nvfp4" else oracle.mxfp4_fake_quant(blk, dst)[0])
            Aq[r, j:j + n] = q[:n]
    Am = oracle.bf16_round(Aq).astype(np.float64)
    Wm = oracle.bf16_round(w.reshape(cout, -1)).astype(np.float64)
    ref = (Am @ Wm.T).reshape(N, OD, OH, OW, cout).transpose(0, 4, 1, 2, 3)
    got = oracle.conv3d(x, w, None, s, plo, phi, d, quant_act=True, act_amax=amax, quant_format=qf, block_size=bs,
                        dst_max=dst)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-11)
    # the block size matters: 16 and the format's size disagree somewhere
    # (when a row holds more than one block of 16)
    if qf == "nvfp4" and Kdim > 16:
        g16 = oracle.conv3d(x, w, None, s, plo, phi, d, quant_act=True, act_amax=amax)
        assert not np.array_equal(g16, got)


def test_block_format_arguments_are_checked():
    x = np.ones((1, 2, 3, 3, 3), np.float32)
    w = np.ones((2, 2, 3, 3, 3), np.float32)
    for kw in (dict(block_size=48), dict(quant_format="mxfp4", block_size=16), dict(quant_format="mxfp4", block_size=32,
                                                                                    dst_max=3.0)):
        with pytest.raises(ValueError):
            oracle.conv3d(x, w, None, (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1), quant_act=True, act_amax=1.0, **kw)

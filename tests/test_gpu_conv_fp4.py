"""GPU parity of the true-FP4 convolution (conv3d_fp4_pack_weights +
conv3d_implicit_gemm_fp4) against the oracle's exact-operand convolution.

- The packed weights are decoded here from the layout the header states
  (codes in the 32-byte-swizzled rows of each image, unsigned E4M3 scale
  bytes in the 512-byte atoms, g_w in the header) and must equal the oracle's
  exact NVFP4 operands of w value for value.
- One-hot weights with power-of-two global scales read the activation operand
  back exactly: the output equals the oracle bit for bit.
- Small shapes (ragged tiles, K not a multiple of 16 or 64, strides,
  dilations, asymmetric padding, two N-tiles, every dtype) are compared on the
  whole output; the full-size layers on sampled rows.  Tolerance as for the
  BF16 path: max|y - y_ref| <= 2e-3 max|y_ref| (plus half an ulp of the
  output dtype) and relative error <= 1e-2 where |y_ref| > 1e-2 max|y_ref|.
- act_amax settings that drive every block into the fallback give exactly
  the bias.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_conv3d_implicit_b200 import api, workloads
from _parity import assert_conv_close, to_np_f32

pytestmark = pytest.mark.gpu

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _e4m3_values():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _decode_packed(wq: api.Fp4Weights):
    """Exact operand values [Cout, K] (float64) from the packed buffer."""
    cout = wq.shape[0]
    K = int(np.prod(wq.shape[1:]))
    plan = api.plan_conv((1, wq.shape[1], 8, 8, 16), wq.shape, 1, tuple(k // 2 for k in wq.shape[2:] for _ in (0, 1)),
                         1, torch.bfloat16, kernel="fp4")
    sub_n, n_sub, n_ntiles = plan["sub_n"], plan["n_sub"], plan["n_ntiles"]
    ks = -(-K // 64)
    n_parts, n_atoms = n_ntiles * n_sub, (sub_n + 127) // 128
    img = sub_n * 32 + n_atoms * 512
    buf = wq.packed.cpu().numpy()
    assert buf.size == 256 + ks * n_parts * img
    g_w = float(buf[:4].view(np.float32)[0])
    e4m3 = _e4m3_values()
    co = np.arange(cout)[:, None]
    kb = np.arange((K + 15) // 16)[None, :]
    part, row = co // sub_n, co % sub_n
    s, bb = kb // 4, kb % 4
    base = 256 + (s * n_parts + part) * img
    code_off = base + row * 32 + ((((bb >> 1) ^ (row >> 2)) & 1) << 4) + (bb & 1) * 8   # [cout, nkb]
    sf_off = base + sub_n * 32 + (row // 128) * 512 + (row % 32) * 16 + ((row // 32) % 4) * 4 + bb
    s8 = e4m3[buf[sf_off]]
    byts = buf[code_off[..., None] + np.arange(8)]                       # [cout, nkb, 8]
    nib = np.stack([byts & 15, byts >> 4], axis=-1).reshape(cout, -1, 16)  # element 2i low nibble
    q = np.where(nib & 8, -1.0, 1.0) * E2M1[nib & 7]
    vals = (q * s8[..., None] * g_w).reshape(cout, -1)[:, :K]
    return vals, buf, g_w


def _exact_rows(w2d, amax):
    out = np.zeros(w2d.shape, np.float64)
    for r in range(w2d.shape[0]):
        for j in range(0, w2d.shape[1], 16):
            n = min(16, w2d.shape[1] - j)
            blk = np.zeros(16, np.float32)
            blk[:n] = w2d[r, j:j + n]
            out[r, j:j + n] = oracle.nvfp4_block_exact(blk, amax)[:n]
    return out


W_SHAPES = [(5, 3, 3, 3, 3), (96, 4, 3, 3, 3), (192, 7, 1, 3, 3), (300, 8, 3, 3, 3), (500, 2, 3, 3, 3),
            (33, 37, 1, 1, 1)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("mode", ["max", "max/50", "1e-6"])
@pytest.mark.parametrize("shape", W_SHAPES)
def test_packed_weights_decode_to_the_oracle_operands(cuda_ok, shape, mode, dtype):
    g = torch.Generator().manual_seed(sum(shape))
    w = (torch.randn(shape, generator=g) * 0.3).to(dtype)
    m = float(w.float().abs().max())
    amax = {"max": m, "max/50": m / 50, "1e-6": 1e-6}[mode]
    wq = api.conv3d_fp4_pack_weights(w.cuda(), torch.tensor([amax], dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    vals, buf, g_w = _decode_packed(wq)
    assert np.float32(g_w) == np.float32(amax) / np.float32(2688.0)
    ref = _exact_rows(w.float().numpy().reshape(shape[0], -1), amax)
    np.testing.assert_array_equal(vals, ref)
    if mode == "1e-6":
        assert not vals.any()


def _run_fp4(inp, stride, plo, phi, dil, w_amax=None, act_amax=None):
    x, w, b = inp["x"], inp["w"], inp["bias"]
    wa = api.act_amax(w) if w_amax is None else torch.tensor([w_amax], dtype=torch.float32, device=x.device)
    aa = inp["act_amax"] if act_amax is None else torch.tensor([act_amax], dtype=torch.float32, device=x.device)
    wq = api.conv3d_fp4_pack_weights(w, wa)
    pad6 = (plo[0], phi[0], plo[1], phi[1], plo[2], phi[2])
    y = api.conv3d_implicit_gemm_fp4(x, wq, b, stride=stride, padding=pad6, dilation=dil, act_amax=aa)
    assert api.check_device_error() == 0
    return y, float(wa.item()), float(aa.item())


def _ref_fp4(inp, stride, plo, phi, dil, w_amax, act_amax, m_list=None):
    x, w, b = inp["x"], inp["w"], inp["bias"]
    return oracle.conv3d_nvfp4(to_np_f32(x), to_np_f32(w), None if b is None else to_np_f32(b), stride, plo, phi, dil,
                               act_amax=act_amax, w_amax=w_amax, m_list=m_list)


# x_shape, cout, kernel, stride, pad_lo, pad_hi, dil (rows of W a multiple of
# 16 bytes in every dtype: W % 8 == 0)
SHAPES = [
    ((1, 16, 4, 16, 16), 16, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1)),   # tiny layer
    ((1, 5, 4, 9, 16), 24, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 1, 1)),     # K = 135: partial block
    ((1, 6, 6, 13, 24), 33, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 2, 2)),    # dilation
    ((2, 5, 5, 9, 32), 20, (3, 3, 3), (1, 2, 2), (1, 1, 1), (1, 1, 1), (1, 1, 1)),     # stride 2
    ((1, 3, 7, 9, 16), 8, (5, 5, 5), (1, 1, 1), (2, 2, 2), (2, 2, 2), (1, 1, 1)),      # 5x5x5, K = 375
    ((1, 8, 3, 6, 8), 500, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1)),     # two N tiles
    ((1, 20, 3, 21, 40), 200, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 1, 1)),  # K = 540, N = 208
    ((1, 8, 3, 8, 32), 192, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1)),    # several subtiles
    ((1, 32, 3, 8, 8), 300, (1, 1, 1), (1, 1, 1), (0, 0, 0), (0, 0, 0), (1, 1, 1)),    # pointwise
    ((1, 7, 4, 9, 16), 19, (1, 3, 3), (1, 1, 1), (0, 1, 1), (0, 1, 1), (1, 1, 1)),     # 1x3x3, K = 63
    ((1, 96, 3, 6, 64), 96, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 1, 1)),    # edge-layer channels
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("case", range(len(SHAPES)))
def test_fp4_conv_small_shapes(cuda_ok, case, dtype):
    xs, cout, k, s, plo, phi, d = SHAPES[case]
    inp = workloads.random_conv_inputs(300 + case, xs, cout, k, dtype=dtype, bias=(case % 2 == 0), device="cuda")
    y, wa, aa = _run_fp4(inp, s, plo, phi, d)
    ref = _ref_fp4(inp, s, plo, phi, d, wa, aa)
    assert_conv_close(to_np_f32(y), ref, f"fp4 case {case} {dtype}", dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
def test_fp4_identity_weight_readout_is_bit_exact(cuda_ok, dtype):
    # one-hot weights of value 2688 * 2^-12 with that value as w_amax: each
    # block's ratio is 448, the code 6 and the operand the weight itself, so
    # y[:, co] is the activation operand of column k(co) times that value;
    # with power-of-two global scales (act_amax = 2688 * 2^-8) every product
    # and the epilogue scaling are exact
    xs, k = (1, 5, 4, 9, 16), (3, 3, 3)
    K = 5 * 27
    g = torch.Generator().manual_seed(41)
    x = (torch.randn(xs, generator=g) * 3).to(dtype)
    wv = 2688.0 * 2.0 ** -12
    cols = list(range(K))
    w = torch.zeros((K,) + (5,) + k)
    w.view(K, K)[torch.arange(K), torch.tensor(cols)] = wv
    inp = {"x": x.cuda(), "w": w.to(dtype).cuda(), "bias": None,
           "act_amax": torch.tensor([2688.0 * 2.0 ** -8], dtype=torch.float32, device="cuda")}
    one, pad = (1, 1, 1), (1, 1, 1)
    y, wa, aa = _run_fp4(inp, one, pad, pad, one, w_amax=wv)
    ref = _ref_fp4(inp, one, pad, pad, one, wa, aa)
    got = to_np_f32(y).astype(np.float64)
    exp = torch.from_numpy(ref).to(dtype).to(torch.float64).numpy()
    assert np.array_equal(got, exp), f"max diff {np.abs(got - exp).max()}"
    assert np.count_nonzero(got) > got.size // 2


@pytest.mark.parametrize("amax", [0.0, 1e-6])
def test_fp4_fallback_blocks_give_the_bias(cuda_ok, amax):
    xs, cout, k = (1, 6, 3, 8, 16), 24, (3, 3, 3)
    inp = workloads.random_conv_inputs(77, xs, cout, k, dtype=torch.bfloat16, bias=True, device="cuda")
    one = (1, 1, 1)
    y, wa, aa = _run_fp4(inp, one, one, one, one, act_amax=amax)
    ref = _ref_fp4(inp, one, one, one, one, wa, aa)
    bias = to_np_f32(inp["bias"]).astype(np.float64)
    assert np.array_equal(ref, np.broadcast_to(bias[None, :, None, None, None], ref.shape))
    assert np.array_equal(to_np_f32(y).astype(np.float64), ref)


def test_fp4_clamped_blocks(cuda_ok):
    # act_amax a fiftieth of max|x|: ratios clamp to 448 and codes saturate
    xs, cout, k = (1, 8, 3, 9, 16), 40, (3, 3, 3)
    inp = workloads.random_conv_inputs(78, xs, cout, k, dtype=torch.bfloat16, bias=True, device="cuda")
    one = (1, 1, 1)
    m = float(inp["x"].float().abs().max())
    y, wa, aa = _run_fp4(inp, one, one, one, one, act_amax=m / 50)
    ref = _ref_fp4(inp, one, one, one, one, wa, aa)
    assert_conv_close(to_np_f32(y), ref, "fp4 clamped", torch.bfloat16)


def test_fp4_rejects_rows_the_tma_cannot_fetch(cuda_ok):
    inp = workloads.random_conv_inputs(79, (1, 4, 3, 8, 11), 8, (3, 3, 3), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(api.Q3DError) as e:
        _run_fp4(inp, (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1))
    assert e.value.status == 7


def _sample_rows(wl, rng, n_random):
    od, oh, ow = wl.out_spatial()
    M = wl.m_gemm
    picks = set(rng.integers(0, M, n_random).tolist())
    picks.update([0, M - 1])
    for n in range(wl.x_shape[0]):
        for d_ in (0, od - 1):
            for h in (0, oh // 2, oh - 1):
                for w_ in (0, 1, ow // 2, ow - 2, ow - 1):
                    picks.add(((n * od + d_) * oh + h) * ow + max(0, w_))
    return np.array(sorted(p for p in picks if 0 <= p < M), dtype=np.int64)


FULL = [n for n in workloads.WORKLOADS if n not in (workloads.SMALL, "wan_hi_192_bf16_noquant")]


@pytest.mark.parametrize("name", FULL)
def test_fp4_full_size_layers_sampled(cuda_ok, name):
    wl = workloads.WORKLOADS[name]
    inp = workloads.make_inputs(wl, device="cuda")
    y, wa, aa = _run_fp4(inp, wl.stride, wl.pad_lo, wl.pad_hi, wl.dil)
    ms = _sample_rows(wl, np.random.default_rng(13), 256)
    ref = _ref_fp4(inp, wl.stride, wl.pad_lo, wl.pad_hi, wl.dil, wa, aa, m_list=ms)
    Co = y.shape[1]
    yf = y.permute(0, 2, 3, 4, 1).reshape(-1, Co)
    got = to_np_f32(yf[torch.from_numpy(ms).cuda()])
    assert_conv_close(got, ref, f"fp4 {name}", wl.dtype)

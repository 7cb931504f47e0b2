"""GPU parity of conv3d_implicit_gemm_ex: the fused activation quantiser's
other formats (NVFP4 with the article's block sizes 32..256, sec. 7.1; MXFP4
from the CANN aclnnFlatQuantV2 page) against the CPU oracle.

The one-hot-weight readout reproduces the quantised im2col matrix A bit for
bit (one nonzero product per output), so every element of the quantiser is
checked exactly; full convolutions are checked with the convolution
acceptance rule."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from quantized_conv3d_implicit_b200 import api, workloads
from _parity import assert_conv_close, bits, to_np_f32

pytestmark = pytest.mark.gpu

DT = {torch.float32: "float32", torch.float16: "float16", torch.bfloat16: "bfloat16"}
FORMATS = [("nvfp4", 32, 0.0), ("nvfp4", 64, 0.0), ("nvfp4", 128, 0.0), ("nvfp4", 256, 0.0),
           ("mxfp4", 32, 0.0), ("mxfp4", 32, 6.0), ("mxfp4", 32, 12.0)]
FIDS = [f"{f}{b}_{d:g}" for f, b, d in FORMATS]


@pytest.mark.parametrize("dtype", list(DT))
@pytest.mark.parametrize("fmt", FORMATS, ids=FIDS)
def test_identity_weight_readout_other_formats(cuda_ok, fmt, dtype):
    qf, bs, dst = fmt
    # K = 11 * 27 = 297: several blocks of every size and a short last one
    xs, k = (1, 11, 4, 7, 12), (3, 3, 3)
    K = 11 * 27
    g = torch.Generator().manual_seed(21)
    x = (torch.randn(xs, generator=g) * 3)
    x[0, 2] *= 40  # blocks with very different maxima
    x = x.to(dtype)
    amax = x.float().abs().max().reshape(1)
    for start in range(0, K, 128):
        cols = list(range(start, min(K, start + 128)))
        w = torch.zeros((len(cols), K), dtype=torch.float32)
        w[torch.arange(len(cols)), torch.tensor(cols)] = 1.0
        w = w.reshape(len(cols), 11, 3, 3, 3).to(dtype)
        y = api.conv3d_implicit_gemm_ex(x.cuda(), w.cuda(), None, 1, (2, 0, 1, 1, 1, 1), 1, act_amax=amax.cuda(),
                                        quant_format=qf, block_size=bs, dst_type_max=dst)
        assert api.check_device_error() == 0
        ref = oracle.conv3d(x.float().numpy(), w.float().numpy(), None, (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 1, 1),
                            quant_act=True, act_amax=float(amax.item()), quant_format=qf, block_size=bs,
                            dst_max=dst)
        assert np.array_equal(bits(y), oracle.round_to_dtype_bits(ref.astype(np.float32), DT[dtype])), start


SHAPES = [
    ((1, 8, 3, 10, 12), 24, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 1, 1)),   # K = 216
    ((2, 5, 5, 9, 11), 20, (3, 3, 3), (1, 2, 2), (1, 1, 1), (1, 1, 1), (1, 1, 1)),    # stride, K = 135
    ((1, 6, 6, 13, 24), 33, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 2, 2)),   # dilation, K = 162
    ((1, 32, 3, 8, 8), 300, (1, 1, 1), (1, 1, 1), (0, 0, 0), (0, 0, 0), (1, 1, 1)),   # pointwise, 2 N tiles
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("fmt", FORMATS, ids=FIDS)
@pytest.mark.parametrize("case", range(len(SHAPES)))
def test_conv_other_formats_small_shapes(cuda_ok, case, fmt, dtype):
    qf, bs, dst = fmt
    xs, cout, k, s, plo, phi, d = SHAPES[case]
    inp = workloads.random_conv_inputs(500 + case, xs, cout, k, dtype=dtype, bias=True, device="cuda", scale=2.0)
    pad6 = (plo[0], phi[0], plo[1], phi[1], plo[2], phi[2])
    y = api.conv3d_implicit_gemm_ex(inp["x"], inp["w"], inp["bias"], s, pad6, d, act_amax=inp["act_amax"],
                                    quant_format=qf, block_size=bs, dst_type_max=dst)
    assert api.check_device_error() == 0
    ref = oracle.conv3d(to_np_f32(inp["x"]), to_np_f32(inp["w"]), to_np_f32(inp["bias"]), s, plo, phi, d,
                        quant_act=True, act_amax=float(inp["act_amax"].item()), quant_format=qf, block_size=bs,
                        dst_max=dst)
    assert_conv_close(to_np_f32(y), ref, f"case {case} {qf}{bs} {dtype}", dtype)


@pytest.mark.parametrize("quant", [False, True])
def test_ex_matches_regular_entry_for_nvfp4_16_and_none(cuda_ok, quant):
    xs, cout, k = (1, 16, 5, 12, 32), 48, (3, 3, 3)
    inp = workloads.random_conv_inputs(61, xs, cout, k, dtype=torch.bfloat16, device="cuda")
    pad6 = (2, 0, 1, 1, 1, 1)
    y = api.conv3d_implicit_gemm_ex(inp["x"], inp["w"], inp["bias"], 1, pad6, 1, act_amax=inp["act_amax"],
                                    quant_format="nvfp4" if quant else "none", block_size=16)
    r = api.conv3d_implicit_gemm(inp["x"], inp["w"], inp["bias"], 1, pad6, 1, act_amax=inp["act_amax"],
                                 quant_act=quant)
    assert api.check_device_error() == 0
    assert torch.equal(y, r)


def test_ex_mxfp4_needs_no_amax(cuda_ok):
    inp = workloads.random_conv_inputs(62, (1, 8, 3, 8, 16), 16, (3, 3, 3), dtype=torch.bfloat16, device="cuda")
    y = api.conv3d_implicit_gemm_ex(inp["x"], inp["w"], None, 1, 1, 1, act_amax=None, quant_format="mxfp4",
                                    block_size=32)
    ref = oracle.conv3d(to_np_f32(inp["x"]), to_np_f32(inp["w"]), None, (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1),
                        quant_act=True, quant_format="mxfp4", block_size=32)
    assert_conv_close(to_np_f32(y), ref, "mxfp4 without amax", torch.bfloat16)


# ---------------------------------------------------------------------------
# The tensor-memory kernel's 32- and 64-column formats (NVFP4 blocks of 32
# and 64, MXFP4): a thread's two 16-column blocks of a K slice form one
# group; for blocks of 64 (A in shared memory) lanes l and l + 16 hold the
# two halves of a row.  Rows of x are a multiple of 16 bytes here, so the
# kernel's tensor maps apply; every shape but the 96-channel one in FP32 has
# a plan with A in shared memory.
# ---------------------------------------------------------------------------

TMEM_FORMATS = [("nvfp4", 32, 0.0), ("nvfp4", 64, 0.0), ("mxfp4", 32, 0.0), ("mxfp4", 32, 6.0), ("mxfp4", 32, 12.0)]
TMEM_FIDS = [f"{f}{b}_{d:g}" for f, b, d in TMEM_FORMATS]


@pytest.fixture(params=["auto", "smem_a"])
def tmem_form(request, monkeypatch):
    """The launcher's choice of A placement, and A in shared memory forced."""
    if request.param == "auto":
        monkeypatch.delenv("Q3D_KERNEL", raising=False)
    else:
        monkeypatch.setenv("Q3D_KERNEL", request.param)
    return request.param


def _readout(x, amax, k, pad6, pad_lo, pad_hi, qf, bs, dst, wscale=1.0):
    """y = A_q[:, cols] * wscale column block by column block (one-hot
    weights), compared bit for bit with the oracle's quantised im2col."""
    dtype = x.dtype
    C = x.shape[1]
    K = C * k[0] * k[1] * k[2]
    for start in range(0, K, 128):
        cols = list(range(start, min(K, start + 128)))
        w = torch.zeros((len(cols), K), dtype=torch.float32)
        w[torch.arange(len(cols)), torch.tensor(cols)] = wscale
        w = w.reshape((len(cols), C) + k).to(dtype)
        assert api.plan_conv(tuple(x.shape), tuple(w.shape), 1, pad6, 1, dtype=dtype, kernel="tmem")["applicable"]
        y = api.conv3d_implicit_gemm_ex(x.cuda(), w.cuda(), None, 1, pad6, 1,
                                        act_amax=None if amax is None else amax.cuda(), quant_format=qf,
                                        block_size=bs, dst_type_max=dst)
        assert api.check_device_error() == 0
        ref = oracle.conv3d(x.float().numpy(), w.float().numpy(), None, (1, 1, 1), pad_lo, pad_hi, (1, 1, 1),
                            quant_act=True, act_amax=0.0 if amax is None else float(amax.item()), quant_format=qf,
                            block_size=bs, dst_max=dst)
        assert np.array_equal(bits(y), oracle.round_to_dtype_bits(ref.astype(np.float32), DT[dtype])), start


@pytest.mark.parametrize("dtype", list(DT))
@pytest.mark.parametrize("fmt", TMEM_FORMATS, ids=TMEM_FIDS)
def test_identity_readout_tensor_memory_kernel(cuda_ok, tmem_form, fmt, dtype):
    qf, bs, dst = fmt
    # K = 11 * 27 = 297: five K slices, the last with one full group and one
    # of 9 columns; channels straddle the halo slots
    xs, k = (1, 11, 4, 7, 16), (3, 3, 3)
    g = torch.Generator().manual_seed(31)
    x = torch.randn(xs, generator=g) * 3
    x[0, 2] *= 40
    x[0, 5, :, 2:5] = 0.0  # all-zero groups
    x = x.to(dtype)
    amax = x.float().abs().max().reshape(1)
    _readout(x, amax, k, (2, 0, 1, 1, 1, 1), (2, 1, 1), (0, 1, 1), qf, bs, dst)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("dst", [0.0, 6.0])
@pytest.mark.parametrize("end", ["small", "large"])
def test_mxfp4_readout_extreme_scales(cuda_ok, tmem_form, end, dst, dtype):
    # channels of very different magnitude (a group spans two channels):
    # scales 2^E at both ends of the range the inputs reach, quantised values
    # down into the subnormals; read out through weights of 2^100 or 2^-100
    # so that every product stays normal and finite
    xs, k = (1, 8, 3, 6, 16), (3, 3, 3)
    g = torch.Generator().manual_seed(37)
    x = torch.randn(xs, generator=g).double()
    exps = [-128, -127, -126, -125, -124, -122, -100, 0] if end == "small" else [0, 60, 100, 118, 120, 122, 123, 124]
    for c, e in enumerate(exps):
        x[0, c] *= 2.0 ** e
    x = x.to(dtype)
    _readout(x, None, k, (1, 1, 1, 1, 1, 1), (1, 1, 1), (1, 1, 1), "mxfp4", 32, dst,
             wscale=2.0 ** (100 if end == "small" else -100))


TMEM_SHAPES = [
    ((1, 11, 4, 7, 16), 41, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 1, 1)),    # K = 297, Cout % 16
    ((1, 6, 6, 13, 24), 33, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 2, 2)),    # W dilation 2
    ((1, 32, 3, 8, 16), 300, (1, 1, 1), (1, 1, 1), (0, 0, 0), (0, 0, 0), (1, 1, 1)),   # pointwise, 2 N tiles
    ((1, 3, 7, 9, 16), 8, (5, 5, 5), (1, 1, 1), (2, 2, 2), (2, 2, 2), (1, 1, 1)),      # 5x5x5, 2 subtiles
    ((1, 8, 3, 8, 32), 192, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1)),    # 2 subtiles, A in smem
    ((2, 5, 5, 9, 32), 20, (3, 3, 3), (1, 2, 2), (1, 1, 1), (1, 1, 1), (1, 1, 1)),     # stride 2
    ((1, 96, 3, 16, 64), 96, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 1, 1)),   # 4 subtiles (bf16)
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("fmt", TMEM_FORMATS, ids=TMEM_FIDS)
@pytest.mark.parametrize("case", range(len(TMEM_SHAPES)))
def test_conv_tensor_memory_kernel_formats(cuda_ok, tmem_form, case, fmt, dtype):
    qf, bs, dst = fmt
    xs, cout, k, s, plo, phi, d = TMEM_SHAPES[case]
    inp = workloads.random_conv_inputs(700 + case, xs, cout, k, dtype=dtype, bias=True, device="cuda", scale=2.0)
    pad6 = (plo[0], phi[0], plo[1], phi[1], plo[2], phi[2])
    assert api.plan_conv(xs, (cout, xs[1]) + k, s, pad6, d, dtype=dtype, kernel="tmem")["applicable"]
    y = api.conv3d_implicit_gemm_ex(inp["x"], inp["w"], inp["bias"], s, pad6, d, act_amax=inp["act_amax"],
                                    quant_format=qf, block_size=bs, dst_type_max=dst)
    assert api.check_device_error() == 0
    ref = oracle.conv3d(to_np_f32(inp["x"]), to_np_f32(inp["w"]), to_np_f32(inp["bias"]), s, plo, phi, d,
                        quant_act=True, act_amax=float(inp["act_amax"].item()), quant_format=qf, block_size=bs,
                        dst_max=dst)
    assert_conv_close(to_np_f32(y), ref, f"case {case} {qf}{bs} {dtype}", dtype)


FULL_FORMAT_LAYERS = ["wan_mid_384_bf16", "edge_full_96_bf16", "down_s122_128to256_fp16"]


@pytest.mark.parametrize("fmt", TMEM_FORMATS[:3], ids=TMEM_FIDS[:3])
@pytest.mark.parametrize("name", FULL_FORMAT_LAYERS)
def test_full_size_layers_other_formats_sampled(cuda_ok, name, fmt):
    """The full-size layers (as the bench times them) with NVFP4 blocks of 32
    and 64 and MXFP4: seeded output rows, every channel, against the oracle
    (the rows at the padding faces and the first and last rows included)."""
    import test_gpu_conv as tg
    qf, bs, dst = fmt
    wl = workloads.WORKLOADS[name]
    inp = workloads.make_inputs(wl, device="cuda")
    pad6 = (wl.pad_lo[0], wl.pad_hi[0], wl.pad_lo[1], wl.pad_hi[1], wl.pad_lo[2], wl.pad_hi[2])
    y = api.conv3d_implicit_gemm_ex(inp["x"], inp["w"], inp["bias"], wl.stride, pad6, wl.dil,
                                    act_amax=inp["act_amax"], quant_format=qf, block_size=bs, dst_type_max=dst)
    assert api.check_device_error() == 0
    ms = tg._sample_rows(wl, np.random.default_rng(17), 256)
    ref = oracle.conv3d(to_np_f32(inp["x"]), to_np_f32(inp["w"]),
                        None if inp["bias"] is None else to_np_f32(inp["bias"]), wl.stride, wl.pad_lo, wl.pad_hi,
                        wl.dil, quant_act=True, act_amax=float(inp["act_amax"].item()), m_list=ms,
                        quant_format=qf, block_size=bs, dst_max=dst)
    Co = y.shape[1]
    got = to_np_f32(y.permute(0, 2, 3, 4, 1).reshape(-1, Co)[torch.from_numpy(ms).cuda()])
    assert_conv_close(got, ref, f"{name} {qf}{bs}", wl.dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("bs", [32, 64])
@pytest.mark.parametrize("mode", ["zero", "max/50", "2688", "1e-6"])
def test_group_readout_amax_edge_cases(cuda_ok, tmem_form, mode, bs, dtype):
    """NVFP4 blocks of 32 and 64 through the group path with the global
    amax at its edges: 0 and 1e-6 (every block takes the 1e-5 fallback),
    max/50 (block maxima above amax: the ratio clamps at 448 and E2M1
    saturates) and 2688 (g = 1): bit-exact against the oracle."""
    xs, k = (1, 11, 4, 7, 16), (3, 3, 3)
    g = torch.Generator().manual_seed(43)
    x = (torch.randn(xs, generator=g) * 3).to(dtype)
    m = float(x.float().abs().max())
    amax = torch.tensor([{"zero": 0.0, "max/50": m / 50.0, "2688": 2688.0, "1e-6": 1e-6}[mode]], dtype=torch.float32)
    _readout(x, amax, k, (2, 0, 1, 1, 1, 1), (2, 1, 1), (0, 1, 1), "nvfp4", bs, 0.0)

"""GPU parity of the implicit-GEMM Conv3D against the CPU oracle.

Small shapes are compared element by element on the whole output; the
full-size layer configurations are compared on a seeded sample of output
rows (every Cout) plus the first and last rows and the rows at the padding
faces.  Tolerance: max|y - y_ref| <= 2e-3 max|y_ref| and per-element
relative error <= 1e-2 where |y_ref| > 1e-2 max|y_ref|.  The identity-weight
readout checks the fused quantiser and the im2col addressing bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_conv3d_implicit_b200 import api, workloads
from _parity import assert_conv_close, bits, to_np_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(params=["auto", "smem_a", "fast", "basic"])
def kernel(request, monkeypatch):
    """Run a test with the library's default kernel choice (the tensor-memory
    kernel where it applies), with the tensor-memory kernel's shared-memory A
    form forced where it applies, with the shared-memory specialised kernel
    forced, and with the general-purpose kernel forced: all must meet the
    same bar."""
    if request.param == "auto":
        monkeypatch.delenv("Q3D_KERNEL", raising=False)
    else:
        monkeypatch.setenv("Q3D_KERNEL", request.param)
    return request.param


def _run(inp, stride, plo, phi, dil, quant):
    x, w, b, amax = inp["x"], inp["w"], inp["bias"], inp["act_amax"]
    pad6 = (plo[0], phi[0], plo[1], phi[1], plo[2], phi[2])
    y = api.conv3d_implicit_gemm(x, w, b, stride=stride, padding=pad6, dilation=dil,
                                 act_amax=amax if quant else None, quant_act=quant)
    assert api.check_device_error() == 0
    return y


def _ref(inp, stride, plo, phi, dil, quant, m_list=None):
    x, w, b, amax = inp["x"], inp["w"], inp["bias"], inp["act_amax"]
    return oracle.conv3d(to_np_f32(x), to_np_f32(w), None if b is None else to_np_f32(b), stride, plo, phi, dil,
                         quant_act=quant, act_amax=float(amax.item()), m_list=m_list)


# x_shape, cout, kernel, stride, pad_lo, pad_hi, dil
SHAPES = [
    ((1, 16, 4, 16, 16), 16, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1)),   # tiny layer
    ((1, 8, 3, 10, 12), 24, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 1, 1)),    # causal pad, K=216 (tail)
    ((2, 5, 5, 9, 11), 20, (3, 3, 3), (1, 2, 2), (1, 1, 1), (1, 1, 1), (1, 1, 1)),     # stride, K=135, Cout%16
    ((1, 6, 6, 13, 14), 33, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 2, 2)),    # dilation
    ((1, 32, 3, 8, 8), 300, (1, 1, 1), (1, 1, 1), (0, 0, 0), (0, 0, 0), (1, 1, 1)),    # pointwise, 2 N tiles
    ((1, 7, 4, 9, 9), 19, (1, 3, 3), (1, 1, 1), (0, 1, 1), (0, 1, 1), (1, 1, 1)),      # 1x3x3, K=63
    ((1, 3, 7, 9, 10), 8, (5, 5, 5), (1, 1, 1), (2, 2, 2), (2, 2, 2), (1, 1, 1)),      # 5x5x5, K=375
    ((1, 4, 5, 8, 8), 16, (3, 3, 3), (2, 3, 1), (0, 1, 2), (1, 0, 0), (2, 1, 3)),      # mixed everything
    ((1, 7, 3, 3, 3), 5, (3, 3, 3), (1, 1, 1), (0, 0, 0), (0, 0, 0), (1, 1, 1)),       # 1x1x1 output, K=189
    ((3, 16, 2, 5, 7), 40, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1)),     # batch 3, M=210
    # rows of x a multiple of 16 bytes (TMA-fed kernels), with ragged tiles
    ((1, 5, 4, 9, 16), 24, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 1, 1)),     # K=135: partial block
    ((1, 6, 6, 13, 24), 33, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 2, 2)),    # dilation
    ((2, 5, 5, 9, 32), 20, (3, 3, 3), (1, 2, 2), (1, 1, 1), (1, 1, 1), (1, 1, 1)),     # stride 2
    ((1, 3, 7, 9, 16), 8, (5, 5, 5), (1, 1, 1), (2, 2, 2), (2, 2, 2), (1, 1, 1)),      # 5x5x5, K=375
    ((1, 8, 3, 6, 8), 500, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1)),     # two N tiles
    ((1, 20, 3, 21, 40), 200, (3, 3, 3), (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 1, 1)),  # K=540, N=208
    ((1, 8, 3, 8, 32), 192, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1)),     # 2 subtiles, 2 A stages
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("quant", [False, True])
@pytest.mark.parametrize("case", range(len(SHAPES)))
def test_conv_small_shapes(cuda_ok, kernel, case, quant, dtype):
    xs, cout, k, s, plo, phi, d = SHAPES[case]
    inp = workloads.random_conv_inputs(100 + case, xs, cout, k, dtype=dtype, bias=(case % 2 == 0), device="cuda")
    y = _run(inp, s, plo, phi, d, quant)
    ref = _ref(inp, s, plo, phi, d, quant)
    assert_conv_close(to_np_f32(y), ref, f"case {case} quant={quant} {dtype}", dtype)


# act_amax settings that reach every branch of the fused quantiser's scale
# step (article sec. 6.2): the tensor's own max|x| (the normal case); 0 (g = 0,
# so the ratio is 0/0 or inf, clamped to 448, and the scale 0 falls back to
# 1.0); a fiftieth of max|x| (blocks whose maximum exceeds act_amax: the ratio
# is clamped to 448 and the E2M1 codes saturate at 6); 2688 = 6 * 448 (g = 1);
# and 1e-6 (every block scale is below 1e-5 and falls back to 1.0).
AMAX_MODES = ("max", "zero", "max/50", "2688", "1e-6")


def _amax_value(mode, x):
    m = float(x.float().abs().max())
    return {"max": m, "zero": 0.0, "max/50": m / 50.0, "2688": 2688.0, "1e-6": 1e-6}[mode]


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("mode", ("noquant",) + AMAX_MODES)
@pytest.mark.parametrize("width", [11, 16])
def test_identity_weight_readout_is_bit_exact(cuda_ok, kernel, mode, dtype, width):
    # one-hot weights: y[:, co] = A[:, k(co)], a single nonzero product per
    # output, so the FP32 accumulator holds the BF16 operand exactly and the
    # whole im2col row (quantised or not) is reproduced bit for bit; W = 16
    # reaches the TMA-fed kernels, W = 11 the general one
    quant = mode != "noquant"
    xs, k = (1, 5, 4, 9, width), (3, 3, 3)
    K = 5 * 27
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(xs, generator=g) * 3).to(dtype)
    amax = torch.tensor([_amax_value(mode if quant else "max", x)], dtype=torch.float32)
    for start in range(0, K, 128):
        cols = list(range(start, min(K, start + 128)))
        w = torch.zeros((len(cols), K), dtype=torch.float32)
        w[torch.arange(len(cols)), torch.tensor(cols)] = 1.0
        w = w.reshape(len(cols), 5, 3, 3, 3).to(dtype)
        inp = dict(x=x.cuda(), w=w.cuda(), bias=None, act_amax=amax.cuda())
        y = _run(inp, (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 1, 1), quant)
        ref = oracle.conv3d(x.float().numpy(), w.float().numpy(), None, (1, 1, 1), (2, 1, 1), (0, 1, 1), (1, 1, 1),
                            quant_act=quant, act_amax=float(amax.item()))
        ref_bits = oracle.round_to_dtype_bits(ref.astype(np.float32), {torch.float32: "float32",
                                                                        torch.float16: "float16",
                                                                        torch.bfloat16: "bfloat16"}[dtype])
        assert np.array_equal(bits(y), ref_bits), start


# shapes of SHAPES that reach the TMA-fed kernels' distinct plans: a partial
# last block, dilation, stride 2, 5x5x5, two N tiles, two subtiles
EDGE_SHAPES = (10, 11, 12, 13, 14, 16)


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("mode", ("zero", "max/50", "2688", "1e-6"))
@pytest.mark.parametrize("case", EDGE_SHAPES)
def test_conv_small_shapes_amax_edge_cases(cuda_ok, kernel, case, mode, dtype):
    xs, cout, k, s, plo, phi, d = SHAPES[case]
    inp = workloads.random_conv_inputs(400 + case, xs, cout, k, dtype=dtype, bias=True, device="cuda", scale=2.0)
    inp["act_amax"] = torch.tensor([_amax_value(mode, inp["x"])], dtype=torch.float32, device="cuda")
    y = _run(inp, s, plo, phi, d, True)
    ref = _ref(inp, s, plo, phi, d, True)
    assert_conv_close(to_np_f32(y), ref, f"case {case} act_amax {mode} {dtype}", dtype)


def test_determinism(cuda_ok, kernel):
    inp = workloads.random_conv_inputs(5, (1, 24, 4, 20, 24), 48, (3, 3, 3), dtype=torch.bfloat16, device="cuda")
    y1 = _run(inp, (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1), True)
    y2 = _run(inp, (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1), True)
    assert torch.equal(y1, y2)


def test_symmetric_entry_point_and_noop(cuda_ok):
    inp = workloads.random_conv_inputs(6, (1, 4, 3, 6, 6), 8, (3, 3, 3), dtype=torch.bfloat16, device="cuda")
    y = api.conv3d_implicit_gemm(inp["x"], inp["w"], inp["bias"], stride=1, padding=1, dilation=1)
    ref = _ref(inp, (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1), False)
    assert_conv_close(to_np_f32(y), ref, "symmetric", torch.bfloat16)
    e = api.conv3d_implicit_gemm(inp["x"][:0], inp["w"], padding=1)
    assert e.shape[0] == 0


@pytest.mark.parametrize("quant", [False, True])
def test_symmetric_c_entry_point_through_ctypes(cuda_ok, quant):
    """conv3d_implicit_gemm with its symmetric pad[3], called straight
    through the C ABI (no binding logic in between), against the oracle."""
    import ctypes
    lib = api.load_library()
    xs, cout, k = (1, 12, 5, 11, 24), 40, (3, 3, 3)
    inp = workloads.random_conv_inputs(77, xs, cout, k, dtype=torch.bfloat16, device="cuda")
    stride, pad, dil = (1, 2, 1), (1, 2, 1), (1, 1, 2)
    oshape = api.out_shape(xs, (cout, xs[1]) + k, stride, pad, dil)
    y = torch.full(oshape, float("nan"), dtype=torch.bfloat16, device="cuda")
    a3 = lambda v: (ctypes.c_int32 * 3)(*v)  # noqa: E731
    tx, tw, tb, ty = api._tensor(inp["x"]), api._tensor(inp["w"]), api._tensor(inp["bias"]), api._tensor(y)
    st = lib.conv3d_implicit_gemm(ctypes.byref(tx), ctypes.byref(tw), ctypes.byref(tb),
                                  inp["act_amax"].data_ptr() if quant else None, a3(stride), a3(pad), a3(dil),
                                  int(quant), ctypes.byref(ty), None)
    assert st == 0, lib.q3d_last_error()
    torch.cuda.synchronize()
    assert api.check_device_error() == 0
    ref = _ref(inp, stride, pad, pad, dil, quant)
    assert_conv_close(to_np_f32(y), ref, f"symmetric C entry quant={quant}", torch.bfloat16)


def _sample_rows(wl, rng, n_random):
    od, oh, ow = wl.out_spatial()
    M = wl.m_gemm
    picks = set(rng.integers(0, M, n_random).tolist())
    picks.update([0, M - 1])
    # rows at the faces of the output volume (padding taps)
    for n in range(wl.x_shape[0]):
        for d in (0, od - 1):
            for h in (0, oh // 2, oh - 1):
                for w_ in (0, 1, ow // 2, ow - 2, ow - 1):
                    picks.add(((n * od + d) * oh + h) * ow + max(0, w_))
    return np.array(sorted(p for p in picks if 0 <= p < M), dtype=np.int64)


@pytest.mark.parametrize("name", [n for n in workloads.WORKLOADS if n != workloads.SMALL])
def test_full_size_layers_sampled(cuda_ok, name):
    wl = workloads.WORKLOADS[name]
    inp = workloads.make_inputs(wl, device="cuda")
    y = _run(inp, wl.stride, wl.pad_lo, wl.pad_hi, wl.dil, wl.quant_act)
    rng = np.random.default_rng(11)
    ms = _sample_rows(wl, rng, 384)
    ref = _ref(inp, wl.stride, wl.pad_lo, wl.pad_hi, wl.dil, wl.quant_act, m_list=ms)
    # gather the same rows from the GPU output [N, Cout, OD, OH, OW]
    N, Co = y.shape[0], y.shape[1]
    yf = y.permute(0, 2, 3, 4, 1).reshape(-1, Co)
    got = to_np_f32(yf[torch.from_numpy(ms).cuda()])
    assert_conv_close(got, ref, name, wl.dtype)


def test_small_workload_full_output(cuda_ok):
    wl = workloads.WORKLOADS[workloads.SMALL]
    inp = workloads.make_inputs(wl, device="cuda")
    y = _run(inp, wl.stride, wl.pad_lo, wl.pad_hi, wl.dil, wl.quant_act)
    ref = _ref(inp, wl.stride, wl.pad_lo, wl.pad_hi, wl.dil, wl.quant_act)
    assert_conv_close(to_np_f32(y), ref, wl.name, wl.dtype)


@pytest.mark.parametrize("quant", [False, True])
def test_single_slice_tiles_many_per_cta(cuda_ok, quant):
    """K = 64 (one K slice per tile, so one transform group has nothing to
    build) and about seven tiles of four halo slots per CTA against an
    11-slot ring: the idle group hands its slots back only as they fill, so
    it cannot lap the ring."""
    xs, cout, k = (1, 64, 32, 64, 256), 32, (1, 1, 1)
    plan = api.plan_conv(xs, (cout, 64) + k, 1, 0, 1, torch.bfloat16, kernel="tmem")
    assert plan["applicable"] and plan["ks"] == 1
    tiles = xs[0] * xs[2] * plan["n_ohb"] * plan["n_owb"] * plan["n_ntiles"]  # 1x1x1, no padding: OD = D
    tiles_per_cta = -(-tiles // 148)
    assert tiles_per_cta * plan["q_slots"] > 2 * plan["ring"]
    inp = workloads.random_conv_inputs(32, xs, cout, k, dtype=torch.bfloat16, device="cuda")
    one, zero = (1, 1, 1), (0, 0, 0)
    y = _run(inp, one, zero, zero, one, quant)
    ref = _ref(inp, one, zero, zero, one, quant)
    assert_conv_close(to_np_f32(y), ref, f"single-slice tiles quant={quant}", torch.bfloat16)

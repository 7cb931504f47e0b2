"""The C ABI: the library loads without a GPU, exports every entry point the
header declares, and validates arguments on the host (before any CUDA call),
so these run on a CPU-only machine with placeholder device pointers that are
never dereferenced."""
import ctypes
import os
import re

import pytest
import torch

from quantized_conv3d_implicit_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("q3d.h", "q3d_testing.h")]


@pytest.fixture(scope="module")
def lib():
    build.build()
    return api.load_library()


def _declared():
    src = "".join(open(h).read() for h in HEADERS)
    return sorted(set(re.findall(r"Q3D_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


def test_header_declares_expected_entry_points():
    assert _declared() == sorted(api.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    assert lib.q3d_version() == 100


FAKE = 0x10000


def T(shape, dtype=2, data=FAKE):
    t = api.Q3DTensor()
    t.data = data
    t.dtype = dtype
    t.ndim = len(shape)
    for i, d in enumerate(shape):
        t.shape[i] = d
    return t


def conv(lib, x, w, out, bias=None, amax=None, stride=(1, 1, 1), plo=(1, 1, 1), phi=(1, 1, 1), dil=(1, 1, 1),
         quant=0):
    arr = lambda v: (ctypes.c_int32 * 3)(*v)  # noqa: E731
    r = lambda t: ctypes.byref(t) if t is not None else None  # noqa: E731
    return lib.conv3d_implicit_gemm_pad2(r(x), r(w), r(bias), amax, arr(stride), arr(plo), arr(phi), arr(dil),
                                         quant, r(out), None)


GOOD = dict(x=((1, 4, 3, 8, 8),), w=((5, 4, 3, 3, 3),), out=((1, 5, 3, 8, 8),))


def good(dtype=2):
    return (T((1, 4, 3, 8, 8), dtype, FAKE), T((5, 4, 3, 3, 3), dtype, FAKE * 16),
            T((1, 5, 3, 8, 8), dtype, FAKE * 256))


def test_null_pointers(lib):
    x, w, out = good()
    assert conv(lib, None, w, out) == 1
    assert conv(lib, x, None, out) == 1
    assert conv(lib, x, w, None) == 1
    assert conv(lib, x, w, out, quant=1) == 1           # quant without act_amax
    assert b"act_amax" in lib.q3d_last_error()
    assert conv(lib, T((1, 4, 3, 8, 8), 2, 0), w, out) == 1


def test_invalid_shapes(lib):
    x, w, out = good()
    assert conv(lib, T((4, 3, 8, 8)), w, out) == 2                    # rank
    assert conv(lib, x, T((5, 3, 3, 3, 3), 2, FAKE * 16), out) == 2   # groups != 1
    assert b"groups" in lib.q3d_last_error()
    assert conv(lib, x, w, T((1, 5, 3, 8, 9), 2, FAKE * 256)) == 2    # wrong out shape
    assert conv(lib, x, w, out, stride=(0, 1, 1)) == 2
    assert conv(lib, x, w, out, dil=(1, 0, 1)) == 2
    assert conv(lib, x, w, out, plo=(-1, 1, 1)) == 2
    big = T((5, 4, 9, 3, 3), 2, FAKE * 16)                            # kernel larger than padded input
    assert conv(lib, x, big, out) == 2
    assert conv(lib, x, w, out, bias=T((4,), 2, FAKE * 4096)) == 2    # bias length != Cout
    alias = T((1, 5, 3, 8, 8), 2, FAKE)                               # out overlaps x
    assert conv(lib, x, w, alias) == 2


def test_dtype_rules(lib):
    x, w, out = good()
    assert conv(lib, x, T((5, 4, 3, 3, 3), 1, FAKE * 16), out) == 3
    assert conv(lib, x, w, T((1, 5, 3, 8, 8), 0, FAKE * 256)) == 3
    assert conv(lib, T((1, 4, 3, 8, 8), 7), w, out) == 3


def test_empty_batch_is_noop(lib):
    x = T((0, 4, 3, 8, 8))
    w = T((5, 4, 3, 3, 3), 2, FAKE * 16)
    out = T((0, 5, 3, 8, 8), 2, FAKE * 256)
    assert conv(lib, x, w, out) == 0


def test_fake_quant_validation(lib):
    r = ctypes.byref
    x = T((3, 7), 2, FAKE)
    out = T((3, 7), 2, FAKE * 256)
    assert lib.fp4_fake_quant(r(x), FAKE * 4096, r(out), None) == 2          # 21 % 16 != 0
    assert lib.fp4_fake_quant(r(T((2, 16))), None, r(T((2, 16), 2, FAKE * 256)), None) == 1
    assert lib.fp4_fake_quant(r(T((2, 16))), FAKE * 4096, r(T((2, 16), 1, FAKE * 256)), None) == 3
    assert lib.fp4_fake_quant(r(T((2, 16))), FAKE * 4096, r(T((16, 2), 2, FAKE * 256)), None) == 2
    assert lib.fp4_fake_quant(r(T((0, 16))), FAKE * 4096, r(T((0, 16), 2, FAKE * 256)), None) == 0


def test_fake_quant_block_size_validation(lib):
    r = ctypes.byref
    x, out = T((4, 64), 2, FAKE), T((4, 64), 2, FAKE * 256)
    for bs in (0, 8, 48, 512, -16):
        assert lib.fp4_fake_quant_bs(r(x), FAKE * 4096, bs, r(out), None) == 2, bs
        assert b"block_size" in lib.q3d_last_error()
    # numel 256: a multiple of 16..256; numel 96 is not a multiple of 64
    assert lib.fp4_fake_quant_bs(r(T((6, 16))), FAKE * 4096, 64, r(T((6, 16), 2, FAKE * 256)), None) == 2
    assert lib.fp4_fake_quant_bs(r(T((0, 64))), FAKE * 4096, 256, r(T((0, 64), 2, FAKE * 256)), None) == 0
    assert lib.fp4_fake_quant_bs(r(x), None, 32, r(out), None) == 1


def conv_sym(lib, x, w, out, pad=(1, 1, 1), amax=None, quant=0):
    arr = lambda v: (ctypes.c_int32 * 3)(*v) if v is not None else None  # noqa: E731
    r = lambda t: ctypes.byref(t) if t is not None else None  # noqa: E731
    return lib.conv3d_implicit_gemm(r(x), r(w), None, amax, arr((1, 1, 1)), arr(pad), arr((1, 1, 1)), quant, r(out),
                                    None)


def test_symmetric_entry_point_validation(lib):
    x, w, out = good()
    assert conv_sym(lib, x, w, out, pad=None) == 1
    assert b"pad" in lib.q3d_last_error()
    assert conv_sym(lib, x, w, out, pad=(-1, 1, 1)) == 2
    assert conv_sym(lib, x, w, T((1, 5, 3, 8, 9), 2, FAKE * 256)) == 2     # out shape for pad 1
    assert conv_sym(lib, x, w, out, quant=1) == 1                           # quant without act_amax
    assert conv_sym(lib, T((0, 4, 3, 8, 8)), w, T((0, 5, 3, 8, 8), 2, FAKE * 256)) == 0


def test_conv_out_shape(lib):
    a3 = lambda t: (ctypes.c_int32 * 3)(*t)  # noqa: E731
    a5 = lambda t: (ctypes.c_int64 * 5)(*t)  # noqa: E731
    o = (ctypes.c_int64 * 5)()
    # causal temporal padding, stride (1, 2, 2), dilation (1, 2, 2)
    st = lib.q3d_conv_out_shape(a5((2, 8, 17, 64, 63)), a5((24, 8, 3, 3, 3)), a3((1, 2, 2)), a3((2, 1, 1)),
                                a3((0, 1, 1)), a3((1, 2, 2)), o)
    assert st == 0
    # floor((I + lo + hi - dil*(k-1) - 1) / s) + 1 along each dim
    assert tuple(o) == (2, 24, 17, 31, 31)
    assert api.out_shape((2, 8, 17, 64, 63), (24, 8, 3, 3, 3), (1, 2, 2), (2, 0, 1, 1, 1, 1), (1, 2, 2)) == \
        (2, 24, 17, 31, 31)
    assert lib.q3d_conv_out_shape(a5((1, 8, 2, 2, 2)), a5((4, 8, 5, 1, 1)), a3((1, 1, 1)), a3((0, 0, 0)),
                                  a3((0, 0, 0)), a3((1, 1, 1)), o) == 2        # empty output
    assert lib.q3d_conv_out_shape(a5((1, 8, 4, 4, 4)), a5((4, 7, 1, 1, 1)), a3((1, 1, 1)), a3((0, 0, 0)),
                                  a3((0, 0, 0)), a3((1, 1, 1)), o) == 2        # groups != 1
    assert lib.q3d_conv_out_shape(None, a5((4, 8, 1, 1, 1)), a3((1, 1, 1)), a3((0, 0, 0)), a3((0, 0, 0)),
                                  a3((1, 1, 1)), o) == 1
    with pytest.raises(api.Q3DError):
        api.out_shape((1, 8, 4, 4, 4), (4, 8, 3, 3, 3), 0, 0, 1)


def test_noalloc_binding_rejects_host_act_amax(lib):
    x = torch.zeros((1, 4, 3, 8, 8), dtype=torch.bfloat16)
    w = torch.zeros((5, 4, 3, 3, 3), dtype=torch.bfloat16)
    y = torch.zeros((1, 5, 3, 8, 8), dtype=torch.bfloat16)
    bad = torch.zeros(1, dtype=torch.float32, device="meta")   # not on x's device
    with pytest.raises(ValueError):
        api.conv3d_implicit_gemm_noalloc(x, w, y, None, 1, 1, 1, act_amax=bad, quant_act=True)
    with pytest.raises(ValueError):
        api.conv3d_implicit_gemm_noalloc(x, w, y, None, 1, 1, 1, act_amax=None, quant_act=True)
    with pytest.raises(ValueError):
        api.conv3d_implicit_gemm(x, w, None, 1, 1, 1, act_amax=torch.zeros(2), quant_act=True, out=y)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_gpu_reports_cuda_error(lib):
    x, w, out = good()
    assert conv(lib, x, w, out) in (4, 5)
    assert lib.q3d_last_error() != b""


def test_python_binding_errors_without_library(tmp_path):
    with pytest.raises(RuntimeError):
        api.load_library(str(tmp_path / "missing.so"))


def test_mxfp4_validation(lib):
    r = ctypes.byref
    x, out = T((4, 64), 2, FAKE), T((4, 64), 2, FAKE * 256)
    assert lib.mxfp4_quantize(None, 0.0, r(out), None, None, None) == 1
    assert lib.mxfp4_quantize(r(x), 0.0, None, None, None, None) == 1          # nothing to write
    for bad in (1.0, 5.5, 12.5, -6.0):
        assert lib.mxfp4_quantize(r(x), bad, r(out), None, None, None) == 2
    assert lib.mxfp4_quantize(r(T((3, 16))), 0.0, r(T((3, 16), 2, FAKE * 256)), None, None, None) == 2   # 48 % 32
    assert lib.mxfp4_quantize(r(x), 0.0, r(T((4, 64), 1, FAKE * 256)), None, None, None) == 3
    assert lib.mxfp4_quantize(r(x), 0.0, None, FAKE + 8, None, None) == 2        # scales inside x
    assert lib.mxfp4_quantize(r(x), 0.0, None, FAKE * 4096, FAKE * 4096 + 4, None) == 2   # scales overlap codes
    assert lib.mxfp4_quantize(r(T((0, 64))), 0.0, None, FAKE * 4096, None, None) == 0


def test_conv_ex_validation(lib):
    x, w, out = good()
    arr = lambda v: (ctypes.c_int32 * 3)(*v)  # noqa: E731
    r = ctypes.byref

    def ex(fmt, bs, dst, amax=FAKE * 4096):
        return lib.conv3d_implicit_gemm_ex(r(x), r(w), None, amax, arr((1, 1, 1)), arr((1, 1, 1)), arr((1, 1, 1)),
                                           arr((1, 1, 1)), fmt, bs, dst, r(out), None)
    assert ex(3, 16, 0.0) == 2 and b"quant_format" in lib.q3d_last_error()
    assert ex(1, 48, 0.0) == 2 and b"block_size" in lib.q3d_last_error()
    assert ex(2, 16, 0.0) == 2
    assert ex(2, 32, 3.0) == 2 and b"dst_type_max" in lib.q3d_last_error()
    assert ex(1, 32, 0.0, amax=None) == 1            # NVFP4 needs act_amax


def _fp4_layout_bytes(shape):
    """The packed-weight size the header documents: 256 + ks * parts * image."""
    cout, K = shape[0], shape[1] * shape[2] * shape[3] * shape[4]
    n_ntiles, n_tile = 1, (cout + 15) // 16 * 16
    if n_tile > 448:
        n_ntiles = -(-cout // 448)
        n_tile = (-(-cout // n_ntiles) + 15) // 16 * 16
    n_sub = -(-n_tile // 256)
    sub_n = (-(-n_tile // n_sub) + 15) // 16 * 16
    img = sub_n * 32 + -(-sub_n // 128) * 512
    return 256 + -(-K // 64) * n_ntiles * n_sub * img


def test_fp4_weight_bytes(lib):
    a5 = lambda v: (ctypes.c_int64 * 5)(*v)  # noqa: E731
    for shape in [(5, 3, 3, 3, 3), (96, 96, 3, 3, 3), (192, 192, 3, 3, 3), (384, 384, 3, 3, 3), (500, 2, 3, 3, 3),
                  (1024, 512, 1, 1, 1), (16, 16, 3, 3, 3), (33, 37, 1, 1, 1)]:
        assert lib.q3d_fp4_weight_bytes(a5(shape)) == _fp4_layout_bytes(shape), shape
        assert api.fp4_weight_bytes(shape) == _fp4_layout_bytes(shape)
    assert lib.q3d_fp4_weight_bytes(a5((0, 3, 3, 3, 3))) == -1
    assert lib.q3d_fp4_weight_bytes(None) == -1


def test_fp4_validation(lib):
    arr = lambda v: (ctypes.c_int32 * 3)(*v)  # noqa: E731
    a5 = lambda v: (ctypes.c_int64 * 5)(*v)  # noqa: E731
    r = ctypes.byref
    w = T((5, 4, 3, 3, 3), 2, FAKE)
    need = _fp4_layout_bytes((5, 4, 3, 3, 3))
    packed = FAKE * 4096
    assert lib.conv3d_fp4_pack_weights(None, FAKE * 8, packed, need, None) == 1
    assert lib.conv3d_fp4_pack_weights(r(w), None, packed, need, None) == 1
    assert lib.conv3d_fp4_pack_weights(r(w), FAKE * 8, None, need, None) == 1
    assert lib.conv3d_fp4_pack_weights(r(w), FAKE * 8, packed, need - 16, None) == 2
    assert lib.conv3d_fp4_pack_weights(r(w), FAKE * 8, packed + 16, need, None) == 2     # alignment
    assert lib.conv3d_fp4_pack_weights(r(w), FAKE * 8, FAKE, need, None) == 2            # overlaps w
    assert lib.conv3d_fp4_pack_weights(r(T((5, 4, 3, 3, 3), 7, FAKE)), FAKE * 8, packed, need, None) == 3
    x, out = T((1, 4, 3, 8, 8), 2, FAKE), T((1, 5, 3, 8, 8), 2, FAKE * 256)
    ws = a5((5, 4, 3, 3, 3))

    def fp4(x=x, pw=packed, ws=ws, amax=FAKE * 8, out=out, plo=(1, 1, 1)):
        return lib.conv3d_implicit_gemm_fp4(r(x) if x is not None else None, pw, ws, None, amax, arr((1, 1, 1)),
                                            arr(plo), arr((1, 1, 1)), arr((1, 1, 1)),
                                            r(out) if out is not None else None, None)
    assert fp4(x=None) == 1
    assert fp4(pw=None) == 1
    assert fp4(ws=None) == 1
    assert fp4(amax=None) == 1
    assert fp4(pw=packed + 16) == 2
    assert fp4(ws=a5((5, 3, 3, 3, 3))) == 2                       # Cin mismatch
    assert fp4(out=T((1, 5, 3, 8, 9), 2, FAKE * 256)) == 2         # wrong out shape
    assert fp4(out=T((1, 5, 3, 8, 8), 2, packed + 64)) == 2        # out overlaps the packed weights
    assert fp4() in (4, 5)                                         # valid: no GPU here


def test_fp4_plans_fit_every_workload():
    from quantized_conv3d_implicit_b200 import workloads
    for name, wl in workloads.WORKLOADS.items():
        ws = (wl.cout, wl.x_shape[1]) + tuple(wl.kernel)
        pad6 = (wl.pad_lo[0], wl.pad_hi[0], wl.pad_lo[1], wl.pad_hi[1], wl.pad_lo[2], wl.pad_hi[2])
        p = api.plan_conv(wl.x_shape, ws, wl.stride, pad6, wl.dil, wl.dtype, kernel="fp4")
        assert p["applicable"], name
        assert p["smem"] <= 232448, name
        # accumulators, then sa scale-factor regions, inside the 512 TMEM columns
        assert p["n_mt"] * p["n_tile"] <= p["sf_col0"], name
        assert p["sf_col0"] + p["sa"] * p["sf_cols"] <= 512, name
        assert p["sf_cols"] == 4 * p["n_mt"] + 4 * -(-p["sub_n"] // 128) * p["n_sub"], name
        # an A stage holds n_mt subtiles of 128 rows x 32 bytes plus a 512-byte scale atom each
        assert p["a_stage_bytes"] >= p["n_mt"] * (4096 + 512) and p["a_stage_bytes"] % 1024 == 0, name
        assert p["b_stage_bytes"] >= p["n_sub"] * (p["sub_n"] * 32 + -(-p["sub_n"] // 128) * 512), name
        assert 2 <= p["sa"] <= 4 and p["sb"] >= 2, name


def test_bf16_plan_choice_per_workload():
    """The launcher's A placement (plan hook field aop): shared memory where
    it frees tensor memory for four subtiles or more A stages (measured
    faster there), tensor memory for the wide layers (measured faster)."""
    from quantized_conv3d_implicit_b200 import workloads
    want = {"edge_full_96_bf16": (1, 4), "wan_hi_192_bf16": (1, 2), "wan_mid_384_bf16": (0, 1),
            "pointwise_512to1024_fp16": (0, 1), "edge_full_96_bf16_dil122": (None, 2)}
    for name, (aop, mt) in want.items():
        wl = workloads.WORKLOADS[name]
        ws = (wl.cout, wl.x_shape[1]) + tuple(wl.kernel)
        pad6 = (wl.pad_lo[0], wl.pad_hi[0], wl.pad_lo[1], wl.pad_hi[1], wl.pad_lo[2], wl.pad_hi[2])
        p = api.plan_conv(wl.x_shape, ws, wl.stride, pad6, wl.dil, wl.dtype, kernel="tmem")
        assert p["applicable"] == 1, name
        if aop is not None:
            assert p["aop"] == aop, (name, p["aop"])
        assert p["n_mt"] == mt, (name, p["n_mt"])
        # accumulators (one or two buffers) fit the 512 columns, A stages beside them in tensor memory
        assert p["acc_bufs"] * p["n_mt"] * p["n_tile"] <= 512
        if p["aop"] == 0:
            assert p["a_col0"] + p["sa"] * p["n_mt"] * 32 <= 512


def test_blocks_of_64_have_a_shared_memory_plan(monkeypatch):
    """NVFP4 blocks of 64 pair two lanes per row, which the tensor-memory
    kernel allows only with A in shared memory: the format's GPU parity
    shapes must have that plan (Q3D_KERNEL=smem_a makes the plan hook report
    it), or the launcher would quietly hand them to the general kernel."""
    monkeypatch.setenv("Q3D_KERNEL", "smem_a")
    shapes = [((1, 11, 4, 7, 16), 41), ((1, 6, 6, 13, 24), 33), ((1, 32, 3, 8, 16), 300), ((1, 3, 7, 9, 16), 8),
              ((1, 8, 3, 8, 32), 192), ((1, 96, 3, 16, 64), 96), ((1, 11, 4, 7, 16), 128),
              ((1, 384, 5, 60, 104), 384)]
    for xs, cout in shapes:
        k = (1, 1, 1) if cout == 300 else (5, 5, 5) if xs[1] == 3 else (3, 3, 3)
        for dt in (torch.bfloat16, torch.float16):
            p = api.plan_conv(xs, (cout, xs[1]) + k, 1, (2, 0, 1, 1, 1, 1), 1, dt, kernel="tmem")
            assert p["applicable"] == 1 and p["aop"] == 1, (xs, cout, dt)

"""Python binding of libq3d.so (include/q3d.h): argument marshalling only.

Every step of the computation runs in the library's sm_100a kernels.  If the
library is missing or cannot be loaded, the calls raise RuntimeError; there is
no CPU or PyTorch fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence, Union

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libq3d.so")

Q3D_F32, Q3D_F16, Q3D_BF16 = 0, 1, 2
_DTYPES = {torch.float32: Q3D_F32, torch.float16: Q3D_F16, torch.bfloat16: Q3D_BF16}

STATUS = {0: "Q3D_OK", 1: "Q3D_ERR_NULLPTR", 2: "Q3D_ERR_INVALID_ARG", 3: "Q3D_ERR_UNSUPPORTED_DTYPE",
          4: "Q3D_ERR_ARCH", 5: "Q3D_ERR_CUDA", 6: "Q3D_ERR_DEVICE_TIMEOUT", 7: "Q3D_ERR_UNSUPPORTED_SHAPE"}

# names of the exported C entry points (checked against include/q3d.h by the tests)
EXPORTS = ("conv3d_implicit_gemm", "conv3d_implicit_gemm_pad2", "conv3d_implicit_gemm_ex",
           "conv3d_implicit_gemm_noalloc",
           "fp4_fake_quant", "fp4_fake_quant_bs", "mxfp4_quantize", "q3d_act_amax", "q3d_last_error",
           "q3d_check_device_error", "q3d_version", "q3d_conv_out_shape", "q3d_selftest_formats",
           "q3d_selftest_ratio", "q3d_selftest_withheld_arrive", "q3d_plan_conv", "q3d_plan_conv_tmem",
           "q3d_fp4_weight_bytes", "conv3d_fp4_pack_weights", "conv3d_implicit_gemm_fp4", "q3d_plan_conv_fp4")


class Q3DTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 5)]


class Q3DError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


_lock = threading.Lock()
_lib = None


def load_library(path: Optional[str] = None):
    """Load libq3d.so (raises RuntimeError when it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"{p} is missing: build it with `python -m quantized_conv3d_implicit_b200.build` "
                               "(there is no fallback implementation)")
        lib = ctypes.CDLL(p)
        T = ctypes.POINTER(Q3DTensor)
        i32x3 = ctypes.POINTER(ctypes.c_int32)
        vp = ctypes.c_void_p
        lib.conv3d_implicit_gemm.restype = ctypes.c_int
        lib.conv3d_implicit_gemm.argtypes = [T, T, T, vp, i32x3, i32x3, i32x3, ctypes.c_int32, T, vp]
        lib.conv3d_implicit_gemm_pad2.restype = ctypes.c_int
        lib.conv3d_implicit_gemm_pad2.argtypes = [T, T, T, vp, i32x3, i32x3, i32x3, i32x3, ctypes.c_int32, T, vp]
        lib.conv3d_implicit_gemm_ex.restype = ctypes.c_int
        lib.conv3d_implicit_gemm_ex.argtypes = [T, T, T, vp, i32x3, i32x3, i32x3, i32x3, ctypes.c_int32,
                                                ctypes.c_int32, ctypes.c_float, T, vp]
        lib.conv3d_implicit_gemm_noalloc.restype = ctypes.c_int
        lib.conv3d_implicit_gemm_noalloc.argtypes = [T, T, T, vp, i32x3, i32x3, i32x3, i32x3, ctypes.c_int32, T, vp]
        lib.fp4_fake_quant.restype = ctypes.c_int
        lib.fp4_fake_quant.argtypes = [T, vp, T, vp]
        lib.fp4_fake_quant_bs.restype = ctypes.c_int
        lib.fp4_fake_quant_bs.argtypes = [T, vp, ctypes.c_int32, T, vp]
        lib.mxfp4_quantize.restype = ctypes.c_int
        lib.mxfp4_quantize.argtypes = [T, ctypes.c_float, T, vp, vp, vp]
        lib.q3d_act_amax.restype = ctypes.c_int
        lib.q3d_act_amax.argtypes = [T, vp, vp]
        lib.q3d_last_error.restype = ctypes.c_char_p
        lib.q3d_last_error.argtypes = []
        lib.q3d_check_device_error.restype = ctypes.c_int
        lib.q3d_check_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
        lib.q3d_version.restype = ctypes.c_int32
        lib.q3d_selftest_formats.restype = ctypes.c_int
        lib.q3d_selftest_formats.argtypes = [vp, ctypes.c_int64, vp, vp, vp]
        lib.q3d_selftest_withheld_arrive.restype = ctypes.c_int
        lib.q3d_selftest_withheld_arrive.argtypes = [T, T, i32x3, i32x3, i32x3, i32x3, T, vp]
        lib.q3d_selftest_ratio.restype = ctypes.c_int
        lib.q3d_selftest_ratio.argtypes = [vp, vp, ctypes.c_int64, vp, vp]
        i64x5 = ctypes.POINTER(ctypes.c_int64)
        lib.q3d_conv_out_shape.restype = ctypes.c_int
        lib.q3d_conv_out_shape.argtypes = [i64x5, i64x5, i32x3, i32x3, i32x3, i32x3, i64x5]
        lib.q3d_fp4_weight_bytes.restype = ctypes.c_int64
        lib.q3d_fp4_weight_bytes.argtypes = [i64x5]
        lib.conv3d_fp4_pack_weights.restype = ctypes.c_int
        lib.conv3d_fp4_pack_weights.argtypes = [T, vp, vp, ctypes.c_int64, vp]
        lib.conv3d_implicit_gemm_fp4.restype = ctypes.c_int
        lib.conv3d_implicit_gemm_fp4.argtypes = [T, vp, i64x5, T, vp, i32x3, i32x3, i32x3, i32x3, T, vp]
        for name in ("q3d_plan_conv", "q3d_plan_conv_tmem", "q3d_plan_conv_fp4"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [i64x5, i64x5, i32x3, i32x3, i32x3, i32x3, ctypes.c_int32,
                           ctypes.POINTER(ctypes.c_int32), ctypes.c_int32]
        if path is None:
            _lib = lib
        return lib


def _tensor(t: Optional[torch.Tensor]) -> Optional[Q3DTensor]:
    if t is None:
        return None
    if t.dtype not in _DTYPES:
        raise Q3DError(3, f"unsupported dtype {t.dtype}")
    if not t.is_contiguous():
        raise Q3DError(2, "tensors must be contiguous")
    s = Q3DTensor()
    s.data = t.data_ptr() if t.numel() > 0 else None
    s.dtype = _DTYPES[t.dtype]
    s.ndim = t.dim()
    for i, d in enumerate(t.shape):
        s.shape[i] = d
    return s


def _ref(s):
    return ctypes.byref(s) if s is not None else None


def _triple(v: Union[int, Sequence[int]]) -> tuple:
    if isinstance(v, int):
        return (v, v, v)
    v = tuple(int(t) for t in v)
    if len(v) != 3:
        raise ValueError("expected an int or a 3-tuple")
    return v


def _pads(padding) -> tuple:
    """int, 3-tuple (symmetric) or 6-tuple (d_lo, d_hi, h_lo, h_hi, w_lo, w_hi)."""
    if isinstance(padding, int):
        return (padding,) * 3, (padding,) * 3
    p = tuple(int(t) for t in padding)
    if len(p) == 3:
        return p, p
    if len(p) == 6:
        return (p[0], p[2], p[4]), (p[1], p[3], p[5])
    raise ValueError("padding must be an int, a 3-tuple or a 6-tuple")


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if stream.cuda_stream != 0 else None


def _check(lib, status: int):
    if status != 0:
        msg = lib.q3d_last_error().decode(errors="replace")
        raise Q3DError(status, msg)


def out_shape(x_shape, w_shape, stride=1, padding=0, dilation=1):
    """[N, Cout, OD, OH, OW] of the convolution, as the library computes it
    (q3d_conv_out_shape); raises Q3DError for an invalid geometry."""
    lib = load_library()
    lo, hi = _pads(padding)
    a3 = lambda t: (ctypes.c_int32 * 3)(*t)  # noqa: E731
    a5 = lambda t: (ctypes.c_int64 * 5)(*[int(v) for v in t])  # noqa: E731
    o = (ctypes.c_int64 * 5)()
    _check(lib, lib.q3d_conv_out_shape(a5(x_shape), a5(w_shape), a3(_triple(stride)), a3(lo), a3(hi),
                                       a3(_triple(dilation)), o))
    return tuple(int(v) for v in o)


def _check_amax(act_amax, x, quant_act):
    if quant_act:
        if act_amax is None:
            raise ValueError("quant_act requires act_amax")
        if act_amax.dtype != torch.float32 or act_amax.numel() != 1 or act_amax.device != x.device:
            raise ValueError("act_amax must be a one-element float32 tensor on x's device")


def conv3d_implicit_gemm(x: torch.Tensor, w: torch.Tensor, bias: Optional[torch.Tensor] = None,
                         stride=1, padding=0, dilation=1, act_amax: Optional[torch.Tensor] = None,
                         quant_act: bool = False, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y = conv3d(x, w) + bias through libq3d (BF16 tensor cores, FP32
    accumulation, result in x.dtype), optionally fake-quantising the
    activation operand to NVFP4 (act_amax: float32 device tensor with one
    element).  padding may be an int, a 3-tuple or a 6-tuple
    (d_lo, d_hi, h_lo, h_hi, w_lo, w_hi); symmetric padding goes through the
    C entry point conv3d_implicit_gemm, asymmetric padding through
    conv3d_implicit_gemm_pad2."""
    lib = load_library()
    lo, hi = _pads(padding)
    if out is None:
        out = torch.empty(out_shape(x.shape, w.shape, stride, padding, dilation), dtype=x.dtype, device=x.device)
    _check_amax(act_amax, x, quant_act)
    arr = lambda t: (ctypes.c_int32 * 3)(*t)  # noqa: E731
    xs, ws, os_, bs = _tensor(x), _tensor(w), _tensor(out), _tensor(bias)
    amax_ptr = act_amax.data_ptr() if (quant_act and act_amax is not None) else None
    if lo == hi:   # symmetric padding: the article's signature (sec. 7.1)
        st = lib.conv3d_implicit_gemm(_ref(xs), _ref(ws), _ref(bs), amax_ptr, arr(_triple(stride)), arr(lo),
                                      arr(_triple(dilation)), int(bool(quant_act)), _ref(os_),
                                      _stream_handle(stream))
    else:
        st = lib.conv3d_implicit_gemm_pad2(_ref(xs), _ref(ws), _ref(bs), amax_ptr, arr(_triple(stride)), arr(lo),
                                           arr(hi), arr(_triple(dilation)), int(bool(quant_act)), _ref(os_),
                                           _stream_handle(stream))
    _check(lib, st)
    return out


QUANT_FORMATS = {"none": 0, "nvfp4": 1, "mxfp4": 2}


def conv3d_implicit_gemm_ex(x: torch.Tensor, w: torch.Tensor, bias: Optional[torch.Tensor] = None,
                            stride=1, padding=0, dilation=1, act_amax: Optional[torch.Tensor] = None,
                            quant_format: str = "nvfp4", block_size: int = 16, dst_type_max: float = 0.0,
                            out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """conv3d_implicit_gemm with the activation quantiser chosen explicitly:
    quant_format "none", "nvfp4" (block_size 16..256, act_amax required) or
    "mxfp4" (block_size 32, power-of-two scales, dst_type_max 0 or 6..12)."""
    lib = load_library()
    lo, hi = _pads(padding)
    if out is None:
        out = torch.empty(out_shape(x.shape, w.shape, stride, padding, dilation), dtype=x.dtype, device=x.device)
    _check_amax(act_amax, x, quant_format == "nvfp4")
    arr = lambda t: (ctypes.c_int32 * 3)(*t)  # noqa: E731
    xs, ws, os_, bs = _tensor(x), _tensor(w), _tensor(out), _tensor(bias)
    amax_ptr = act_amax.data_ptr() if (quant_format == "nvfp4" and act_amax is not None) else None
    st = lib.conv3d_implicit_gemm_ex(_ref(xs), _ref(ws), _ref(bs), amax_ptr, arr(_triple(stride)), arr(lo), arr(hi),
                                     arr(_triple(dilation)), QUANT_FORMATS[quant_format], int(block_size),
                                     float(dst_type_max), _ref(os_), _stream_handle(stream))
    _check(lib, st)
    return out


class Fp4Weights:
    """Weights packed for conv3d_implicit_gemm_fp4: the device buffer (uint8)
    and the original [Cout, Cin, kd, kh, kw] shape."""

    def __init__(self, packed: torch.Tensor, shape):
        self.packed = packed
        self.shape = tuple(int(v) for v in shape)


def fp4_weight_bytes(w_shape) -> int:
    """Bytes of the packed NVFP4 weights of a [Cout, Cin, kd, kh, kw] tensor."""
    lib = load_library()
    n = lib.q3d_fp4_weight_bytes((ctypes.c_int64 * 5)(*[int(v) for v in w_shape]))
    if n < 0:
        raise ValueError("w_shape must have five positive extents")
    return int(n)


def conv3d_fp4_pack_weights(w: torch.Tensor, w_amax: torch.Tensor, stream=None) -> Fp4Weights:
    """Quantise w to NVFP4 operands (blocks of 16 along K, global scale
    w_amax / 2688; w_amax a one-element float32 tensor on w's device) into a
    new packed buffer for conv3d_implicit_gemm_fp4."""
    lib = load_library()
    _check_amax(w_amax, w, True)
    n = fp4_weight_bytes(w.shape)
    packed = torch.empty(n, dtype=torch.uint8, device=w.device)
    ws = _tensor(w)
    _check(lib, lib.conv3d_fp4_pack_weights(_ref(ws), w_amax.data_ptr(), packed.data_ptr(), n,
                                            _stream_handle(stream)))
    return Fp4Weights(packed, w.shape)


def conv3d_implicit_gemm_fp4(x: torch.Tensor, wq: Fp4Weights, bias: Optional[torch.Tensor] = None, stride=1,
                             padding=0, dilation=1, act_amax: Optional[torch.Tensor] = None,
                             out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The true-FP4 convolution: activations quantised to NVFP4 with act_amax,
    weights packed by conv3d_fp4_pack_weights, block-scaled FP4 tensor-core
    products with FP32 accumulation, result in x.dtype."""
    lib = load_library()
    lo, hi = _pads(padding)
    if wq.packed.device != x.device:
        raise ValueError("the packed weights must be on x's device")
    if out is None:
        out = torch.empty(out_shape(x.shape, wq.shape, stride, padding, dilation), dtype=x.dtype, device=x.device)
    _check_amax(act_amax, x, True)
    arr = lambda t: (ctypes.c_int32 * 3)(*t)  # noqa: E731
    xs, os_, bs = _tensor(x), _tensor(out), _tensor(bias)
    st = lib.conv3d_implicit_gemm_fp4(_ref(xs), wq.packed.data_ptr(), (ctypes.c_int64 * 5)(*wq.shape), _ref(bs),
                                      act_amax.data_ptr(), arr(_triple(stride)), arr(lo), arr(hi),
                                      arr(_triple(dilation)), _ref(os_), _stream_handle(stream))
    _check(lib, st)
    return out


def conv3d_implicit_gemm_noalloc(x: torch.Tensor, w: torch.Tensor, out: torch.Tensor,
                                 bias: Optional[torch.Tensor] = None, stride=1, padding=0, dilation=1,
                                 act_amax: Optional[torch.Tensor] = None, quant_act: bool = False,
                                 stream=None) -> torch.Tensor:
    """conv3d_implicit_gemm through the C entry point that allocates no
    device memory (weights needing conversion are staged in the library's
    fixed 16 MiB area per device).  `out` must be preallocated."""
    lib = load_library()
    lo, hi = _pads(padding)
    _check_amax(act_amax, x, quant_act)
    arr = lambda t: (ctypes.c_int32 * 3)(*t)  # noqa: E731
    xs, ws, os_, bs = _tensor(x), _tensor(w), _tensor(out), _tensor(bias)
    amax_ptr = act_amax.data_ptr() if quant_act else None
    st = lib.conv3d_implicit_gemm_noalloc(_ref(xs), _ref(ws), _ref(bs), amax_ptr, arr(_triple(stride)), arr(lo),
                                          arr(hi), arr(_triple(dilation)), int(bool(quant_act)), _ref(os_),
                                          _stream_handle(stream))
    _check(lib, st)
    return out


def fp4_fake_quant(x: torch.Tensor, amax: torch.Tensor, out: Optional[torch.Tensor] = None,
                   stream=None, block_size: int = 16) -> torch.Tensor:
    """NVFP4 fake-quantisation through libq3d: consecutive blocks of
    block_size (16, 32, 64, 128 or 256) elements, each with its own E4M3
    scale.  block_size 16 calls fp4_fake_quant, the others fp4_fake_quant_bs."""
    lib = load_library()
    if out is None:
        out = torch.empty_like(x)
    if amax.dtype != torch.float32 or amax.numel() != 1 or amax.device != x.device:
        raise ValueError("amax must be a one-element float32 tensor on x's device")
    xs, os_ = _tensor(x), _tensor(out)
    if block_size == 16:
        st = lib.fp4_fake_quant(_ref(xs), amax.data_ptr(), _ref(os_), _stream_handle(stream))
    else:
        st = lib.fp4_fake_quant_bs(_ref(xs), amax.data_ptr(), int(block_size), _ref(os_), _stream_handle(stream))
    _check(lib, st)
    return out


def mxfp4_quantize(x: torch.Tensor, dst_type_max: float = 0.0, out: Optional[torch.Tensor] = None,
                   want_out: bool = True, want_codes: bool = True, stream=None):
    """MXFP4 through libq3d: groups of 32 elements with a power-of-two E8M0
    scale.  Returns (dequantised tensor or None, E8M0 scale bytes [numel/32],
    packed E2M1 codes [numel/2] or None)."""
    lib = load_library()
    if want_out and out is None:
        out = torch.empty_like(x)
    n = x.numel()
    scales = torch.empty(n // 32, dtype=torch.uint8, device=x.device)
    codes = torch.empty(n // 2, dtype=torch.uint8, device=x.device) if want_codes else None
    xs = _tensor(x)
    os_ = _tensor(out) if want_out else None
    st = lib.mxfp4_quantize(_ref(xs), float(dst_type_max), _ref(os_), scales.data_ptr() if n else None,
                            codes.data_ptr() if (codes is not None and n) else None, _stream_handle(stream))
    _check(lib, st)
    return (out if want_out else None), scales, codes


def act_amax(x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """max |x| over all elements as a one-element float32 device tensor (0 for
    an empty x), computed on the device by libq3d; pass it on as act_amax."""
    lib = load_library()
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    if out.dtype != torch.float32 or out.numel() != 1:
        raise ValueError("out must be a one-element float32 tensor")
    xs = _tensor(x if x.dim() > 0 else x.reshape(1))
    st = lib.q3d_act_amax(_ref(xs), out.data_ptr(), _stream_handle(stream))
    _check(lib, st)
    return out


def check_device_error(stream=None) -> int:
    """Synchronise the stream and return the device error bits (0 = none);
    raises Q3DError when a bounded device wait gave up."""
    lib = load_library()
    bits = ctypes.c_uint32(0)
    st = lib.q3d_check_device_error(_stream_handle(stream), ctypes.byref(bits))
    _check(lib, st)
    return bits.value


def selftest_formats(v: torch.Tensor, stream=None):
    """Test hook: device E2M1 and E4M3 conversions of float32 values."""
    lib = load_library()
    assert v.dtype == torch.float32 and v.is_cuda and v.is_contiguous()
    e2m1 = torch.empty_like(v)
    e4m3 = torch.empty_like(v)
    st = lib.q3d_selftest_formats(v.data_ptr(), v.numel(), e2m1.data_ptr(), e4m3.data_ptr(), _stream_handle(stream))
    _check(lib, st)
    return e2m1, e4m3


def selftest_withheld_arrive(x: torch.Tensor, w: torch.Tensor, out: torch.Tensor, stride=1, padding=0,
                             dilation=1, stream=None):
    """Test hook of the bounded waits: the convolution with one hand-back
    arrival withheld in CTA 0, so that CTA's MMA wait gives up and it aborts
    (see q3d_testing.h)."""
    lib = load_library()
    lo, hi = _pads(padding)
    a3 = lambda t: (ctypes.c_int32 * 3)(*t)  # noqa: E731
    st = lib.q3d_selftest_withheld_arrive(_ref(_tensor(x)), _ref(_tensor(w)), a3(_triple(stride)), a3(lo), a3(hi),
                                          a3(_triple(dilation)), _ref(_tensor(out)), _stream_handle(stream))
    _check(lib, st)


def selftest_ratio(bmax: torch.Tensor, t: torch.Tensor, stream=None) -> torch.Tensor:
    """Test hook: the device's min(bmax / t, 448) of the block-scale step."""
    lib = load_library()
    for v in (bmax, t):
        assert v.dtype == torch.float32 and v.is_cuda and v.is_contiguous()
    assert bmax.shape == t.shape
    out = torch.empty_like(bmax)
    st = lib.q3d_selftest_ratio(bmax.data_ptr(), t.data_ptr(), bmax.numel(), out.data_ptr(), _stream_handle(stream))
    _check(lib, st)
    return out


PLAN_FIELDS = ("applicable", "TH", "TW", "n_mt", "groups", "n_tile", "n_ntiles", "n_sub", "sub_n", "ks", "c_slot",
               "q_slots", "ring", "sa", "sb", "tmem_cols", "smem", "n_ohb", "n_owb", "vec", "w_box", "h_ext", "kd_ext")


def plan_conv(x_shape, w_shape, stride=1, padding=0, dilation=1, dtype=torch.bfloat16, kernel="fast") -> dict:
    """Test hook (host only): the tiling/pipeline plan of the shared-memory
    specialised kernel (kernel="fast"), of the tensor-memory kernel
    (kernel="tmem", four more fields: a_col0, aop = where A lives (0 tensor
    memory, 1 shared memory), acc_bufs, hb_wait = halo hand-backs wait for
    the slot's fill) or of its NVFP4-operand variant
    (kernel="fp4", six more: sf_col0, sf_cols, a_stage_bytes, b_stage_bytes,
    acc_bufs, hb_wait)."""
    lib = load_library()
    lo, hi = _pads(padding)
    a3 = lambda t: (ctypes.c_int32 * 3)(*t)  # noqa: E731
    a5 = lambda t: (ctypes.c_int64 * 5)(*[int(v) for v in t])  # noqa: E731
    out = (ctypes.c_int32 * 32)()
    fn = {"tmem": lib.q3d_plan_conv_tmem, "fp4": lib.q3d_plan_conv_fp4}.get(kernel, lib.q3d_plan_conv)
    st = fn(a5(x_shape), a5(w_shape), a3(_triple(stride)), a3(lo), a3(hi), a3(_triple(dilation)), _DTYPES[dtype],
            out, 32)
    _check(lib, st)
    extra = {"tmem": ("a_col0", "aop", "acc_bufs", "hb_wait"), "fp4": ("sf_col0", "sf_cols", "a_stage_bytes", "b_stage_bytes", "acc_bufs", "hb_wait")}
    fields = PLAN_FIELDS + extra.get(kernel, ())
    return dict(zip(fields, list(out)[:len(fields)]))


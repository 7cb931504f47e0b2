"""CPU oracle for the Conv3D implicit GEMM with fused NVFP4 activation fake-quant.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` are the only
callers.  The product path (``quantized_conv3d_implicit_b200``) never imports
this package, and this package never imports the product.

The arithmetic lives in ``q3d_oracle.c`` (plain C, compiled with gcc,
``-ffp-contract=off``, no fast-math); this module only marshals numpy arrays.
Every function states the passage of the Model-Optimizer "Conv3D Implicit
GEMM CUDA kernel" article it follows (sections 5.1, 6.1-6.4, 7.1).

The MXFP4 functions follow the CANN aclnnFlatQuantV2 page instead (its
per-group route with E2M1 output, steps 3 and 4).

The NVFP4-operand functions (``nvfp4_block_exact``, ``nvfp4_exact``,
``conv3d_nvfp4``) define the true-FP4 variant: the same codes and block
scales, the operand value q * s8 * g taken exactly.

Parity pins: tests/test_oracle_formats.py, tests/test_oracle_fake_quant.py,
tests/test_oracle_conv.py, tests/test_oracle_mxfp4.py,
tests/test_oracle_nvfp4_exact.py.  No function here is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "q3d_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

DTYPE_CODES = {"float32": 0, "float16": 1, "bfloat16": 2}


def build(force: bool = False) -> str:
    """Compile q3d_oracle.c into liboracle.so next to it (gcc, -O2, no fast-math)."""
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-pthread", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            f32, i64, i32p = ctypes.c_float, ctypes.c_int64, ctypes.POINTER(ctypes.c_int32)
            vp = ctypes.c_void_p
            lib.oracle_e2m1_rne_sat.restype = f32
            lib.oracle_e2m1_rne_sat.argtypes = [f32]
            lib.oracle_e4m3_rne_sat.restype = f32
            lib.oracle_e4m3_rne_sat.argtypes = [f32]
            lib.oracle_bf16_round.restype = f32
            lib.oracle_bf16_round.argtypes = [f32]
            lib.oracle_fq_block.restype = None
            lib.oracle_fq_block.argtypes = [vp, ctypes.c_int, f32, vp]
            lib.oracle_fp4_fake_quant.restype = ctypes.c_int
            lib.oracle_fp4_fake_quant.argtypes = [vp, i64, f32, vp]
            lib.oracle_fp4_fake_quant_bs.restype = ctypes.c_int
            lib.oracle_fp4_fake_quant_bs.argtypes = [vp, i64, f32, ctypes.c_int, vp]
            lib.oracle_mx_scale_exp.restype = ctypes.c_int
            lib.oracle_mx_scale_exp.argtypes = [f32, f32]
            lib.oracle_mxfp4_block.restype = ctypes.c_int
            lib.oracle_mxfp4_block.argtypes = [vp, ctypes.c_int, f32, vp, vp]
            lib.oracle_mxfp4_fake_quant.restype = ctypes.c_int
            lib.oracle_mxfp4_fake_quant.argtypes = [vp, i64, f32, vp, vp, vp]
            lib.oracle_act_amax.restype = f32
            lib.oracle_act_amax.argtypes = [vp, i64]
            lib.oracle_round_to_dtype_bits.restype = None
            lib.oracle_round_to_dtype_bits.argtypes = [vp, i64, ctypes.c_int, vp]
            lib.oracle_out_dim.restype = i64
            lib.oracle_out_dim.argtypes = [i64] * 6
            lib.oracle_conv3d_ex.restype = ctypes.c_int
            lib.oracle_conv3d_ex.argtypes = [vp, i64, i64, i64, i64, i64, vp, i64, i64, i64, i64, vp,
                                             i32p, i32p, i32p, i32p, ctypes.c_int, ctypes.c_int, f32, f32,
                                             vp, i64, ctypes.c_int, vp]
            lib.oracle_nvfp4_block_exact.restype = None
            lib.oracle_nvfp4_block_exact.argtypes = [vp, ctypes.c_int, f32, vp]
            lib.oracle_nvfp4_exact.restype = ctypes.c_int
            lib.oracle_nvfp4_exact.argtypes = [vp, i64, f32, vp]
            lib.oracle_conv3d_nvfp4.restype = ctypes.c_int
            lib.oracle_conv3d_nvfp4.argtypes = [vp, i64, i64, i64, i64, i64, vp, i64, i64, i64, i64, vp,
                                                i32p, i32p, i32p, i32p, f32, f32, vp, i64, ctypes.c_int, vp]
            lib.oracle_conv3d.restype = ctypes.c_int
            lib.oracle_conv3d.argtypes = ([vp, i64, i64, i64, i64, i64, vp, i64, i64, i64, i64, vp,
                                           i32p, i32p, i32p, i32p, ctypes.c_int, f32, vp, i64,
                                           ctypes.c_int, vp])
            _lib = lib
    return _lib


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------------------
# scalar formats (article sec. 6.1, 6.2; RNE as fixed by the specification)
# ---------------------------------------------------------------------------

def e2m1(a) -> np.ndarray:
    """Nearest E2M1 value (grid of sec. 6.1), ties to even code, saturating at 6."""
    lib = _load()
    a = _f32(a)
    return np.array([lib.oracle_e2m1_rne_sat(float(v)) for v in a.ravel()], dtype=np.float32).reshape(a.shape)


def e4m3(r) -> np.ndarray:
    """Nearest E4M3FN value (with subnormals), ties to even code, saturating at 448 (sec. 6.2)."""
    lib = _load()
    r = _f32(r)
    return np.array([lib.oracle_e4m3_rne_sat(float(v)) for v in r.ravel()], dtype=np.float32).reshape(r.shape)


def bf16_round(v) -> np.ndarray:
    """Round-to-nearest-even to bfloat16, returned as float32 values (sec. 3)."""
    lib = _load()
    v = _f32(v)
    return np.array([lib.oracle_bf16_round(float(t)) for t in v.ravel()], dtype=np.float32).reshape(v.shape)


def round_to_dtype_bits(v, dtype: str) -> np.ndarray:
    """Raw storage bits of float32 values rounded (RNE) to dtype: uint32 for
    float32, uint16 for float16/bfloat16."""
    lib = _load()
    v = _f32(v)
    code = DTYPE_CODES[dtype]
    out = np.empty(v.shape, dtype=np.uint32 if code == 0 else np.uint16)
    lib.oracle_round_to_dtype_bits(_ptr(v), v.size, code, _ptr(out))
    return out


# ---------------------------------------------------------------------------
# fake-quantisation (sec. 6.2-6.4)
# ---------------------------------------------------------------------------

def fq_block(v, act_amax: float) -> np.ndarray:
    """One NVFP4 block (1..16 values; shorter blocks act as zero-filled)."""
    lib = _load()
    v = _f32(v)
    assert 1 <= v.size <= 16
    out = np.empty_like(v)
    lib.oracle_fq_block(_ptr(v), int(v.size), float(np.float32(act_amax)), _ptr(out))
    return out


def fp4_fake_quant(x, amax: float) -> np.ndarray:
    """Standalone fake-quant of sec. 6.4 on the fp32 values of x (any shape,
    numel % 16 == 0): binary32 outputs before the cast back to x's dtype."""
    lib = _load()
    x = _f32(x)
    if x.size % 16:
        raise ValueError("numel must be a multiple of 16")
    out = np.empty_like(x)
    rc = lib.oracle_fp4_fake_quant(_ptr(x), x.size, float(np.float32(amax)), _ptr(out))
    assert rc == 0
    return out


def fp4_fake_quant_bs(x, amax: float, block_size: int) -> np.ndarray:
    """Standalone fake-quant with the article's other block sizes (sec. 7.1,
    7.3: 16, 32, 64, 128 or 256; numel a multiple of it): binary32 outputs
    before the cast back to x's dtype."""
    lib = _load()
    x = _f32(x)
    out = np.empty_like(x)
    rc = lib.oracle_fp4_fake_quant_bs(_ptr(x), x.size, float(np.float32(amax)), int(block_size), _ptr(out))
    if rc != 0:
        raise ValueError("block_size must be 16, 32, 64, 128 or 256 and divide numel")
    return out


# ---------------------------------------------------------------------------
# MXFP4 (the CANN aclnnFlatQuantV2 page: per-group route, steps 3 and 4)
# ---------------------------------------------------------------------------

def mx_scale_exp(amax: float, dst_max: float = 0.0) -> int:
    """Shared exponent E of an MXFP4 group (scale 2^E) from its |v| maximum:
    floor(log2 amax) - 2 when dst_max is 0, else the exponent of
    amax / dst_max rounded up when that quotient is not a power of two."""
    return int(_load().oracle_mx_scale_exp(float(np.float32(amax)), float(np.float32(dst_max))))


def mxfp4_block(v, dst_max: float = 0.0):
    """One group (1..32 values): (dequantised binary32 values, signed 4-bit
    codes, E)."""
    lib = _load()
    v = _f32(v)
    out = np.empty_like(v)
    codes = np.empty(v.shape, np.uint8)
    e = lib.oracle_mxfp4_block(_ptr(v), int(v.size), float(np.float32(dst_max)), _ptr(out),
                               codes.ctypes.data_as(ctypes.c_void_p))
    return out, codes, int(e)


def mxfp4_fake_quant(x, dst_max: float = 0.0):
    """MXFP4 over the fp32 values of x (numel % 32 == 0, groups of 32
    consecutive elements): (dequantised binary32 values in x's shape, E8M0
    scale bytes [numel / 32], signed 4-bit codes [numel])."""
    lib = _load()
    x = _f32(x)
    out = np.empty_like(x)
    scales = np.empty(x.size // 32, np.uint8)
    codes = np.empty(x.size, np.uint8)
    rc = lib.oracle_mxfp4_fake_quant(_ptr(x), x.size, float(np.float32(dst_max)), _ptr(out),
                                     scales.ctypes.data_as(ctypes.c_void_p), codes.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError("numel must be a multiple of 32 and dst_max 0 or in [6, 12]")
    return out, scales, codes


def act_amax(x) -> np.float32:
    """max |x| over the fp32 values of x (0 for an empty x): the global amax
    of sec. 7.2 / 8.3, as one binary32 value."""
    lib = _load()
    x = _f32(x)
    return np.float32(lib.oracle_act_amax(_ptr(x), x.size))


def fp4_fake_quant_bits(x, amax: float, dtype: str) -> np.ndarray:
    """Standalone fake-quant with the result stored in dtype (RNE), as raw bits."""
    return round_to_dtype_bits(fp4_fake_quant(x, amax), dtype)


# ---------------------------------------------------------------------------
# convolution (sec. 5.1, 7.1)
# ---------------------------------------------------------------------------

def out_dims(in_dhw, k_dhw, stride, pad_lo, pad_hi, dil):
    lib = _load()
    return tuple(int(lib.oracle_out_dim(int(in_dhw[i]), int(k_dhw[i]), int(stride[i]), int(pad_lo[i]),
                                        int(pad_hi[i]), int(dil[i]))) for i in range(3))


QUANT_FORMATS = {"nvfp4": 1, "mxfp4": 2}


def conv3d(x, w, bias=None, stride=(1, 1, 1), pad_lo=(0, 0, 0), pad_hi=None, dil=(1, 1, 1),
           quant_act: bool = False, act_amax: float = 0.0, m_list=None, nthreads: int = 0,
           quant_format: str = "nvfp4", block_size: int = 16, dst_max: float = 0.0) -> np.ndarray:
    """Reference convolution in binary64 over BF16 (and, with quant_act,
    fake-quantised) operands.  quant_format "nvfp4": blocks of block_size
    (16, 32, 64, 128, 256) consecutive K elements of each A row with E4M3
    scales and the global scale act_amax / (6*448) (the article, sec. 6 and
    7.1); "mxfp4": groups of 32 with power-of-two scales and dst_max (the
    CANN aclnnFlatQuantV2 page).  A short last block acts as zero-filled.

    x: [N, C, D, H, W] values (any float dtype, taken exactly as float32);
    w: [Cout, C, KD, KH, KW]; bias: [Cout] or None.
    Returns [N, Cout, OD, OH, OW] float64, or, when m_list is given, the
    [len(m_list), Cout] rows for those flattened output positions
    m = ((n*OD + od)*OH + oh)*OW + ow.
    """
    lib = _load()
    x = _f32(x)
    w = _f32(w)
    if pad_hi is None:
        pad_hi = pad_lo
    N, C, D, H, W = x.shape
    Cout, Cw, KD, KH, KW = w.shape
    assert Cw == C
    b = None if bias is None else _f32(bias)
    arr = lambda t: (ctypes.c_int32 * 3)(*[int(v) for v in t])  # noqa: E731
    OD, OH, OW = out_dims((D, H, W), (KD, KH, KW), stride, pad_lo, pad_hi, dil)
    if min(OD, OH, OW) <= 0:
        raise ValueError("oracle_conv3d: invalid arguments or empty output")
    M = N * OD * OH * OW
    if m_list is None:
        ml = None
        n_m = M
    else:
        ml = np.ascontiguousarray(np.asarray(m_list, dtype=np.int64))
        n_m = ml.size
    y = np.empty((n_m, Cout), dtype=np.float64)
    qfmt = QUANT_FORMATS[quant_format] if quant_act else 0
    rc = lib.oracle_conv3d_ex(_ptr(x), N, C, D, H, W, _ptr(w), Cout, KD, KH, KW,
                              None if b is None else _ptr(b),
                              arr(stride), arr(pad_lo), arr(pad_hi), arr(dil), qfmt, int(block_size),
                              float(np.float32(act_amax)), float(np.float32(dst_max)),
                              None if ml is None else _ptr(ml), n_m, int(nthreads), _ptr(y))
    if rc != 0:
        raise ValueError("oracle_conv3d: invalid arguments")
    if m_list is None:
        return y.reshape(N, OD, OH, OW, Cout).transpose(0, 4, 1, 2, 3).copy()
    return y


# ---------------------------------------------------------------------------
# NVFP4 operands taken exactly: the true-FP4 product (formats of sec. 6.1,
# 6.2; weights quantised along K as in sec. 7.2)
# ---------------------------------------------------------------------------

def nvfp4_block_exact(v, amax: float) -> np.ndarray:
    """One block of up to 16 values as exact NVFP4 operand values
    sign * q * s8 * g (float64); the same codes and E4M3 scale as
    ``fq_block``, and zero for a block that takes the 1.0 fallback scale."""
    lib = _load()
    v = _f32(v)
    assert 1 <= v.size <= 16
    out = np.empty(v.size, dtype=np.float64)
    lib.oracle_nvfp4_block_exact(_ptr(v), v.size, float(np.float32(amax)), _ptr(out))
    return out


def nvfp4_exact(x, amax: float) -> np.ndarray:
    """A flat tensor in consecutive blocks of 16, each as ``nvfp4_block_exact``."""
    lib = _load()
    x = _f32(x)
    out = np.empty(x.shape, dtype=np.float64)
    if lib.oracle_nvfp4_exact(_ptr(x), x.size, float(np.float32(amax)), _ptr(out)) != 0:
        raise ValueError("nvfp4_exact: numel must be a multiple of 16")
    return out


def conv3d_nvfp4(x, w, bias=None, stride=(1, 1, 1), pad_lo=(0, 0, 0), pad_hi=None, dil=(1, 1, 1),
                 act_amax: float = 0.0, w_amax: float = 0.0, m_list=None, nthreads: int = 0) -> np.ndarray:
    """The true-FP4 convolution: every A row and every weight row quantised
    to NVFP4 operands in blocks of 16 consecutive K elements (act_amax and
    w_amax give the two global scales), multiplied exactly and summed in
    binary64, plus the bias.  Shapes and m_list as in ``conv3d``."""
    lib = _load()
    x = _f32(x)
    w = _f32(w)
    if pad_hi is None:
        pad_hi = pad_lo
    N, C, D, H, W = x.shape
    Cout, Cw, KD, KH, KW = w.shape
    assert Cw == C
    b = None if bias is None else _f32(bias)
    arr = lambda t: (ctypes.c_int32 * 3)(*[int(v) for v in t])  # noqa: E731
    OD, OH, OW = out_dims((D, H, W), (KD, KH, KW), stride, pad_lo, pad_hi, dil)
    if min(OD, OH, OW) <= 0:
        raise ValueError("oracle_conv3d_nvfp4: invalid arguments or empty output")
    M = N * OD * OH * OW
    if m_list is None:
        ml = None
        n_m = M
    else:
        ml = np.ascontiguousarray(np.asarray(m_list, dtype=np.int64))
        n_m = ml.size
    y = np.empty((n_m, Cout), dtype=np.float64)
    rc = lib.oracle_conv3d_nvfp4(_ptr(x), N, C, D, H, W, _ptr(w), Cout, KD, KH, KW,
                                 None if b is None else _ptr(b),
                                 arr(stride), arr(pad_lo), arr(pad_hi), arr(dil),
                                 float(np.float32(act_amax)), float(np.float32(w_amax)),
                                 None if ml is None else _ptr(ml), n_m, int(nthreads), _ptr(y))
    if rc != 0:
        raise ValueError("oracle_conv3d_nvfp4: invalid arguments")
    if m_list is None:
        return y.reshape(N, OD, OH, OW, Cout).transpose(0, 4, 1, 2, 3).copy()
    return y

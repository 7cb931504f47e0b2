"""GPU parity of mxfp4_quantize (the CANN aclnnFlatQuantV2 page's MXFP4
per-group route): the dequantised tensor, the E8M0 scale bytes and the
packed E2M1 codes are bit-exact against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from quantized_conv3d_implicit_b200 import api, workloads
from _parity import bits

pytestmark = pytest.mark.gpu

DTYPES = {torch.float32: "float32", torch.float16: "float16", torch.bfloat16: "bfloat16"}


def _groups(seed, ngroups, dtype):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(ngroups, 32, generator=g)
    # spread the group scales over many binades, plus zero, tiny and grid groups
    x *= torch.exp2(torch.randint(-20, 20, (ngroups, 1), generator=g).float())
    x[::9] = 0
    x[5::13] *= 1e-30
    grid = torch.tensor([0, 0.5, 1, 1.5, 2, 3, 4, 6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -6.0] * 2)
    x[7::17] = grid
    return x.to(dtype).reshape(-1)


def _check(x_dev, dst, out, scales, codes):
    xf = x_dev.float().cpu().numpy()
    ref, ref_s, ref_c = oracle.mxfp4_fake_quant(xf, dst)
    dt = DTYPES[x_dev.dtype]
    if out is not None:
        assert np.array_equal(bits(out), oracle.round_to_dtype_bits(ref, dt))
    assert np.array_equal(scales.cpu().numpy(), ref_s)
    if codes is not None:
        packed = (ref_c[0::2] | (ref_c[1::2] << 4)).astype(np.uint8)
        assert np.array_equal(codes.cpu().numpy(), packed)


@pytest.mark.parametrize("dtype", list(DTYPES))
@pytest.mark.parametrize("dst", [0.0, 6.0, 8.5, 12.0])
def test_mxfp4_bit_exact(cuda_ok, dtype, dst):
    # 1001 groups: the last warp spans a partial range
    x = _groups(1, 1001, dtype).cuda()
    out, scales, codes = api.mxfp4_quantize(x, dst)
    torch.cuda.synchronize()
    _check(x, dst, out, scales, codes)


@pytest.mark.parametrize("dtype", list(DTYPES))
def test_mxfp4_unaligned_inplace_and_partial_outputs(cuda_ok, dtype):
    x = _groups(2, 400, dtype).cuda()
    for off in (32, 1):           # an offset of one element is misaligned for every dtype
        xs = x[off: off + 32 * 390]
        out, scales, codes = api.mxfp4_quantize(xs, 6.0)
        _check(xs, 6.0, out, scales, codes)
    # codes and scales only, then the dequantised tensor only, then in place
    _, scales, codes = api.mxfp4_quantize(x, 0.0, want_out=False)
    _check(x, 0.0, None, scales, codes)
    out, scales, codes = api.mxfp4_quantize(x, 0.0, want_codes=False)
    _check(x, 0.0, out, scales, None)
    z = x.clone()
    api.mxfp4_quantize(z, 0.0, out=z)
    ref = oracle.round_to_dtype_bits(oracle.mxfp4_fake_quant(x.float().cpu().numpy(), 0.0)[0], DTYPES[dtype])
    assert np.array_equal(bits(z), ref)


def test_mxfp4_argument_errors(cuda_ok):
    x = torch.zeros(96, device="cuda")
    with pytest.raises(api.Q3DError):
        api.mxfp4_quantize(torch.zeros(48, device="cuda"))       # numel % 32
    for bad in (1.0, 13.0, -6.0):
        with pytest.raises(api.Q3DError):
            api.mxfp4_quantize(x, bad)
    out, scales, codes = api.mxfp4_quantize(torch.zeros(0, device="cuda"))
    assert scales.numel() == 0


def test_mxfp4_on_a_full_layer_input(cuda_ok):
    inp = workloads.make_inputs("wan_mid_384_bf16", device="cuda")
    x = inp["x"].reshape(-1)
    out, scales, codes = api.mxfp4_quantize(x, 0.0)
    torch.cuda.synchronize()
    rng = np.random.default_rng(9)
    ng = x.numel() // 32
    for s in np.unique(np.concatenate([[0, ng - 2048], rng.integers(0, ng - 2048, 16)])):
        lo, hi = int(s) * 32, (int(s) + 2048) * 32
        _check(x[lo:hi], 0.0, out[lo:hi], scales[int(s): int(s) + 2048], codes[lo // 2: hi // 2])
    assert api.check_device_error() == 0

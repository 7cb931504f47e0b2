"""GPU parity of the standalone NVFP4 fake-quantisation and of the device
format conversions: bit-exact against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from quantized_conv3d_implicit_b200 import api, workloads
from _parity import bits

pytestmark = pytest.mark.gpu

DTYPES = {torch.float32: "float32", torch.float16: "float16", torch.bfloat16: "bfloat16"}


def _sweep_values():
    rng = np.random.default_rng(0)
    parts = []
    # every E2M1 / E4M3 midpoint with 64 neighbours on each side
    g = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    e4 = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mids = np.concatenate([(g[:-1] + g[1:]) / 2, (e4[:-1] + e4[1:]) / 2, [6.0, 448.0, 0.0]]).astype(np.float32)
    for mid in mids:
        u = mid.view(np.uint32).astype(np.int64)
        parts.append((np.arange(u - 64, u + 65).clip(0, 0x7F7FFFFF)).astype(np.uint32).view(np.float32))
    parts.append(rng.uniform(0, 8, 200000).astype(np.float32))
    parts.append(np.exp(rng.uniform(np.log(1e-12), np.log(1e4), 200000)).astype(np.float32))
    v = np.concatenate(parts)
    return np.concatenate([v, -v])


def test_device_format_conversions_match_oracle(cuda_ok):
    v = _sweep_values()
    e2, e4 = api.selftest_formats(torch.from_numpy(v).cuda())
    assert np.array_equal(e2.cpu().numpy().view(np.uint32), oracle.e2m1(v).view(np.uint32))
    assert np.array_equal(e4.cpu().numpy().view(np.uint32), oracle.e4m3(np.abs(v)).view(np.uint32))


def _blocks(seed, nblocks, dtype):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(nblocks, 16, generator=g)
    # adversarial blocks: outliers, zero blocks, tiny blocks, exact grid points, ties
    x[::7] *= 20
    x[3::11] = 0
    x[5::13] *= 1e-6
    grid = torch.tensor([0, 0.5, 1, 1.5, 2, 3, 4, 6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -6.0])
    x[9::17] = grid
    return x.to(dtype)


@pytest.mark.parametrize("dtype", list(DTYPES))
@pytest.mark.parametrize("amax_mode", ["max", "zero", "small", "pow2"])
def test_fake_quant_bit_exact(cuda_ok, dtype, amax_mode):
    x = _blocks(1, 4096, dtype)
    xm = float(x.float().abs().max())
    amax = {"max": xm, "zero": 0.0, "small": xm / 50, "pow2": 2688.0}[amax_mode]
    amax_t = torch.tensor([amax], dtype=torch.float32)
    y = api.fp4_fake_quant(x.cuda(), amax_t.cuda())
    torch.cuda.synchronize()
    ref = oracle.fp4_fake_quant_bits(x.float().numpy(), np.float32(amax), DTYPES[dtype])
    assert np.array_equal(bits(y).reshape(-1), ref.reshape(-1))


@pytest.mark.parametrize("dtype", list(DTYPES))
def test_fake_quant_unaligned_and_inplace(cuda_ok, dtype):
    x = _blocks(2, 1000, dtype).reshape(-1).cuda()
    amax = x.float().abs().max().reshape(1)
    # views starting 16 and 8 elements in keep 16-byte alignment for 16-bit
    # types; a view starting 1 element in is misaligned for every dtype
    for off in (16, 8, 1):
        xs = x[off: off + 16 * 500]
        y = api.fp4_fake_quant(xs, amax)
        ref = oracle.fp4_fake_quant_bits(xs.float().cpu().numpy(), np.float32(amax.item()), DTYPES[dtype])
        assert np.array_equal(bits(y), ref), off
    # in place
    z = x.clone()
    api.fp4_fake_quant(z, amax, out=z)
    ref = oracle.fp4_fake_quant_bits(x.float().cpu().numpy(), np.float32(amax.item()), DTYPES[dtype])
    assert np.array_equal(bits(z), ref)


def test_fake_quant_empty_and_ranks(cuda_ok):
    amax = torch.ones(1, device="cuda")
    e = torch.empty(0, 16, device="cuda", dtype=torch.bfloat16)
    assert api.fp4_fake_quant(e, amax).numel() == 0
    x5 = _blocks(3, 64, torch.bfloat16).reshape(2, 4, 2, 4, 16).cuda()
    y5 = api.fp4_fake_quant(x5, amax)
    ref = oracle.fp4_fake_quant_bits(x5.float().cpu().numpy(), np.float32(1.0), "bfloat16")
    assert np.array_equal(bits(y5), ref)
    with pytest.raises(api.Q3DError):
        api.fp4_fake_quant(torch.zeros(17, device="cuda"), amax)


@pytest.mark.parametrize("name", ["wan_mid_384_bf16", "down_s122_128to256_fp16", "edge_full_96_bf16"])
def test_fake_quant_full_size_workload_inputs(cuda_ok, name):
    # the whole activation tensor of a layer: GPU vs oracle on a seeded
    # sample of 64 contiguous ranges of 4096 blocks plus the first and last
    inp = workloads.make_inputs(name, device="cuda")
    x, amax = inp["x"], inp["act_amax"]
    y = api.fp4_fake_quant(x, amax)
    torch.cuda.synchronize()
    xf, yf = x.reshape(-1), y.reshape(-1)
    nb = xf.numel() // 16
    rng = np.random.default_rng(7)
    starts = np.unique(np.concatenate([[0, max(0, nb - 4096)], rng.integers(0, max(1, nb - 4096), 64)]))
    dt = DTYPES[x.dtype]
    for s in starts:
        lo, hi = int(s) * 16, min(nb, int(s) + 4096) * 16
        ref = oracle.fp4_fake_quant_bits(xf[lo:hi].float().cpu().numpy(), np.float32(amax.item()), dt)
        assert np.array_equal(bits(yf[lo:hi]), ref), (name, s)
    assert api.check_device_error() == 0

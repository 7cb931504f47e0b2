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


def _ratio_divisors():
    """6 g for a spread of act_amax: powers of two, mantissas next to 1 and 2,
    log-uniform values, and the smallest amax for which the ratio decides
    anything (below it every block scale falls back to 1.0)."""
    rng = np.random.default_rng(3)
    t = [2.0 ** e for e in (-22, -10, -3, 0, 1, 5, 20)]
    t += [np.float32(1.0).view(np.uint32) + d for d in (1, 2, 3)]
    t += [np.float32(2.0).view(np.uint32) - d for d in (1, 2, 3)]
    t = [np.uint32(v).view(np.float32) if isinstance(v, (int, np.integer)) else v for v in t]
    t += list(np.exp(rng.uniform(np.log(1.4e-7), np.log(1e6), 40)))
    t += [6.0 * (6e-5 / 2688.0), 6.0 * (448.0 / 2688.0), 6.0 * (1.0 / 2688.0)]
    return np.array(t, np.float32)


def _ratio_ref(a, t):
    with np.errstate(all="ignore"):
        r = a / t  # IEEE binary32 division, correctly rounded
    return np.where(np.isnan(r), np.float32(448.0), np.minimum(r, np.float32(448.0))).astype(np.float32)


def test_device_scale_ratio_is_correctly_rounded(cuda_ok):
    """The block maximum over 6 g that feeds the E4M3 scale rounding equals
    the correctly rounded binary32 quotient (clamped to 448) for every
    non-negative finite BF16 maximum over a spread of divisors, for random
    binary32 maxima, and in the degenerate cases amax = 0 and 0 / t.  Near
    binary32 underflow (quotients below 2^-64) only the E4M3 decision is
    fixed: E4M3 rounds everything below 2^-10 to zero, so there both values
    must lie below 2^-10."""
    bf = (np.arange(0, 0x7F80, dtype=np.uint32) << 16).view(np.float32)  # all finite bf16 >= 0
    t = _ratio_divisors()
    a = np.tile(bf, t.size)
    tt = np.repeat(t, bf.size)
    rng = np.random.default_rng(4)
    ar = rng.integers(0, 0x7F800000, 1_000_000, dtype=np.uint32).view(np.float32)  # any finite binary32
    tr = np.exp(rng.uniform(np.log(1.4e-7), np.log(1e6), ar.size)).astype(np.float32)
    # maxima whose quotient lands where it decides the E4M3 code (2^-11 .. 2^10)
    td = np.exp(rng.uniform(np.log(1.4e-7), np.log(1e6), 2_000_000)).astype(np.float32)
    ad = (td.astype(np.float64) * np.exp2(rng.uniform(-11, 10, td.size))).astype(np.float32)
    a = np.concatenate([a, ar, ad, np.array([0.0, 1.0, 3e38, 0.0], np.float32)])
    tt = np.concatenate([tt, tr, td, np.array([0.0, 0.0, 0.0, 1.0], np.float32)])
    out = api.selftest_ratio(torch.from_numpy(a).cuda(), torch.from_numpy(tt).cuda()).cpu().numpy()
    ref = _ratio_ref(a, tt)
    tiny = ref < np.float32(2.0 ** -64)
    assert np.all(out[tiny] < np.float32(2.0 ** -10)) and np.all(out[tiny] >= 0)
    assert np.count_nonzero((ref >= np.float32(2.0 ** -10)) & (ref < np.float32(448.0))) > 1_500_000
    bad = np.flatnonzero((out.view(np.uint32) != ref.view(np.uint32)) & ~tiny)
    assert bad.size == 0, (bad.size, a[bad[:5]], tt[bad[:5]], out[bad[:5]], ref[bad[:5]])


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


# --- the article's other block sizes (sec. 7.1: fp4_block_size 16..256) ---

BLOCK_SIZES = (16, 32, 64, 128, 256)


def _ref_bs(x, amax, bs, dt):
    return oracle.round_to_dtype_bits(oracle.fp4_fake_quant_bs(x, np.float32(amax), bs), dt)


@pytest.mark.parametrize("dtype", list(DTYPES))
@pytest.mark.parametrize("bs", BLOCK_SIZES)
@pytest.mark.parametrize("amax_mode", ["max", "zero", "small"])
def test_fake_quant_block_sizes_bit_exact(cuda_ok, dtype, bs, amax_mode):
    # 1007 blocks: a numel that is a multiple of bs but not of 512 elements
    # (the span of one warp), so the last warp holds a partial span
    x = _blocks(11, 1007 * bs // 16, dtype).reshape(-1)
    xm = float(x.float().abs().max())
    amax = {"max": xm, "zero": 0.0, "small": xm / 50}[amax_mode]
    y = api.fp4_fake_quant(x.cuda(), torch.tensor([amax], dtype=torch.float32).cuda(), block_size=bs)
    torch.cuda.synchronize()
    assert np.array_equal(bits(y), _ref_bs(x.float().numpy(), amax, bs, DTYPES[dtype]))


@pytest.mark.parametrize("dtype", list(DTYPES))
@pytest.mark.parametrize("bs", (32, 256))
def test_fake_quant_block_sizes_unaligned_and_inplace(cuda_ok, dtype, bs):
    x = _blocks(12, 300 * bs // 16 + 1, dtype).reshape(-1).cuda()
    amax = x.float().abs().max().reshape(1)
    n = 299 * bs
    for off in (16, 1):
        xs = x[off: off + n]
        y = api.fp4_fake_quant(xs, amax, block_size=bs)
        assert np.array_equal(bits(y), _ref_bs(xs.float().cpu().numpy(), amax.item(), bs, DTYPES[dtype])), off
    z = x[:n].clone()
    api.fp4_fake_quant(z, amax, out=z, block_size=bs)
    assert np.array_equal(bits(z), _ref_bs(x[:n].float().cpu().numpy(), amax.item(), bs, DTYPES[dtype]))


def test_fake_quant_block_size_errors_and_empty(cuda_ok):
    amax = torch.ones(1, device="cuda")
    with pytest.raises(api.Q3DError):
        api.fp4_fake_quant(torch.zeros(96, device="cuda"), amax, block_size=64)
    with pytest.raises(api.Q3DError):
        api.fp4_fake_quant(torch.zeros(96, device="cuda"), amax, block_size=48)
    assert api.fp4_fake_quant(torch.empty(0, device="cuda"), amax, block_size=256).numel() == 0


def test_fake_quant_block_128_on_a_full_layer_input(cuda_ok):
    # the article's default block size on a whole activation tensor, sampled
    inp = workloads.make_inputs("wan_mid_384_bf16", device="cuda")
    x, amax = inp["x"].reshape(-1), inp["act_amax"]
    y = api.fp4_fake_quant(x, amax, block_size=128)
    torch.cuda.synchronize()
    rng = np.random.default_rng(8)
    nb = x.numel() // 128
    for s in np.unique(np.concatenate([[0, nb - 512], rng.integers(0, nb - 512, 32)])):
        lo, hi = int(s) * 128, (int(s) + 512) * 128
        assert np.array_equal(bits(y[lo:hi]), _ref_bs(x[lo:hi].float().cpu().numpy(), amax.item(), 128,
                                                       "bfloat16")), s
    assert api.check_device_error() == 0

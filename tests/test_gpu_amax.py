"""GPU parity of the device-side global amax (q3d_act_amax): bit-exact
against the CPU oracle over dtypes, ragged and empty sizes, misaligned
pointers, adversarial values, an input larger than L2 and the full-size
layer input; and the amax it writes drives the fused quantiser exactly as a
host-supplied one does."""
import numpy as np
import pytest
import torch

import oracle
from quantized_conv3d_implicit_b200 import api, workloads

pytestmark = pytest.mark.gpu

DTYPES = [torch.float32, torch.float16, torch.bfloat16]


def _check(x: torch.Tensor):
    got = api.act_amax(x)
    torch.cuda.synchronize()
    ref = oracle.act_amax(x.float().cpu().numpy())
    g = got.cpu().numpy().astype(np.float32)
    assert g.view(np.uint32)[0] == ref.view(np.uint32), (x.dtype, x.numel(), g[0], ref)


def _rand(n, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    v = torch.randn(n, generator=g) * torch.exp(torch.empty(n).uniform_(-6, 6, generator=g))
    return v.to(dtype)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("n", [0, 1, 7, 8, 9, 15, 16, 17, 1023, 4097, (1 << 20) + 5])
def test_amax_sizes(cuda_ok, dtype, n):
    _check(_rand(n, dtype, n).cuda())


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("offset", [1, 3])
def test_amax_misaligned_pointer(cuda_ok, dtype, offset):
    buf = _rand(100_003 + offset, dtype, 11).cuda()
    x = buf[offset:]
    assert x.data_ptr() % 16 != 0
    _check(x)


@pytest.mark.parametrize("dtype", DTYPES)
def test_amax_adversarial(cuda_ok, dtype):
    n = 40_007  # the vector part, a ragged tail, several CTAs
    base = _rand(n, dtype, 5)
    cases = []
    for pos in (0, 1, n // 2, n - 9, n - 1):        # maximum at the head, inside, in the tail
        x = base.clone()
        x[pos] = -1e4 if dtype != torch.float16 else -6e4
        cases.append(x)
    cases.append(torch.full((n,), -0.0, dtype=dtype))               # only negative zeros -> +0
    cases.append(torch.zeros(n, dtype=dtype))
    tiny = {torch.float32: 1e-44, torch.float16: 6e-8, torch.bfloat16: 1e-40}[dtype]
    cases.append(torch.full((n,), tiny, dtype=dtype) * torch.tensor([-1.0, 1.0]).repeat(n // 2 + 1)[:n].to(dtype))
    x = base.clone()
    x[123] = float("-inf")
    cases.append(x)
    for x in cases:
        _check(x.cuda())


def test_amax_larger_than_l2(cuda_ok):
    x = _rand(72 << 20, torch.bfloat16, 9)  # 151 MB > 126 MB L2
    x[-3] = 123.0
    _check(x.cuda())


@pytest.mark.parametrize("name", ["wan_mid_384_bf16", "down_s122_128to256_fp16"])
def test_amax_full_size_layer_input(cuda_ok, name):
    wl = workloads.WORKLOADS[name]
    inp = workloads.make_inputs(wl, device="cuda")
    got = api.act_amax(inp["x"])
    torch.cuda.synchronize()
    assert torch.equal(got.cpu(), inp["act_amax"].cpu().reshape(1))
    _check(inp["x"])


@pytest.mark.parametrize("dtype", DTYPES)
def test_device_amax_drives_the_quantiser(cuda_ok, dtype):
    g = torch.Generator().manual_seed(3)
    x = torch.randn(1, 16, 3, 10, 16, generator=g).to(dtype).cuda()
    w = (torch.randn(24, 16, 3, 3, 3, generator=g) / 20).to(dtype).cuda()
    host = torch.tensor([float(x.float().abs().max())], dtype=torch.float32).cuda()
    dev = api.act_amax(x)
    assert torch.equal(dev, host)
    y_dev = api.conv3d_implicit_gemm(x, w, None, 1, 1, 1, dev, True)
    y_host = api.conv3d_implicit_gemm(x, w, None, 1, 1, 1, host, True)
    torch.cuda.synchronize()
    assert torch.equal(y_dev, y_host)
    fq_dev = api.fp4_fake_quant(x, dev)
    fq_host = api.fp4_fake_quant(x, host)
    torch.cuda.synchronize()
    assert torch.equal(fq_dev, fq_host)

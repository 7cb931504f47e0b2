"""GPU tests of conv3d_implicit_gemm_noalloc, the entry point that stages
weights in the library's fixed device area instead of allocating.

Each case calls the no-alloc entry point twice in a row on one stream (with
different weights, so the second call overwrites the staging area the first
one read) and compares both results with the regular entry point
conv3d_implicit_gemm_pad2 bit for bit: both run the same kernels on the same
BF16 weights, so any difference would be a staging fault.  The file
is named to be collected last, so the cases also run after every other GPU
test in the same process; they are written to pass alone in a fresh process
as well.
"""
import pytest
import torch

from quantized_conv3d_implicit_b200 import api, workloads

pytestmark = pytest.mark.gpu

STAGING_BYTES = 16 << 20

# (x shape, Cout, kernel, stride, 6-tuple padding, dilation, dtype, quant)
CASES = [
    # F16 weights: always converted, so always staged
    ((1, 24, 6, 20, 40), 64, (3, 3, 3), (1, 1, 1), (2, 0, 1, 1, 1, 1), (1, 1, 1), torch.float16, True),
    # BF16 with K = 3*27 = 81, not a multiple of 8: staged
    ((2, 3, 5, 17, 33), 40, (3, 3, 3), (1, 2, 2), (1, 1, 1, 1, 1, 1), (1, 1, 1), torch.bfloat16, True),
    # F32, no quantisation, dilation
    ((1, 16, 7, 12, 24), 48, (3, 3, 3), (1, 1, 1), (2, 2, 2, 2, 2, 2), (1, 2, 2), torch.float32, False),
    # BF16 with K % 8 == 0: weights read in place, no staging
    ((1, 32, 4, 10, 16), 96, (3, 3, 3), (1, 1, 1), (1, 1, 1, 1, 1, 1), (1, 1, 1), torch.bfloat16, True),
]


def _inputs(seed, xs, cout, k, dtype):
    d = workloads.random_conv_inputs(seed, xs, cout, k, dtype, bias=True, device="cuda")
    return d["x"], d["w"], d["bias"], d["act_amax"]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_noalloc_matches_regular_entry_twice_in_a_row(cuda_ok, case):
    xs, cout, k, s, pad6, d, dtype, quant = CASES[case]
    x1, w1, b1, a1 = _inputs(100 + case, xs, cout, k, dtype)
    _, w2, b2, _ = _inputs(200 + case, xs, cout, k, dtype)
    oshape = api.out_shape(x1.shape, w1.shape, s, pad6, d)
    y1 = torch.full(oshape, float("nan"), dtype=dtype, device="cuda")
    y2 = torch.full(oshape, float("nan"), dtype=dtype, device="cuda")
    # two no-alloc calls back to back on the same stream
    api.conv3d_implicit_gemm_noalloc(x1, w1, y1, b1, s, pad6, d, act_amax=a1, quant_act=quant)
    api.conv3d_implicit_gemm_noalloc(x1, w2, y2, b2, s, pad6, d, act_amax=a1, quant_act=quant)
    r1 = api.conv3d_implicit_gemm(x1, w1, b1, s, pad6, d, act_amax=a1, quant_act=quant)
    r2 = api.conv3d_implicit_gemm(x1, w2, b2, s, pad6, d, act_amax=a1, quant_act=quant)
    assert api.check_device_error() == 0
    assert torch.equal(y1, r1), "no-alloc call 1 differs from the regular entry point"
    assert torch.equal(y2, r2), "no-alloc call 2 differs from the regular entry point"
    assert not torch.equal(y1, y2)


def test_noalloc_rejects_weights_beyond_the_staging_area(cuda_ok):
    # F16 [1024, 512, 3, 3, 3]: staged BF16 copy 1024 * 13824 * 2 bytes > 16 MiB
    x = torch.zeros((1, 512, 3, 3, 8), dtype=torch.float16, device="cuda")
    w = torch.zeros((1024, 512, 3, 3, 3), dtype=torch.float16, device="cuda")
    assert 1024 * 13824 * 2 > STAGING_BYTES
    y = torch.full(api.out_shape(x.shape, w.shape, 1, 1, 1), 7.0, dtype=torch.float16, device="cuda")
    with pytest.raises(api.Q3DError) as ei:
        api.conv3d_implicit_gemm_noalloc(x, w, y, None, 1, 1, 1)
    assert ei.value.status == 7 and "16777216" in str(ei.value)
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())  # nothing was enqueued


def test_noalloc_in_place_bf16_weights_have_no_size_limit(cuda_ok):
    # BF16 [1024, 512, 3, 3, 3] with K % 8 == 0 is read in place (no staging)
    x, w, b, amax = _inputs(300, (1, 512, 3, 4, 8), 1024, (3, 3, 3), torch.bfloat16)
    y = torch.empty(api.out_shape(x.shape, w.shape, 1, 1, 1), dtype=torch.bfloat16, device="cuda")
    api.conv3d_implicit_gemm_noalloc(x, w, y, b, 1, 1, 1, act_amax=amax, quant_act=True)
    r = api.conv3d_implicit_gemm(x, w, b, 1, 1, 1, act_amax=amax, quant_act=True)
    assert api.check_device_error() == 0
    assert torch.equal(y, r)


def _captured_node_types(call):
    """Capture `call(stream)` on a fresh stream into a CUDA graph (relaxed
    mode, never launched) and return the types of the graph's nodes."""
    from cuda.bindings import runtime as rt

    err, s = rt.cudaStreamCreateWithFlags(rt.cudaStreamNonBlocking)
    assert err == rt.cudaError_t.cudaSuccess
    ts = torch.cuda.ExternalStream(int(s))
    try:
        err, = rt.cudaStreamBeginCapture(s, rt.cudaStreamCaptureMode.cudaStreamCaptureModeRelaxed)
        assert err == rt.cudaError_t.cudaSuccess
        call(ts)
        err, graph = rt.cudaStreamEndCapture(s)
        assert err == rt.cudaError_t.cudaSuccess
        err, _, n = rt.cudaGraphGetNodes(graph, 0)
        assert err == rt.cudaError_t.cudaSuccess
        err, nodes, n = rt.cudaGraphGetNodes(graph, n)
        assert err == rt.cudaError_t.cudaSuccess
        types = []
        for nd in nodes[:n]:
            err, t = rt.cudaGraphNodeGetType(nd)
            assert err == rt.cudaError_t.cudaSuccess
            types.append(t)
        rt.cudaGraphDestroy(graph)
        return types
    finally:
        rt.cudaStreamDestroy(s)


def test_noalloc_enqueues_no_allocation(cuda_ok):
    """The property the entry point exists for: with weights that must be
    staged (F16), the regular entry point's captured work contains a
    stream-ordered allocation and the no-alloc one's does not."""
    from cuda.bindings import runtime as rt

    xs, cout, k, s, pad6, d, dtype, quant = CASES[0]
    x, w, b, a = _inputs(400, xs, cout, k, dtype)
    oshape = api.out_shape(x.shape, w.shape, s, pad6, d)
    y = torch.empty(oshape, dtype=dtype, device="cuda")
    # first calls outside any capture (the no-alloc area's address is looked up once)
    api.conv3d_implicit_gemm_noalloc(x, w, y, b, s, pad6, d, act_amax=a, quant_act=quant)
    api.conv3d_implicit_gemm(x, w, b, s, pad6, d, act_amax=a, quant_act=quant, out=y)
    assert api.check_device_error() == 0
    alloc = rt.cudaGraphNodeType.cudaGraphNodeTypeMemAlloc
    regular = _captured_node_types(lambda st: api.conv3d_implicit_gemm(x, w, b, s, pad6, d, act_amax=a,
                                                                      quant_act=quant, out=y, stream=st))
    noalloc = _captured_node_types(lambda st: api.conv3d_implicit_gemm_noalloc(x, w, y, b, s, pad6, d, act_amax=a,
                                                                              quant_act=quant, stream=st))
    assert alloc in regular          # the check can see an allocation
    assert alloc not in noalloc
    assert rt.cudaGraphNodeType.cudaGraphNodeTypeKernel in noalloc
    torch.cuda.synchronize()
    assert api.check_device_error() == 0

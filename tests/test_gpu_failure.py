"""The bounded waits on the GPU: a withheld arrival makes one wait give up.

q3d_selftest_withheld_arrive runs a convolution on the tensor-memory kernel
with one of the four arrivals of CTA 0's first accumulator hand-back
withheld, so that CTA's MMA issuer waits for a phase that never completes.
The first of the waits that depend on the withheld arrival to reach the
library's limit (2 s) gives up -- the transform warps' wait for a free A
stage (they run ahead of the MMA and start waiting first) or the MMA
issuer's wait for the accumulator -- records its site bit in the device
error word and aborts the CTA; every role waits for its copies in flight
and the launch ends.  Nothing faults, traps or spins without a bound.  The
host then reads Q3D_ERR_DEVICE_TIMEOUT with only such site bits (none from
a wait for a copy to land or from the final drain), the word is cleared,
and the next convolution is correct."""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
from quantized_conv3d_implicit_b200 import api, workloads
from _parity import assert_conv_close, to_np_f32

pytestmark = pytest.mark.gpu

# site bits of the waits downstream of the withheld arrival: producers waiting
# for a free stage or slot, transform warps for a free A stage, the epilogue
# for an accumulator, the MMA issuer for a free accumulator
DOWNSTREAM = (1 << 0) | (1 << 3) | (1 << 4) | (1 << 5) | (1 << 7)


def test_withheld_arrival_times_out_and_the_context_stays_usable(cuda_ok):
    lib = api.load_library()
    assert api.check_device_error() == 0                 # start from a clear word
    # more tiles than CTAs times accumulator buffers: CTA 0 reuses accumulator
    # buffer 0 (two buffers with this plan: CTA 0 has a third tile)
    xs, cout, k = (1, 16, 16, 128, 128), 32, (3, 3, 3)
    plan = api.plan_conv(xs, (cout, 16) + k, 1, 1, 1, torch.bfloat16, kernel="tmem")
    assert plan["applicable"] == 1
    assert xs[2] * plan["n_ohb"] * plan["n_owb"] * plan["n_ntiles"] > 2 * 148
    inp = workloads.random_conv_inputs(71, xs, cout, k, dtype=torch.bfloat16, bias=False, device="cuda")
    y = torch.empty(api.out_shape(xs, (cout, 16) + k, 1, 1, 1), dtype=torch.bfloat16, device="cuda")
    t0 = time.time()
    api.selftest_withheld_arrive(inp["x"], inp["w"], y, 1, 1, 1)
    bits = ctypes.c_uint32(0)
    st = lib.q3d_check_device_error(None, ctypes.byref(bits))
    elapsed = time.time() - t0
    assert st == 6, lib.q3d_last_error()                 # Q3D_ERR_DEVICE_TIMEOUT
    assert bits.value != 0 and (bits.value & ~DOWNSTREAM) == 0, hex(bits.value)
    assert 1.5 < elapsed < 60.0                           # the 2 s limit, then the drain
    # the word was cleared and the context still works
    assert api.check_device_error() == 0
    y2 = api.conv3d_implicit_gemm(inp["x"], inp["w"], None, 1, 1, 1)
    assert api.check_device_error() == 0
    # sampled output rows (every Cout), the first and last included
    M = y2.numel() // cout
    ms = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(3).integers(0, M, 400)]))
    ref = oracle.conv3d(to_np_f32(inp["x"]), to_np_f32(inp["w"]), None, (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1),
                        m_list=ms)
    got = to_np_f32(y2.permute(0, 2, 3, 4, 1).reshape(-1, cout)[torch.from_numpy(ms).cuda()])
    assert_conv_close(got, ref, "after the timeout", torch.bfloat16)


def test_withheld_arrival_rejects_problems_it_cannot_exercise(cuda_ok):
    # a single tile per CTA: the withheld hand-back would never be waited for
    xs, cout, k = (1, 16, 2, 8, 16), 16, (3, 3, 3)
    inp = workloads.random_conv_inputs(72, xs, cout, k, dtype=torch.bfloat16, bias=False, device="cuda")
    y = torch.empty(api.out_shape(xs, (cout, 16) + k, 1, 1, 1), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(api.Q3DError) as ei:
        api.selftest_withheld_arrive(inp["x"], inp["w"], y, 1, 1, 1)
    assert ei.value.status == 2
    assert api.check_device_error() == 0

"""Shared helpers for the GPU parity tests (comparison rules only)."""
import numpy as np
import torch

# significand bits (including the implicit one) of each output dtype
_SIG_BITS = {torch.float32: 24, torch.float16: 11, torch.bfloat16: 8}


def half_ulp(y_ref: np.ndarray, dtype) -> np.ndarray:
    """Half a unit in the last place of |y_ref| in the output dtype: the
    error that storing an exact result in that dtype can add."""
    if dtype is None:
        return np.zeros_like(y_ref)
    p = _SIG_BITS[dtype]
    a = np.abs(y_ref)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    if dtype == torch.float16:
        e = np.maximum(e, -14.0)   # subnormal spacing
    return np.where(a > 0, np.exp2(e - p), 0.0)


def assert_conv_close(y_gpu, y_ref, what="", dtype=None):
    """Acceptance for convolution outputs against the oracle:
    max|y - y_ref| <= 2e-3 * max|y_ref| and per-element relative error
    <= 1e-2 wherever |y_ref| > 1e-2 * max|y_ref|, both measured on the
    computed value: the half-ulp of the output dtype (the result has to be
    returned in x's dtype) is added to the absolute bound."""
    y = np.asarray(y_gpu, dtype=np.float64)
    r = np.asarray(y_ref, dtype=np.float64)
    assert y.shape == r.shape, (y.shape, r.shape)
    if r.size == 0:
        return
    ymax = np.abs(r).max()
    err = np.abs(y - r)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    bound = 2e-3 * ymax + half_ulp(r, dtype) + 1e-30
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} elements over the bound; worst err {err.max():.3e}, "
                           f"2e-3*max|y_ref| = {2e-3 * ymax:.3e}")
    big = np.abs(r) > 1e-2 * ymax
    if big.any():
        rel = err[big] / np.abs(r[big])
        assert rel.max() <= 1e-2, f"{what}: max rel err {rel.max():.3e} on |y_ref| > 1e-2 max"


def to_np_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float32).cpu().numpy()


def bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy().view(np.uint32)
    return t.view(torch.int16).numpy().view(np.uint16)

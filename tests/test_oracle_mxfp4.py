"""Pins of the MXFP4 oracle (the CANN aclnnFlatQuantV2 page's per-group
route: groups of 32, power-of-two E8M0 scale, the dstTypeMax rule).

Pinned by hand-derived worked examples (tests/golden/mxfp4_worked_examples.txt),
the exponent's closed forms through numpy's frexp, and invariants that a
dropped round-up, a wrong emax, a wrong tie rule or a lost sign each break:
nearest-grid-point brute force, power-of-two covariance, sign symmetry,
idempotence, code/scale consistency and the argument rules."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mxfp4_worked_examples.txt")
GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _num(s):
    return float.fromhex(s) if "0x" in s else float(s)


def _load_golden():
    cases, cur = [], None
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip() if not line.lstrip().startswith("#") else ""
        if not line:
            continue
        key, val = (t.strip() for t in line.split(":", 1))
        if key == "name":
            cur = {"name": val}
            cases.append(cur)
        elif key in ("in", "out"):
            cur[key] = np.array([_num(t) for t in val.split()], np.float32)
        else:
            cur[key] = _num(val)
    return cases


CASES = _load_golden()


def test_golden_file_parsed():
    assert len(CASES) == 11
    for c in CASES:
        assert c["in"].size == c["out"].size <= 32, c["name"]


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_worked_examples(case):
    v = np.zeros(32, np.float32)
    v[:case["in"].size] = case["in"]
    out, codes, e = oracle.mxfp4_block(v, case["dst_max"])
    assert e == case["exp"]
    want = np.zeros(32, np.float32)
    want[:case["out"].size] = case["out"]
    assert np.array_equal(out.view(np.uint32), want.view(np.uint32)), (out[:case["out"].size], case["out"])


def _rand_groups(seed, n, spread=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, 32)).astype(np.float32)
    if spread:
        x *= np.exp2(rng.integers(-30, 30, (n, 1))).astype(np.float32)
    x[::9] = 0.0
    x[4::13, :5] = 0.0
    return x


def _expected_exp(amax, dst):
    """E from the page's formulas, computed through numpy's frexp (x = m 2^e,
    m in [0.5, 1)): floor(log2 x) = e - 1, and ceil(log2 S) = e - 1 when m is
    0.5 exactly, else e."""
    if dst == 0:
        if amax == 0 or amax < np.float32(2.0 ** -126):
            return -127
        m, e = np.frexp(np.float64(amax))
        return max(-127, int(e) - 1 - 2)
    s = np.float32(amax) / np.float32(dst)          # binary32 quotient, as the page computes S
    if s == 0 or s < np.float32(2.0 ** -126):
        return -127
    m, e = np.frexp(np.float64(s))
    return int(e) - 1 if m == 0.5 else int(e)


@pytest.mark.parametrize("dst", [0.0, 6.0, 8.0, 12.0])
def test_exponent_closed_forms(dst):
    x = _rand_groups(1, 3000)
    amax = np.abs(x).max(axis=1)
    extra = np.array([1.0, 2.0, 6.0, 7.999, 8.0, 2.0 ** -126, 2.0 ** -127, 2.0 ** 120, 3e38], np.float32)
    for a in np.concatenate([amax, extra]):
        assert oracle.mx_scale_exp(a, dst) == _expected_exp(a, dst), (a, dst)


@pytest.mark.parametrize("dst", [0.0, 6.0, 10.0])
def test_nearest_grid_point_brute_force(dst):
    """Every output is the grid point q * 2^E nearest to v (ties to the even
    code, |v| / 2^E above 6 saturating), with E from the exponent rule."""
    x = _rand_groups(2, 400)
    out, scales, codes = oracle.mxfp4_fake_quant(x.reshape(-1), dst)
    out = out.reshape(x.shape)
    for g in range(x.shape[0]):
        e = int(scales[g]) - 127
        assert e == _expected_exp(np.abs(x[g]).max(), dst)
        a = np.abs(x[g].astype(np.float64)) * 2.0 ** -e
        d = np.abs(a[:, None] - GRID[None, :])
        best = d.min(axis=1, keepdims=True)
        cand = d == best
        # ties: the even code of the two nearest
        idx = np.where(cand.sum(axis=1) > 1, np.argmax(cand & (np.arange(8) % 2 == 0), axis=1), np.argmin(d, axis=1))
        q = np.where(a >= 6.0, 6.0, GRID[idx])
        want = np.copysign(q * 2.0 ** e, x[g]).astype(np.float32)
        assert np.array_equal(out[g].view(np.uint32), want.view(np.uint32)), g


@pytest.mark.parametrize("dst", [0.0, 6.0])
def test_invariants(dst):
    x = _rand_groups(3, 500).reshape(-1)
    out, scales, codes = oracle.mxfp4_fake_quant(x, dst)
    # sign symmetry
    o2, s2, _ = oracle.mxfp4_fake_quant(-x, dst)
    assert np.array_equal(o2, -out) and np.array_equal(s2, scales)
    # power-of-two covariance (scales that stay clear of the E8M0 limits)
    xs = (x * np.float32(2.0 ** 5)).astype(np.float32)
    o3, s3, _ = oracle.mxfp4_fake_quant(xs, dst)
    ok = (scales.astype(int) > 10) & (scales.astype(int) < 240)
    okel = np.repeat(ok, 32)
    assert np.array_equal(o3[okel], (out * np.float32(32.0))[okel])
    assert np.array_equal(s3[ok].astype(int), scales[ok].astype(int) + 5)
    # idempotence: a quantised group quantises to itself
    o4, _, _ = oracle.mxfp4_fake_quant(out, dst)
    assert np.array_equal(o4, out)
    # codes and scales give the outputs back
    e = np.repeat(scales.astype(np.int64) - 127, 32)
    mag = GRID[codes & 7]
    back = np.where(codes & 8, -mag, mag) * np.exp2(e.astype(np.float64))
    assert np.array_equal(back.astype(np.float32), out)
    # dstTypeMax 6 rounds the scale up: nothing saturates
    if dst == 6.0:
        assert np.all(np.abs(x.astype(np.float64)) * np.exp2(-e.astype(np.float64)) <= 6.0)


def test_argument_rules():
    with pytest.raises(ValueError):
        oracle.mxfp4_fake_quant(np.zeros(48, np.float32), 0.0)
    for bad in (1.0, 5.9, 12.5, -6.0):
        with pytest.raises(ValueError):
            oracle.mxfp4_fake_quant(np.zeros(32, np.float32), bad)
    out, scales, codes = oracle.mxfp4_fake_quant(np.zeros(0, np.float32), 0.0)
    assert out.size == 0 and scales.size == 0
